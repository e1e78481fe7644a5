// qsa_sparse_decode: softmax attention of every Q head over the selected
// micro-blocks (plus the causal tail) of its query, on the uncompressed BF16
// K/V, written as split-KV partials (o, lse).
//
// Source: [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section
// "Wat de pull request daadwerkelijk verandert" (final softmax and value
// aggregation on the uncompressed K and V; the split read is combined
// afterwards); [CANN] "Qwen4-Exp QSA komt naar Huawei's Ascend ...", sections
// "Wat de pull request daadwerkelijk toevoegt" (D256 scale, zero output for
// fully masked rows) and "Negen tests ..." (causal tail remainders 0..3).
//
// Work decomposition.  Each (query, KV head) pair owns K+1 unit slots: the K
// selection slots (one micro-block of 4 tokens each: its 4 K rows and 4 V rows
// of one KV head form one contiguous 4 KiB run in the cache) and the tail slot.  All slots, query
// major, are cut into fixed chunks; one CTA per chunk, so every SM gets the
// same number of slots whatever the batch shape.  The part of a pair inside a
// chunk is a "segment"; each segment yields one split partial.
//
// CTA = 8 consumer warps + 2 copy warps + a lookup warp, 1 CTA per SM.
//   lookup warp: walks the CTA's units 32 at a time (selection -> page table),
//     four batches per round, and writes their source offsets into an 8-batch
//     descriptor queue, so the dependent selection and page-table loads run
//     ahead of the copies.
//   copy warps: tile T (4 units) belongs to copy warp T % 2, which moves each
//     unit's 4 KiB with 16-byte cp.async copies (every lane 8 per unit) into
//     an 8-stage shared-memory ring; each lane then arrives on the stage's
//     mbarrier when its copies land (cp.async.mbarrier.arrive.noinc).  With
//     one issuing thread per SM (a 1-D bulk copy per unit) random 4 KiB
//     gathers stayed near half the HBM rate on B200; spreading the issue over
//     the lanes of more warps is what raises the gather rate.
//   consumers: 4 pairs of warps; tile T (16 tokens) belongs to pair T % 4.
//     Each warp of a pair computes S = Q K^T over its half of the 256 dims
//     (mma.sync m16n8k16, M = 16 Q-head rows of the KV group, fp32
//     accumulate) and the pair swaps the partial sums through shared memory,
//     so both hold the whole S; both run the same online softmax, and each
//     accumulates O += P V for its half of the 256 output dims, which halves
//     the accumulator registers and lets 8 consumer warps keep the copies
//     fed.  At the end of a segment the 4 pairs merge their (m, l, O) in two
//     steps through shared memory and write the partial.
// FP8 e4m3 K/V (template F8): 2 KiB units, a 16-stage ring of 8 KiB tiles, K
// and V widened to FP16 in registers, FP16 MMAs.
// Shared-memory layouts are skewed so that every 16-byte fragment read is
// bank-conflict free (micro-block slots 4128 B apart, Q rows 576 B apart).
#include "qsa_common.cuh"

namespace {

using namespace qsa;

constexpr int kConsumerWarps = 8;                 // 4 pairs
constexpr int kPairs = kConsumerWarps / 2;
constexpr int kCopyWarps = 2;
constexpr int kCopyWarp0 = kConsumerWarps;                // warps 8, 9
constexpr int kLookupWarp = kConsumerWarps + kCopyWarps;  // warp 10
constexpr int kThreads = (kLookupWarp + 1) * 32;
constexpr int kConsumerThreads = kConsumerWarps * 32;
// A stage is reused by tile T + kStages; with kStages a multiple of the consumer
// pair count and tile T owned by pair T % 4, that tile's owner is the pair that
// consumed tile T, so no mbarrier wait can ever skip a phase (a parity wait can
// only name the current phase or the one before it).
constexpr int kUnitsPerTile = 4;
constexpr int kBatch = 32;                                             // units per lookup batch
constexpr int kRound = 4;                                              // lookup batches resolved together
constexpr int kDescSlots = 2 * kRound;                                 // lookup batches in flight
constexpr int kQRowStride = kHeadDim * 2 + 64;                         // 576
constexpr int kQBufBytes = 16 * kQRowStride;
constexpr int kCombRow = kHeadDim + 4;                                 // floats
constexpr int kCombBytes = 2 * 16 * kCombRow * 4;                      // two warps' O

// Shared-memory layout for BF16 (F8 = false) or FP8 e4m3 (F8 = true) K/V.
// A unit (one micro-block of one KV head) is 4 K rows then 4 V rows: 4 KiB in
// BF16, 2 KiB in FP8; the FP8 ring has twice the stages for the same bytes.
template <bool F8>
struct Lay {
  static constexpr int kStages = F8 ? 16 : 8;
  static constexpr int kHalfBytes = kRatio * kHeadDim * (F8 ? 1 : 2);  // 4 K (or V) rows
  static constexpr int kUnitBytes = 2 * kHalfBytes;
  static constexpr int kSlotStride = kUnitBytes + 32;                  // 16-B bank-group skew of 2
  static constexpr int kStageBytes = kUnitsPerTile * kSlotStride;
  static constexpr int kOffRing = 0;
  static constexpr int kOffQ = kOffRing + kStages * kStageBytes;
  static constexpr int kOffComb = kOffQ + kQBufBytes;
  static constexpr int kOffML = kOffComb + kCombBytes;
  static constexpr int kOffX = kOffML + kPairs * 16 * 2 * 4;              // S exchange: [pair][parity][half][lane][8]
  static constexpr int kOffDescOff = kOffX + kPairs * 2 * 2 * 32 * 8 * 4;
  static constexpr int kOffDescRows = kOffDescOff + kDescSlots * kBatch * 8;
  static constexpr int kOffMeta = kOffDescRows + kDescSlots * kBatch * 4;
  static constexpr int kOffBar = (kOffMeta + kStages * 4 + 7) & ~7;
  static constexpr int kNumBars = 2 * kStages + 2 * kDescSlots;
  static constexpr int kOffAbort = kOffBar + kNumBars * 8;
  static constexpr int kSmemBytes = kOffAbort + 16;
  static_assert(kSmemBytes <= 232448, "shared memory budget");
  static_assert(kStages % kPairs == 0 && kStages % kCopyWarps == 0, "tile ownership must repeat with the stage ring");
};

#define QSA_DECODE_LAYOUT                                   \
  using LY = Lay<F8>;                                       \
  constexpr int kStages = LY::kStages;                      \
  constexpr int kHalfBytes = LY::kHalfBytes;                \
  constexpr int kUnitBytes = LY::kUnitBytes;                \
  constexpr int kSlotStride = LY::kSlotStride;              \
  constexpr int kStageBytes = LY::kStageBytes;              \
  constexpr int kOffRing = LY::kOffRing;                    \
  constexpr int kOffQ = LY::kOffQ;                          \
  constexpr int kOffComb = LY::kOffComb;                    \
  constexpr int kOffML = LY::kOffML;                        \
  constexpr int kOffX = LY::kOffX;                          \
  constexpr int kOffDescOff = LY::kOffDescOff;              \
  constexpr int kOffDescRows = LY::kOffDescRows;            \
  constexpr int kOffMeta = LY::kOffMeta;                    \
  constexpr int kOffBar = LY::kOffBar;                      \
  constexpr int kOffAbort = LY::kOffAbort;                  \
  (void)kStages; (void)kHalfBytes; (void)kUnitBytes; (void)kSlotStride; (void)kStageBytes; (void)kOffRing; \
  (void)kOffQ; (void)kOffComb; (void)kOffML; (void)kOffX; (void)kOffDescOff; (void)kOffDescRows; (void)kOffMeta;      \
  (void)kOffBar; (void)kOffAbort
// full barrier: the 32 lanes' copy-completion arrivals + the owning copy warp's
// lane 0, whose plain (release) arrival publishes the stage's row mask
constexpr int kFullArrivals = 33;
constexpr uint64_t kWaitLimitNs = 2000000000ull;  // 2 s
constexpr int kBarConsumers = 1;                  // named barrier id
constexpr uint64_t kNoCopy = ~0ull;

struct DecodeArgs {
  const uint8_t* kv_bytes;
  const int32_t* bt;
  int32_t num_pages, max_seqs, mpps, hkv;
  const __nv_bfloat16* q;
  int32_t hq, G;
  const int32_t* q_seq;
  const int32_t* q_pos;
  const int32_t* sel;
  const int32_t* count;
  int32_t K;
  float scale_log2;
  int64_t chunk;
  int64_t total_slots;
  int32_t max_splits;
  float* part_o;
  float* part_lse;
  // in-kernel merge (all three null: partials only): per (query, KV group) the
  // number of its splits written so far, zero on entry and on exit
  int32_t* pair_done;
  __nv_bfloat16* out;  // [nq][hq][256]
  float* lse;          // [nq][hq]
  int32_t* st;
};

struct Seg {
  int q, g, split;
  int u0, u1;  // unit slots [u0, u1) of the pair
  int seq, nb, t;
  int n_main;  // selected blocks in the segment
  int n_valid, n_tiles;
  bool has_tail, last_of_pair, query_ok;
};

// Segment of pair `pair` inside chunk [x0, x1).  Identical in every warp.
__device__ __forceinline__ Seg make_seg(const DecodeArgs& a, int64_t pair, int64_t x0, int64_t x1, bool report) {
  Seg s;
  const int64_t n_slots = (int64_t)a.K + 1;
  const int64_t base = pair * n_slots;
  s.q = (int)(pair / a.hkv);
  s.g = (int)(pair % a.hkv);
  s.split = (int)(blockIdx.x - base / a.chunk);
  s.u0 = (int)(max(x0, base) - base);
  s.u1 = (int)(min(x1, base + n_slots) - base);
  s.last_of_pair = s.u1 == (int)n_slots;
  // the three per-query loads are independent: issued together, one latency
  s.seq = a.q_seq[s.q];
  const int p = a.q_pos[s.q];
  const int cnt_raw = a.count[s.q];
  s.query_ok = s.seq >= 0 && s.seq < a.max_seqs && p >= 0 && (int64_t)p < (int64_t)a.mpps * kPage;
  if (!s.query_ok) {
    if (report) flag(a.st, (s.seq < 0 || s.seq >= a.max_seqs) ? QSA_DEV_BAD_SEQ : QSA_DEV_BAD_POS);
    s.nb = 0;
    s.t = 0;
  } else {
    s.nb = (p + 1) / kRatio;
    s.t = (p + 1) % kRatio;
  }
  int cnt = s.query_ok ? cnt_raw : 0;
  const int cap = min(a.K, s.nb);
  if (cnt < 0 || cnt > cap) {
    if (report) flag(a.st, QSA_DEV_BAD_COUNT);
    cnt = cnt < 0 ? 0 : cap;
  }
  s.n_main = max(0, min(s.u1, cnt) - s.u0);
  s.has_tail = s.u0 <= a.K && a.K < s.u1 && s.t > 0;
  s.n_valid = s.n_main + (s.has_tail ? 1 : 0);
  s.n_tiles = (s.n_valid + kUnitsPerTile - 1) / kUnitsPerTile;
  return s;
}

// ------------------------------------------------------------------ producers

// Walk the CTA's segments in 32-unit batches (identical in both producer warps).
struct BatchIter {
  int64_t pair, last_pair, x0, x1;
  int ub;
  Seg s;
};

__device__ __forceinline__ bool iter_begin(const DecodeArgs& a, BatchIter& it, int64_t x0, int64_t x1) {
  const int64_t n_slots = (int64_t)a.K + 1;
  it.x0 = x0;
  it.x1 = x1;
  it.pair = x0 / n_slots;
  it.last_pair = (x1 - 1) / n_slots;
  it.ub = 0;
  it.s = make_seg(a, it.pair, x0, x1, false);
  while (it.s.n_valid == 0) {
    if (++it.pair > it.last_pair) return false;
    it.s = make_seg(a, it.pair, x0, x1, false);
  }
  return true;
}

__device__ __forceinline__ bool iter_next(const DecodeArgs& a, BatchIter& it) {
  it.ub += kBatch;
  while (it.ub >= it.s.n_valid) {
    if (++it.pair > it.last_pair) return false;
    it.s = make_seg(a, it.pair, it.x0, it.x1, false);
    it.ub = 0;
  }
  return true;
}

// bounded wait used by the producer warps: lane 0 polls, the warp agrees
__device__ __forceinline__ bool warp_wait(const DecodeArgs& a, uint32_t bar, uint32_t parity, volatile int* abort_flag) {
  const int lane = threadIdx.x & 31;
  int ok = 1;
  if (lane == 0) {
    ok = 0;
    if (mbar_try_wait(bar, parity)) {
      ok = 1;
    } else {
      const uint64_t t0 = global_timer_ns();
      for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) {
          ok = 1;
          break;
        }
        if ((it & 255u) == 255u) {
          if (*abort_flag) break;
          if (global_timer_ns() - t0 > kWaitLimitNs) {
            flag(a.st, QSA_DEV_TIMEOUT);
            *abort_flag = 1;
            break;
          }
        }
      }
    }
  }
  ok = __shfl_sync(0xffffffffu, ok, 0);
  __syncwarp();  // orders every lane after lane 0's acquire
  return ok != 0;
}

// warp-uniform read of the abort flag
__device__ __forceinline__ bool warp_aborted(volatile int* abort_flag) {
  int v = 0;
  if ((threadIdx.x & 31) == 0) v = *abort_flag;
  return __shfl_sync(0xffffffffu, v, 0) != 0;
}

// Where a lookup warp publishes the unit descriptors of each 32-unit batch.
struct LookupQueue {
  uint64_t* d_off;       // [kDescSlots][kBatch] byte offset of the unit in the K/V pages (kNoCopy: none)
  uint32_t* d_rows;      // [kDescSlots][kBatch] mask of the unit's valid rows
  uint32_t bar_dfull;    // kDescSlots mbarriers: batch written
  uint32_t bar_dempty;   // kDescSlots mbarriers: batch taken by every copy warp
  volatile int* abort_flag;
  uint32_t unit_bytes;
};

// Resolves kRound batches per round: the selection loads of all of them are
// issued together, then the page-table loads, so a round costs two dependent
// global-load latencies for 4 x 32 units.  The CTA's first selection entries
// are loaded before the per-query loads return (their address needs only the
// chunk's geometry), so the first round costs one latency less.
__device__ void lookup_run(const DecodeArgs& a, const LookupQueue& L, int64_t x0, int64_t x1) {
  const int lane = threadIdx.x & 31;
  uint64_t* d_off = L.d_off;
  uint32_t* d_rows = L.d_rows;
  const uint32_t bar_dfull = L.bar_dfull, bar_dempty = L.bar_dempty;
  volatile int* abort_flag = L.abort_flag;
  const int64_t n_slots = (int64_t)a.K + 1;
  const int64_t pair0 = x0 / n_slots;
  const int q_first = (int)(pair0 / a.hkv);
  const int u_first = (int)(x0 - pair0 * n_slots);
  int j_first = 0;
  if (u_first + lane < a.K) j_first = a.sel[(size_t)q_first * a.K + u_first + lane];
  bool first_round = true;
  BatchIter it;
  bool have = iter_begin(a, it, x0, x1);
  int b = 0;
  while (have) {
    int nr = 0;
    int q[kRound], seq[kRound], nb[kRound], t[kRound], sel_base[kRound], g[kRound], i_main[kRound], i_valid[kRound];
#pragma unroll
    for (int r = 0; r < kRound; ++r) {
      if (have) {  // warp-uniform
        const Seg& sg = it.s;
        q[r] = sg.q;
        g[r] = sg.g;
        seq[r] = sg.seq;
        nb[r] = sg.nb;
        t[r] = sg.t;
        sel_base[r] = sg.u0 + it.ub;
        i_main[r] = sg.n_main - it.ub;   // this batch's units below i_main are selected blocks
        i_valid[r] = sg.n_valid - it.ub; // ... below i_valid are valid (the tail last)
        nr = r + 1;
        have = iter_next(a, it);
      }
    }
    // 1. selection entries of every batch in the round (independent loads)
    int j[kRound];
    bool ok[kRound];
#pragma unroll
    for (int r = 0; r < kRound; ++r) {
      ok[r] = false;
      j[r] = 0;
      if (r < nr && lane < i_valid[r]) {
        if (lane < i_main[r]) {
          j[r] = (first_round && r == 0 && q[r] == q_first && sel_base[r] == u_first)
                     ? j_first
                     : a.sel[(size_t)q[r] * a.K + sel_base[r] + lane];
          ok[r] = true;
        } else {
          j[r] = nb[r];
          ok[r] = true;
        }
      }
    }
    first_round = false;
#pragma unroll
    for (int r = 0; r < kRound; ++r) {
      if (ok[r] && lane < i_main[r] && (j[r] < 0 || j[r] >= nb[r])) {
        flag(a.st, QSA_DEV_BAD_SEL);
        ok[r] = false;
      }
    }
    // 2. page-table entries (independent loads)
    int phys[kRound];
#pragma unroll
    for (int r = 0; r < kRound; ++r) phys[r] = ok[r] ? a.bt[(int64_t)seq[r] * a.mpps + j[r] / kBlocksPerPage] : -1;
    // 3. publish each batch's descriptors once its queue slot is free
#pragma unroll
    for (int r = 0; r < kRound; ++r) {
      if (r >= nr) break;
      const int bb = b + r;
      const int slot = bb % kDescSlots;
      if (bb >= kDescSlots && !warp_wait(a, bar_dempty + slot * 8, (uint32_t)((bb / kDescSlots - 1) & 1), abort_flag))
        return;
      if (warp_aborted(abort_flag)) return;
      uint64_t off = kNoCopy;
      uint32_t rows = 0;
      if (ok[r]) {
        if (phys[r] < 0 || phys[r] >= a.num_pages) {
          flag(a.st, QSA_DEV_BAD_PAGE);
        } else {
          off = (((uint64_t)phys[r] * a.hkv + g[r]) * kBlocksPerPage + (uint64_t)(j[r] % kBlocksPerPage)) *
                L.unit_bytes;  // bytes
          rows = lane < i_main[r] ? 0xFu : (1u << t[r]) - 1u;
        }
      }
      d_off[slot * kBatch + lane] = off;
      d_rows[slot * kBatch + lane] = rows;
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_dfull + slot * 8);
    }
    b += nr;
  }
}

template <bool F8>
__device__ void lookup_warp(const DecodeArgs& a, uint8_t* smem, int64_t x0, int64_t x1) {
  QSA_DECODE_LAYOUT;
  LookupQueue L;
  L.d_off = reinterpret_cast<uint64_t*>(smem + kOffDescOff);
  L.d_rows = reinterpret_cast<uint32_t*>(smem + kOffDescRows);
  L.bar_dfull = smem_u32(smem + kOffBar) + 2 * kStages * 8;
  L.bar_dempty = L.bar_dfull + kDescSlots * 8;
  L.abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  L.unit_bytes = kUnitBytes;
  lookup_run(a, L, x0, x1);
}

template <bool F8>
__device__ void copy_warp(const DecodeArgs& a, uint8_t* smem, int64_t x0, int64_t x1, int cw) {
  QSA_DECODE_LAYOUT;
  const int lane = threadIdx.x & 31;
  const uint32_t ring = smem_u32(smem + kOffRing);
  const uint32_t bar_full = smem_u32(smem + kOffBar);
  const uint32_t bar_empty = bar_full + kStages * 8;
  const uint32_t bar_dfull = bar_full + 2 * kStages * 8;
  const uint32_t bar_dempty = bar_dfull + kDescSlots * 8;
  const uint64_t* d_off = reinterpret_cast<const uint64_t*>(smem + kOffDescOff);
  const uint32_t* d_rows = reinterpret_cast<const uint32_t*>(smem + kOffDescRows);
  uint32_t* meta = reinterpret_cast<uint32_t*>(smem + kOffMeta);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  const uint64_t policy = l2_policy_evict_first();
  const char* kv = reinterpret_cast<const char*>(a.kv_bytes);
  int64_t T = 0;
  BatchIter it;
  bool have = iter_begin(a, it, x0, x1);
  for (int b = 0; have; ++b, have = iter_next(a, it)) {
    const int slot = b % kDescSlots;
    if (!warp_wait(a, bar_dfull + slot * 8, (uint32_t)((b / kDescSlots) & 1), abort_flag)) break;
    const uint64_t off = d_off[slot * kBatch + lane];
    const uint32_t rows = d_rows[slot * kBatch + lane];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_dempty + slot * 8);  // both copy warps arrive
    const int n_units = min(kBatch, it.s.n_valid - it.ub);
    const int tiles = (n_units + kUnitsPerTile - 1) / kUnitsPerTile;
    bool stop = false;
    for (int tb = 0; tb < tiles; ++tb, ++T) {
      if ((int)(T % kCopyWarps) != cw) continue;
      const int stage = (int)(T % kStages);
      if (T >= kStages && !warp_wait(a, bar_empty + stage * 8, (uint32_t)((T / kStages - 1) & 1), abort_flag)) {
        stop = true;
        break;
      }
      if (warp_aborted(abort_flag)) {
        stop = true;
        break;
      }
      const bool mine = (lane >> 2) == tb && lane < n_units;
      const uint32_t rowmask = __reduce_or_sync(0xffffffffu, mine ? (rows << ((lane & 3) * 4)) : 0u);
      const uint32_t dst = ring + stage * kStageBytes + lane * 16;
#pragma unroll
      for (int u = 0; u < kUnitsPerTile; ++u) {
        const uint64_t uoff = __shfl_sync(0xffffffffu, off, (tb * kUnitsPerTile + u) & 31);
        if (tb * kUnitsPerTile + u < n_units && uoff != kNoCopy) {
          const char* src = kv + uoff + lane * 16;
#pragma unroll
          for (int c = 0; c < kUnitBytes / 512; ++c) cp_async16(dst + u * kSlotStride + c * 512, src + c * 512, policy);
        }
      }
      if (lane == 0) {
        meta[stage] = rowmask;
        mbar_arrive(bar_full + stage * 8);
      }
      cp_async_arrive_noinc(bar_full + stage * 8);
    }
    if (stop) break;
  }
  // Never leave the CTA with copies in flight.
  cp_async_wait_all();
  __syncwarp();
}

// ------------------------------------------------------------------ consumers

__device__ __forceinline__ bool consumer_wait(const DecodeArgs& a, uint32_t bar, uint32_t parity,
                                              volatile int* abort_flag) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        flag(a.st, QSA_DEV_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

// Log-sum-exp merge of the nspl splits of pair (q, g) into out / lse, by the
// `nthreads` threads (a multiple of 32) of the CTA that wrote the pair's last
// split: thread t owns dims 4 (t % 64) .. + 3 of every row of the group it
// visits (rows t / 64, t / 64 + nthreads / 64, ... with 64 or more threads;
// with 32, dims 4t .. + 3 and 128 + 4t .. + 3 of every row).  The arithmetic is
// that of qsa_combine (same order over the splits), so the result is the same
// bit for bit.  Partials of other CTAs are read from L2.
__device__ __forceinline__ void merge_pair(const DecodeArgs& a, int q, int g, int nspl, int tid,
                                           int nthreads = kConsumerThreads) {
  const int G = a.G;
  const int per = nthreads >= 64 ? nthreads / 64 : 1;  // rows visited at once
  for (int idx = nthreads >= 64 ? tid >> 6 : 0; idx < G * (nthreads >= 64 ? 1 : 2); idx += per) {
    const int r = nthreads >= 64 ? idx : idx >> 1;
    const int c4 = nthreads >= 64 ? (tid & 63) : (tid & 31) + 32 * (idx & 1);
    const int h = g * G + r;
    const float* pl = a.part_lse + (size_t)q * a.max_splits * a.hq + h;
    const float* po = a.part_o + ((size_t)q * a.max_splits * a.hq + h) * kHeadDim + 4 * c4;
    float lse_v;
    const float4 res = merge_row(
        nspl, [&](int sp) { return __ldcg(pl + (size_t)sp * a.hq); },
        [&](int sp) { return __ldcg(reinterpret_cast<const float4*>(po + (size_t)sp * a.hq * kHeadDim)); }, lse_v);
    uint2 o;
    o.x = pack_bf16(res.x, res.y);
    o.y = pack_bf16(res.z, res.w);
    reinterpret_cast<uint2*>(a.out + ((size_t)q * a.hq + h) * kHeadDim)[c4] = o;
    if (c4 == 0) a.lse[(size_t)q * a.hq + h] = lse_v;
  }
}

template <bool F8>
__device__ void consumers(const DecodeArgs& a, uint8_t* smem, int64_t x0, int64_t x1) {
  QSA_DECODE_LAYOUT;
  const int tid = threadIdx.x;  // 0..255
  const int warp = tid >> 5, lane = tid & 31;
  const int cp = warp >> 1;     // consumer pair: owns tiles T with T % 4 == cp
  const int half = warp & 1;    // output dims [128 * half, 128 * half + 128)
  const int gq = lane >> 2, tq = lane & 3;
  const uint32_t ring = smem_u32(smem + kOffRing);
  const uint32_t bar_full = smem_u32(smem + kOffBar);
  const uint32_t bar_empty = bar_full + kStages * 8;
  const uint32_t* meta = reinterpret_cast<const uint32_t*>(smem + kOffMeta);
  float* comb = reinterpret_cast<float*>(smem + kOffComb);
  float* ml = reinterpret_cast<float*>(smem + kOffML);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + kOffAbort);
  const int64_t n_slots = (int64_t)a.K + 1;
  const int G = a.G;

  // K tile: S column n = gq of n-tile j is token (slot ks, row 2j + ke); the
  // lane holds dims 32i + 8tq .. + 7 of it for k-step pair i (Q likewise)
  constexpr int kRowBytes = kHalfBytes / kRatio;  // one K or V row: 512 B BF16, 256 B FP8
  constexpr int kElt = kRowBytes / kHeadDim;
  const int ke = gq & 1;
  const int ks = ((gq >> 1) + 2 * ke) & 3;
  const uint32_t k_off = ks * kSlotStride + ke * kRowBytes + tq * 8 * kElt;
  // S/P columns held by this lane: n = 2tq + e -> (slot (tq + 2e) & 3, row 2j + e)
  const int ps0 = tq, ps1 = (tq + 2) & 3;
  // V tokens of the PV B fragment: (ps0,row0) (ps1,row1) (ps0,row2) (ps1,row3); this
  // warp reads V chunks 8qq + gq for qq in {2 half, 2 half + 1}
  const uint32_t vh = kHalfBytes + half * 128 * kElt;
  const uint32_t v_off0 = ps0 * kSlotStride + vh + 0 * kRowBytes + gq * 8 * kElt;
  const uint32_t v_off1 = ps1 * kSlotStride + vh + 1 * kRowBytes + gq * 8 * kElt;
  const uint32_t v_off2 = ps0 * kSlotStride + vh + 2 * kRowBytes + gq * 8 * kElt;
  const uint32_t v_off3 = ps1 * kSlotStride + vh + 3 * kRowBytes + gq * 8 * kElt;
  const int vb0 = ps0 * 4 + 0, vb1 = ps1 * 4 + 1, vb2 = ps0 * 4 + 2, vb3 = ps1 * 4 + 3;

  int64_t T_base = 0;
  for (int64_t pair = x0 / n_slots; pair <= (x1 - 1) / n_slots; ++pair) {
    const Seg s = make_seg(a, pair, x0, x1, tid == 0);
    const uint32_t qb = smem_u32(smem + kOffQ);  // the merge barriers of the last segment order reuse
    // ---- stage Q rows of this KV group (rows >= G are zero); FP8 K/V takes
    // FP16 operands, so Q is converted (exact for normal BF16 values within +-65504)
    for (int idx = tid; idx < 16 * 32; idx += kConsumerThreads) {
      const int row = idx >> 5, c = idx & 31;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (row < G) v = ldg_nc(a.q + ((size_t)s.q * a.hq + (size_t)s.g * G + row) * kHeadDim + c * 8);
      if (!s.query_ok) v = make_uint4(0, 0, 0, 0);
      if constexpr (F8) {
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) w[e] = pack_f16_sat(__uint_as_float(w[e] << 16), __uint_as_float(w[e] & 0xffff0000u));
        v = make_uint4(w[0], w[1], w[2], w[3]);
      }
      sts128(qb + row * kQRowStride + c * 16, v);
    }
    named_bar_sync(kBarConsumers, kConsumerThreads);

    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

    // tile T (counted over the whole chunk) belongs to pair T % 4
    const int first_ti = (int)(((int64_t)cp - T_base % kPairs + kPairs) % kPairs);
    for (int ti = first_ti; ti < s.n_tiles; ti += kPairs) {
      const int64_t T = T_base + ti;
      const int stage = (int)(T % kStages);
      if (!*abort_flag) consumer_wait(a, bar_full + stage * 8, (uint32_t)((T / kStages) & 1), abort_flag);
      __syncwarp();  // reconverge before the warp-wide mma.sync
      const uint32_t mask = meta[stage];
      const uint32_t kb = ring + stage * kStageBytes;

      // ---- S = Q K^T : two n-tiles of 8 tokens; this warp sums its half of the
      // 256 dims (k-steps 8 half .. 8 half + 7) and the pair exchanges the partial
      // sums in shared memory (a + b == b + a, so both warps hold the same S)
      float sa[2][4], sb[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int c = 0; c < 4; ++c) sa[j][c] = sb[j][c] = 0.f;
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const int i = 4 * half + ii;
        const uint4 qa = lds128(qb + gq * kQRowStride + (4 * i + tq) * 16);
        const uint4 qc = lds128(qb + (gq + 8) * kQRowStride + (4 * i + tq) * 16);
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float(&acc)[4] = (ii & 1) ? sb[j] : sa[j];
          if constexpr (F8) {
            const uint4 kk = e4m3x8_to_f16x8(lds64(kb + k_off + j * 2 * kRowBytes + i * 32));
            mma_f16_16816(acc, qa.x, qc.x, qa.y, qc.y, kk.x, kk.y);
            mma_f16_16816(acc, qa.z, qc.z, qa.w, qc.w, kk.z, kk.w);
          } else {
            const uint4 kk = lds128(kb + k_off + j * 2 * kRowBytes + i * 64);
            mma_bf16_16816(acc, qa.x, qc.x, qa.y, qc.y, kk.x, kk.y);
            mma_bf16_16816(acc, qa.z, qc.z, qa.w, qc.w, kk.z, kk.w);
          }
        }
      }
      {
        float* xb = reinterpret_cast<float*>(smem + kOffX) + ((cp * 2 + (int)((T / kPairs) & 1)) * 2) * 256;
        float4* mine = reinterpret_cast<float4*>(xb + (half * 32 + lane) * 8);
        const float4 p0 = make_float4(sa[0][0] + sb[0][0], sa[0][1] + sb[0][1], sa[0][2] + sb[0][2], sa[0][3] + sb[0][3]);
        const float4 p1 = make_float4(sa[1][0] + sb[1][0], sa[1][1] + sb[1][1], sa[1][2] + sb[1][2], sa[1][3] + sb[1][3]);
        mine[0] = p0;
        mine[1] = p1;
        named_bar_sync(2 + cp, 64);  // the pair's two warps
        const float4* other = reinterpret_cast<const float4*>(xb + ((1 - half) * 32 + lane) * 8);
        const float4 o0 = other[0], o1 = other[1];
        sa[0][0] = p0.x + o0.x; sa[0][1] = p0.y + o0.y; sa[0][2] = p0.z + o0.z; sa[0][3] = p0.w + o0.w;
        sa[1][0] = p1.x + o1.x; sa[1][1] = p1.y + o1.y; sa[1][2] = p1.z + o1.z; sa[1][3] = p1.w + o1.w;
#pragma unroll
        for (int j = 0; j < 2; ++j)
#pragma unroll
          for (int c = 0; c < 4; ++c) sb[j][c] = 0.f;
      }
      // ---- mask, online softmax (base-2 logits)
      float z[2][4];
      float r0 = -INFINITY, r1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const bool v0 = (mask >> (ps0 * 4 + 2 * j)) & 1u;      // column 2tq   -> (ps0, row 2j)
        const bool v1 = (mask >> (ps1 * 4 + 2 * j + 1)) & 1u;  // column 2tq+1 -> (ps1, row 2j+1)
        z[j][0] = v0 ? (sa[j][0] + sb[j][0]) * a.scale_log2 : -INFINITY;
        z[j][1] = v1 ? (sa[j][1] + sb[j][1]) * a.scale_log2 : -INFINITY;
        z[j][2] = v0 ? (sa[j][2] + sb[j][2]) * a.scale_log2 : -INFINITY;
        z[j][3] = v1 ? (sa[j][3] + sb[j][3]) * a.scale_log2 : -INFINITY;
        r0 = fmaxf(r0, fmaxf(z[j][0], z[j][1]));
        r1 = fmaxf(r1, fmaxf(z[j][2], z[j][3]));
      }
      r0 = fmaxf(r0, __shfl_xor_sync(0xffffffffu, r0, 1));
      r1 = fmaxf(r1, __shfl_xor_sync(0xffffffffu, r1, 1));
      r0 = fmaxf(r0, __shfl_xor_sync(0xffffffffu, r0, 2));
      r1 = fmaxf(r1, __shfl_xor_sync(0xffffffffu, r1, 2));
      const float mn0 = fmaxf(m0, r0), mn1 = fmaxf(m1, r1);
      // a tile whose units were all rejected as bad data keeps every logit at -inf
      const float sub0 = mn0 == -INFINITY ? 0.f : mn0, sub1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = exp2f(m0 - sub0), al1 = exp2f(m1 - sub1);
      m0 = mn0;
      m1 = mn1;
      float pr[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        pr[j][0] = exp2f(z[j][0] - sub0);
        pr[j][1] = exp2f(z[j][1] - sub0);
        pr[j][2] = exp2f(z[j][2] - sub1);
        pr[j][3] = exp2f(z[j][3] - sub1);
      }
      l0 = l0 * al0 + ((pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]));
      l1 = l1 * al1 + ((pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]));
      if (al0 != 1.f || al1 != 1.f) {
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          o[nt][0] *= al0;
          o[nt][1] *= al0;
          o[nt][2] *= al1;
          o[nt][3] *= al1;
        }
      }
      // BF16 K/V: P = hi + lo, both BF16, so the PV product keeps ~17
      // significant bits of every weight (BF16 alone, 8 bits, is too coarse for
      // short token sets).  FP8 K/V: P in FP16 (11 bits) against e4m3 V (4 bits).
      uint32_t pa[4], pl[4];
      if constexpr (F8) {
        pa[0] = pack_f16_sat(pr[0][0], pr[0][1]);
        pa[1] = pack_f16_sat(pr[0][2], pr[0][3]);
        pa[2] = pack_f16_sat(pr[1][0], pr[1][1]);
        pa[3] = pack_f16_sat(pr[1][2], pr[1][3]);
        pl[0] = pl[1] = pl[2] = pl[3] = 0u;
      } else {
        split_bf16(pr[0][0], pr[0][1], pa[0], pl[0]);
        split_bf16(pr[0][2], pr[0][3], pa[1], pl[1]);
        split_bf16(pr[1][0], pr[1][1], pa[2], pl[2]);
        split_bf16(pr[1][2], pr[1][3], pa[3], pl[3]);
      }

      // ---- O += P V for this warp's 128 dims: 16 n-tiles, k = the tile's 16 tokens
      const bool full = mask == 0xffffu;
      const bool ok0 = (mask >> vb0) & 1u, ok1 = (mask >> vb1) & 1u;
      const bool ok2 = (mask >> vb2) & 1u, ok3 = (mask >> vb3) & 1u;
#pragma unroll
      for (int qh = 0; qh < 2; ++qh) {
        uint4 x0v, x1v, x2v, x3v;
        if constexpr (F8) {
          x0v = e4m3x8_to_f16x8(lds64(kb + v_off0 + qh * 64));
          x1v = e4m3x8_to_f16x8(lds64(kb + v_off1 + qh * 64));
          x2v = e4m3x8_to_f16x8(lds64(kb + v_off2 + qh * 64));
          x3v = e4m3x8_to_f16x8(lds64(kb + v_off3 + qh * 64));
        } else {
          x0v = lds128(kb + v_off0 + qh * 128);
          x1v = lds128(kb + v_off1 + qh * 128);
          x2v = lds128(kb + v_off2 + qh * 128);
          x3v = lds128(kb + v_off3 + qh * 128);
        }
        if (!full) {  // masked rows may hold stale or never-written data
          if (!ok0) x0v = make_uint4(0, 0, 0, 0);
          if (!ok1) x1v = make_uint4(0, 0, 0, 0);
          if (!ok2) x2v = make_uint4(0, 0, 0, 0);
          if (!ok3) x3v = make_uint4(0, 0, 0, 0);
        }
        const uint32_t a0[4] = {x0v.x, x0v.y, x0v.z, x0v.w};
        const uint32_t a1[4] = {x1v.x, x1v.y, x1v.z, x1v.w};
        const uint32_t a2[4] = {x2v.x, x2v.y, x2v.z, x2v.w};
        const uint32_t a3[4] = {x3v.x, x3v.y, x3v.z, x3v.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint32_t lo01 = __byte_perm(a0[r], a1[r], 0x5410);
          const uint32_t hi01 = __byte_perm(a0[r], a1[r], 0x7632);
          const uint32_t lo23 = __byte_perm(a2[r], a3[r], 0x5410);
          const uint32_t hi23 = __byte_perm(a2[r], a3[r], 0x7632);
          if constexpr (F8) {
            mma_f16_16816(o[qh * 8 + 2 * r], pa[0], pa[1], pa[2], pa[3], lo01, lo23);
            mma_f16_16816(o[qh * 8 + 2 * r + 1], pa[0], pa[1], pa[2], pa[3], hi01, hi23);
          } else {
            mma_bf16_16816(o[qh * 8 + 2 * r], pa[0], pa[1], pa[2], pa[3], lo01, lo23);
            mma_bf16_16816(o[qh * 8 + 2 * r + 1], pa[0], pa[1], pa[2], pa[3], hi01, hi23);
            mma_bf16_16816(o[qh * 8 + 2 * r], pl[0], pl[1], pl[2], pl[3], lo01, lo23);
            mma_bf16_16816(o[qh * 8 + 2 * r + 1], pl[0], pl[1], pl[2], pl[3], hi01, hi23);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty + stage * 8);  // both warps of the pair arrive
    }
    T_base += s.n_tiles;

    // ---- merge the 4 pairs' (m, l, O) and write the split partial
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (half == 0 && tq == 0) {  // both warps of a pair hold the same m and l
      ml[(cp * 16 + gq) * 2 + 0] = m0;
      ml[(cp * 16 + gq) * 2 + 1] = l0;
      ml[(cp * 16 + gq + 8) * 2 + 0] = m1;
      ml[(cp * 16 + gq + 8) * 2 + 1] = l1;
    }
    named_bar_sync(kBarConsumers, kConsumerThreads);
    // this pair's weight for rows gq / gq+8, and the merged lse of those rows
    float fac[2], lse_row[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int row = gq + 8 * hr;
      const float mine = hr ? m1 : m0;
      float M = -INFINITY;
      for (int w = 0; w < kPairs; ++w) M = fmaxf(M, ml[(w * 16 + row) * 2]);
      fac[hr] = 0.f;
      lse_row[hr] = -INFINITY;
      if (M != -INFINITY) {
        float L = 0.f;
        for (int w = 0; w < kPairs; ++w) {
          const float mw = ml[(w * 16 + row) * 2];
          if (mw != -INFINITY) L += ml[(w * 16 + row) * 2 + 1] * exp2f(mw - M);
        }
        fac[hr] = mine != -INFINITY ? exp2f(mine - M) / L : 0.f;
        lse_row[hr] = (M + log2f(L)) * 0.69314718055994530942f;
      }
    }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      o[nt][0] *= fac[0];
      o[nt][1] *= fac[0];
      o[nt][2] *= fac[1];
      o[nt][3] *= fac[1];
    }
    // local n-tile 8qh + w8 holds dims 128half + 64qh + 16tq + w8 (c0/c2) and + 8 (c1/c3)
    auto store_rows = [&](float* base, int row_stride) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int row = gq + 8 * hr;
        if (row >= G) continue;
        const int c = 2 * hr;
#pragma unroll
        for (int qh = 0; qh < 2; ++qh) {
          float4* d4 = reinterpret_cast<float4*>(base + (size_t)row * row_stride + 128 * half + 64 * qh + 16 * tq);
          d4[0] = make_float4(o[qh * 8 + 0][c], o[qh * 8 + 1][c], o[qh * 8 + 2][c], o[qh * 8 + 3][c]);
          d4[1] = make_float4(o[qh * 8 + 4][c], o[qh * 8 + 5][c], o[qh * 8 + 6][c], o[qh * 8 + 7][c]);
          d4[2] = make_float4(o[qh * 8 + 0][c + 1], o[qh * 8 + 1][c + 1], o[qh * 8 + 2][c + 1], o[qh * 8 + 3][c + 1]);
          d4[3] = make_float4(o[qh * 8 + 4][c + 1], o[qh * 8 + 5][c + 1], o[qh * 8 + 6][c + 1], o[qh * 8 + 7][c + 1]);
        }
      }
    };
    auto add_rows = [&](const float* base) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int row = gq + 8 * hr;
        if (row >= G) continue;
        const int c = 2 * hr;
#pragma unroll
        for (int qh = 0; qh < 2; ++qh) {
          const float4* s4 = reinterpret_cast<const float4*>(base + row * kCombRow + 128 * half + 64 * qh + 16 * tq);
          const float4 x0 = s4[0], x1 = s4[1], x2 = s4[2], x3 = s4[3];
          o[qh * 8 + 0][c] += x0.x; o[qh * 8 + 1][c] += x0.y; o[qh * 8 + 2][c] += x0.z; o[qh * 8 + 3][c] += x0.w;
          o[qh * 8 + 4][c] += x1.x; o[qh * 8 + 5][c] += x1.y; o[qh * 8 + 6][c] += x1.z; o[qh * 8 + 7][c] += x1.w;
          o[qh * 8 + 0][c + 1] += x2.x; o[qh * 8 + 1][c + 1] += x2.y; o[qh * 8 + 2][c + 1] += x2.z;
          o[qh * 8 + 3][c + 1] += x2.w;
          o[qh * 8 + 4][c + 1] += x3.x; o[qh * 8 + 5][c + 1] += x3.y; o[qh * 8 + 6][c + 1] += x3.z;
          o[qh * 8 + 7][c + 1] += x3.w;
        }
      }
    };
    // merge step 1: pairs 2, 3 hand their O to pairs 0, 1; step 2: pair 1 to pair 0
    if (cp >= 2) store_rows(comb + (cp - 2) * 16 * kCombRow, kCombRow);
    named_bar_sync(kBarConsumers, kConsumerThreads);
    if (cp < 2) add_rows(comb + cp * 16 * kCombRow);
    named_bar_sync(kBarConsumers, kConsumerThreads);
    if (cp == 1) store_rows(comb, kCombRow);
    named_bar_sync(kBarConsumers, kConsumerThreads);
    const size_t row0 = ((size_t)s.q * a.max_splits + s.split) * a.hq + (size_t)s.g * G;
    if (cp == 0) {
      add_rows(comb);
      store_rows(a.part_o + row0 * kHeadDim, kHeadDim);
      if (half == 0 && tq == 0) {
        if (gq < G) a.part_lse[row0 + gq] = lse_row[0];
        if (gq + 8 < G) a.part_lse[row0 + gq + 8] = lse_row[1];
      }
    }
    if (s.last_of_pair) {  // slots this pair never reaches: empty splits
      for (int sp = s.split + 1; sp < a.max_splits; ++sp) {
        const size_t r0 = ((size_t)s.q * a.max_splits + sp) * a.hq + (size_t)s.g * G;
        for (int idx = tid; idx < G * 64; idx += kConsumerThreads)
          *reinterpret_cast<float4*>(a.part_o + (r0 + (idx >> 6)) * kHeadDim + (idx & 63) * 4) =
              make_float4(0.f, 0.f, 0.f, 0.f);
        for (int row = tid; row < G; row += kConsumerThreads) a.part_lse[r0 + row] = -INFINITY;
      }
    }
    if (a.pair_done) {
      // The CTA that writes a pair's last split merges the pair: every writer
      // fences its partial stores, one thread counts the split (device-scope
      // atomic) and fences again before the merge reads the other splits.
      __threadfence();
      named_bar_sync(kBarConsumers, kConsumerThreads);
      volatile int* last_flag = reinterpret_cast<volatile int*>(ml);  // ml is free until the next segment ends
      const int64_t base = pair * n_slots;
      const int nspl = (int)((base + n_slots - 1) / a.chunk - base / a.chunk) + 1;
      if (tid == 0) {
        const int done = atomicAdd(a.pair_done + pair, 1);
        const bool last = done == nspl - 1;
        if (last) a.pair_done[pair] = 0;  // every other split has counted: ready for the next call
        __threadfence();
        *last_flag = last ? 1 : 0;
      }
      named_bar_sync(kBarConsumers, kConsumerThreads);
      const bool last = *last_flag != 0;
      named_bar_sync(kBarConsumers, kConsumerThreads);  // the flag is read before ml is written again
      if (last) merge_pair(a, s.q, s.g, nspl, tid);
    }
  }
}

template <bool F8>
__global__ void __launch_bounds__(kThreads, 1) sparse_decode_kernel(DecodeArgs a) {
  QSA_DECODE_LAYOUT;
  extern __shared__ __align__(128) uint8_t smem[];
  pdl_launch_dependents();
  const int64_t x0 = (int64_t)blockIdx.x * a.chunk;
  const int64_t x1 = min(x0 + a.chunk, a.total_slots);
  if (threadIdx.x == 0) {
    const uint32_t bf = smem_u32(smem + kOffBar);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(bf + i * 8, kFullArrivals);      // full: copy completions + row mask published
      mbar_init(bf + (kStages + i) * 8, 2);      // empty: both warps of the owning pair
    }
    for (int i = 0; i < kDescSlots; ++i) {
      mbar_init(bf + (2 * kStages + i) * 8, 1);               // descriptors written (lookup warp)
      mbar_init(bf + (2 * kStages + kDescSlots + i) * 8, kCopyWarps);  // descriptors taken (copy warps)
    }
    *reinterpret_cast<volatile int*>(smem + kOffAbort) = 0;
    fence_mbar_init();
  }
  pdl_wait_previous();  // the selection and counts come from the previous kernel
  __syncthreads();
  if (x0 >= x1) return;
  const int warp = threadIdx.x >> 5;
  if (warp >= kCopyWarp0 && warp < kCopyWarp0 + kCopyWarps)
    copy_warp<F8>(a, smem, x0, x1, warp - kCopyWarp0);
  else if (warp == kLookupWarp)
    lookup_warp<F8>(a, smem, x0, x1);
  else
    consumers<F8>(a, smem, x0, x1);
}

template <bool F8>
int launch_decode(const DecodeArgs& a, int64_t grid, void* stream) {
  constexpr int kSmem = Lay<F8>::kSmemBytes;
  cudaError_t e = cudaFuncSetAttribute(sparse_decode_kernel<F8>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  return qsa_host::launch(sparse_decode_kernel<F8>, dim3((unsigned)grid), dim3(kThreads), kSmem,
                          static_cast<cudaStream_t>(stream), a);
}

// ================================================================== BF16 form
//
// The BF16 cache stores each micro-block of one KV head as one 4 KiB run:
// [4 dim atoms][8 rows: K 0-3, V 0-3][64 elements], the 16-byte chunk c of row
// r at chunk position c ^ r (128-byte swizzle); the copy warps move each
// selected run to its shared-memory slot as it is, with 16-byte cp.async
// copies from every lane (bulk copies of whole runs, one per run, kept fewer
// bytes in flight per SM on B200: about 29 GB/s per SM against 43 for the
// 16-byte copies, whatever the ring depth).
// The consumers are those of the mma.sync form, with fragment addresses
// chosen for the swizzled rows so that every 16-byte fragment read of a warp is
// bank-conflict free:
//   * S n-tile j, column n is token (unit 2j + (n & 1), row (n >> 1) ^ (n & 1));
//     for k-step pair i the lane reads chunk 8 (i >> 1) + 2 tq + (i & 1) of it
//     (the contraction index is permuted identically in Q and K);
//   * the PV B fragment's k index 2tq + (L & 1) + 8 (L >> 1) is then token
//     (unit L, row tq ^ (L & 1)); lane gq reads dims chunk
//     kappa(gq) = (gq >> 1) | ((gq & 1) << 2) of each 64-dim group, so output
//     column n of an n-tile is dim 8 kappa(n) + the n-tile's offset.
// Q fragments stay in registers for a whole segment.
namespace sdb {

constexpr int kUnitsPerTileB = 4;                       // 16 tokens
constexpr int kStagesB = 8;
constexpr int kUnitBytesB = 4096;
constexpr int kStageBytesB = kUnitsPerTileB * kUnitBytesB;  // 16 KiB
constexpr int kCopyWarp0B = kConsumerWarps;             // warps 8, 9
constexpr int kLookupWarpB = kConsumerWarps + kCopyWarps;  // warp 10
constexpr int kThreadsB = (kLookupWarpB + 1) * 32;
constexpr int kOffComb = kStagesB * kStageBytesB;
constexpr int kOffMLB = kOffComb + kCombBytes;
constexpr int kOffXB = kOffMLB + kPairs * 16 * 2 * 4;
constexpr int kOffDescOffB = kOffXB + kPairs * 2 * 2 * 32 * 8 * 4;
constexpr int kOffDescRowsB = kOffDescOffB + kDescSlots * kBatch * 8;
constexpr int kOffMetaB = kOffDescRowsB + kDescSlots * kBatch * 4;
constexpr int kOffBarB = (kOffMetaB + kStagesB * 4 + 7) & ~7;
constexpr int kNumBarsB = 2 * kStagesB + 2 * kDescSlots;
constexpr int kOffAbortB = kOffBarB + kNumBarsB * 8;
constexpr int kSmemUsedB = kOffAbortB + 16;
constexpr int kSmemBytesB = kSmemUsedB + 128;           // slack to align the ring to 128 B
static_assert(kSmemBytesB <= 232448, "shared memory budget");
static_assert(kStagesB % kPairs == 0 && kStagesB % kCopyWarps == 0, "tile ownership must repeat with the stage ring");

struct Ctx {
  uint8_t* smem;   // 128-B aligned
  uint32_t ring;   // its shared address
  uint32_t bar;    // full[kStagesB], empty[kStagesB], dfull[kDescSlots], dempty[kDescSlots]
  volatile int* abort_flag;
};

// ------------------------------------------------------------------ copy warps

// Tile T (4 runs) belongs to copy warp T % 2; every lane copies 16 bytes of each
// 512-byte eighth of each run and arrives on the stage's mbarrier when its copies
// land (cp.async.mbarrier.arrive.noinc); lane 0 also publishes the row mask.
__device__ void copy_run(const DecodeArgs& a, const Ctx& c, int64_t x0, int64_t x1, int cw) {
  const int lane = threadIdx.x & 31;
  const uint64_t* d_off = reinterpret_cast<const uint64_t*>(c.smem + kOffDescOffB);
  const uint32_t* d_rows = reinterpret_cast<const uint32_t*>(c.smem + kOffDescRowsB);
  uint32_t* meta = reinterpret_cast<uint32_t*>(c.smem + kOffMetaB);
  const uint32_t bar_full = c.bar, bar_empty = c.bar + kStagesB * 8;
  const uint32_t bar_dfull = c.bar + 2 * kStagesB * 8, bar_dempty = bar_dfull + kDescSlots * 8;
  const uint64_t policy = l2_policy_evict_first();
  const char* kv = reinterpret_cast<const char*>(a.kv_bytes);
  int64_t T = 0;
  BatchIter it;
  bool have = iter_begin(a, it, x0, x1);
  for (int b = 0; have; ++b, have = iter_next(a, it)) {
    const int slot = b % kDescSlots;
    if (!warp_wait(a, bar_dfull + slot * 8, (uint32_t)((b / kDescSlots) & 1), c.abort_flag)) break;
    const uint64_t off = d_off[slot * kBatch + lane];
    const uint32_t rows = d_rows[slot * kBatch + lane];
    __syncwarp();
    if (lane == 0) mbar_arrive(bar_dempty + slot * 8);  // both copy warps arrive
    const int n_units = min(kBatch, it.s.n_valid - it.ub);
    const int tiles = (n_units + kUnitsPerTileB - 1) / kUnitsPerTileB;
    bool stop = false;
    for (int tb = 0; tb < tiles; ++tb, ++T) {
      if ((int)(T % kCopyWarps) != cw) continue;
      const int stage = (int)(T % kStagesB);
      if (T >= kStagesB && !warp_wait(a, bar_empty + stage * 8, (uint32_t)((T / kStagesB - 1) & 1), c.abort_flag)) {
        stop = true;
        break;
      }
      if (warp_aborted(c.abort_flag)) {
        stop = true;
        break;
      }
      const bool mine = (lane >> 2) == tb && lane < n_units;
      const uint32_t rowmask = __reduce_or_sync(0xffffffffu, mine ? (rows << ((lane & 3) * 4)) : 0u);
      const uint32_t dst = c.ring + (uint32_t)stage * kStageBytesB + lane * 16;
#pragma unroll
      for (int u = 0; u < kUnitsPerTileB; ++u) {
        const uint64_t uoff = __shfl_sync(0xffffffffu, off, (tb * kUnitsPerTileB + u) & 31);
        if (tb * kUnitsPerTileB + u < n_units && uoff != kNoCopy) {
          const char* src = kv + uoff + lane * 16;
#pragma unroll
          for (int q8 = 0; q8 < kUnitBytesB / 512; ++q8) cp_async16(dst + u * kUnitBytesB + q8 * 512, src + q8 * 512, policy);
        }
      }
      if (lane == 0) {
        meta[stage] = rowmask;
        mbar_arrive(bar_full + stage * 8);
      }
      cp_async_arrive_noinc(bar_full + stage * 8);
    }
    if (stop) break;
  }
  // Never leave the CTA with copies in flight.
  cp_async_wait_all();
  __syncwarp();
}

// ------------------------------------------------------------------ consumers

__device__ void consumers(const DecodeArgs& a, const Ctx& c, int64_t x0, int64_t x1) {
  const int tid = threadIdx.x;  // 0..255
  const int warp = tid >> 5, lane = tid & 31;
  const int cp = warp >> 1;     // consumer pair: owns tiles T with T % 4 == cp
  const int half = warp & 1;    // output dims [128 * half, 128 * half + 128)
  const int gq = lane >> 2, tq = lane & 3;
  const uint32_t bar_full = c.bar, bar_empty = c.bar + kStagesB * 8;
  const uint32_t* meta = reinterpret_cast<const uint32_t*>(c.smem + kOffMetaB);
  float* comb = reinterpret_cast<float*>(c.smem + kOffComb);
  float* ml = reinterpret_cast<float*>(c.smem + kOffMLB);
  volatile int* abort_flag = c.abort_flag;
  const int64_t n_slots = (int64_t)a.K + 1;
  const int G = a.G;

  // K fragment of S n-tile j: token (unit 2j + (gq & 1), row kr); byte offsets of its
  // chunk 8 (i >> 1) + 2 tq + (i & 1) for the warp's k-step pairs i = 4 half + ii
  const int kr = (gq >> 1) ^ (gq & 1);
  uint32_t koff[4];
#pragma unroll
  for (int ii = 0; ii < 4; ++ii) {
    const int i = 4 * half + ii;
    const int ch = 8 * (i >> 1) + 2 * tq + (i & 1);
    koff[ii] = (uint32_t)((gq & 1) * kUnitBytesB + (ch >> 3) * 1024 + kr * 128 + (((ch & 7) ^ kr) << 4));
  }
  // V loads L = 0..3: token (unit L, row tq ^ (L & 1)) = smem row 4 + that, chunk
  // kappa(gq) of the 64-dim group 2 half + qh
  const int kap = (gq >> 1) | ((gq & 1) << 2);
  uint32_t voff[4];
#pragma unroll
  for (int L = 0; L < 4; ++L) {
    const int vr = kRatio + (tq ^ (L & 1));
    voff[L] = (uint32_t)(L * kUnitBytesB + (2 * half) * 1024 + vr * 128 + ((kap ^ vr) << 4));
  }
  // mask bits of the lane's S columns 2tq + e of n-tile j: token (unit 2j + e, row tq ^ e)
  const int mb00 = 0 * 4 + tq, mb01 = 1 * 4 + (tq ^ 1), mb10 = 2 * 4 + tq, mb11 = 3 * 4 + (tq ^ 1);

  int64_t T_base = 0;
  for (int64_t pair = x0 / n_slots; pair <= (x1 - 1) / n_slots; ++pair) {
    const Seg s = make_seg(a, pair, x0, x1, tid == 0);
    const int n_tiles = (s.n_valid + kUnitsPerTileB - 1) / kUnitsPerTileB;
    // ---- Q fragments of this KV group (rows >= G are zero), for the whole segment
    uint4 qa[4], qc[4];
    {
      const __nv_bfloat16* qrow = a.q + ((size_t)s.q * a.hq + (size_t)s.g * G) * kHeadDim;
      const bool ra = s.query_ok && gq < G, rc = s.query_ok && gq + 8 < G;
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
        const int i = 4 * half + ii;
        const int ch = 8 * (i >> 1) + 2 * tq + (i & 1);
        qa[ii] = ra ? ldg_nc(qrow + (size_t)gq * kHeadDim + ch * 8) : make_uint4(0, 0, 0, 0);
        qc[ii] = rc ? ldg_nc(qrow + (size_t)(gq + 8) * kHeadDim + ch * 8) : make_uint4(0, 0, 0, 0);
      }
    }

    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;
    float o[16][4];
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

    // tile T (counted over the whole chunk) belongs to pair T % 4
    const int first_ti = (int)(((int64_t)cp - T_base % kPairs + kPairs) % kPairs);
    for (int ti = first_ti; ti < n_tiles; ti += kPairs) {
      const int64_t T = T_base + ti;
      const int stage = (int)(T % kStagesB);
      if (!*abort_flag) consumer_wait(a, bar_full + stage * 8, (uint32_t)((T / kStagesB) & 1), abort_flag);
      __syncwarp();  // reconverge before the warp-wide mma.sync
      const uint32_t mask = meta[stage];
      const uint32_t kb = c.ring + (uint32_t)stage * kStageBytesB;

      // ---- S = Q K^T over this warp's half of the dims; the pair swaps the partial sums
      float sa[2][4], sb[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) sa[j][e] = sb[j][e] = 0.f;
#pragma unroll
      for (int ii = 0; ii < 4; ++ii) {
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          float(&acc)[4] = (ii & 1) ? sb[j] : sa[j];
          const uint4 kk = lds128(kb + j * 2 * kUnitBytesB + koff[ii]);
          mma_bf16_16816(acc, qa[ii].x, qc[ii].x, qa[ii].y, qc[ii].y, kk.x, kk.y);
          mma_bf16_16816(acc, qa[ii].z, qc[ii].z, qa[ii].w, qc[ii].w, kk.z, kk.w);
        }
      }
      {
        float* xb = reinterpret_cast<float*>(c.smem + kOffXB) + ((cp * 2 + (int)((T / kPairs) & 1)) * 2) * 256;
        float4* mine = reinterpret_cast<float4*>(xb + (half * 32 + lane) * 8);
        const float4 p0 = make_float4(sa[0][0] + sb[0][0], sa[0][1] + sb[0][1], sa[0][2] + sb[0][2], sa[0][3] + sb[0][3]);
        const float4 p1 = make_float4(sa[1][0] + sb[1][0], sa[1][1] + sb[1][1], sa[1][2] + sb[1][2], sa[1][3] + sb[1][3]);
        mine[0] = p0;
        mine[1] = p1;
        named_bar_sync(2 + cp, 64);  // the pair's two warps
        const float4* other = reinterpret_cast<const float4*>(xb + ((1 - half) * 32 + lane) * 8);
        const float4 o0 = other[0], o1 = other[1];
        sa[0][0] = p0.x + o0.x; sa[0][1] = p0.y + o0.y; sa[0][2] = p0.z + o0.z; sa[0][3] = p0.w + o0.w;
        sa[1][0] = p1.x + o1.x; sa[1][1] = p1.y + o1.y; sa[1][2] = p1.z + o1.z; sa[1][3] = p1.w + o1.w;
      }
      // ---- mask, online softmax (base-2 logits)
      float z[2][4];
      float r0 = -INFINITY, r1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const bool v0 = (mask >> (j ? mb10 : mb00)) & 1u;  // column 2tq
        const bool v1 = (mask >> (j ? mb11 : mb01)) & 1u;  // column 2tq + 1
        z[j][0] = v0 ? sa[j][0] * a.scale_log2 : -INFINITY;
        z[j][1] = v1 ? sa[j][1] * a.scale_log2 : -INFINITY;
        z[j][2] = v0 ? sa[j][2] * a.scale_log2 : -INFINITY;
        z[j][3] = v1 ? sa[j][3] * a.scale_log2 : -INFINITY;
        r0 = fmaxf(r0, fmaxf(z[j][0], z[j][1]));
        r1 = fmaxf(r1, fmaxf(z[j][2], z[j][3]));
      }
      r0 = fmaxf(r0, __shfl_xor_sync(0xffffffffu, r0, 1));
      r1 = fmaxf(r1, __shfl_xor_sync(0xffffffffu, r1, 1));
      r0 = fmaxf(r0, __shfl_xor_sync(0xffffffffu, r0, 2));
      r1 = fmaxf(r1, __shfl_xor_sync(0xffffffffu, r1, 2));
      const float mn0 = fmaxf(m0, r0), mn1 = fmaxf(m1, r1);
      // a tile whose units were all rejected as bad data keeps every logit at -inf
      const float sub0 = mn0 == -INFINITY ? 0.f : mn0, sub1 = mn1 == -INFINITY ? 0.f : mn1;
      const float al0 = exp2f(m0 - sub0), al1 = exp2f(m1 - sub1);
      m0 = mn0;
      m1 = mn1;
      float pr[2][4];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        pr[j][0] = exp2f(z[j][0] - sub0);
        pr[j][1] = exp2f(z[j][1] - sub0);
        pr[j][2] = exp2f(z[j][2] - sub1);
        pr[j][3] = exp2f(z[j][3] - sub1);
      }
      l0 = l0 * al0 + ((pr[0][0] + pr[0][1]) + (pr[1][0] + pr[1][1]));
      l1 = l1 * al1 + ((pr[0][2] + pr[0][3]) + (pr[1][2] + pr[1][3]));
      if (al0 != 1.f || al1 != 1.f) {
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          o[nt][0] *= al0;
          o[nt][1] *= al0;
          o[nt][2] *= al1;
          o[nt][3] *= al1;
        }
      }
      // P = hi + lo, both BF16, so the PV product keeps ~17 significant bits of
      // every weight (BF16 alone, 8 bits, is too coarse for short token sets)
      uint32_t pa[4], pl[4];
      split_bf16(pr[0][0], pr[0][1], pa[0], pl[0]);
      split_bf16(pr[0][2], pr[0][3], pa[1], pl[1]);
      split_bf16(pr[1][0], pr[1][1], pa[2], pl[2]);
      split_bf16(pr[1][2], pr[1][3], pa[3], pl[3]);

      // ---- O += P V for this warp's 128 dims: 16 n-tiles, k = the tile's 16 tokens
      // V load L reads token (unit L, row tq ^ (L & 1)); rows outside the selection
      // may hold stale or never-written data and are zeroed
      const bool full = mask == 0xffffu;
      const bool ok0 = (mask >> (0 * 4 + tq)) & 1u, ok1 = (mask >> (1 * 4 + (tq ^ 1))) & 1u;
      const bool ok2 = (mask >> (2 * 4 + tq)) & 1u, ok3 = (mask >> (3 * 4 + (tq ^ 1))) & 1u;
#pragma unroll
      for (int qh = 0; qh < 2; ++qh) {
        uint4 x0v = lds128(kb + voff[0] + qh * 1024);
        uint4 x1v = lds128(kb + voff[1] + qh * 1024);
        uint4 x2v = lds128(kb + voff[2] + qh * 1024);
        uint4 x3v = lds128(kb + voff[3] + qh * 1024);
        if (!full) {
          if (!ok0) x0v = make_uint4(0, 0, 0, 0);
          if (!ok1) x1v = make_uint4(0, 0, 0, 0);
          if (!ok2) x2v = make_uint4(0, 0, 0, 0);
          if (!ok3) x3v = make_uint4(0, 0, 0, 0);
        }
        const uint32_t a0[4] = {x0v.x, x0v.y, x0v.z, x0v.w};
        const uint32_t a1[4] = {x1v.x, x1v.y, x1v.z, x1v.w};
        const uint32_t a2[4] = {x2v.x, x2v.y, x2v.z, x2v.w};
        const uint32_t a3[4] = {x3v.x, x3v.y, x3v.z, x3v.w};
#pragma unroll
        for (int r = 0; r < 4; ++r) {
          const uint32_t lo01 = __byte_perm(a0[r], a1[r], 0x5410);
          const uint32_t hi01 = __byte_perm(a0[r], a1[r], 0x7632);
          const uint32_t lo23 = __byte_perm(a2[r], a3[r], 0x5410);
          const uint32_t hi23 = __byte_perm(a2[r], a3[r], 0x7632);
          mma_bf16_16816(o[qh * 8 + 2 * r], pa[0], pa[1], pa[2], pa[3], lo01, lo23);
          mma_bf16_16816(o[qh * 8 + 2 * r + 1], pa[0], pa[1], pa[2], pa[3], hi01, hi23);
          mma_bf16_16816(o[qh * 8 + 2 * r], pl[0], pl[1], pl[2], pl[3], lo01, lo23);
          mma_bf16_16816(o[qh * 8 + 2 * r + 1], pl[0], pl[1], pl[2], pl[3], hi01, hi23);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_empty + stage * 8);  // both warps of the pair arrive
    }
    T_base += n_tiles;

    // ---- merge the 4 pairs' (m, l, O) and write the split partial
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    if (half == 0 && tq == 0) {  // both warps of a pair hold the same m and l
      ml[(cp * 16 + gq) * 2 + 0] = m0;
      ml[(cp * 16 + gq) * 2 + 1] = l0;
      ml[(cp * 16 + gq + 8) * 2 + 0] = m1;
      ml[(cp * 16 + gq + 8) * 2 + 1] = l1;
    }
    named_bar_sync(kBarConsumers, kConsumerThreads);
    // this pair's weight for rows gq / gq+8, and the merged lse of those rows
    float fac[2], lse_row[2];
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      const int row = gq + 8 * hr;
      const float mine = hr ? m1 : m0;
      float M = -INFINITY;
      for (int w = 0; w < kPairs; ++w) M = fmaxf(M, ml[(w * 16 + row) * 2]);
      fac[hr] = 0.f;
      lse_row[hr] = -INFINITY;
      if (M != -INFINITY) {
        float L = 0.f;
        for (int w = 0; w < kPairs; ++w) {
          const float mw = ml[(w * 16 + row) * 2];
          if (mw != -INFINITY) L += ml[(w * 16 + row) * 2 + 1] * exp2f(mw - M);
        }
        fac[hr] = mine != -INFINITY ? exp2f(mine - M) / L : 0.f;
        lse_row[hr] = (M + log2f(L)) * 0.69314718055994530942f;
      }
    }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      o[nt][0] *= fac[0];
      o[nt][1] *= fac[0];
      o[nt][2] *= fac[1];
      o[nt][3] *= fac[1];
    }
    // n-tile 8 qh + e, column 2tq + f holds dim 128 half + 64 qh + 8 kappa(2tq + f) + e,
    // kappa(2tq) = tq and kappa(2tq + 1) = tq + 4
    auto store_rows = [&](float* base, int row_stride) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int row = gq + 8 * hr;
        if (row >= G) continue;
        const int cc = 2 * hr;
#pragma unroll
        for (int qh = 0; qh < 2; ++qh) {
#pragma unroll
          for (int f = 0; f < 2; ++f) {
            float4* d4 = reinterpret_cast<float4*>(base + (size_t)row * row_stride + 128 * half + 64 * qh + 32 * f + 8 * tq);
            d4[0] = make_float4(o[qh * 8 + 0][cc + f], o[qh * 8 + 1][cc + f], o[qh * 8 + 2][cc + f], o[qh * 8 + 3][cc + f]);
            d4[1] = make_float4(o[qh * 8 + 4][cc + f], o[qh * 8 + 5][cc + f], o[qh * 8 + 6][cc + f], o[qh * 8 + 7][cc + f]);
          }
        }
      }
    };
    auto add_rows = [&](const float* base) {
#pragma unroll
      for (int hr = 0; hr < 2; ++hr) {
        const int row = gq + 8 * hr;
        if (row >= G) continue;
        const int cc = 2 * hr;
#pragma unroll
        for (int qh = 0; qh < 2; ++qh) {
#pragma unroll
          for (int f = 0; f < 2; ++f) {
            const float4* s4 = reinterpret_cast<const float4*>(base + row * kCombRow + 128 * half + 64 * qh + 32 * f + 8 * tq);
            const float4 x0 = s4[0], x1 = s4[1];
            o[qh * 8 + 0][cc + f] += x0.x; o[qh * 8 + 1][cc + f] += x0.y;
            o[qh * 8 + 2][cc + f] += x0.z; o[qh * 8 + 3][cc + f] += x0.w;
            o[qh * 8 + 4][cc + f] += x1.x; o[qh * 8 + 5][cc + f] += x1.y;
            o[qh * 8 + 6][cc + f] += x1.z; o[qh * 8 + 7][cc + f] += x1.w;
          }
        }
      }
    };
    // merge step 1: pairs 2, 3 hand their O to pairs 0, 1; step 2: pair 1 to pair 0
    if (cp >= 2) store_rows(comb + (cp - 2) * 16 * kCombRow, kCombRow);
    named_bar_sync(kBarConsumers, kConsumerThreads);
    if (cp < 2) add_rows(comb + cp * 16 * kCombRow);
    named_bar_sync(kBarConsumers, kConsumerThreads);
    if (cp == 1) store_rows(comb, kCombRow);
    named_bar_sync(kBarConsumers, kConsumerThreads);
    const size_t row0 = ((size_t)s.q * a.max_splits + s.split) * a.hq + (size_t)s.g * G;
    if (cp == 0) {
      add_rows(comb);
      store_rows(a.part_o + row0 * kHeadDim, kHeadDim);
      if (half == 0 && tq == 0) {
        if (gq < G) a.part_lse[row0 + gq] = lse_row[0];
        if (gq + 8 < G) a.part_lse[row0 + gq + 8] = lse_row[1];
      }
    }
    if (s.last_of_pair) {  // slots this pair never reaches: empty splits
      for (int sp = s.split + 1; sp < a.max_splits; ++sp) {
        const size_t r0 = ((size_t)s.q * a.max_splits + sp) * a.hq + (size_t)s.g * G;
        for (int idx = tid; idx < G * 64; idx += kConsumerThreads)
          *reinterpret_cast<float4*>(a.part_o + (r0 + (idx >> 6)) * kHeadDim + (idx & 63) * 4) =
              make_float4(0.f, 0.f, 0.f, 0.f);
        for (int row = tid; row < G; row += kConsumerThreads) a.part_lse[r0 + row] = -INFINITY;
      }
    }
    if (a.pair_done) {
      // The CTA that writes a pair's last split merges the pair: every writer
      // fences its partial stores, one thread counts the split (device-scope
      // atomic) and fences again before the merge reads the other splits.
      __threadfence();
      named_bar_sync(kBarConsumers, kConsumerThreads);
      volatile int* last_flag = reinterpret_cast<volatile int*>(ml);  // ml is free until the next segment ends
      const int64_t base = pair * n_slots;
      const int nspl = (int)((base + n_slots - 1) / a.chunk - base / a.chunk) + 1;
      if (tid == 0) {
        const int done = atomicAdd(a.pair_done + pair, 1);
        const bool last = done == nspl - 1;
        if (last) a.pair_done[pair] = 0;  // every other split has counted: ready for the next call
        __threadfence();
        *last_flag = last ? 1 : 0;
      }
      named_bar_sync(kBarConsumers, kConsumerThreads);
      const bool last = *last_flag != 0;
      named_bar_sync(kBarConsumers, kConsumerThreads);  // the flag is read before ml is written again
      if (last) merge_pair(a, s.q, s.g, nspl, tid);
    } else {
      named_bar_sync(kBarConsumers, kConsumerThreads);  // comb and ml are read before the next segment writes them
    }
  }
}

__global__ void __launch_bounds__(kThreadsB, 1) sparse_decode_bf16_kernel(DecodeArgs a) {
  extern __shared__ __align__(128) uint8_t smem_raw[];
  pdl_launch_dependents();
  Ctx c;
  c.ring = (smem_u32(smem_raw) + 127u) & ~127u;
  c.smem = smem_raw + (c.ring - smem_u32(smem_raw));
  c.bar = c.ring + kOffBarB;
  c.abort_flag = reinterpret_cast<volatile int*>(c.smem + kOffAbortB);
  const int64_t x0 = (int64_t)blockIdx.x * a.chunk;
  const int64_t x1 = min(x0 + a.chunk, a.total_slots);
  if (threadIdx.x == 0) {
    for (int i = 0; i < kStagesB; ++i) {
      mbar_init(c.bar + i * 8, kFullArrivals);        // full: copy completions + row mask published
      mbar_init(c.bar + (kStagesB + i) * 8, 2);       // empty: both warps of the owning pair
    }
    for (int i = 0; i < kDescSlots; ++i) {
      mbar_init(c.bar + (2 * kStagesB + i) * 8, 1);               // descriptors written (lookup warp)
      mbar_init(c.bar + (2 * kStagesB + kDescSlots + i) * 8, kCopyWarps);  // descriptors taken (copy warps)
    }
    *c.abort_flag = 0;
    fence_mbar_init();
  }
  pdl_wait_previous();  // the selection and counts come from the previous kernel
  __syncthreads();
  if (x0 >= x1) return;
  const int warp = threadIdx.x >> 5;
  if (warp >= kCopyWarp0B && warp < kCopyWarp0B + kCopyWarps) {
    copy_run(a, c, x0, x1, warp - kCopyWarp0B);
  } else if (warp == kLookupWarpB) {
    LookupQueue L;
    L.d_off = reinterpret_cast<uint64_t*>(c.smem + kOffDescOffB);
    L.d_rows = reinterpret_cast<uint32_t*>(c.smem + kOffDescRowsB);
    L.bar_dfull = c.bar + 2 * kStagesB * 8;
    L.bar_dempty = L.bar_dfull + kDescSlots * 8;
    L.abort_flag = c.abort_flag;
    L.unit_bytes = kUnitBytesB;
    lookup_run(a, L, x0, x1);
  } else {
    consumers(a, c, x0, x1);
  }
}

int launch(const DecodeArgs& a, int64_t grid, void* stream) {
  cudaError_t e = cudaFuncSetAttribute(sparse_decode_bf16_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytesB);
  if (e != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  return qsa_host::launch(sparse_decode_bf16_kernel, dim3((unsigned)grid), dim3(kThreadsB), kSmemBytesB,
                          static_cast<cudaStream_t>(stream), a);
}

}  // namespace sdb

}  // namespace

int32_t qsa_splits_bound(int32_t k, int32_t chunk);

namespace {

int decode_call(const qsa_cache_t* cache, const void* q, int32_t nq, int32_t hq, const int32_t* q_seq,
                const int32_t* q_pos, const int32_t* sel, const int32_t* count, int32_t k, float scale,
                int32_t chunk_units, int32_t max_splits, float* part_o, float* part_lse, int32_t* pair_done,
                void* out, float* lse, int32_t* dev_status, void* stream) {
  if (!cache || nq < 0 || hq < 1 || k < 0 || k > QSA_MAX_TOPK || chunk_units < 1 || max_splits < 1)
    return QSA_ERR_INVALID_ARG;
  if (!(scale > 0.f) || !(scale < 3.0e38f)) return QSA_ERR_INVALID_ARG;
  const qsa_cache_t& c = *cache;
  if (c.num_kv_heads < 1 || hq % c.num_kv_heads != 0) return QSA_ERR_INVALID_ARG;
  if (hq / c.num_kv_heads > QSA_MAX_GROUP) return QSA_ERR_UNSUPPORTED;
  if (max_splits < qsa_splits_bound(k, chunk_units)) return QSA_ERR_INVALID_ARG;
  if (c.kv_dtype != QSA_KV_BF16 && c.kv_dtype != QSA_KV_FP8_E4M3) return QSA_ERR_UNSUPPORTED;
  if (nq == 0) return QSA_OK;
  if (!c.kv_pages || !c.block_table || !q || !q_seq || !q_pos || !count || !part_o || !part_lse ||
      (k > 0 && !sel))
    return QSA_ERR_INVALID_ARG;
  if (c.num_pages < 1 || c.max_seqs < 1 || c.max_pages_per_seq < 1) return QSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(c.kv_pages) |
       reinterpret_cast<uintptr_t>(q) | reinterpret_cast<uintptr_t>(part_o)) & 15u)
    return QSA_ERR_INVALID_ARG;
  DecodeArgs a;
  a.kv_bytes = static_cast<const uint8_t*>(c.kv_pages);
  a.bt = c.block_table;
  a.num_pages = c.num_pages;
  a.max_seqs = c.max_seqs;
  a.mpps = c.max_pages_per_seq;
  a.hkv = c.num_kv_heads;
  a.q = static_cast<const __nv_bfloat16*>(q);
  a.hq = hq;
  a.G = hq / c.num_kv_heads;
  a.q_seq = q_seq;
  a.q_pos = q_pos;
  a.sel = sel;
  a.count = count;
  a.K = k;
  a.scale_log2 = scale * 1.44269504088896340736f;
  a.chunk = chunk_units;
  a.total_slots = (int64_t)nq * c.num_kv_heads * ((int64_t)k + 1);
  a.max_splits = max_splits;
  a.part_o = part_o;
  a.part_lse = part_lse;
  a.pair_done = pair_done;
  a.out = static_cast<__nv_bfloat16*>(out);
  a.lse = lse;
  a.st = dev_status;
  const int64_t grid = (a.total_slots + a.chunk - 1) / a.chunk;
  if (grid > 0x7fffffff) return QSA_ERR_UNSUPPORTED;
  if (c.kv_dtype == QSA_KV_FP8_E4M3) return launch_decode<true>(a, grid, stream);
  return sdb::launch(a, grid, stream);
}

}  // namespace

extern "C" int qsa_sparse_decode(const qsa_cache_t* cache, const void* q, int32_t nq, int32_t hq,
                                 const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel,
                                 const int32_t* count, int32_t k, float scale, int32_t chunk_units,
                                 int32_t max_splits, float* part_o, float* part_lse, int32_t* dev_status,
                                 void* stream) {
  return decode_call(cache, q, nq, hq, q_seq, q_pos, sel, count, k, scale, chunk_units, max_splits, part_o, part_lse,
                     nullptr, nullptr, nullptr, dev_status, stream);
}

extern "C" int qsa_sparse_attention(const qsa_cache_t* cache, const void* q, int32_t nq, int32_t hq,
                                    const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel,
                                    const int32_t* count, int32_t k, float scale, int32_t chunk_units,
                                    int32_t max_splits, float* part_o, float* part_lse, int32_t* pair_done,
                                    void* out, float* lse, int32_t* dev_status, void* stream) {
  if (nq > 0 && (!pair_done || !out || !lse)) return QSA_ERR_INVALID_ARG;
  if (reinterpret_cast<uintptr_t>(out) & 7u) return QSA_ERR_INVALID_ARG;
  return decode_call(cache, q, nq, hq, q_seq, q_pos, sel, count, k, scale, chunk_units, max_splits, part_o, part_lse,
                     pair_done, out, lse, dev_status, stream);
}
