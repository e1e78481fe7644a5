// qsa_topk_blocks: per query, the best min(K, nb_q) blocks under (score desc,
// index asc), emitted sorted by block index ascending.
//
// Source: [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section
// "Wat de pull request daadwerkelijk verandert" (keep the best 512 blocks);
// the tie-break (lower index first) and ascending output order are the fixed
// readings.
//
// One CTA per query, order-preserving uint32 keys of the fp32 scores.
// Common path (two passes over the scores, both L2-resident):
//   1. a 13-bit histogram finds the bin b holding the K-th largest key;
//   2. one more pass keeps every key above bin b and gathers bin b's keys
//      (with their indices) into shared memory; a bitonic sort of those
//      candidates on (key desc, index asc) picks the rest exactly; the K chosen
//      indices are emitted in ascending order from a shared-memory bitmap.
// Heavy ties (bin b larger than the candidate buffer) take the general path:
// three histogram passes (12 + 12 + 8 bits) find the exact K-th key T, and an
// ordered compaction (warp ballots over contiguous index ranges plus a prefix
// over warps) emits every key > T and the lowest-index keys == T.
// Integer counters only: the result does not depend on atomic order.
#include "qsa_common.cuh"

namespace {

using namespace qsa;

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

struct TopkArgs {
  const float* scores;
  int64_t ld;
  const int32_t* q_pos;
  int32_t K;
  int32_t* sel;
  int32_t* count;
  int32_t* st;
};

// Block-wide: find the bin b (scanning from the top) with
// sum_{i > b} hist[i] < remaining <= sum_{i >= b} hist[i].
__device__ void find_bin(const uint32_t* hist, int nbins, uint32_t remaining, uint32_t* wsum, int* out_bin,
                         uint32_t* out_above) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = nbins >= kThreads ? nbins / kThreads : 1;
  const int lo = tid * per;
  uint32_t local = 0;
  if (lo < nbins)
    for (int i = 0; i < per; ++i) local += hist[lo + i];
  // inclusive suffix sum within the warp (lanes above)
  uint32_t suf = local;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, suf, d);
    if (lane + d < 32) suf += v;
  }
  if (lane == 0) wsum[warp] = suf;  // warp total
  __syncthreads();
  uint32_t after_warps = 0;
  for (int w = warp + 1; w < kWarps; ++w) after_warps += wsum[w];
  uint32_t cum = after_warps + (suf - local);  // everything in bins above my range
  if (lo < nbins) {
    for (int i = per - 1; i >= 0; --i) {
      const uint32_t h = hist[lo + i];
      if (cum < remaining && remaining <= cum + h) {
        *out_bin = lo + i;
        *out_above = cum;
      }
      cum += h;
    }
  }
  __syncthreads();
}

constexpr int kBits1 = 13;
constexpr int kBins1 = 1 << kBits1;       // first-pass histogram
constexpr int kCandCap = 4096;           // bin-b candidates held in shared memory
constexpr int kMaxBlocks = 65536;        // bitmap capacity of the fast path (blocks per query)
constexpr int kUnroll = 8;
// dynamic shared memory layout
constexpr int kOffHist = 0;                                   // u32 [kBins1]
constexpr int kOffCand = kOffHist + kBins1 * 4;               // u64 [kCandCap]
constexpr int kOffBitmap = kOffCand + kCandCap * 8;           // u32 [kMaxBlocks / 32]
constexpr int kSmemBytes = kOffBitmap + kMaxBlocks / 8;

__device__ __forceinline__ void load_keys(const float* s, int i0, int n, uint32_t (&key)[kUnroll]) {
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const int i = i0 + u * kThreads;
    key[u] = i < n ? float_key(s[i]) : 0u;
  }
}

// General path: exact K-th key by three radix passes, then ordered compaction.
__device__ void topk_general(const float* s, int n, int K, int32_t* out, uint32_t* hist, uint32_t* wsum,
                             uint32_t* wgt, uint32_t* weq, int* s_bin, uint32_t* s_above) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t prefix = 0, mask = 0, remaining = (uint32_t)K;
  const int shifts[3] = {20, 8, 0};
  const int bits[3] = {12, 12, 8};
  for (int pass = 0; pass < 3; ++pass) {
    const int nbins = 1 << bits[pass];
    const int sh = shifts[pass];
    for (int i = tid; i < nbins; i += kThreads) hist[i] = 0;
    __syncthreads();
    for (int i0 = tid; i0 < n; i0 += kThreads * kUnroll) {
      uint32_t key[kUnroll];
      load_keys(s, i0, n, key);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (i0 + u * kThreads < n && (key[u] & mask) == prefix) atomicAdd(&hist[(key[u] >> sh) & (nbins - 1)], 1u);
    }
    __syncthreads();
    find_bin(hist, nbins, remaining, wsum, s_bin, s_above);
    prefix |= (uint32_t)*s_bin << sh;
    mask |= (uint32_t)(nbins - 1) << sh;
    remaining -= *s_above;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const uint32_t need_eq = remaining;  // keys equal to T to keep, lowest index first
  const int span = (((n + kWarps - 1) / kWarps) + 31) & ~31;
  const int beg = warp * span;
  const int end = min(n, beg + span);
  uint32_t c_gt = 0, c_eq = 0;
  for (int i = beg + lane; i < end; i += 32) {
    const uint32_t key = float_key(s[i]);
    c_gt += key > T;
    c_eq += key == T;
  }
  c_gt = __reduce_add_sync(0xffffffffu, c_gt);
  c_eq = __reduce_add_sync(0xffffffffu, c_eq);
  if (lane == 0) {
    wgt[warp] = c_gt;
    weq[warp] = c_eq;
  }
  __syncthreads();
  uint32_t eq_before = 0, sel_before = 0;
  for (int w = 0; w < warp; ++w) {
    const uint32_t take_eq = need_eq > eq_before ? min(need_eq - eq_before, weq[w]) : 0u;
    sel_before += wgt[w] + take_eq;
    eq_before += weq[w];
  }
  const uint32_t lt = (1u << lane) - 1u;
  for (int i0 = beg; i0 < end; i0 += 32) {
    const int i = i0 + lane;
    uint32_t key = 0;
    if (i < end) key = float_key(s[i]);
    const bool is_gt = i < end && key > T;
    const bool is_eq = i < end && key == T;
    const uint32_t b_eq = __ballot_sync(0xffffffffu, is_eq);
    const uint32_t rank = eq_before + __popc(b_eq & lt);
    const bool take = is_gt || (is_eq && rank < need_eq);
    const uint32_t b_take = __ballot_sync(0xffffffffu, take);
    if (take) out[sel_before + __popc(b_take & lt)] = i;
    sel_before += __popc(b_take);
    eq_before += __popc(b_eq);
  }
}

__global__ void __launch_bounds__(kThreads) topk_kernel(TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint32_t* hist = reinterpret_cast<uint32_t*>(smem + kOffHist);
  uint64_t* cand = reinterpret_cast<uint64_t*>(smem + kOffCand);
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + kOffBitmap);
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t wgt[kWarps], weq[kWarps];
  __shared__ int s_bin;
  __shared__ uint32_t s_above, s_ncand;

  const int q = blockIdx.x;
  const int tid = threadIdx.x;
  const int p = a.q_pos[q];
  int64_t nb = p >= 0 ? (int64_t)(p + 1) / kRatio : 0;
  if (p < 0 && tid == 0) flag(a.st, QSA_DEV_BAD_POS);
  if (nb > a.ld) {
    if (tid == 0) flag(a.st, QSA_DEV_SCORES_LD);
    nb = a.ld;
  }
  const int K = a.K;
  int32_t* out = a.sel + (size_t)q * K;
  if (K == 0) {
    if (tid == 0) a.count[q] = 0;
    return;
  }
  if (nb <= K) {  // every visible block is kept
    for (int i = tid; i < K; i += kThreads) out[i] = i < nb ? i : -1;
    if (tid == 0) a.count[q] = (int32_t)nb;
    return;
  }
  const int n = (int)nb;
  const float* s = a.scores + (size_t)q * a.ld;
  if (tid == 0) a.count[q] = K;

  if (n > kMaxBlocks) {
    topk_general(s, n, K, out, hist, wsum, wgt, weq, &s_bin, &s_above);
    return;
  }
  // ---- pass 1: 13-bit histogram
  for (int i = tid; i < kBins1; i += kThreads) hist[i] = 0;
  for (int i = tid; i < (n + 31) / 32; i += kThreads) bitmap[i] = 0;
  if (tid == 0) s_ncand = 0;
  __syncthreads();
  constexpr int kShift1 = 32 - kBits1;
  const int lane = tid & 31;
  const uint32_t lt = (1u << lane) - 1u;
  const int n_pad = (n + kThreads * kUnroll - 1) / (kThreads * kUnroll) * (kThreads * kUnroll);
  for (int i0 = tid; i0 < n_pad; i0 += kThreads * kUnroll) {  // warp-uniform trip count
    uint32_t key[kUnroll];
    load_keys(s, i0, n, key);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      // scores crowd into few bins: one atomic per distinct bin per warp
      const bool live = i0 + u * kThreads < n;
      const uint32_t bin = live ? (key[u] >> kShift1) : 0xffffffffu;
      const uint32_t peers = __match_any_sync(0xffffffffu, bin);
      if (live && (peers & lt) == 0) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
    }
  }
  __syncthreads();
  find_bin(hist, kBins1, (uint32_t)K, wsum, &s_bin, &s_above);
  const uint32_t b1 = (uint32_t)s_bin;
  const uint32_t above = s_above;
  const uint32_t in_bin = hist[b1];
  if (in_bin > kCandCap) {  // heavy ties: general path (uniform decision)
    __syncthreads();
    topk_general(s, n, K, out, hist, wsum, wgt, weq, &s_bin, &s_above);
    return;
  }
  // ---- pass 2: keep keys above bin b1, gather bin b1's candidates
  for (int i0 = tid; i0 < n_pad; i0 += kThreads * kUnroll) {
    uint32_t key[kUnroll];
    load_keys(s, i0, n, key);
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      // the warp's 32 lanes hold the 32 consecutive indices of one bitmap word
      const int i = i0 + u * kThreads;
      const bool live = i < n;
      const uint32_t bin = key[u] >> kShift1;
      const uint32_t above_w = __ballot_sync(0xffffffffu, live && bin > b1);
      const uint32_t cand_w = __ballot_sync(0xffffffffu, live && bin == b1);
      if (lane == 0 && i < n) bitmap[i >> 5] = above_w;
      uint32_t base = 0;
      if (lane == 0 && cand_w) base = atomicAdd(&s_ncand, (uint32_t)__popc(cand_w));
      base = __shfl_sync(0xffffffffu, base, 0);
      if (cand_w & (1u << lane))
        cand[base + __popc(cand_w & lt)] = ((uint64_t)key[u] << 32) | (uint32_t)(0xffffffffu - (uint32_t)i);
    }
  }
  __syncthreads();
  // ---- exact order inside bin b1: bitonic sort descending on (key, -index)
  int P = 1;
  while (P < (int)in_bin) P <<= 1;
  for (int i = in_bin + tid; i < P; i += kThreads) cand[i] = 0;  // pads sort last
  __syncthreads();
  for (int k = 2; k <= P; k <<= 1) {
    for (int j = k >> 1; j > 0; j >>= 1) {
      for (int i = tid; i < P; i += kThreads) {
        const int ixj = i ^ j;
        if (ixj > i) {
          const uint64_t x = cand[i], y = cand[ixj];
          const bool desc = (i & k) == 0;
          if (desc ? (x < y) : (x > y)) {
            cand[i] = y;
            cand[ixj] = x;
          }
        }
      }
      __syncthreads();
    }
  }
  const uint32_t take = (uint32_t)K - above;
  for (uint32_t t = tid; t < take; t += kThreads) {
    const int i = (int)(0xffffffffu - (uint32_t)(cand[t] & 0xffffffffu));
    atomicOr(&bitmap[i >> 5], 1u << (i & 31));
  }
  __syncthreads();
  // ---- ascending emission from the bitmap: per-thread word runs + block scan
  const int words = (n + 31) / 32;
  const int per = (words + kThreads - 1) / kThreads;
  const int w0 = tid * per;
  uint32_t cnt = 0;
  for (int w = w0; w < min(words, w0 + per); ++w) cnt += __popc(bitmap[w]);
  // exclusive prefix over threads (warp shuffles + warp totals)
  const int warp = tid >> 5;
  uint32_t inc = cnt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += v;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  uint32_t base = inc - cnt;
  for (int w = 0; w < warp; ++w) base += wsum[w];
  for (int w = w0; w < min(words, w0 + per); ++w) {
    uint32_t bits = bitmap[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      out[base++] = w * 32 + b;
    }
  }
}

}  // namespace

extern "C" int qsa_topk_blocks(const float* scores, int64_t scores_ld, const int32_t* q_pos, int32_t nq, int32_t k,
                               int32_t* sel, int32_t* count, int32_t* dev_status, void* stream) {
  if (nq < 0 || k < 0 || k > QSA_MAX_TOPK || scores_ld < 1) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!scores || !q_pos || !count || (k > 0 && !sel)) return QSA_ERR_INVALID_ARG;
  TopkArgs a{scores, scores_ld, q_pos, k, sel, count, dev_status};
  if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  topk_kernel<<<(unsigned)nq, kThreads, kSmemBytes, static_cast<cudaStream_t>(stream)>>>(a);
  return qsa_host::launch_status();
}
