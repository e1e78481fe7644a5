// qsa_index_scores: s[q][j] = sum_h w[q][h] * ReLU(q_idx[q][h] . kc[j]) for every
// complete micro-block j < nb_q visible to query q.
//
// Source: [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section
// "Wat de pull request daadwerkelijk verandert" (the indexer scores the
// micro-blocks) and [CANN] "Qwen4-Exp QSA komt naar Huawei's Ascend ...",
// section "Waarom QSA het lastige onderdeel is, in cijfers" (multi-query
// indexer sharing one key head, head dim 128).  The ReLU-weighted head sum is
// the fixed scoring reading.
//
// HBM-bound stream over the side cache (256 B per block).  Each warp owns whole
// 4 KiB kc pages (16 blocks x 128 dims): every lane issues 16-byte loads that
// land directly in mma.sync m16n8k16 A fragments (rows = the page's 16
// blocks, K = 128 dims, N = the 8 indexer heads), index_page.cuh.
#include <cuda.h>
#include <cudaTypedefs.h>

#include "index_page.cuh"

namespace {

using namespace qsa;

constexpr int kWarps = 8;
// Each warp scores a run of pages_per_warp pages (2 at a time), a CTA 8 such
// runs.  The host sizes the run (4 to 16 pages) so the grid keeps about six
// waves of resident CTAs: fewer, longer CTAs when the block table is wide
// and many of its chunks hold no pages of a shorter query, more and shorter
// ones when every chunk is full.
constexpr int kMinPagesPerWarp = 4, kMaxPagesPerWarp = 16;

struct ScoreArgs {
  const __nv_bfloat16* kc;
  const int32_t* bt;
  int32_t num_pages, max_seqs, mpps;
  const __nv_bfloat16* q_idx;
  const float* w;
  const int32_t* q_seq;
  const int32_t* q_pos;
  float* scores;
  int64_t ld;
  int32_t chunks_per_query;
  int32_t pages_per_warp;
  int32_t* st;
};

__global__ void __launch_bounds__(kWarps * 32) index_scores_kernel(ScoreArgs a) {
  pdl_launch_dependents();
  const int q = blockIdx.x / a.chunks_per_query;
  const int chunk = blockIdx.x % a.chunks_per_query;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;

  // The query's sequence, position, indexer query and page ids are inputs that
  // no kernel of this library writes: they are loaded before waiting for the
  // preceding kernel, so only the side-cache pages are read after the wait.
  const int seq = a.q_seq[q];
  const int p = a.q_pos[q];
  const bool bad = seq < 0 || seq >= a.max_seqs || p < 0 || (int64_t)p >= (int64_t)a.mpps * kPage;
  int64_t nb = bad ? 0 : (p + 1) / kRatio;
  const bool ld_over = nb > a.ld;
  if (ld_over) nb = a.ld;
  const int npg = (int)((nb + kBlocksPerPage - 1) / kBlocksPerPage);
  const int ppw = a.pages_per_warp;
  const int pg0 = chunk * (kWarps * ppw) + warp * ppw;
  IdxQuery Q{};
  int myphys = -1;
  if (!bad && pg0 < npg) {
    Q = load_idx_query(a.q_idx, a.w, q);
    if (lane < ppw && pg0 + lane < npg) myphys = a.bt[(int64_t)seq * a.mpps + pg0 + lane];
  }
  pdl_wait_previous();
  if (bad) {
    if (chunk == 0 && threadIdx.x == 0) flag(a.st, (seq < 0 || seq >= a.max_seqs) ? QSA_DEV_BAD_SEQ : QSA_DEV_BAD_POS);
    return;
  }
  if (ld_over && chunk == 0 && threadIdx.x == 0) flag(a.st, QSA_DEV_SCORES_LD);
  if (pg0 >= npg) return;
  float* srow = a.scores + (size_t)q * a.ld;

#pragma unroll
  for (int pp = 0; pp < ppw; pp += 2) {
    uint4 ra[2][4], rb[2][4];
    int phys[2];
    bool ok[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      phys[k] = __shfl_sync(0xffffffffu, myphys, pp + k);
      ok[k] = (pg0 + pp + k < npg) && phys[k] >= 0 && phys[k] < a.num_pages;
      if (ok[k]) load_idx_page(a.kc, phys[k], ra[k], rb[k]);
    }
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int pg = pg0 + pp + k;
      if (pg >= npg) continue;
      const int64_t blk_lo = (int64_t)pg * kBlocksPerPage + g;
      const int64_t blk_hi = blk_lo + 8;
      if (!ok[k]) {  // page-table miss: these blocks can never be read
        if (lane == 0) flag(a.st, QSA_DEV_BAD_PAGE);
        if (t == 0 && blk_lo < nb) srow[blk_lo] = -INFINITY;
        if (t == 1 && blk_hi < nb) srow[blk_hi] = -INFINITY;
        continue;
      }
      float s_lo, s_hi;
      score_idx_page(ra[k], rb[k], Q, s_lo, s_hi);
      if (t == 0 && blk_lo < nb) srow[blk_lo] = s_lo;
      if (t == 1 && blk_hi < nb) srow[blk_hi] = s_hi;
    }
  }
}

// ---------------------------------------------------------------------------
// Query-tiled variant for calls with many queries per sequence (chunked
// prefill / extend): the queries of one sequence all read the same side cache,
// so the work is a dense contraction [queries x 8 heads] x 128 x [blocks] and
// a CTA of 32 consecutive queries reads each 128-block kc tile once for all of
// them.  Queries of a CTA that belong to different sequences are handled by
// one pass per distinct sequence.

constexpr int kTQ = 32;                   // queries per CTA
constexpr int kTB = 128;                  // blocks per kc tile
constexpr int kTChunkBlocks = 8192;       // blocks per CTA (gridDim.y splits longer rows)

struct TiledArgs {
  const __nv_bfloat16* kc;
  const int32_t* bt;
  int32_t num_pages, max_seqs, mpps;
  const __nv_bfloat16* q_idx;
  const float* w;
  const int32_t* q_seq;
  const int32_t* q_pos;
  int32_t nq;
  float* scores;
  int64_t ld;
  int32_t bulk;  // score rows 16-byte aligned (base and pitch): scores leave by bulk copies
  int32_t* st;
  CUtensorMap tm_kc;  // kc_pages as [num_pages * 16 rows][128 dims], boxes of 16 rows x 64 dims, 128-B swizzle
  CUtensorMap tm_q;   // q_idx as [nq * 8 rows][128 dims], boxes of 256 rows x 64 dims, 128-B swizzle
};

// ---------------------------------------------------------------------------
// The contraction runs on the 5th-generation tensor cores (tcgen05): per
// 128-block kc tile, D[block][query*8 + head] = kc[block] .
// q_idx[query][head] for the CTA's 32 queries, accumulated in tensor memory
// (M = 128 blocks, N = 256, K = 128 dims in 8 steps of 16).  One TMEM lane per
// block, so the w * ReLU head sum of a (query, block) score stays inside one
// thread.
//   warps 0-7  epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (the lane
//              quadrant a warp may access) and the columns of queries
//              16 (w / 4) .. + 15, sums the heads, stages the scores in shared
//              memory and stores each query's 32 consecutive scores with one
//              128-byte bulk copy (cp.async.bulk from this CTA; element stores
//              when the caller's score rows are not 16-byte aligned)
//   warp 8     TMEM allocation (512 columns: two accumulator buffers) and the
//              MMA issue (one elected thread), tcgen05.commit to mbarriers
//   warp 9     producer: tensor-map copies (one thread issues them) into the
//              K-major 128-byte-swizzled operand layout (8-row x 128-byte
//              atoms 1 KiB apart; dims 64 .. 127 one operand-height further):
//              the q_idx operand once, then per kc tile its 8 pages x 2 halves
//              of 16 rows x 64 dims, completing on the stage mbarrier by byte
//              count (4-stage ring).  Each tile's page ids are loaded while the
//              tile before it is copied.  Tensor-map copies move a tile with 16
//              requests where 16-byte copies needed 2,048, which had capped the
//              tile rate at about 19 GB/s per SM.
// All waits are bounded; on expiry the CTA records QSA_DEV_TIMEOUT, stops
// issuing work, drains what it issued and frees its tensor memory.

constexpr int kUStages = 4;
constexpr int kUTileBytes = kTB * kIdxDim * 2;                 // 32 KiB: one operand of 128 rows
constexpr int kUEpiWarps = 8, kUMmaWarp = 8, kUProdWarp0 = 9, kUProdWarps = 1;
constexpr int kUThreads = (kUProdWarp0 + kUProdWarps) * 32;    // 320
constexpr int kUEpiQ = kTQ * 4 / kUEpiWarps;                    // queries per epilogue warp: 16
constexpr int kUN = kTQ * kIdxHeads;                           // 256: MMA N = the CTA's queries x heads
constexpr int kUBBytes = kUN * kIdxDim * 2;                    // 64 KiB: the q_idx operand
constexpr int kUAcc = 2;                                       // accumulator buffers in tensor memory
constexpr int kUTmemCols = kUAcc * kUN;
constexpr int kUOffB = 0;                                      // q_idx operand (256 rows)
constexpr int kUOffA = kUOffB + kUBBytes;                      // kc ring
constexpr int kUOffW = kUOffA + kUStages * kUTileBytes;        // [32][8] weights
constexpr int kUOffMeta = kUOffW + kTQ * kIdxHeads * 4;        // t_seq[32], t_nb[32], t_list[32], count, tmem, abort
constexpr int kUOffBar = (kUOffMeta + (3 * kTQ + 4) * 4 + 7) & ~7;
constexpr int kUNumBars = 2 * kUStages + 2 * kUAcc + 2;        // full/empty per stage, acc full/empty, b_full, done
constexpr int kUStageFloats = kUEpiQ * 32;                     // one epilogue warp's 32 rows x 16 queries
constexpr int kUOffStage = (kUOffBar + kUNumBars * 8 + 127) & ~127;  // 2 x 4 warps score staging buffers
constexpr int kUSmem = kUOffStage + 2 * kUEpiWarps * kUStageFloats * 4 + 1024;  // + room to align the base to 1 KiB
constexpr uint32_t kUIdesc = (1u << 4)                       // D: fp32
                           | (1u << 7) | (1u << 10)          // A, B: bf16
                           | ((uint32_t)(kUN >> 3) << 17)    // N = 256
                           | ((uint32_t)(128 >> 4) << 24);   // M = 128
constexpr uint64_t kUWaitNs = 2000000000ull;

// shared-memory matrix descriptor: K-major, 128-byte swizzle (8 rows x 128 B atoms, 1 KiB apart)
__device__ __forceinline__ uint64_t umma_desc_sw128(uint32_t saddr) {
  uint64_t d = 0;
  d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
  d |= (uint64_t)(16u >> 4) << 16;     // leading byte offset: unused by this layout
  d |= (uint64_t)(1024u >> 4) << 32;   // stride byte offset: between 8-row groups
  d |= (uint64_t)1u << 46;             // descriptor version for sm_100
  d |= (uint64_t)2u << 61;             // 128-byte swizzle
  return d;
}
// descriptor advance for 16-element K step ks of a `rows`-row operand: 64-dim halves
// `rows` x 128 B apart, 32 B per step inside a half (in 16-byte units)
template <int rows>
__device__ __forceinline__ uint64_t ksteps(int ks) {
  return (uint64_t)(((ks >> 2) * rows * 128 + (ks & 3) * 32) >> 4);
}

// 2-D tensor-map copy into this CTA's shared memory, completing on an mbarrier
__device__ __forceinline__ void tma2d(uint32_t sdst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(sdst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(bar)
      : "memory");
}

__device__ __forceinline__ void umma_f16(uint32_t tmem_d, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      ::"r"(tmem_d), "l"(a), "l"(b), "r"(idesc), "r"(acc), "r"(0), "r"(0), "r"(0), "r"(0));
}
__device__ __forceinline__ void umma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
// bulk copy shared -> global (16-byte aligned addresses, size a multiple of 16), tracked per thread in groups
__device__ __forceinline__ void bulk_s2g(void* gdst, uint32_t ssrc, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;" ::"l"(gdst), "r"(ssrc), "r"(bytes)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// all but this thread's most recent group have finished reading their shared-memory source
__device__ __forceinline__ void bulk_wait_read1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
// every group of this thread has completed its writes
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void reg_fence16(uint32_t (&r)[16]) {
  asm volatile("" : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]), "+r"(r[6]), "+r"(r[7]),
               "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]), "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]));
}
// bounded mbarrier wait shared by all roles; false once the CTA aborted
__device__ __forceinline__ bool uwait(uint32_t bar, uint32_t parity, volatile int* abort_flag, int32_t* st) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u) {
      if (*abort_flag) return false;
      if (global_timer_ns() - t0 > kUWaitNs) {
        flag(st, QSA_DEV_TIMEOUT);
        *abort_flag = 1;
        return false;
      }
    }
  }
}

__global__ void __launch_bounds__(kUThreads, 1) index_scores_umma_kernel(const __grid_constant__ TiledArgs a) {
  pdl_launch_dependents();
  extern __shared__ __align__(128) uint8_t usmem[];
  uint8_t* smem = usmem + (((smem_u32(usmem) + 1023u) & ~1023u) - smem_u32(usmem));  // 1 KiB aligned
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int32_t* t_seq = reinterpret_cast<int32_t*>(smem + kUOffMeta);
  int32_t* t_nb = t_seq + kTQ;
  int32_t* t_list = t_nb + kTQ;
  int32_t* t_cnt = t_list + kTQ;
  uint32_t* t_tmem = reinterpret_cast<uint32_t*>(t_cnt + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(t_cnt + 2);
  float* t_w = reinterpret_cast<float*>(smem + kUOffW);
  const uint32_t sb = smem_u32(smem);
  const uint32_t bar0 = sb + kUOffBar;
  const uint32_t bar_full = bar0, bar_empty = bar0 + kUStages * 8;
  const uint32_t bar_accf = bar0 + 2 * kUStages * 8, bar_acce = bar_accf + kUAcc * 8;
  const uint32_t bar_bfull = bar_acce + kUAcc * 8, bar_done = bar_bfull + 8;
  const int q0 = blockIdx.x * kTQ;
  const int64_t blk_lo = (int64_t)blockIdx.y * kTChunkBlocks;

  if (tid == 0) {
    for (int i = 0; i < kUStages; ++i) {
      mbar_init(bar_full + i * 8, 1);  // the producer's arrive with the tile's byte count
      mbar_init(bar_empty + i * 8, 1);
    }
    for (int i = 0; i < kUAcc; ++i) {
      mbar_init(bar_accf + i * 8, 1);
      mbar_init(bar_acce + i * 8, kUEpiWarps * 32);
    }
    mbar_init(bar_bfull, 1);
    mbar_init(bar_done, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kUMmaWarp) {  // tensor memory for two 128 x 256 fp32 accumulators
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(t_tmem)),
                 "r"(kUTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait_previous();
  if (tid < kTQ) {
    const int q = q0 + tid;
    int seq = -1, nb = 0;
    if (q < a.nq) {
      seq = a.q_seq[q];
      const int p = a.q_pos[q];
      if (seq < 0 || seq >= a.max_seqs || p < 0 || (int64_t)p >= (int64_t)a.mpps * kPage) {
        if (blockIdx.y == 0) flag(a.st, (seq < 0 || seq >= a.max_seqs) ? QSA_DEV_BAD_SEQ : QSA_DEV_BAD_POS);
        seq = -1;
      } else {
        int64_t n = (p + 1) / kRatio;
        if (n > a.ld) {
          if (blockIdx.y == 0) flag(a.st, QSA_DEV_SCORES_LD);
          n = a.ld;
        }
        nb = (int)n;
      }
    }
    t_seq[tid] = seq;
    t_nb[tid] = nb;
  }
  if (tid < kTQ * kIdxHeads) {
    const int q = q0 + tid / kIdxHeads;
    t_w[tid] = q < a.nq ? a.w[(size_t)q * kIdxHeads + tid % kIdxHeads] : 0.f;
  }
  __syncthreads();
  if (tid == 0) {
    int n = 0;
    for (int i = 0; i < kTQ; ++i) {
      const int sq = t_seq[i];
      if (sq < 0) continue;
      bool seen = false;
      for (int j = 0; j < n; ++j) seen |= t_list[j] == sq;
      if (!seen) t_list[n++] = sq;
    }
    *t_cnt = n;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *t_tmem;
  const int nseq = *t_cnt;

  // the (sequence pass, tile) order every role walks
  auto pass_range = [&](int si, int64_t& B0, int64_t& B1) {
    const int S = t_list[si];
    int nb_max = 0;
    for (int i = 0; i < kTQ; ++i)
      if (t_seq[i] == S) nb_max = max(nb_max, t_nb[i]);
    B0 = blk_lo;
    B1 = min((int64_t)nb_max, blk_lo + kTChunkBlocks);
  };

  if (warp >= kUProdWarp0) {
    // ---------------- producer warp: tensor-map copies, issued by lane 0.  The q_idx
    // operand (two 256-row x 64-dim boxes; rows past nq * 8 read as zero) once, then
    // per kc tile 8 pages x 2 halves of 16 rows x 64 dims.  A tile's page ids are
    // loaded (lane p: page p) while the tile before it is copied; a rejected page
    // reads rows past the tensor, which arrive as zeros.
    if (lane == 0) {
      mbar_arrive_expect_tx(bar_bfull, (uint32_t)kUBBytes);
      tma2d(sb + kUOffB, &a.tm_q, 0, q0 * kIdxHeads, bar_bfull);
      tma2d(sb + kUOffB + kUN * 128, &a.tm_q, 64, q0 * kIdxHeads, bar_bfull);
    }
    int j = 0;
    for (int si = 0; si < nseq && !*abort_flag; ++si) {
      int64_t B0, B1;
      pass_range(si, B0, B1);
      const int S = t_list[si];
      auto load_ids = [&](int64_t tb0) {
        const int64_t bp = tb0 + (int64_t)kBlocksPerPage * lane;
        return (lane < kTB / kBlocksPerPage && bp < B1) ? __ldg(a.bt + (int64_t)S * a.mpps + bp / kBlocksPerPage) : -1;
      };
      int phys = load_ids(B0);
      bool ok_all = true;
      for (int64_t b0 = B0; b0 < B1; b0 += kTB, ++j) {
        const int stage = j % kUStages;
        int okw = 1;
        if (lane == 0 && j >= kUStages)
          okw = uwait(bar_empty + stage * 8, (uint32_t)((j / kUStages - 1) & 1), abort_flag, a.st) ? 1 : 0;
        okw = __shfl_sync(0xffffffffu, okw, 0);
        __syncwarp();
        if (!okw) {
          ok_all = false;
          break;
        }
        const int next = load_ids(b0 + kTB);
        const bool good = phys >= 0 && phys < a.num_pages;
        if (lane < kTB / kBlocksPerPage && !good && b0 + (int64_t)kBlocksPerPage * lane < B1) flag(a.st, QSA_DEV_BAD_PAGE);
        const int y = good ? phys * kBlocksPerPage : a.num_pages * kBlocksPerPage;
        const uint32_t tile = sb + kUOffA + stage * kUTileBytes;
        if (lane == 0) mbar_arrive_expect_tx(bar_full + stage * 8, (uint32_t)kUTileBytes);
#pragma unroll
        for (int p = 0; p < kTB / kBlocksPerPage; ++p) {
          const int yp = __shfl_sync(0xffffffffu, y, p);
          if (lane == 0) {
            tma2d(tile + p * kBlocksPerPage * 128, &a.tm_kc, 0, yp, bar_full + stage * 8);
            tma2d(tile + kTB * 128 + p * kBlocksPerPage * 128, &a.tm_kc, 64, yp, bar_full + stage * 8);
          }
        }
        phys = next;
      }
      if (!ok_all) break;
    }
    // every copy this warp issued has landed before the CTA moves on (the last
    // tile of each stage and the q_idx operand; bounded, as every wait here)
    if (lane == 0) {
      (void)mbar_wait_bounded(bar_bfull, 0, kUWaitNs);
      for (int t = j - kUStages < 0 ? 0 : j - kUStages; t < j; ++t)
        (void)mbar_wait_bounded(bar_full + (t % kUStages) * 8, (uint32_t)((t / kUStages) & 1), kUWaitNs);
    }
    __syncwarp();
  } else if (warp == kUMmaWarp) {
    // ---------------- MMA issue (one thread)
    if (lane == 0) {
      bool ok = uwait(bar_bfull, 0, abort_flag, a.st);
      const uint64_t bdesc0 = umma_desc_sw128(sb + kUOffB);
      int j = 0;
      for (int si = 0; si < nseq && ok; ++si) {
        int64_t B0, B1;
        pass_range(si, B0, B1);
        for (int64_t b0 = B0; b0 < B1 && ok; b0 += kTB, ++j) {
          const int stage = j % kUStages, acc = j % kUAcc;
          if (!uwait(bar_full + stage * 8, (uint32_t)((j / kUStages) & 1), abort_flag, a.st)) { ok = false; break; }
          if (j >= kUAcc && !uwait(bar_acce + acc * 8, (uint32_t)((j / kUAcc - 1) & 1), abort_flag, a.st)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc0 = umma_desc_sw128(sb + kUOffA + stage * kUTileBytes);
#pragma unroll
          for (int ks = 0; ks < kIdxDim / 16; ++ks)  // per 16-element K step: rows * 32 B, in 16-B units
            umma_f16(tmem + acc * kUN, adesc0 + ksteps<kTB>(ks), bdesc0 + ksteps<kUN>(ks), kUIdesc, ks > 0 ? 1u : 0u);
          umma_commit(bar_empty + stage * 8);  // the kc stage is free once these MMAs finish
          umma_commit(bar_accf + acc * 8);     // the accumulator is ready
        }
      }
      umma_commit(bar_done);  // every MMA issued above has completed when this fires
      mbar_wait_bounded(bar_done, 0, kUWaitNs);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue: warp w reads TMEM lanes 32 (w % 4) .. + 31 (rows) and the
    // columns of queries 16 (w / 4) .. + 15
    const int qd = warp & 3, qh = warp >> 2;
    const int row = 32 * qd + lane;
    int j = 0;
    for (int si = 0; si < nseq; ++si) {
      int64_t B0, B1;
      pass_range(si, B0, B1);
      const int S = t_list[si];
      for (int64_t b0 = B0; b0 < B1; b0 += kTB, ++j) {
        const int acc = j % kUAcc;
        const int64_t b = b0 + row;
        // a block on a rejected page scores -inf (its kc rows were zero-filled)
        const int phys = b < B1 ? a.bt[(int64_t)S * a.mpps + b / kBlocksPerPage] : 0;
        if (!uwait(bar_accf + acc * 8, (uint32_t)((j / kUAcc) & 1), abort_flag, a.st)) goto epi_done;
        tc_fence_after();
        float sc[kUEpiQ];
        const uint32_t taddr = tmem + acc * kUN + ((uint32_t)(32 * qd) << 16) + (uint32_t)(qh * kUEpiQ * kIdxHeads);
#pragma unroll
        for (int h8 = 0; h8 < kUEpiQ / 8; ++h8) {  // 4 loads of two queries (16 columns) each, then one wait
          uint32_t r[4][16];
#pragma unroll
          for (int u = 0; u < 4; ++u) tmem_ld16(taddr + (h8 * 4 + u) * 16, r[u]);
          tmem_wait_ld();
#pragma unroll
          for (int u = 0; u < 4; ++u) reg_fence16(r[u]);
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int k = 0; k < 2; ++k) {
              const int ql = 2 * (h8 * 4 + u) + k;
              const int qg = qh * kUEpiQ + ql;
              const float4 wa = *reinterpret_cast<const float4*>(t_w + qg * kIdxHeads);
              const float4 wb = *reinterpret_cast<const float4*>(t_w + qg * kIdxHeads + 4);
              const float wv[8] = {wa.x, wa.y, wa.z, wa.w, wb.x, wb.y, wb.z, wb.w};
              float s = 0.f;
#pragma unroll
              for (int hd = 0; hd < kIdxHeads; ++hd) s += wv[hd] * relu(__uint_as_float(r[u][8 * k + hd]));
              sc[ql] = s;
            }
        }
        tc_fence_before();
        mbar_arrive(bar_acce + acc * 8);  // this thread is done reading the accumulator
        const bool bad = b < B1 && (phys < 0 || phys >= a.num_pages);
        if (a.bulk) {
          float* stg = reinterpret_cast<float*>(smem + kUOffStage) + ((j & 1) * kUEpiWarps + warp) * kUStageFloats;
          bulk_wait_read1();
          __syncwarp();
#pragma unroll
          for (int ql = 0; ql < kUEpiQ; ++ql) stg[ql * 32 + lane] = bad ? -INFINITY : sc[ql];
          fence_async_smem();
          __syncwarp();
          const int64_t bw = b0 + 32 * qd;
          if (lane < kUEpiQ) {
            const int qg = qh * kUEpiQ + lane;
            const int nbq = t_nb[qg];
            if (t_seq[qg] == S && bw < nbq) {
              float* dst = a.scores + (size_t)(q0 + qg) * a.ld + bw;
              if (bw + 32 <= nbq) {
                bulk_s2g(dst, smem_u32(stg + lane * 32), 128u);
              } else {
                for (int i = 0; i < nbq - bw; ++i) dst[i] = stg[lane * 32 + i];
              }
            }
          }
          bulk_commit();
        } else {
#pragma unroll
          for (int ql = 0; ql < kUEpiQ; ++ql) {
            const int qg = qh * kUEpiQ + ql;
            if (t_seq[qg] == S && b < t_nb[qg])
              a.scores[(size_t)(q0 + qg) * a.ld + b] = bad ? -INFINITY : sc[ql];
          }
        }
      }
    }
  epi_done:;
    bulk_wait_all();  // the scores are written before the CTA ends
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kUMmaWarp) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kUTmemCols) : "memory");
  }
}

bool aligned(const void* p, unsigned a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// The two tensor maps of the query-tiled kernel (the driver's encoder is looked
// up once through the runtime).  Both views are [rows][128 dims] BF16 with rows
// 256 B apart; boxes of 64 dims (128 B, the swizzle span) by 16 rows (one kc
// page) or 256 rows (the 32 queries x 8 heads of a CTA).
bool encode_maps(TiledArgs& t, const void* kc, int32_t num_pages, const void* q_idx, int32_t nq) {
  static PFN_cuTensorMapEncodeTiled_v12000 enc = nullptr;
  if (!enc) {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || !f) {
      (void)cudaGetLastError();
      return false;
    }
    enc = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  }
  const cuuint64_t strides[1] = {(cuuint64_t)kIdxDim * 2};
  const cuuint32_t es[2] = {1, 1};
  const cuuint64_t kdims[2] = {(cuuint64_t)kIdxDim, (cuuint64_t)num_pages * kBlocksPerPage};
  const cuuint32_t kbox[2] = {64, (cuuint32_t)kBlocksPerPage};
  const cuuint64_t qdims[2] = {(cuuint64_t)kIdxDim, (cuuint64_t)nq * kIdxHeads};
  const cuuint32_t qbox[2] = {64, (cuuint32_t)kUN};
  return enc(&t.tm_kc, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(kc), kdims, strides, kbox, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS &&
         enc(&t.tm_q, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(q_idx), qdims, strides, qbox, es,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

extern "C" int qsa_index_scores(const qsa_cache_t* cache, const void* q_idx, const float* w, const int32_t* q_seq,
                                const int32_t* q_pos, int32_t nq, float* scores, int64_t scores_ld,
                                int32_t* dev_status, void* stream) {
  if (!cache || nq < 0 || scores_ld < 1) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!cache->kc_pages || !cache->block_table || !q_idx || !w || !q_seq || !q_pos || !scores)
    return QSA_ERR_INVALID_ARG;
  if (cache->num_pages < 1 || cache->max_seqs < 1 || cache->max_pages_per_seq < 1) return QSA_ERR_INVALID_ARG;
  if (!aligned(cache->kc_pages, 16) || !aligned(q_idx, 16)) return QSA_ERR_INVALID_ARG;
  ScoreArgs a;
  a.kc = static_cast<const __nv_bfloat16*>(cache->kc_pages);
  a.bt = cache->block_table;
  a.num_pages = cache->num_pages;
  a.max_seqs = cache->max_seqs;
  a.mpps = cache->max_pages_per_seq;
  a.q_idx = static_cast<const __nv_bfloat16*>(q_idx);
  a.w = w;
  a.q_seq = q_seq;
  a.q_pos = q_pos;
  a.scores = scores;
  a.ld = scores_ld;
  // Many queries per sequence (chunked prefill): the query-tiled contraction,
  // while every row coordinate of its tensor maps fits 32 bits.
  const bool coords_fit = (int64_t)cache->num_pages * kBlocksPerPage + kBlocksPerPage <= 0x7fffffff &&
                          (int64_t)nq * kIdxHeads + kUN <= 0x7fffffff;
  if ((int64_t)nq >= 8 * (int64_t)cache->max_seqs && nq >= kTQ && coords_fit) {
    TiledArgs t;
    t.kc = static_cast<const __nv_bfloat16*>(cache->kc_pages);
    t.bt = cache->block_table;
    t.num_pages = cache->num_pages;
    t.max_seqs = cache->max_seqs;
    t.mpps = cache->max_pages_per_seq;
    t.q_idx = static_cast<const __nv_bfloat16*>(q_idx);
    t.w = w;
    t.q_seq = q_seq;
    t.q_pos = q_pos;
    t.nq = nq;
    t.scores = scores;
    t.ld = scores_ld;
    t.bulk = (reinterpret_cast<uintptr_t>(scores) & 15u) == 0 && (scores_ld & 3) == 0;
    t.st = dev_status;
    int64_t max_blocks = (int64_t)cache->max_pages_per_seq * kBlocksPerPage;
    if (scores_ld < max_blocks) max_blocks = scores_ld;
    const int64_t gy = (max_blocks + kTChunkBlocks - 1) / kTChunkBlocks;
    const int64_t gx = ((int64_t)nq + kTQ - 1) / kTQ;
    if (gy > 65535 || gx > 0x7fffffff) return QSA_ERR_UNSUPPORTED;
    if (!encode_maps(t, cache->kc_pages, cache->num_pages, q_idx, nq)) return QSA_ERR_CUDA;
    if (cudaFuncSetAttribute(index_scores_umma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kUSmem) !=
        cudaSuccess) {
      (void)cudaGetLastError();
      return QSA_ERR_CUDA;
    }
    return qsa_host::launch(index_scores_umma_kernel, dim3((unsigned)gx, (unsigned)gy), dim3(kUThreads),
                            (size_t)kUSmem, static_cast<cudaStream_t>(stream), t);
  }
  // the most kc pages any query can see is the block-table width
  int64_t max_pages = cache->max_pages_per_seq;
  const int64_t ld_pages = (scores_ld + kBlocksPerPage - 1) / kBlocksPerPage;
  if (ld_pages < max_pages) max_pages = ld_pages;
  // run length: the longest that still leaves about six waves of resident CTAs
  int ppw = kMinPagesPerWarp;
  {
    int dev = 0, sms = 0, per_sm = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, index_scores_kernel, kWarps * 32, 0) != cudaSuccess) {
      (void)cudaGetLastError();
      return QSA_ERR_CUDA;
    }
    const int64_t slots = (int64_t)sms * (per_sm > 0 ? per_sm : 1);
    while (ppw < kMaxPagesPerWarp) {
      const int64_t ctas = (int64_t)nq * ((max_pages + kWarps * 2 * ppw - 1) / (kWarps * 2 * ppw));
      if (ctas < 6 * slots) break;
      ppw *= 2;
    }
  }
  a.pages_per_warp = ppw;
  a.chunks_per_query = (int32_t)((max_pages + kWarps * ppw - 1) / (kWarps * ppw));
  a.st = dev_status;
  const int64_t grid = (int64_t)nq * a.chunks_per_query;
  if (grid > 0x7fffffff) return QSA_ERR_UNSUPPORTED;
  return qsa_host::launch(index_scores_kernel, dim3((unsigned)grid), dim3(kWarps * 32), 0,
                          static_cast<cudaStream_t>(stream), a);
}
