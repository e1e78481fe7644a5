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
// blocks, K = 128 dims, N = the 8 indexer heads).  The contraction dimension
// is permuted consistently in A and B so that each lane reads whole 16-byte
// chunks: lane (g, t) holds dims of chunks 4i+t (i = 0..3) of rows g and g+8.
#include "qsa_common.cuh"

namespace {

using namespace qsa;

constexpr int kWarps = 8;
constexpr int kPagesPerWarp = 4;
constexpr int kPagesPerCta = kWarps * kPagesPerWarp;  // 32 pages = 512 blocks = 128 KiB

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
  int32_t* st;
};

__device__ __forceinline__ float relu(float x) { return x > 0.f ? x : 0.f; }

__global__ void __launch_bounds__(kWarps * 32) index_scores_kernel(ScoreArgs a) {
  pdl_launch_dependents();
  pdl_wait_previous();
  const int q = blockIdx.x / a.chunks_per_query;
  const int chunk = blockIdx.x % a.chunks_per_query;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, t = lane & 3;

  const int seq = a.q_seq[q];
  const int p = a.q_pos[q];
  if (seq < 0 || seq >= a.max_seqs || p < 0 || (int64_t)p >= (int64_t)a.mpps * kPage) {
    if (chunk == 0 && threadIdx.x == 0) flag(a.st, (seq < 0 || seq >= a.max_seqs) ? QSA_DEV_BAD_SEQ : QSA_DEV_BAD_POS);
    return;
  }
  int64_t nb = (p + 1) / kRatio;
  if (nb > a.ld) {
    if (chunk == 0 && threadIdx.x == 0) flag(a.st, QSA_DEV_SCORES_LD);
    nb = a.ld;
  }
  const int npg = (int)((nb + kBlocksPerPage - 1) / kBlocksPerPage);
  const int pg0 = chunk * kPagesPerCta + warp * kPagesPerWarp;
  if (pg0 >= npg) return;

  // B fragments: indexer query head g, chunks 4i+t of its 128 dims.
  uint4 qb[4];
  const __nv_bfloat16* qrow = a.q_idx + ((size_t)q * kIdxHeads + g) * kIdxDim;
#pragma unroll
  for (int i = 0; i < 4; ++i) qb[i] = ldg_nc(qrow + (4 * i + t) * 8);
  const float w0 = a.w[q * kIdxHeads + 2 * t];
  const float w1 = a.w[q * kIdxHeads + 2 * t + 1];

  int myphys = -1;
  if (lane < kPagesPerWarp && pg0 + lane < npg) myphys = a.bt[(int64_t)seq * a.mpps + pg0 + lane];
  float* srow = a.scores + (size_t)q * a.ld;

#pragma unroll
  for (int pp = 0; pp < kPagesPerWarp; pp += 2) {
    uint4 ra[2][4], rb[2][4];
    int phys[2];
    bool ok[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      phys[k] = __shfl_sync(0xffffffffu, myphys, pp + k);
      ok[k] = (pg0 + pp + k < npg) && phys[k] >= 0 && phys[k] < a.num_pages;
      if (ok[k]) {
        const __nv_bfloat16* base = a.kc + (size_t)phys[k] * kBlocksPerPage * kIdxDim;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          ra[k][i] = ldg_stream(base + (size_t)g * kIdxDim + (4 * i + t) * 8);
          rb[k][i] = ldg_stream(base + (size_t)(g + 8) * kIdxDim + (4 * i + t) * 8);
        }
      }
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
      float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        mma_bf16_16816(acc, ra[k][i].x, rb[k][i].x, ra[k][i].y, rb[k][i].y, qb[i].x, qb[i].y);
        mma_bf16_16816(acc, ra[k][i].z, rb[k][i].z, ra[k][i].w, rb[k][i].w, qb[i].z, qb[i].w);
      }
      // acc: (block g, heads 2t, 2t+1), (block g+8, heads 2t, 2t+1)
      float s_lo = w0 * relu(acc[0]) + w1 * relu(acc[1]);
      float s_hi = w0 * relu(acc[2]) + w1 * relu(acc[3]);
      s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
      s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
      s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
      s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
      if (t == 0 && blk_lo < nb) srow[blk_lo] = s_lo;
      if (t == 1 && blk_hi < nb) srow[blk_hi] = s_hi;
    }
  }
}

// ---------------------------------------------------------------------------
// Query-tiled variant for calls with many queries per sequence (chunked
// prefill / extend): the queries of one sequence all read the same side cache,
// so the work is a dense contraction [queries x 8 heads] x 128 x [blocks] and
// a CTA of 16 consecutive queries reads each kc tile once for all of them.
// Warp w holds, for the whole kernel, the A fragments of its 16 rows (queries
// 2w and 2w+1, 8 heads each); 128-block kc tiles stream through a 3-stage
// shared-memory ring (16-byte cp.async, rows padded to 272 B so the 16-byte
// fragment reads are bank-conflict free); per 8-block n-tile: 8 mma.sync, then
// w * ReLU and the sum over the 8 heads by a 3-step butterfly across the lanes.
// Queries of the tile that belong to other sequences are handled by further
// passes over their own pages (one pass per distinct sequence of the tile).

constexpr int kTQ = 16;                   // queries per CTA
constexpr int kTB = 128;                  // blocks per kc tile
constexpr int kTStages = 3;
constexpr int kTRow = kIdxDim * 2 + 16;   // 272 B: padded kc row in shared memory
constexpr int kTTileBytes = kTB * kTRow;
constexpr int kTChunkBlocks = 2048;       // blocks per CTA (gridDim.y splits longer rows)
constexpr int kTSmem = kTStages * kTTileBytes + kTStages * kTB + 4 * kTQ * 4 + 64;

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
  int32_t* st;
};

__device__ __forceinline__ void cp_async16_zfill_skip(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__global__ void __launch_bounds__(kWarps * 32, 2) index_scores_tiled_kernel(TiledArgs a) {
  pdl_launch_dependents();
  pdl_wait_previous();
  extern __shared__ __align__(16) uint8_t smem[];
  uint8_t* badrow = smem + kTStages * kTTileBytes;                           // [stage][128]
  int32_t* t_seq = reinterpret_cast<int32_t*>(badrow + kTStages * kTB);      // [16] sequence of each query (-1: none)
  int32_t* t_nb = t_seq + kTQ;                                               // [16] visible blocks
  int32_t* t_list = t_nb + kTQ;                                              // [16] distinct sequences
  int32_t* t_cnt = t_list + kTQ;                                             // [1]  how many
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, t = lane & 3;
  const int q0 = blockIdx.x * kTQ;
  const int64_t blk_lo = (int64_t)blockIdx.y * kTChunkBlocks;

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

  // A fragments: rows g -> (query 2w, head g), g + 8 -> (query 2w + 1, head g);
  // chunk 4i + t of each 128-dim row (the contraction index permuted as in B)
  const int qa = q0 + 2 * warp, qb = qa + 1;
  uint4 fa[4], fb[4];
  float wa = 0.f, wb = 0.f;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    fa[i] = qa < a.nq ? ldg_nc(a.q_idx + ((size_t)qa * kIdxHeads + g) * kIdxDim + (4 * i + t) * 8) : make_uint4(0, 0, 0, 0);
    fb[i] = qb < a.nq ? ldg_nc(a.q_idx + ((size_t)qb * kIdxHeads + g) * kIdxDim + (4 * i + t) * 8) : make_uint4(0, 0, 0, 0);
  }
  if (qa < a.nq) wa = a.w[qa * kIdxHeads + g];
  if (qb < a.nq) wb = a.w[qb * kIdxHeads + g];
  __syncthreads();
  const int nseq = *t_cnt;
  const uint32_t ring = smem_u32(smem);

  for (int si = 0; si < nseq; ++si) {
    const int S = t_list[si];
    int nb_max = 0;
    for (int i = 0; i < kTQ; ++i)
      if (t_seq[i] == S) nb_max = max(nb_max, t_nb[i]);
    const int64_t B0 = blk_lo, B1 = min((int64_t)nb_max, blk_lo + kTChunkBlocks);
    if (B0 >= B1) continue;  // uniform
    const int ntile = (int)((B1 - B0 + kTB - 1) / kTB);
    const bool mine_a = qa < a.nq && t_seq[2 * warp] == S;
    const bool mine_b = qb < a.nq && t_seq[2 * warp + 1] == S;
    const int nb_a = t_nb[2 * warp], nb_b = t_nb[2 * warp + 1];

    auto load_tile = [&](int j) {
      const int stage = j % kTStages;
      const int64_t b0 = B0 + (int64_t)j * kTB;
#pragma unroll
      for (int k = 0; k < (kTB * 16) / (kWarps * 32); ++k) {  // 8 x 16 B per thread
        const int e = tid + k * kWarps * 32;
        const int r = e >> 4, c = e & 15;
        const int64_t b = b0 + r;
        const uint32_t dst = ring + stage * kTTileBytes + r * kTRow + c * 16;
        bool bad = false;
        if (b < B1) {
          const int phys = a.bt[(int64_t)S * a.mpps + b / kBlocksPerPage];
          if (phys >= 0 && phys < a.num_pages) {
            cp_async16_zfill_skip(dst, a.kc + ((size_t)phys * kBlocksPerPage + b % kBlocksPerPage) * kIdxDim + c * 8);
          } else {
            bad = true;
            sts128(dst, make_uint4(0, 0, 0, 0));
          }
        } else {
          sts128(dst, make_uint4(0, 0, 0, 0));
        }
        if (c == 0) {
          badrow[stage * kTB + r] = bad ? 1 : 0;
          if (bad) flag(a.st, QSA_DEV_BAD_PAGE);
        }
      }
    };

#pragma unroll
    for (int j = 0; j < kTStages - 1; ++j) {
      if (j < ntile) load_tile(j);
      cp_async_commit();
    }
    for (int j = 0; j < ntile; ++j) {
      cp_async_wait_group<kTStages - 2>();
      __syncthreads();  // tile j visible to all; every warp is done with tile j - 1
      if (j + kTStages - 1 < ntile) load_tile(j + kTStages - 1);
      cp_async_commit();
      const int stage = j % kTStages;
      const uint32_t tile = ring + stage * kTTileBytes;
      const int64_t b0 = B0 + (int64_t)j * kTB;
      if (!mine_a && !mine_b) continue;
#pragma unroll 2
      for (int nt = 0; nt < kTB / 8; ++nt) {
        float s0[4] = {0.f, 0.f, 0.f, 0.f}, s1[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const uint4 kb = lds128(tile + (nt * 8 + g) * kTRow + (4 * i + t) * 16);
          float(&acc)[4] = (i & 1) ? s1 : s0;
          mma_bf16_16816(acc, fa[i].x, fb[i].x, fa[i].y, fb[i].y, kb.x, kb.y);
          mma_bf16_16816(acc, fa[i].z, fb[i].z, fa[i].w, fb[i].w, kb.z, kb.w);
        }
        // (row g | g + 8, block 2t | 2t + 1) -> w * ReLU, then the sum over the 8 heads
        const float v0 = wa * relu(s0[0] + s1[0]), v1 = wa * relu(s0[1] + s1[1]);
        const float v2 = wb * relu(s0[2] + s1[2]), v3 = wb * relu(s0[3] + s1[3]);
        const bool up4 = (g & 4) != 0, up2 = (g & 2) != 0;
        float x0 = up4 ? v2 : v0, x1 = up4 ? v3 : v1;
        x0 += __shfl_xor_sync(0xffffffffu, up4 ? v0 : v2, 16);
        x1 += __shfl_xor_sync(0xffffffffu, up4 ? v1 : v3, 16);
        float z = up2 ? x1 : x0;
        z += __shfl_xor_sync(0xffffffffu, up2 ? x0 : x1, 8);
        z += __shfl_xor_sync(0xffffffffu, z, 4);
        // lanes with g even hold query (g & 4 ? qb : qa), block nt * 8 + 2t + (g >> 1 & 1)
        if ((g & 1) == 0) {
          const int r = nt * 8 + 2 * t + ((g >> 1) & 1);
          const int64_t b = b0 + r;
          const bool for_b = up4;
          const int q = for_b ? qb : qa;
          const int nbq = for_b ? nb_b : nb_a;
          if ((for_b ? mine_b : mine_a) && b < nbq)
            a.scores[(size_t)q * a.ld + b] = badrow[stage * kTB + r] ? -INFINITY : z;
        }
      }
    }
    cp_async_wait_group<0>();
    __syncthreads();  // the ring is free before the next sequence's pass
  }
}

bool aligned(const void* p, unsigned a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

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
  // Many queries per sequence (chunked prefill): the query-tiled contraction.
  if ((int64_t)nq >= 8 * (int64_t)cache->max_seqs && nq >= kTQ) {
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
    t.st = dev_status;
    int64_t max_blocks = (int64_t)cache->max_pages_per_seq * kBlocksPerPage;
    if (scores_ld < max_blocks) max_blocks = scores_ld;
    const int64_t gy = (max_blocks + kTChunkBlocks - 1) / kTChunkBlocks;
    const int64_t gx = ((int64_t)nq + kTQ - 1) / kTQ;
    if (gy > 65535 || gx > 0x7fffffff) return QSA_ERR_UNSUPPORTED;
    if (cudaFuncSetAttribute(index_scores_tiled_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kTSmem) !=
        cudaSuccess) {
      (void)cudaGetLastError();
      return QSA_ERR_CUDA;
    }
    return qsa_host::launch(index_scores_tiled_kernel, dim3((unsigned)gx, (unsigned)gy), dim3(kWarps * 32),
                            (size_t)kTSmem, static_cast<cudaStream_t>(stream), t);
  }
  // the most kc pages any query can see is the block-table width
  int64_t max_pages = cache->max_pages_per_seq;
  const int64_t ld_pages = (scores_ld + kBlocksPerPage - 1) / kBlocksPerPage;
  if (ld_pages < max_pages) max_pages = ld_pages;
  a.chunks_per_query = (int32_t)((max_pages + kPagesPerCta - 1) / kPagesPerCta);
  a.st = dev_status;
  const int64_t grid = (int64_t)nq * a.chunks_per_query;
  if (grid > 0x7fffffff) return QSA_ERR_UNSUPPORTED;
  return qsa_host::launch(index_scores_kernel, dim3((unsigned)grid), dim3(kWarps * 32), 0,
                          static_cast<cudaStream_t>(stream), a);
}
