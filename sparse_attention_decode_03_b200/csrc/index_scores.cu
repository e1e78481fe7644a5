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
