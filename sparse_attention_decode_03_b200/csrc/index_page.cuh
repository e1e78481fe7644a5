// One warp scores one 4 KiB side-cache page (16 micro-blocks x 128 dims) for
// one query: s[j] = sum_h w[h] * ReLU(q_idx[h] . kc[j]) over the 8 indexer
// heads, on mma.sync m16n8k16 (A = the page's 16 blocks, B = the 8 heads).
// Shared by the standalone indexer (index_scores.cu) and the fused indexer +
// selection kernel (index_topk.cu), so the two produce identical scores.
//
// Fragment layout: lane (g, t) = (lane / 4, lane % 4) holds dims of 16-byte
// chunks 4i + t (i = 0..3) of page rows g and g + 8 (A) and of head g (B); the
// contraction dimension is permuted the same way in A and B, so every lane
// reads whole 16-byte chunks.
#pragma once
#include "qsa_common.cuh"

namespace qsa {

QSA_DEVINL float relu(float x) { return x > 0.f ? x : 0.f; }

struct IdxQuery {
  uint4 qb[4];  // B fragments: head g, chunks 4i + t
  float w0, w1; // head weights 2t and 2t + 1
};

QSA_DEVINL IdxQuery load_idx_query(const __nv_bfloat16* q_idx, const float* w, int q) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  IdxQuery Q;
  const __nv_bfloat16* qrow = q_idx + ((size_t)q * kIdxHeads + g) * kIdxDim;
#pragma unroll
  for (int i = 0; i < 4; ++i) Q.qb[i] = ldg_nc(qrow + (4 * i + t) * 8);
  Q.w0 = w[q * kIdxHeads + 2 * t];
  Q.w1 = w[q * kIdxHeads + 2 * t + 1];
  return Q;
}

// A fragments of page `phys` (rows g and g + 8), streamed past L1.
QSA_DEVINL void load_idx_page(const __nv_bfloat16* kc, int phys, uint4 (&ra)[4], uint4 (&rb)[4]) {
  const int lane = threadIdx.x & 31, g = lane >> 2, t = lane & 3;
  const __nv_bfloat16* base = kc + (size_t)phys * kBlocksPerPage * kIdxDim;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    ra[i] = ldg_stream(base + (size_t)g * kIdxDim + (4 * i + t) * 8);
    rb[i] = ldg_stream(base + (size_t)(g + 8) * kIdxDim + (4 * i + t) * 8);
  }
}

// Scores of page rows g (s_lo) and g + 8 (s_hi), summed over the heads in
// every lane of the quad.
QSA_DEVINL void score_idx_page(const uint4 (&ra)[4], const uint4 (&rb)[4], const IdxQuery& Q, float& s_lo,
                               float& s_hi) {
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    mma_bf16_16816(acc, ra[i].x, rb[i].x, ra[i].y, rb[i].y, Q.qb[i].x, Q.qb[i].y);
    mma_bf16_16816(acc, ra[i].z, rb[i].z, ra[i].w, rb[i].w, Q.qb[i].z, Q.qb[i].w);
  }
  // acc: (block g, heads 2t, 2t+1), (block g+8, heads 2t, 2t+1)
  s_lo = Q.w0 * relu(acc[0]) + Q.w1 * relu(acc[1]);
  s_hi = Q.w0 * relu(acc[2]) + Q.w1 * relu(acc[3]);
  s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 1);
  s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 1);
  s_lo += __shfl_xor_sync(0xffffffffu, s_lo, 2);
  s_hi += __shfl_xor_sync(0xffffffffu, s_hi, 2);
}

}  // namespace qsa
