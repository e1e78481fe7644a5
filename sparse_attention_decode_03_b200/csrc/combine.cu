// qsa_combine: log-sum-exp merge of the split-KV partials of every (query, Q head).
//
// Source: [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section
// "Wat de pull request daadwerkelijk verandert" (after the split read the
// attention results are combined); [CANN] "Qwen4-Exp QSA komt naar Huawei's
// Ascend ...", section "Wat de pull request daadwerkelijk toevoegt" (fully
// masked rows keep the zero-output convention).
//
// One CTA per query; thread d owns output dim d of every head, so every read of
// part_o and every write of out is a coalesced row.  The split weights
// exp(lse_s - lse) are computed once per (query, head) in shared memory.
#include "qsa_common.cuh"

namespace {

using namespace qsa;

constexpr int kThreads = kHeadDim;  // 256
constexpr int kMaxSplitHeads = 8192;  // max_splits * hq held in shared memory

__global__ void __launch_bounds__(kThreads) combine_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_lse, int S, int hq,
                                                           __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  __shared__ float wt[kMaxSplitHeads];   // [S][hq] split weights
  __shared__ float s_lse[QSA_MAX_GROUP * 64];
  const int q = blockIdx.x;
  const int tid = threadIdx.x;
  const float* pl = part_lse + (size_t)q * S * hq;
  for (int h = tid; h < hq; h += kThreads) {
    float M = -INFINITY;
    for (int s = 0; s < S; ++s) M = fmaxf(M, pl[s * hq + h]);
    if (M == -INFINITY) {
      for (int s = 0; s < S; ++s) wt[s * hq + h] = 0.f;
      s_lse[h] = -INFINITY;
      continue;
    }
    float L = 0.f;
    for (int s = 0; s < S; ++s) {
      const float v = pl[s * hq + h];
      const float e = v == -INFINITY ? 0.f : expf(v - M);
      wt[s * hq + h] = e;
      L += e;
    }
    const float inv = 1.f / L;
    for (int s = 0; s < S; ++s) wt[s * hq + h] *= inv;
    s_lse[h] = M + logf(L);
  }
  __syncthreads();
  for (int h = 0; h < hq; ++h) {
    float acc = 0.f;
    for (int s = 0; s < S; ++s) {
      const float wgt = wt[s * hq + h];
      if (wgt != 0.f) acc += wgt * part_o[(((size_t)q * S + s) * hq + h) * kHeadDim + tid];
    }
    out[((size_t)q * hq + h) * kHeadDim + tid] = __float2bfloat16_rn(acc);
  }
  for (int h = tid; h < hq; h += kThreads) lse[(size_t)q * hq + h] = s_lse[h];
}

}  // namespace

extern "C" int qsa_combine(const float* part_o, const float* part_lse, int32_t nq, int32_t max_splits, int32_t hq,
                           void* out, float* lse, void* stream) {
  if (nq < 0 || max_splits < 1 || hq < 1) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!part_o || !part_lse || !out || !lse) return QSA_ERR_INVALID_ARG;
  if (hq > QSA_MAX_GROUP * 64 || (int64_t)max_splits * hq > kMaxSplitHeads) return QSA_ERR_UNSUPPORTED;
  combine_kernel<<<(unsigned)nq, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(
      part_o, part_lse, max_splits, hq, static_cast<__nv_bfloat16*>(out), lse);
  return qsa_host::launch_status();
}
