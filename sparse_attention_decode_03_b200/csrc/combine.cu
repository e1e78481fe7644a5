// qsa_combine: log-sum-exp merge of the split-KV partials of every (query, Q head).
//
// Source: [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section
// "Wat de pull request daadwerkelijk verandert" (after the split read the
// attention results are combined); [CANN] "Qwen4-Exp QSA komt naar Huawei's
// Ascend ...", section "Wat de pull request daadwerkelijk toevoegt" (fully
// masked rows keep the zero-output convention).
//
#include "qsa_common.cuh"

namespace {

using namespace qsa;

constexpr int kThreads = kHeadDim / 4;  // 64: four output dims per thread

// One CTA per (query, head).  Each thread recomputes the S split weights (S
// lse values, broadcast from L1) and accumulates its 4 dims over the splits
// with independent 16-byte loads.
__global__ void __launch_bounds__(kThreads) combine_kernel(const float* __restrict__ part_o,
                                                           const float* __restrict__ part_lse, int S, int hq,
                                                           __nv_bfloat16* __restrict__ out, float* __restrict__ lse) {
  pdl_launch_dependents();
  pdl_wait_previous();
  const int qh = blockIdx.x;
  const int q = qh / hq, h = qh % hq;
  const int tid = threadIdx.x;
  const float* pl = part_lse + (size_t)q * S * hq + h;
  float M = -INFINITY;
  for (int s = 0; s < S; ++s) M = fmaxf(M, pl[(size_t)s * hq]);
  uint2* dst = reinterpret_cast<uint2*>(out + (size_t)qh * kHeadDim) + tid;
  if (M == -INFINITY) {  // every split empty: zero output, lse = -inf
    *dst = make_uint2(0u, 0u);
    if (tid == 0) lse[qh] = -INFINITY;
    return;
  }
  float L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  const float4* po = reinterpret_cast<const float4*>(part_o + ((size_t)q * S * hq + h) * kHeadDim) + tid;
  const size_t split_stride = (size_t)hq * kHeadDim / 4;
#pragma unroll 4
  for (int s = 0; s < S; ++s) {
    const float v = pl[(size_t)s * hq];
    if (v == -INFINITY) continue;
    const float e = expf(v - M);
    const float4 x = po[s * split_stride];
    L += e;
    acc.x += e * x.x;
    acc.y += e * x.y;
    acc.z += e * x.z;
    acc.w += e * x.w;
  }
  const float inv = 1.f / L;
  uint2 o;
  o.x = pack_bf16(acc.x * inv, acc.y * inv);
  o.y = pack_bf16(acc.z * inv, acc.w * inv);
  *dst = o;
  if (tid == 0) lse[qh] = M + logf(L);
}

}  // namespace

extern "C" int qsa_combine(const float* part_o, const float* part_lse, int32_t nq, int32_t max_splits, int32_t hq,
                           void* out, float* lse, void* stream) {
  if (nq < 0 || max_splits < 1 || hq < 1) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!part_o || !part_lse || !out || !lse) return QSA_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(part_o) & 15u) || (reinterpret_cast<uintptr_t>(out) & 7u)) return QSA_ERR_INVALID_ARG;
  const int64_t grid = (int64_t)nq * hq;
  if (grid > 0x7fffffff) return QSA_ERR_UNSUPPORTED;
  return qsa_host::launch(combine_kernel, dim3((unsigned)grid), dim3(kThreads), 0, static_cast<cudaStream_t>(stream),
                          part_o, part_lse, max_splits, hq, static_cast<__nv_bfloat16*>(out), lse);
}
