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

struct CombineArgs {
  const float* part_o;
  const float* part_lse;
  int S, hq;
  int64_t o_q, o_s;  // element strides of part_o between queries / splits (heads: 256)
  int64_t l_q, l_s;  // element strides of part_lse between queries / splits (heads: 1)
  void* out;         // bf16 or fp32 [nq][hq][256]
  float* lse;
};

// One CTA per (query, head).  Each thread owns 4 dims; the split loads are
// issued together (merge_row).
template <bool F32Out>
__global__ void __launch_bounds__(kThreads) combine_kernel(CombineArgs a) {
  pdl_launch_dependents();
  pdl_wait_previous();
  const int qh = blockIdx.x;
  const int q = qh / a.hq, h = qh % a.hq;
  const int tid = threadIdx.x;
  const float* pl = a.part_lse + q * a.l_q + h;
  const float* po = a.part_o + q * a.o_q + (int64_t)h * kHeadDim + 4 * tid;
  float lse_v;
  const float4 res = merge_row(
      a.S, [&](int s) { return pl[s * a.l_s]; },
      [&](int s) { return *reinterpret_cast<const float4*>(po + s * a.o_s); }, lse_v);
  if constexpr (F32Out) {
    reinterpret_cast<float4*>(static_cast<float*>(a.out) + (size_t)qh * kHeadDim)[tid] = res;
  } else {
    uint2 o;
    o.x = pack_bf16(res.x, res.y);
    o.y = pack_bf16(res.z, res.w);
    reinterpret_cast<uint2*>(static_cast<__nv_bfloat16*>(a.out) + (size_t)qh * kHeadDim)[tid] = o;
  }
  if (tid == 0) a.lse[qh] = lse_v;
}

}  // namespace

extern "C" int qsa_combine_strided(const float* part_o, const float* part_lse, int32_t nq, int32_t nsplits,
                                   int32_t hq, int64_t o_q_stride, int64_t o_split_stride, int64_t lse_q_stride,
                                   int64_t lse_split_stride, void* out, int32_t out_dtype, float* lse, void* stream) {
  if (nq < 0 || nsplits < 1 || hq < 1) return QSA_ERR_INVALID_ARG;
  if (out_dtype != QSA_OUT_BF16 && out_dtype != QSA_OUT_F32) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!part_o || !part_lse || !out || !lse) return QSA_ERR_INVALID_ARG;
  if (o_q_stride < 0 || o_split_stride < 0 || lse_q_stride < 0 || lse_split_stride < 0 || (o_q_stride & 3) ||
      (o_split_stride & 3))
    return QSA_ERR_INVALID_ARG;
  const uintptr_t out_align = out_dtype == QSA_OUT_F32 ? 15u : 7u;
  if ((reinterpret_cast<uintptr_t>(part_o) & 15u) || (reinterpret_cast<uintptr_t>(out) & out_align))
    return QSA_ERR_INVALID_ARG;
  const int64_t grid = (int64_t)nq * hq;
  if (grid > 0x7fffffff) return QSA_ERR_UNSUPPORTED;
  const CombineArgs a{part_o, part_lse, nsplits, hq, o_q_stride, o_split_stride, lse_q_stride, lse_split_stride, out,
                      lse};
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  return out_dtype == QSA_OUT_F32
             ? qsa_host::launch(combine_kernel<true>, dim3((unsigned)grid), dim3(kThreads), 0, s, a)
             : qsa_host::launch(combine_kernel<false>, dim3((unsigned)grid), dim3(kThreads), 0, s, a);
}

extern "C" int qsa_combine(const float* part_o, const float* part_lse, int32_t nq, int32_t max_splits, int32_t hq,
                           void* out, float* lse, void* stream) {
  if (nq < 0 || max_splits < 1 || hq < 1) return QSA_ERR_INVALID_ARG;
  const int64_t S = max_splits, H = hq;
  return qsa_combine_strided(part_o, part_lse, nq, max_splits, hq, S * H * kHeadDim, H * kHeadDim, S * H, H, out,
                             QSA_OUT_BF16, lse, stream);
}
