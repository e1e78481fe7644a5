// qsa_topk_blocks: per query, the best min(K, nb_q) blocks under (score desc,
// index asc), emitted sorted by block index ascending.
//
// Source: [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section
// "Wat de pull request daadwerkelijk verandert" (keep the best 512 blocks);
// the tie-break (lower index first) and ascending output order are the fixed
// readings.
//
// Order-preserving uint32 keys of the fp32 scores; one CTA of 1024 threads per
// query.  A histogram pass over a whole row costs about one cycle per key of
// one SM's shared-memory atomics, so only small sets are histogrammed:
//   1. threshold: 1024 keys sampled at a regular stride are histogrammed (12-bit
//      window from their highest differing bit); T0 is the lower edge of the
//      bin where the count from the top reaches r = K*1024/n plus a margin of
//      three standard deviations, so that about r*n/1024 >= K keys are >= T0;
//   2. candidates: each warp streams its contiguous 1/32 of the row (16-byte
//      loads) and appends the keys >= T0 with their indices to its own
//      shared-memory list, in index order (ballots and a warp scan);
//   3. exact select among the candidates: radix passes (12-bit windows from
//      the candidates' highest differing bit, shared-memory atomics) give a
//      prefix T under a mask with "every key above T, and the first `need`
//      keys equal to T in index order" = the top K;
//   4. ordered output: warp totals scanned once, then each warp writes its
//      kept indices in order.
// If the sample misleads (fewer than K candidates, or more than a warp's list
// holds) the CTA instead runs the general exact path: three radix passes over
// the row in global memory and an ordered compaction.  Integer counters only:
// the result does not depend on atomic order.
#include "topk_select.cuh"

namespace {

using namespace qsa;

// Block sizes: 1024 threads (few queries: one query's latency is the step's)
// or 256 threads (many queries: more CTAs resident per SM, more throughput).
// Every function below is templated on the block size kThreads.
constexpr int kThreadsLarge = 1024, kThreadsSmall = 256;

struct TopkArgs {
  const float* scores;
  int64_t ld;
  const int32_t* q_pos;
  int32_t K;
  int32_t* sel;
  int32_t* count;
  int32_t* st;
};

constexpr int kBatch = 8;  // 128-key chunks a warp loads at once

// Load the chunks c0 + u*128 (u < kBatch) of [., hi): lane holds keys 4*lane .. 4*lane+3 of each.
__device__ __forceinline__ void load_batch(const float* s, int c0, int hi, bool vec, float4 (&v)[kBatch]) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int u = 0; u < kBatch; ++u) {
    const int i0 = c0 + u * 128 + 4 * lane;
    if (vec && i0 + 3 < hi) {
      v[u] = __ldg(reinterpret_cast<const float4*>(s + i0));
    } else {
      v[u].x = i0 + 0 < hi ? __ldg(s + i0 + 0) : 0.f;
      v[u].y = i0 + 1 < hi ? __ldg(s + i0 + 1) : 0.f;
      v[u].z = i0 + 2 < hi ? __ldg(s + i0 + 2) : 0.f;
      v[u].w = i0 + 3 < hi ? __ldg(s + i0 + 3) : 0.f;
    }
  }
}


template <int kThreads>
__global__ void __launch_bounds__(kThreads, kThreads == kThreadsLarge ? 1 : 4) topk_kernel(TopkArgs a) {
  constexpr int kWarps = kThreads / 32;
  constexpr int kSPer = kSample / kThreads;  // sample keys per thread
  pdl_launch_dependents();
  extern __shared__ __align__(16) uint8_t smem_raw[];
  TopkSmem<kWarps>& S = *reinterpret_cast<TopkSmem<kWarps>*>(smem_raw);
  const int q = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p = a.q_pos[q];  // an input no kernel of this library writes: read before the wait
  pdl_wait_previous();
  int64_t nb = p >= 0 ? (int64_t)(p + 1) / kRatio : 0;
  if (tid == 0 && p < 0) flag(a.st, QSA_DEV_BAD_POS);
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
  if (tid == 0) a.count[q] = K;
  const int n = (int)min(nb, (int64_t)0x7fffffff);
  const float* s = a.scores + (size_t)q * a.ld;

  // Each warp owns a contiguous segment of the row (a multiple of 128 keys).
  // Its first kBatch x 128 keys are loaded now, so that their latency hides
  // behind the threshold phase.
  const int seg = (int)(((int64_t)n + kWarps * 128 - 1) / (kWarps * 128)) * 128;
  const int w_lo = min(n, warp * seg), w_hi = min(n, w_lo + seg);
  const bool vec = (reinterpret_cast<uintptr_t>(s) & 15u) == 0;
  float4 v[kBatch];
  load_batch(s, w_lo, w_hi, vec, v);

  // ---- 1. threshold T0 from a regular sample
  const int ns = min(n, kSample);
  uint32_t ks[kSPer];
#pragma unroll
  for (int u = 0; u < kSPer; ++u) {
    const int i = u * kThreads + tid;
    // position i * n / ns; ns is either n (every key) or the constant kSample
    const int64_t pos = ns < kSample ? (int64_t)i : (int64_t)i * n / kSample;
    ks[u] = i < ns ? float_key(__ldg(s + pos)) : 0u;
  }
  const uint32_t T0 = sample_threshold<kThreads>(ks, ns, n, K, S);

  // ---- 2. candidates: keys >= T0, per warp over its segment, in index order.
  // The scores are compared as floats with T0's float bound; only the
  // candidates' keys are computed.
  const float thr = key_floor(T0);
  uint32_t cnt = 0;
  for (int c0 = w_lo; c0 < w_hi; c0 += kBatch * 128) {
    if (c0 != w_lo) load_batch(s, c0, w_hi, vec, v);
#pragma unroll
    for (int u = 0; u < kBatch; ++u) {
      const int i0 = c0 + u * 128 + 4 * lane;
      const float x[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
      const bool f[4] = {i0 < w_hi && x[0] >= thr, i0 + 1 < w_hi && x[1] >= thr, i0 + 2 < w_hi && x[2] >= thr,
                         i0 + 3 < w_hi && x[3] >= thr};
      append4_by(S, warp, cnt, [&](int c) { return float_key(x[c]); }, i0, f);
    }
  }
  if (lane == 0) S.wcnt[warp] = cnt > kCap ? kCap + 1 : cnt;
  __syncthreads();
  uint32_t total = 0;
  bool overflow = false;
  for (int w = 0; w < kWarps; ++w) {
    total += S.wcnt[w];
    overflow |= S.wcnt[w] > kCap;
  }
  if (overflow || total < (uint32_t)K) {  // block-uniform
    topk_general<kThreads>(s, n, K, out, S.hist, S.wsum, S.wgt, S.weq, &S.bin, &S.above);
    return;
  }
  select_from_lists<kThreads>(S, K, out);
}

template <int kThreads>
int launch_topk(const TopkArgs& a, int32_t nq, void* stream) {
  const int smem = (int)sizeof(TopkSmem<kThreads / 32>);
  if (cudaFuncSetAttribute(topk_kernel<kThreads>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  return qsa_host::launch(topk_kernel<kThreads>, dim3((unsigned)nq), dim3(kThreads), (size_t)smem,
                          static_cast<cudaStream_t>(stream), a);
}

}  // namespace

extern "C" int qsa_topk_blocks(const float* scores, int64_t scores_ld, const int32_t* q_pos, int32_t nq, int32_t k,
                               int32_t* sel, int32_t* count, int32_t* dev_status, void* stream) {
  if (nq < 0 || k < 0 || k > QSA_MAX_TOPK || scores_ld < 1) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!scores || !q_pos || !count || (k > 0 && !sel)) return QSA_ERR_INVALID_ARG;
  TopkArgs a{scores, scores_ld, q_pos, k, sel, count, dev_status};
  int dev = 0, sms = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  // few queries (at most two 1024-thread CTAs per SM): the large block, lowest latency per query;
  // many: 256-thread blocks, several resident per SM, more queries in flight
  const bool large = (int64_t)nq <= 2 * (int64_t)sms;
  return large ? launch_topk<kThreadsLarge>(a, nq, stream) : launch_topk<kThreadsSmall>(a, nq, stream);
}
