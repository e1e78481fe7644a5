// qsa_topk_blocks: per query, the best min(K, nb_q) blocks under (score desc,
// index asc), emitted sorted by block index ascending.
//
// Source: [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section
// "Wat de pull request daadwerkelijk verandert" (keep the best 512 blocks);
// the tie-break (lower index first) and ascending output order are the fixed
// readings.
//
// One CTA per query.  Deterministic radix select on order-preserving uint32
// keys of the fp32 scores: three histogram passes (12 + 12 + 8 bits, integer
// shared-memory counters) find the exact key T of the K-th largest score; a
// final ordered compaction (warp ballots over contiguous index ranges plus a
// prefix over warps) emits every key > T and the lowest-index keys == T.
#include "qsa_common.cuh"

namespace {

using namespace qsa;

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kMaxBins = 4096;

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

__global__ void __launch_bounds__(kThreads) topk_kernel(TopkArgs a) {
  __shared__ uint32_t hist[kMaxBins];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t wgt[kWarps], weq[kWarps];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;

  const int q = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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

  uint32_t prefix = 0, mask = 0, remaining = (uint32_t)K;
  const int shifts[3] = {20, 8, 0};
  const int bits[3] = {12, 12, 8};
  for (int pass = 0; pass < 3; ++pass) {
    const int nbins = 1 << bits[pass];
    const int sh = shifts[pass];
    for (int i = tid; i < nbins; i += kThreads) hist[i] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kThreads) {
      const uint32_t key = float_key(s[i]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> sh) & (nbins - 1)], 1u);
    }
    __syncthreads();
    find_bin(hist, nbins, remaining, wsum, &s_bin, &s_above);
    prefix |= (uint32_t)s_bin << sh;
    mask |= (uint32_t)(nbins - 1) << sh;
    remaining -= s_above;
    __syncthreads();
  }
  const uint32_t T = prefix;
  const uint32_t need_eq = remaining;  // keys equal to T to keep, lowest index first

  // ordered compaction: warp w owns the contiguous index range [w*span, (w+1)*span)
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
  if (tid == 0) a.count[q] = K;
}

}  // namespace

extern "C" int qsa_topk_blocks(const float* scores, int64_t scores_ld, const int32_t* q_pos, int32_t nq, int32_t k,
                               int32_t* sel, int32_t* count, int32_t* dev_status, void* stream) {
  if (nq < 0 || k < 0 || k > QSA_MAX_TOPK || scores_ld < 1) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!scores || !q_pos || !count || (k > 0 && !sel)) return QSA_ERR_INVALID_ARG;
  TopkArgs a{scores, scores_ld, q_pos, k, sel, count, dev_status};
  topk_kernel<<<(unsigned)nq, kThreads, 0, static_cast<cudaStream_t>(stream)>>>(a);
  return qsa_host::launch_status();
}
