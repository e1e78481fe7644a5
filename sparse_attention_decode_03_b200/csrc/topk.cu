// qsa_topk_blocks: per query, the best min(K, nb_q) blocks under (score desc,
// index asc), emitted sorted by block index ascending.
//
// Source: [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section
// "Wat de pull request daadwerkelijk verandert" (keep the best 512 blocks);
// the tie-break (lower index first) and ascending output order are the fixed
// readings.
//
// Order-preserving uint32 keys of the fp32 scores.  One thread-block cluster
// of 8 CTAs per query (decode batches have only 32-64 queries, so a single CTA
// per query leaves the per-key work on too few SMs).  CTA r of the cluster owns
// the r-th contiguous eighth of the row and keeps its keys in shared memory
// after one vectorised read.  Then:
//   1. cluster-wide min / max key (distributed shared memory);
//   2. radix select with adaptive 11-bit windows starting at the highest bit
//      where the keys differ (scores share their top exponent bits): every CTA
//      histograms its slice, the 8 histograms are summed through distributed
//      shared memory, and each CTA finds the same bin; this yields the exact
//      K-th largest key T;
//   3. each CTA ranks its keys == T in index order (word ballots, a block scan
//      and the counts of the lower-ranked CTAs) and keeps the lowest-index
//      ones, then writes its selected indices, in ascending order, at the
//      offset given by the lower-ranked CTAs' counts.
// Rows longer than 65,536 blocks take the general path in the cluster's first
// CTA: three radix passes over the scores (12 + 12 + 8 bits) and an ordered
// compaction with warp ballots.
// Integer counters only: the result does not depend on atomic order.
#include "qsa_common.cuh"

#include <cooperative_groups.h>

namespace {

using namespace qsa;

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

struct TopkArgs {
  const float* scores;
  int64_t ld;
  const int32_t* q_pos;
  int32_t K;
  int32_t fast_cap;  // blocks per query the shared-memory path holds
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

constexpr int kCluster = 8;                    // CTAs per query
constexpr int kCThreads = 512;                 // threads per cluster CTA
constexpr int kCWarps = kCThreads / 32;
constexpr int kSliceCap = 8192;                // keys per CTA on the cluster path
constexpr int kMaxFast = kCluster * kSliceCap; // 65,536 blocks per query
constexpr int kUnroll = 8;
constexpr int kWin = 11;                       // radix window bits
constexpr int kWinBins = 1 << kWin;

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

// Shared-memory histogram increment.  A warp whose live lanes all hit one bin
// (common when scores crowd together) adds once; otherwise per-lane atomics.
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool live) {
  const uint32_t act = __ballot_sync(0xffffffffu, live);
  if (act == 0) return;
  const int leader = __ffs(act) - 1;
  const uint32_t b0 = __shfl_sync(0xffffffffu, bin, leader);
  if (__all_sync(0xffffffffu, !live || bin == b0)) {
    if ((threadIdx.x & 31) == leader) atomicAdd(&hist[b0], (uint32_t)__popc(act));
  } else if (live) {
    atomicAdd(&hist[bin], 1u);
  }
}

// Bin b of a merged histogram (every thread returns the same) with
// sum_{i > b} hist[i] < remaining <= sum_{i >= b} hist[i]; *above = sum_{i > b}.
__device__ int cluster_find_bin(const uint32_t* hist, int nbins, uint32_t remaining, uint32_t* wsum, int* s_bin,
                                uint32_t* s_above, uint32_t* above) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (nbins + kCThreads - 1) / kCThreads;
  const int lo = tid * per;
  uint32_t local = 0;
  for (int i = 0; i < per; ++i)
    if (lo + i < nbins) local += hist[lo + i];
  uint32_t suf = local;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, suf, d);
    if (lane + d < 32) suf += v;
  }
  if (lane == 0) wsum[warp] = suf;
  __syncthreads();
  uint32_t cum = suf - local;
  for (int w = warp + 1; w < kCWarps; ++w) cum += wsum[w];
  for (int i = per - 1; i >= 0; --i) {
    if (lo + i >= nbins) continue;
    const uint32_t h = hist[lo + i];
    if (cum < remaining && remaining <= cum + h) {
      *s_bin = lo + i;
      *s_above = cum;
    }
    cum += h;
  }
  __syncthreads();
  *above = *s_above;
  return *s_bin;
}

// Block-wide exclusive prefix of one value per thread; returns the block total.
__device__ uint32_t block_exclusive(uint32_t v, uint32_t* wsum, uint32_t* prefix) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t inc = v;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += x;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  uint32_t base = inc - v, total = 0;
  for (int w = 0; w < kCWarps; ++w) {
    if (w < warp) base += wsum[w];
    total += wsum[w];
  }
  __syncthreads();
  *prefix = base;
  return total;
}

__global__ void __cluster_dims__(kCluster, 1, 1) __launch_bounds__(kCThreads) topk_kernel(TopkArgs a) {
  namespace cg = cooperative_groups;
  cg::cluster_group cluster = cg::this_cluster();
  extern __shared__ __align__(16) uint32_t keys[];  // [kSliceCap] this CTA's slice of keys (dynamic)
  __shared__ uint32_t hist[kWinBins];    // this slice's histogram
  __shared__ uint32_t merged[kWinBins];  // the cluster's histogram (written by all 8 CTAs)
  __shared__ uint32_t wgt_cnt[kSliceCap / 32], weq_cnt[kSliceCap / 32];
  __shared__ uint32_t wsum[kCWarps];
  __shared__ uint32_t pub[4];  // published per CTA: min key, max key, #keys > T, #keys == T
  __shared__ int s_bin;
  __shared__ uint32_t s_above;

  const int rank = (int)cluster.block_rank();
  const int q = blockIdx.x / kCluster;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p = a.q_pos[q];
  int64_t nb = p >= 0 ? (int64_t)(p + 1) / kRatio : 0;
  if (rank == 0 && tid == 0 && p < 0) flag(a.st, QSA_DEV_BAD_POS);
  if (nb > a.ld) {
    if (rank == 0 && tid == 0) flag(a.st, QSA_DEV_SCORES_LD);
    nb = a.ld;
  }
  const int K = a.K;
  int32_t* out = a.sel + (size_t)q * K;
  // uniform early exits (every CTA of the cluster takes the same branch, before any cluster barrier)
  if (K == 0) {
    if (rank == 0 && tid == 0) a.count[q] = 0;
    return;
  }
  if (nb <= K) {  // every visible block is kept
    if (rank == 0) {
      for (int i = tid; i < K; i += kCThreads) out[i] = i < nb ? i : -1;
      if (tid == 0) a.count[q] = (int32_t)nb;
    }
    return;
  }
  const int n = (int)nb;
  const float* s = a.scores + (size_t)q * a.ld;
  if (n > kMaxFast) {  // selection written by topk_long_kernel, launched after this one
    if (rank == 0 && tid == 0) a.count[q] = K;
    return;
  }
  if (rank == 0 && tid == 0) a.count[q] = K;
  // ---- slice of this CTA: [lo, hi)
  const int per_cta = (n + kCluster - 1) / kCluster;
  const int lo = min(n, rank * per_cta), hi = min(n, lo + per_cta);
  const int m = hi - lo;
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  for (int i0 = tid; i0 < m; i0 += kCThreads * kUnroll) {  // kUnroll independent loads in flight
    uint32_t kv[kUnroll];
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i = i0 + u * kCThreads;
      kv[u] = i < m ? float_key(__ldg(s + lo + i)) : 0u;
    }
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const int i = i0 + u * kCThreads;
      if (i < m) {
        keys[i] = kv[u];
        kmin = min(kmin, kv[u]);
        kmax = max(kmax, kv[u]);
      }
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    wsum[warp] = kmin;
    hist[warp] = kmax;
  }
  __syncthreads();
  if (tid == 0) {
    uint32_t mn = 0xffffffffu, mx = 0u;
    for (int w = 0; w < kCWarps; ++w) {
      mn = min(mn, wsum[w]);
      mx = max(mx, hist[w]);
    }
    pub[0] = mn;
    pub[1] = mx;
  }
  cluster.sync();
  kmin = 0xffffffffu;
  kmax = 0u;
  for (int r = 0; r < kCluster; ++r) {
    const uint32_t* rp = cluster.map_shared_rank(pub, r);
    kmin = min(kmin, rp[0]);
    kmax = max(kmax, rp[1]);
  }
  // ---- radix select over the bits where the keys differ
  uint32_t prefix = kmin, remaining = (uint32_t)K;
  int hb = kmin == kmax ? -1 : 31 - __clz(kmin ^ kmax);
  if (hb >= 0) prefix &= (hb >= 31) ? 0u : ~((2u << hb) - 1u);
  while (hb >= 0) {
    const int wlo = hb >= kWin - 1 ? hb - (kWin - 1) : 0;
    const uint32_t nbins = 1u << (hb - wlo + 1);
    const uint32_t hmask = (hb >= 31) ? 0u : ~((2u << hb) - 1u);
    for (int i = tid; i < (int)nbins; i += kCThreads) hist[i] = 0;
    __syncthreads();
    for (int i0 = tid; i0 < ((m + 31) & ~31); i0 += kCThreads) {
      const bool live0 = i0 < m;
      const uint32_t key = live0 ? keys[i0] : 0u;
      hist_add(hist, (key >> wlo) & (nbins - 1), live0 && (key & hmask) == (prefix & hmask));
    }
    cluster.sync();  // every slice histogram complete
    // reduce-scatter + all-gather: this CTA sums bins [rank * nbins / 8, ...) over
    // the 8 slices and writes the sums into every CTA's merged histogram
    {
      const int span = (int)nbins / kCluster > 0 ? (int)nbins / kCluster : 1;
      const int b0 = rank * span;
      for (int bin = b0 + tid; bin < min((int)nbins, b0 + span); bin += kCThreads) {
        uint32_t v[kCluster];
#pragma unroll
        for (int r = 0; r < kCluster; ++r) v[r] = cluster.map_shared_rank(hist, r)[bin];  // independent loads
        uint32_t sum = 0;
#pragma unroll
        for (int r = 0; r < kCluster; ++r) sum += v[r];
#pragma unroll
        for (int r = 0; r < kCluster; ++r) cluster.map_shared_rank(merged, r)[bin] = sum;
      }
      if ((int)nbins < kCluster) {  // tiny windows: rank 0 alone
        if (rank == 0)
          for (int bin = tid; bin < (int)nbins; bin += kCThreads) {
            uint32_t sum = 0;
            for (int r = 0; r < kCluster; ++r) sum += cluster.map_shared_rank(hist, r)[bin];
            for (int r = 0; r < kCluster; ++r) cluster.map_shared_rank(merged, r)[bin] = sum;
          }
      }
    }
    cluster.sync();  // merged histogram complete everywhere; slice histograms free
    uint32_t above;
    const int b = cluster_find_bin(merged, (int)nbins, remaining, wsum, &s_bin, &s_above, &above);
    prefix |= (uint32_t)b << wlo;
    remaining -= above;
    hb = wlo - 1;
  }
  const uint32_t T = prefix;          // the K-th largest key
  const uint32_t need_eq = remaining;  // keys equal to T to keep, lowest index first
  // ---- ordered output.  Per 32-key word: counts of keys > T and == T (ballots)
  const int words = (m + 31) >> 5;
  const uint32_t lt = (1u << lane) - 1u;
  for (int w = warp; w < words; w += kCWarps) {
    const int i = (w << 5) + lane;
    const uint32_t k = i < m ? keys[i] : 0u;
    const uint32_t gt = __ballot_sync(0xffffffffu, i < m && k > T);
    const uint32_t eq = __ballot_sync(0xffffffffu, i < m && k == T);
    if (lane == 0) {
      wgt_cnt[w] = __popc(gt);
      weq_cnt[w] = __popc(eq);
    }
  }
  __syncthreads();
  // slice totals, published for the higher-ranked CTAs
  uint32_t g_loc = tid < words ? wgt_cnt[tid] : 0u, e_loc = tid < words ? weq_cnt[tid] : 0u;
  uint32_t e_pre;
  const uint32_t e_tot = block_exclusive(e_loc, wsum, &e_pre);
  uint32_t g_pre;
  const uint32_t g_tot = block_exclusive(g_loc, wsum, &g_pre);
  if (tid == 0) {
    pub[2] = g_tot;
    pub[3] = e_tot;
  }
  cluster.sync();
  uint32_t eq_before = 0, sel_before = 0;
  for (int r = 0; r < rank; ++r) {
    const uint32_t* rp = cluster.map_shared_rank(pub, r);
    const uint32_t take_eq = need_eq > eq_before ? min(need_eq - eq_before, rp[3]) : 0u;
    sel_before += rp[2] + take_eq;
    eq_before += rp[3];
  }
  cluster.sync();  // remote reads of pub done before any CTA exits
  // per word: ties before it (index order), keys it keeps, and its first output slot
  uint32_t eqb = eq_before + e_pre;
  const uint32_t take_w = tid < words ? (need_eq > eqb ? min(need_eq - eqb, e_loc) : 0u) + g_loc : 0u;
  uint32_t sel_pre;
  block_exclusive(take_w, wsum, &sel_pre);
  if (tid < words) {
    weq_cnt[tid] = eqb;                    // ties before this word
    wgt_cnt[tid] = sel_before + sel_pre;   // first output slot of this word
  }
  __syncthreads();
  for (int w = warp; w < words; w += kCWarps) {
    const int i = (w << 5) + lane;
    const uint32_t k = i < m ? keys[i] : 0u;
    const bool is_gt = i < m && k > T;
    const bool is_eq = i < m && k == T;
    const uint32_t eq = __ballot_sync(0xffffffffu, is_eq);
    const bool take = is_gt || (is_eq && weq_cnt[w] + __popc(eq & lt) < need_eq);
    const uint32_t tk = __ballot_sync(0xffffffffu, take);
    if (take) out[wgt_cnt[w] + __popc(tk & lt)] = lo + i;
  }
}

// Rows longer than the cluster path holds: one CTA per such query.
__global__ void __launch_bounds__(kThreads) topk_long_kernel(TopkArgs a) {
  __shared__ uint32_t hist[4096];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t wgt[kWarps], weq[kWarps];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;
  const int q = blockIdx.x;
  const int p = a.q_pos[q];
  int64_t nb = p >= 0 ? (int64_t)(p + 1) / kRatio : 0;
  if (nb > a.ld) nb = a.ld;
  if (a.K == 0 || nb <= kMaxFast) return;  // handled by the cluster kernel
  topk_general(a.scores + (size_t)q * a.ld, (int)nb, a.K, a.sel + (size_t)q * a.K, hist, wsum, wgt, weq, &s_bin,
               &s_above);
}

}  // namespace

extern "C" int qsa_topk_blocks(const float* scores, int64_t scores_ld, const int32_t* q_pos, int32_t nq, int32_t k,
                               int32_t* sel, int32_t* count, int32_t* dev_status, void* stream) {
  if (nq < 0 || k < 0 || k > QSA_MAX_TOPK || scores_ld < 1) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!scores || !q_pos || !count || (k > 0 && !sel)) return QSA_ERR_INVALID_ARG;
  TopkArgs a{scores, scores_ld, q_pos, k, kMaxFast, sel, count, dev_status};
  const cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSliceCap * 4) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  topk_kernel<<<(unsigned)((int64_t)nq * kCluster), kCThreads, kSliceCap * 4, st>>>(a);
  int rc = qsa_host::launch_status();
  if (rc != QSA_OK) return rc;
  if (scores_ld > kMaxFast) topk_long_kernel<<<(unsigned)nq, kThreads, 0, st>>>(a);
  return qsa_host::launch_status();
}
