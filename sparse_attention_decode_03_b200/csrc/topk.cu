// qsa_topk_blocks: per query, the best min(K, nb_q) blocks under (score desc,
// index asc), emitted sorted by block index ascending.
//
// Source: [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section
// "Wat de pull request daadwerkelijk verandert" (keep the best 512 blocks);
// the tie-break (lower index first) and ascending output order are the fixed
// readings.
//
// One CTA per query, order-preserving uint32 keys of the fp32 scores.
// Common path (rows up to 65,536 blocks): ONE vectorised read of the scores
// (L2-resident), then shared memory.
//   1. read the row once: keep every key's high 16 bits in shared memory and
//      the row's min / max key;
//   2. radix select with adaptive 11-bit windows starting at the highest bit
//      where the keys differ (scores share their top exponent bits, so fixed
//      top-bit bins would all land in a couple of bins): each window is a
//      shared-memory histogram of the keys that still match the prefix; bits
//      below 16 are fetched from L2 for those keys only.  The result is the
//      exact K-th largest key T;
//   3. a word-wise ballot pass writes a bitmap of keys > T and counts keys == T
//      per 32 indices; a block scan ranks the ties in index order and the
//      lowest-index ones are added;
//   4. the K indices are emitted in ascending order from the bitmap.
// Longer rows take the general path: three radix passes over the scores
// (12 + 12 + 8 bits) and an ordered compaction with warp ballots.
// Integer counters only: the result does not depend on atomic order.
#include "qsa_common.cuh"

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

constexpr int kMaxFast = 65536;          // blocks per query on the shared-memory path
constexpr int kUnroll = 8;
constexpr int kWin = 11;                 // radix window bits

__device__ __forceinline__ void load_keys(const float* s, int i0, int n, uint32_t (&key)[kUnroll]) {
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const int i = i0 + u * kThreads;
    key[u] = i < n ? float_key(s[i]) : 0u;
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

// In-place exclusive scan of v[0..m) (m <= 4 * kThreads), block-wide.
__device__ void block_exclusive_scan(uint32_t* v, int m, uint32_t* wsum) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (m + kThreads - 1) / kThreads;
  const int lo = tid * per;
  uint32_t loc[4] = {0, 0, 0, 0};
  uint32_t sum = 0;
  for (int k = 0; k < per; ++k)
    if (lo + k < m) {
      loc[k] = v[lo + k];
      sum += loc[k];
    }
  uint32_t inc = sum;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t x = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += x;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  uint32_t base = inc - sum;
  for (int w = 0; w < warp; ++w) base += wsum[w];
  for (int k = 0; k < per; ++k)
    if (lo + k < m) {
      v[lo + k] = base;
      base += loc[k];
    }
  __syncthreads();
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

__global__ void __launch_bounds__(kThreads) topk_kernel(TopkArgs a) {
  extern __shared__ __align__(16) uint8_t smem[];
  __shared__ uint32_t hist[4096];
  __shared__ uint32_t wsum[kWarps];
  __shared__ uint32_t wgt[kWarps], weq[kWarps];
  __shared__ uint32_t wmin[kWarps], wmax[kWarps];
  __shared__ int s_bin;
  __shared__ uint32_t s_above;

  const int q = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt = (1u << lane) - 1u;
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
  if (tid == 0) a.count[q] = K;
  if (n > a.fast_cap) {
    topk_general(s, n, K, out, hist, wsum, wgt, weq, &s_bin, &s_above);
    return;
  }
  const int words = (n + 31) >> 5;
  uint16_t* hi16 = reinterpret_cast<uint16_t*>(smem);                             // [fast_cap]
  uint32_t* bitmap = reinterpret_cast<uint32_t*>(smem + (size_t)a.fast_cap * 2);  // [fast_cap / 32]
  uint32_t* wcnt = bitmap + a.fast_cap / 32;                                       // [fast_cap / 32]

  // ---- 1. one read of the row: high halves to shared memory, min / max key
  uint32_t kmin = 0xffffffffu, kmax = 0u;
  if ((reinterpret_cast<uintptr_t>(s) & 15u) == 0) {
    const int n4 = n >> 2;
    const float4* s4 = reinterpret_cast<const float4*>(s);
    constexpr int kU4 = 4;
    for (int j0 = tid; j0 < n4; j0 += kThreads * kU4) {
      float4 v[kU4];
#pragma unroll
      for (int u = 0; u < kU4; ++u)
        if (j0 + u * kThreads < n4) v[u] = __ldg(s4 + j0 + u * kThreads);
#pragma unroll
      for (int u = 0; u < kU4; ++u) {
        const int j = j0 + u * kThreads;
        if (j >= n4) continue;
        const uint32_t k0 = float_key(v[u].x), k1 = float_key(v[u].y), k2 = float_key(v[u].z), k3 = float_key(v[u].w);
        kmin = min(kmin, min(min(k0, k1), min(k2, k3)));
        kmax = max(kmax, max(max(k0, k1), max(k2, k3)));
        uint2 h;
        h.x = (k0 >> 16) | (k1 & 0xffff0000u);
        h.y = (k2 >> 16) | (k3 & 0xffff0000u);
        *reinterpret_cast<uint2*>(hi16 + 4 * j) = h;
      }
    }
    for (int i = (n4 << 2) + tid; i < n; i += kThreads) {
      const uint32_t k = float_key(s[i]);
      kmin = min(kmin, k);
      kmax = max(kmax, k);
      hi16[i] = (uint16_t)(k >> 16);
    }
  } else {
    for (int i = tid; i < n; i += kThreads) {
      const uint32_t k = float_key(s[i]);
      kmin = min(kmin, k);
      kmax = max(kmax, k);
      hi16[i] = (uint16_t)(k >> 16);
    }
  }
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  if (lane == 0) {
    wmin[warp] = kmin;
    wmax[warp] = kmax;
  }
  __syncthreads();
  kmin = 0xffffffffu;
  kmax = 0u;
  for (int w = 0; w < kWarps; ++w) {
    kmin = min(kmin, wmin[w]);
    kmax = max(kmax, wmax[w]);
  }
  // ---- 2. radix select over the bits where the keys differ
  uint32_t prefix = kmin, remaining = (uint32_t)K;
  int hb = kmin == kmax ? -1 : 31 - __clz(kmin ^ kmax);  // highest differing bit
  if (hb >= 0) prefix &= ~((2u << hb) - 1u);               // (2u << 31) wraps to 0: all bits cleared
  while (hb >= 0) {
    const int lo = hb >= kWin - 1 ? hb - (kWin - 1) : 0;
    const uint32_t nbins = 1u << (hb - lo + 1);
    const uint32_t hmask = (hb >= 31) ? 0u : ~((2u << hb) - 1u);  // bits above the window
    for (int i = tid; i < (int)nbins; i += kThreads) hist[i] = 0;
    __syncthreads();
    if (lo >= 16) {  // window inside the high halves: shared memory only
      for (int i0 = tid; i0 < ((n + 31) & ~31); i0 += kThreads) {
        const bool live0 = i0 < n;
        const uint32_t key = live0 ? ((uint32_t)hi16[i0] << 16) : 0u;
        const bool live = live0 && (key & hmask) == (prefix & hmask);
        hist_add(hist, (key >> lo) & (nbins - 1), live);
      }
    } else {  // low bits: fetch the full key of the keys still matching the prefix
      const uint32_t hm16 = hmask >> 16, hp16 = (prefix & hmask) >> 16;
      for (int i0 = tid; i0 < ((n + 31) & ~31); i0 += kThreads) {
        const bool live0 = i0 < n && ((uint32_t)hi16[min(i0, n - 1)] & hm16) == hp16;
        const uint32_t key = live0 ? float_key(s[i0]) : 0u;
        const bool live = live0 && (key & hmask) == (prefix & hmask);
        hist_add(hist, (key >> lo) & (nbins - 1), live);
      }
    }
    __syncthreads();
    find_bin(hist, (int)nbins, remaining, wsum, &s_bin, &s_above);
    prefix |= (uint32_t)s_bin << lo;
    remaining -= s_above;
    hb = lo - 1;
  }
  const uint32_t T = prefix;          // the K-th largest key
  const uint32_t need_eq = remaining;  // keys equal to T to keep, lowest index first
  const uint32_t T16 = T >> 16;
  // ---- 3. bitmap of keys > T, per-word counts of keys == T
  for (int w = warp; w < words; w += kWarps) {
    const int i = (w << 5) + lane;
    const bool live = i < n;
    const uint32_t h = live ? hi16[i] : 0u;
    const bool tie16 = live && h == T16;
    const uint32_t key = tie16 ? float_key(s[i]) : 0u;
    const uint32_t gt = __ballot_sync(0xffffffffu, live && (h > T16 || (tie16 && key > T)));
    const uint32_t eq = __ballot_sync(0xffffffffu, tie16 && key == T);
    if (lane == 0) {
      bitmap[w] = gt;
      wcnt[w] = __popc(eq);
    }
  }
  __syncthreads();
  block_exclusive_scan(wcnt, words, wsum);
  for (int w = warp; w < words; w += kWarps) {
    const int i = (w << 5) + lane;
    const bool tie16 = i < n && hi16[i] == T16;
    const bool e = tie16 && float_key(s[i]) == T;
    const uint32_t eq = __ballot_sync(0xffffffffu, e);
    const bool take = e && wcnt[w] + __popc(eq & lt) < need_eq;
    const uint32_t tk = __ballot_sync(0xffffffffu, take);
    if (lane == 0 && tk) bitmap[w] |= tk;
  }
  __syncthreads();
  // ---- 4. ascending emission from the bitmap: per-thread word runs + block scan
  const int per = (words + kThreads - 1) / kThreads;
  const int w0 = tid * per;
  uint32_t cnt = 0;
  for (int w = w0; w < min(words, w0 + per); ++w) cnt += __popc(bitmap[w]);
  uint32_t inc = cnt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t v = __shfl_up_sync(0xffffffffu, inc, d);
    if (lane >= d) inc += v;
  }
  if (lane == 31) wsum[warp] = inc;
  __syncthreads();
  uint32_t base = inc - cnt;
  for (int w = 0; w < warp; ++w) base += wsum[w];
  for (int w = w0; w < min(words, w0 + per); ++w) {
    uint32_t bits = bitmap[w];
    while (bits) {
      const int b = __ffs(bits) - 1;
      bits &= bits - 1;
      out[base++] = w * 32 + b;
    }
  }
}

}  // namespace

extern "C" int qsa_topk_blocks(const float* scores, int64_t scores_ld, const int32_t* q_pos, int32_t nq, int32_t k,
                               int32_t* sel, int32_t* count, int32_t* dev_status, void* stream) {
  if (nq < 0 || k < 0 || k > QSA_MAX_TOPK || scores_ld < 1) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!scores || !q_pos || !count || (k > 0 && !sel)) return QSA_ERR_INVALID_ARG;
  // shared-memory path sized for this call's rows: 2 B of key prefix + 8 B per 32 blocks
  const int32_t fast_cap = (int32_t)((scores_ld < kMaxFast ? (scores_ld + 1023) / 1024 * 1024 : kMaxFast));
  TopkArgs a{scores, scores_ld, q_pos, k, fast_cap, sel, count, dev_status};
  const size_t smem = (size_t)fast_cap * 2 + (size_t)fast_cap / 32 * 4 * 2;
  if (cudaFuncSetAttribute(topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  topk_kernel<<<(unsigned)nq, kThreads, smem, static_cast<cudaStream_t>(stream)>>>(a);
  return qsa_host::launch_status();
}
