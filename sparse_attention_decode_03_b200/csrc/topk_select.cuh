// Block-wide pieces of the deterministic top-K block selection, shared by
// the standalone selection kernel (topk.cu) and the fused indexer + selection
// kernel (index_topk.cu).  Keys are the order-preserving uint32 images of the
// fp32 scores (float_key); every count is an integer, so no result depends on
// the order of shared-memory atomics.
#pragma once
#include "qsa_common.cuh"

namespace qsa {

// Block-wide: find the bin b (scanning from the top) with
// sum_{i > b} hist[i] < remaining <= sum_{i >= b} hist[i].
template <int kThreads>
__device__ void find_bin(const uint32_t* hist, int nbins, uint32_t remaining, uint32_t* wsum, int* out_bin,
                         uint32_t* out_above) {
  constexpr int kWarps = kThreads / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = nbins >= kThreads ? nbins / kThreads : 1;  // a power of two
  const int lo = tid * per;
  uint32_t local = 0;
  if (lo < nbins)  // lane-rotated order, as in top_bin
    for (int i = 0; i < per; ++i) local += hist[lo + ((i + lane) & (per - 1))];
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
  if (lo < nbins && cum < remaining && remaining <= cum + local) {
    for (int i = per - 1; i >= 0; --i) {
      const uint32_t h = hist[lo + i];
      if (cum < remaining && remaining <= cum + h) {
        *out_bin = lo + i;
        *out_above = cum;
        break;
      }
      cum += h;
    }
  }
  __syncthreads();
}

constexpr int kUnroll = 8;

template <int kThreads>
__device__ __forceinline__ void load_keys(const float* s, int i0, int n, uint32_t (&key)[kUnroll]) {
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const int i = i0 + u * kThreads;
    key[u] = i < n ? float_key(s[i]) : 0u;
  }
}

// General path: exact K-th key by three radix passes, then ordered compaction.
template <int kThreads>
__device__ void topk_general(const float* s, int n, int K, int32_t* out, uint32_t* hist, uint32_t* wsum,
                             uint32_t* wgt, uint32_t* weq, int* s_bin, uint32_t* s_above) {
  constexpr int kWarps = kThreads / 32;
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
      load_keys<kThreads>(s, i0, n, key);
#pragma unroll
      for (int u = 0; u < kUnroll; ++u)
        if (i0 + u * kThreads < n && (key[u] & mask) == prefix) atomicAdd(&hist[(key[u] >> sh) & (nbins - 1)], 1u);
    }
    __syncthreads();
    find_bin<kThreads>(hist, nbins, remaining, wsum, s_bin, s_above);
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

constexpr int kSample = 1024;   // keys sampled for the threshold (one per thread)
constexpr int kCap = 256;       // candidates one warp's list holds
constexpr int kWin = 12;        // radix window bits
constexpr int kWinBins = 1 << kWin;

template <int kWarps, int kListCap = kCap>
struct TopkSmem {
  static constexpr int kList = kListCap;
  uint32_t ckey[kWarps][kListCap];  // candidate keys, per warp, in index order
  uint32_t cidx[kWarps][kListCap];  // their block indices
  uint32_t hist[kWinBins];
  uint32_t wcnt[kWarps];        // candidates per warp (kListCap + 1: overflow)
  uint32_t wgt[kWarps], weq[kWarps], wslot[kWarps], weqb[kWarps];
  uint32_t wsum[kWarps];
  uint32_t red[2 * kWarps];
  int bin;
  uint32_t above;
  uint32_t nsmall;              // keys gathered from a small final bin
  uint32_t skey[32], sidx[32];  // those keys and their block indices
  uint32_t scut, sneed;         // the exact cut key, and how many keys equal to it are kept
};

// Add 1 to hist[bin] for every live lane.  Plain shared-memory atomics: the
// hardware serialises lanes that hit the same bin, which costs less than
// aggregating them with __match_any_sync first (measured on B200).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool live) {
  if (live) atomicAdd(&hist[bin], 1u);
}

// Block-wide min and max of one value per thread.
template <int kThreads>
__device__ __forceinline__ void block_minmax(uint32_t& mn, uint32_t& mx, uint32_t* red) {
  constexpr int kWarps = kThreads / 32;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (lane == 0) {
    red[warp] = mn;
    red[kWarps + warp] = mx;
  }
  __syncthreads();
  mn = __reduce_min_sync(0xffffffffu, lane < kWarps ? red[lane] : 0xffffffffu);
  mx = __reduce_max_sync(0xffffffffu, lane < kWarps ? red[kWarps + lane] : 0u);
  __syncthreads();
}

// The bin b of hist[0..nbins) (counting from the top) with
// sum_{>b} < remaining <= sum_{>=b}; *above = sum_{>b}.  Same result in every thread.
template <int kThreads, class Smem>
__device__ int top_bin(const uint32_t* hist, int nbins, uint32_t remaining, Smem& S,
                       uint32_t* above) {
  constexpr int kWarps = kThreads / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int per = (nbins + kThreads - 1) / kThreads;  // a power of two, as nbins and kThreads are
  const int b0 = tid * per;
  uint32_t local = 0;
  // Each thread sums its per consecutive bins in a lane-rotated order: in the
  // plain order up to min(per, 32) lanes of a warp would hit one bank at once.
  for (int jj = 0; jj < per; ++jj) {
    const int j = (jj + lane) & (per - 1);
    if (b0 + j < nbins) local += hist[b0 + j];
  }
  uint32_t suf = local;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, suf, d);
    if (lane + d < 32) suf += v;
  }
  if (lane == 0) S.wsum[warp] = suf;
  __syncthreads();
  // sum of the totals of the warps above mine: a suffix scan across lanes
  const uint32_t wt = lane < kWarps ? S.wsum[lane] : 0u;
  uint32_t wsuf = wt;
#pragma unroll
  for (int d = 1; d < 32; d <<= 1) {
    const uint32_t v = __shfl_down_sync(0xffffffffu, wsuf, d);
    if (lane + d < 32) wsuf += v;
  }
  uint32_t cum = suf - local + (__shfl_sync(0xffffffffu, wsuf, warp) - __shfl_sync(0xffffffffu, wt, warp));
  if (cum < remaining && remaining <= cum + local) {  // the one thread whose bins hold the target
    for (int j = per - 1; j >= 0; --j) {
      if (b0 + j >= nbins) continue;
      const uint32_t h = hist[b0 + j];
      if (cum < remaining && remaining <= cum + h) {
        S.bin = b0 + j;
        S.above = cum;
        break;
      }
      cum += h;
    }
  }
  __syncthreads();
  const int b = S.bin;
  *above = S.above;
  __syncthreads();  // S.bin / S.above / hist read everywhere before reuse
  return b;
}

// Append lane's flagged keys (f0..f3 of idx0..idx0+3) to this warp's list, in
// index order.  A lane flags 0..4 keys, so the exclusive prefix of the counts
// over the lanes comes from three ballots (one per bit of the count) and
// popcounts, with no chain of shuffles.
template <class Smem, class KeyAt>
__device__ __forceinline__ void append4_by(Smem& S, int warp, uint32_t& cnt, KeyAt key_at, int idx0,
                                           const bool (&f)[4]) {
  const int lane = threadIdx.x & 31;
  const uint32_t nc = (uint32_t)f[0] + f[1] + f[2] + f[3];
  const uint32_t b0 = __ballot_sync(0xffffffffu, nc & 1u);
  const uint32_t b1 = __ballot_sync(0xffffffffu, nc & 2u);
  const uint32_t b2 = __ballot_sync(0xffffffffu, nc & 4u);
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t pos = cnt + __popc(b0 & lt) + 2u * __popc(b1 & lt) + 4u * __popc(b2 & lt);
#pragma unroll
  for (int c = 0; c < 4; ++c)
    if (f[c]) {
      if (pos < Smem::kList) {
        S.ckey[warp][pos] = key_at(c);  // computed for flagged keys only
        S.cidx[warp][pos] = (uint32_t)(idx0 + c);
      }
      ++pos;
    }
  cnt += __popc(b0) + 2u * __popc(b1) + 4u * __popc(b2);
}

// The same, for keys already held as keys.
template <class Smem>
__device__ __forceinline__ void append4(Smem& S, int warp, uint32_t& cnt, const uint32_t (&k)[4], int idx0,
                                        const bool (&f)[4]) {
  append4_by(S, warp, cnt, [&](int c) { return k[c]; }, idx0, f);
}

// Step 1: a threshold T0 such that about r >= K keys of the n-key row are
// >= T0, from ns keys sampled at a regular stride (thread tid holds samples
// u * kThreads + tid in ks[u]).  The samples are histogrammed over a kWin-bit
// window below their highest differing bit; T0 is the lower edge of the bin
// where the count from the top reaches r = K * ns / n plus three standard
// deviations.  Same result in every thread.
template <int kThreads, int kSPer, class Smem>
__device__ uint32_t sample_threshold(const uint32_t (&ks)[kSPer], int ns, int n, int K, Smem& S) {
  const int tid = threadIdx.x;
  uint32_t smin = 0xffffffffu, smax = 0u;
#pragma unroll
  for (int u = 0; u < kSPer; ++u)
    if (u * kThreads + tid < ns) {
      smin = min(smin, ks[u]);
      smax = max(smax, ks[u]);
    }
  block_minmax<kThreads>(smin, smax, S.red);
  uint32_t r;
  if (ns == n) {
    r = (uint32_t)K;
  } else {
    const float e = (float)K * (float)ns / (float)n;
    r = (uint32_t)min((float)ns, ceilf(e + 3.f * sqrtf(e) + 2.f));
  }
  uint32_t T0 = smin;
  if (smin != smax) {
    const int hb = 31 - __clz(smin ^ smax);
    const int wlo = hb >= kWin - 1 ? hb - (kWin - 1) : 0;
    const int nbins = 1 << (hb - wlo + 1);
    const uint32_t mhi = hb >= 31 ? 0u : ~((2u << hb) - 1u);
    for (int i = tid; i < nbins; i += kThreads) S.hist[i] = 0;
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kSPer; ++u) hist_add(S.hist, (ks[u] >> wlo) & (uint32_t)(nbins - 1), u * kThreads + tid < ns);
    __syncthreads();
    uint32_t above;
    const int b = top_bin<kThreads>(S.hist, nbins, r, S, &above);
    T0 = (smin & mhi) | ((uint32_t)b << wlo);
  }
  return T0;
}

// The end of the exact select when the bin that holds the K-th key has at most
// 32 keys: they are gathered (warp ballots, any order) and one warp ranks them
// under (key desc, index asc), a total order, so the lane whose rank is
// remaining - 1 holds the exact cut key whatever the gathering order.  On
// return T is that key, M all ones and remaining the number of keys equal to
// it that are kept (lowest index first).  Replaces the radix passes over the
// lower bits.
template <class Smem>
__device__ void small_bin_cut(Smem& S, const uint32_t* ck, const uint32_t* ci, uint32_t mycnt, uint32_t mr,
                              uint32_t& T, uint32_t& M, uint32_t& remaining) {
  const int tid = threadIdx.x, lane = tid & 31;
  for (uint32_t j = lane; j < mr; j += 32) {
    const bool in = j < mycnt && (ck[j] & M) == T;
    const uint32_t b = __ballot_sync(0xffffffffu, in);
    uint32_t base = 0;
    if (lane == 0 && b) base = atomicAdd(&S.nsmall, (uint32_t)__popc(b));
    base = __shfl_sync(0xffffffffu, base, 0);
    if (in) {
      const uint32_t at = base + __popc(b & ((1u << lane) - 1u));
      S.skey[at] = ck[j];
      S.sidx[at] = ci[j];
    }
  }
  __syncthreads();
  if (tid < 32) {
    const uint32_t n = S.nsmall;  // the bin's count, at most 32
    const uint32_t key = lane < (int)n ? S.skey[lane] : 0u;
    const uint32_t idx = lane < (int)n ? S.sidx[lane] : 0xffffffffu;
    uint32_t rank = 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const uint32_t kj = __shfl_sync(0xffffffffu, key, j), ij = __shfl_sync(0xffffffffu, idx, j);
      rank += (j < (int)n && (kj > key || (kj == key && ij < idx))) ? 1u : 0u;
    }
    const uint32_t cut = __ballot_sync(0xffffffffu, lane < (int)n && rank == remaining - 1u);
    const uint32_t Tk = __shfl_sync(0xffffffffu, key, __ffs(cut) - 1);
    const uint32_t above = __popc(__ballot_sync(0xffffffffu, lane < (int)n && key > Tk));
    if (lane == 0) {
      S.scut = Tk;
      S.sneed = remaining - above;
    }
  }
  __syncthreads();
  T = S.scut;
  M = 0xffffffffu;
  remaining = S.sneed;
}

// Steps 3 and 4: the exact top K among the candidates in the per-warp lists
// S.ckey / S.cidx (S.wcnt[w] entries in list w; each list in block-index
// order and the lists in index order by warp), written to out[0..K) in index
// order.  Radix passes (kWin-bit windows from the candidates' highest
// differing bit) give a prefix T under a mask M with "every key above T, and
// the first `need` keys equal to T in index order" = the top K.
template <int kThreads, class Smem>
__device__ void select_from_lists(Smem& S, int K, int32_t* out) {
  constexpr int kWarps = kThreads / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t mycnt = S.wcnt[warp];
  const uint32_t* ck = S.ckey[warp];
  const uint32_t* ci = S.cidx[warp];
  const uint32_t mr = (mycnt + 31) & ~31u;
  if (tid == 0) S.nsmall = 0;  // ordered before small_bin_cut by the barriers of block_minmax

  // ---- 3. exact select among the candidates
  uint32_t cmin = 0xffffffffu, cmax = 0u;
  for (uint32_t j = lane; j < mycnt; j += 32) {
    cmin = min(cmin, ck[j]);
    cmax = max(cmax, ck[j]);
  }
  block_minmax<kThreads>(cmin, cmax, S.red);
  uint32_t T = cmin, M = 0xffffffffu, remaining = (uint32_t)K;
  int hb = cmin == cmax ? -1 : 31 - __clz(cmin ^ cmax);
  if (hb >= 0) {
    M = hb >= 31 ? 0u : ~((2u << hb) - 1u);
    T = cmin & M;
  }
  while (hb >= 0) {
    const int wlo = hb >= kWin - 1 ? hb - (kWin - 1) : 0;
    const int nbins = 1 << (hb - wlo + 1);
    for (int i = tid; i < nbins; i += kThreads) S.hist[i] = 0;
    __syncthreads();
    for (uint32_t j = lane; j < mr; j += 32) {
      const uint32_t key = j < mycnt ? ck[j] : 0u;
      hist_add(S.hist, (key >> wlo) & (uint32_t)(nbins - 1), j < mycnt && (key & M) == T);
    }
    __syncthreads();
    uint32_t above;
    const int b = top_bin<kThreads>(S.hist, nbins, remaining, S, &above);
    const uint32_t in_bin = S.hist[b];
    remaining -= above;
    T |= (uint32_t)b << wlo;
    M |= (uint32_t)(nbins - 1) << wlo;
    __syncthreads();
    if (remaining == in_bin) break;  // the whole bin is kept: its order does not matter
    if (in_bin <= 32 && wlo > 0) {   // few keys left: rank them in one warp
      small_bin_cut(S, ck, ci, mycnt, mr, T, M, remaining);
      break;
    }
    hb = wlo - 1;
  }
  const uint32_t need = remaining;  // keys equal to T (under M) to keep, lowest index first

  // ---- 4. ordered output
  const uint32_t lt = (1u << lane) - 1u;
  uint32_t g = 0, e = 0;
  for (uint32_t j = lane; j < mr; j += 32) {
    const uint32_t k = j < mycnt ? ck[j] & M : 0u;
    g += __popc(__ballot_sync(0xffffffffu, j < mycnt && k > T));
    e += __popc(__ballot_sync(0xffffffffu, j < mycnt && k == T));
  }
  if (lane == 0) {
    S.wgt[warp] = g;
    S.weq[warp] = e;
  }
  __syncthreads();
  if (warp == 0) {  // warp totals -> ties before each warp, first output slot of each warp
    const uint32_t ew = lane < kWarps ? S.weq[lane] : 0u, gw = lane < kWarps ? S.wgt[lane] : 0u;
    uint32_t einc = ew;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, einc, d);
      if (lane >= d) einc += x;
    }
    const uint32_t eqb = einc - ew;
    const uint32_t take = gw + (need > eqb ? min(need - eqb, ew) : 0u);
    uint32_t tinc = take;
#pragma unroll
    for (int d = 1; d < 32; d <<= 1) {
      const uint32_t x = __shfl_up_sync(0xffffffffu, tinc, d);
      if (lane >= d) tinc += x;
    }
    if (lane < kWarps) {
      S.weqb[lane] = eqb;
      S.wslot[lane] = tinc - take;
    }
  }
  __syncthreads();
  uint32_t eqb = S.weqb[warp], slot = S.wslot[warp];
  for (uint32_t j = lane; j < mr; j += 32) {
    const uint32_t k = j < mycnt ? ck[j] & M : 0u;
    const bool is_gt = j < mycnt && k > T;
    const bool is_eq = j < mycnt && k == T;
    const uint32_t eqm = __ballot_sync(0xffffffffu, is_eq);
    const bool keep = is_gt || (is_eq && eqb + __popc(eqm & lt) < need);
    const uint32_t kb = __ballot_sync(0xffffffffu, keep);
    if (keep) out[slot + __popc(kb & lt)] = (int32_t)ci[j];
    slot += __popc(kb);
    eqb += __popc(eqm);
  }
}

}  // namespace qsa
