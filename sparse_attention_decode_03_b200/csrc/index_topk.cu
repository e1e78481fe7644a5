// qsa_index_topk: the indexer scores and the top-K block selection of a decode
// step in one kernel.  Same results as qsa_index_scores followed by
// qsa_topk_blocks (identical scores; the selection is exact, so it does not
// depend on how it is reached).
//
// Source: [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section
// "Wat de pull request daadwerkelijk verandert" (the indexer scores every
// micro-block, the best 512 are kept); the ReLU-weighted head sum, the
// tie-break (lower index first) and the ascending output order are the fixed
// readings shared with the two separate calls.
//
// One thread-block cluster of kFC = 8 CTAs per query.  CTA r of the cluster
// owns the r-th of 8 equal runs of the query's side-cache pages (its slice):
//   A. scores: its 8 warps stream the run's 4 KiB pages (index_page.cuh), keep
//      each block's order-preserving score key in shared memory and write the
//      fp32 score to the caller's scores row.  The CTA then stores the keys of
//      the 1024 regularly spaced sample positions that fall in its slice into
//      the sample array of every CTA of the cluster (distributed shared
//      memory; stores, so nobody waits on a remote round trip).
//   cluster barrier 1: every CTA holds all 1024 samples.
//   B. 1. every CTA derives the same threshold T0 from the samples
//         (topk_select.cuh: about K * n / 1024 plus three standard deviations
//         of the keys are >= T0);
//      2. every CTA lists its slice's keys >= T0 per warp, in index order,
//         then stores the CTA's list, in order, into the leader CTA's
//         gather list number r, with its length;
//   cluster barrier 2: the leader (rank 0) holds the whole row's candidates
//      as 8 lists, one per warp, in block-index order; the others leave.
//      3. the leader runs the exact select and the ordered output on them.
//   If the sample misleads (fewer than K candidates, or more than a list
//   holds) the leader runs the general exact path over the scores row the
//   cluster wrote to global memory.
// The cluster barriers are hardware barriers that every CTA reaches on the
// same path: a query's validity, nb and K are the same in all its CTAs.  An
// arrive at the start and its wait before the first remote store make sure
// every CTA of the cluster is running before its shared memory is written;
// no CTA touches a peer's shared memory after barrier 2.
#include "index_page.cuh"
#include "topk_select.cuh"

namespace {

using namespace qsa;

constexpr int kFC = 8;                    // CTAs per query (one cluster)
constexpr int kFThreads = 256;
constexpr int kFWarps = kFThreads / 32;
constexpr int kFLocal = 256;              // candidates one warp of a CTA lists
constexpr int kFList = 512;               // candidates one CTA hands to the leader
constexpr int kFSPer = kSample / kFThreads;
static_assert(kFWarps == kFC, "the leader's warp w selects from the list of CTA w");

using FSmem = TopkSmem<kFWarps, kFList>;  // leader: gather lists (ckey/cidx/wcnt) + selection scratch

struct LocalLists {
  static constexpr int kList = kFLocal;
  uint32_t ckey[kFWarps][kFLocal];
  uint32_t cidx[kFWarps][kFLocal];
};

struct FusedArgs {
  const __nv_bfloat16* kc;
  const int32_t* bt;
  int32_t num_pages, max_seqs, mpps;
  const __nv_bfloat16* q_idx;
  const float* w;
  const int32_t* q_seq;
  const int32_t* q_pos;
  float* scores;
  int64_t ld;
  int32_t K;
  int32_t* sel;
  int32_t* count;
  int32_t slice_pages;  // pages per CTA the shared memory holds
  int32_t* st;
};

// dynamic shared memory: FSmem | LocalLists | samples | page ids [slice_pages] | keys [slice_pages * 16]
constexpr size_t kFOffLocal = (sizeof(FSmem) + 15) & ~(size_t)15;
constexpr size_t kFOffSamp = kFOffLocal + sizeof(LocalLists);
constexpr size_t kFOffIds = kFOffSamp + kSample * 4;
static_assert(kFOffIds % 16 == 0, "16-byte aligned page ids and keys");

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// All threads of all CTAs of the cluster; orders shared and global memory
// accesses before it (release) against those after it (acquire).
__device__ __forceinline__ void cluster_barrier() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.aligned;" ::: "memory"); }

// 32-bit store into the shared memory of CTA `rank` of this cluster, at the
// offset `p` has in this CTA.
__device__ __forceinline__ void st_cluster(void* p, uint32_t rank, uint32_t v) {
  uint32_t remote;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(remote) : "r"(smem_u32(p)), "r"(rank));
  asm volatile("st.shared::cluster.u32 [%0], %1;" ::"r"(remote), "r"(v) : "memory");
}

// Bulk prefetch of `bytes` (a multiple of 16, 16-byte aligned) into L2.
__device__ __forceinline__ void l2_prefetch_bulk(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__global__ void __launch_bounds__(kFThreads, 2) index_topk_kernel(FusedArgs a) {
  extern __shared__ __align__(16) uint8_t smem_raw[];
  FSmem& S = *reinterpret_cast<FSmem*>(smem_raw);
  LocalLists& LL = *reinterpret_cast<LocalLists*>(smem_raw + kFOffLocal);
  uint32_t* samp = reinterpret_cast<uint32_t*>(smem_raw + kFOffSamp);
  int32_t* ids = reinterpret_cast<int32_t*>(smem_raw + kFOffIds);
  uint32_t* keys = reinterpret_cast<uint32_t*>(ids + a.slice_pages);  // slice_pages % 4 == 0: 16-B aligned

  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int q = blockIdx.x / kFC;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int K = a.K;
  int32_t* out = a.sel + (size_t)q * K;

  // The query's sequence, position, indexer query and page ids are inputs that
  // no kernel of this library writes: they are loaded before waiting for the
  // preceding kernel, so only the side-cache pages are read after the wait.
  const int seq = a.q_seq[q];
  const int p = a.q_pos[q];
  const bool bad = seq < 0 || seq >= a.max_seqs || p < 0 || (int64_t)p >= (int64_t)a.mpps * kPage;
  int64_t nb = bad ? 0 : (p + 1) / kRatio;
  const bool ld_over = nb > a.ld;
  if (ld_over) nb = a.ld;
  const int n = (int)nb;
  const int npg = (n + kBlocksPerPage - 1) / kBlocksPerPage;
  const int pps = (npg + kFC - 1) / kFC;  // pages per CTA (<= slice_pages: the host sizes the slice)
  const int slice = pps * kBlocksPerPage;  // blocks per CTA
  const int pg_lo = (int)rank * pps;
  const int np_cta = max(0, min(npg, pg_lo + pps) - pg_lo);
  const int b_lo = pg_lo * kBlocksPerPage;
  const int m = max(0, min(n, b_lo + slice) - b_lo);  // blocks (keys) in this CTA's slice
  const bool selecting = K > 0 && n > K;             // cluster-uniform
  IdxQuery Q{};
  if (!bad) {
    for (int i = tid; i < np_cta; i += kFThreads) ids[i] = a.bt[(int64_t)seq * a.mpps + pg_lo + i];
    if (np_cta > 0) Q = load_idx_query(a.q_idx, a.w, q);
  }
  pdl_wait_previous();
  if (bad) {
    // the whole cluster leaves here, before any cluster barrier operation
    if (leader) {
      if (tid == 0) {
        flag(a.st, (seq < 0 || seq >= a.max_seqs) ? QSA_DEV_BAD_SEQ : QSA_DEV_BAD_POS);
        a.count[q] = 0;
      }
      for (int i = tid; i < K; i += kFThreads) out[i] = -1;
    }
    return;
  }
  cluster_arrive_relaxed();  // this CTA is running (waited for before the first remote store)
  if (ld_over && leader && tid == 0) flag(a.st, QSA_DEV_SCORES_LD);

  // ---------------- A. scores of this CTA's pages
  __syncthreads();  // the page ids are in shared memory
  {
    float* srow = a.scores + (size_t)q * a.ld;
    for (int pp = 2 * warp; pp < np_cta; pp += 2 * kFWarps) {  // warp-uniform
      uint4 ra[2][4], rb[2][4];
      bool ok[2];
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int pl = pp + k;
        const int phys = pl < np_cta ? ids[pl] : -1;
        ok[k] = pl < np_cta && phys >= 0 && phys < a.num_pages;
        if (ok[k]) load_idx_page(a.kc, phys, ra[k], rb[k]);
      }
      // the warp's next two pages go to L2 now (lanes 0 and 1, one bulk
      // prefetch of 4 KiB each): the next loads find them there, and the
      // bytes in flight per SM are no longer bounded by these registers
      if (lane < 2) {
        const int pn = pp + 2 * kFWarps + lane;
        const int phys = pn < np_cta ? ids[pn] : -1;
        if (phys >= 0 && phys < a.num_pages)
          l2_prefetch_bulk(a.kc + (size_t)phys * kBlocksPerPage * kIdxDim, kBlocksPerPage * kIdxDim * 2);
      }
#pragma unroll
      for (int k = 0; k < 2; ++k) {
        const int pl = pp + k;
        if (pl >= np_cta) continue;
        const int blk_lo = (pg_lo + pl) * kBlocksPerPage + g;  // rows g and g + 8 of the page
        const int blk_hi = blk_lo + 8;
        float s_lo = -INFINITY, s_hi = -INFINITY;  // a block on a rejected page scores -inf
        if (ok[k]) {
          score_idx_page(ra[k], rb[k], Q, s_lo, s_hi);
        } else if (lane == 0) {
          flag(a.st, QSA_DEV_BAD_PAGE);
        }
        if (t == 0 && blk_lo < n) {
          srow[blk_lo] = s_lo;
          keys[blk_lo - b_lo] = float_key(s_lo);
        }
        if (t == 1 && blk_hi < n) {
          srow[blk_hi] = s_hi;
          keys[blk_hi - b_lo] = float_key(s_hi);
        }
      }
    }
  }
  // The cluster barriers below are release/acquire at cluster scope for every
  // state space: the scores row written here is visible to the leader's
  // fallback path after them, without a device-wide fence.
  __syncthreads();  // this CTA's keys are in shared memory
  cluster_wait();   // every CTA of the cluster is running
  const int ns = min(n, kSample);
  if (selecting) {
    // the samples at positions i * n / ns that lie in this slice, to every CTA
    for (int i = tid; i < ns; i += kFThreads) {
      const int pos = ns < kSample ? i : (int)((int64_t)i * n / kSample);  // ns is n or the constant kSample
      if (pos >= b_lo && pos < b_lo + m) {
        const uint32_t kv = keys[pos - b_lo];
#pragma unroll
        for (int c = 0; c < kFC; ++c) st_cluster(samp + i, (uint32_t)c, kv);
      }
    }
  }
  cluster_barrier();  // 1: the samples are everywhere

  if (!selecting) {  // every visible block is kept
    if (leader) {
      for (int i = tid; i < K; i += kFThreads) out[i] = i < n ? i : -1;
      if (tid == 0) a.count[q] = min(n, K);
    }
    return;
  }
  if (leader && tid == 0) a.count[q] = K;

  // ---------------- B1. threshold from the regular sample of the whole row
  uint32_t ks[kFSPer];
#pragma unroll
  for (int u = 0; u < kFSPer; ++u) {
    const int i = u * kFThreads + tid;
    ks[u] = i < ns ? samp[i] : 0u;
  }
  const uint32_t T0 = sample_threshold<kFThreads>(ks, ns, n, K, S);

  // ---------------- B2. this CTA's candidates, per warp over a contiguous segment, in index order
  {
    const int seg = ((m + kFWarps * 128 - 1) / (kFWarps * 128)) * 128;
    const int w_lo = min(m, warp * seg), w_hi = min(m, w_lo + seg);
    uint32_t cnt = 0;
    for (int c0 = w_lo; c0 < w_hi; c0 += 128) {  // warp-uniform trip count
      const int i0 = c0 + 4 * lane;
      uint32_t k[4] = {0u, 0u, 0u, 0u};
      if (i0 + 3 < w_hi) {
        const uint4 v = *reinterpret_cast<const uint4*>(keys + i0);
        k[0] = v.x;
        k[1] = v.y;
        k[2] = v.z;
        k[3] = v.w;
      } else {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (i0 + c < w_hi) k[c] = keys[i0 + c];
      }
      const bool f[4] = {i0 < w_hi && k[0] >= T0, i0 + 1 < w_hi && k[1] >= T0, i0 + 2 < w_hi && k[2] >= T0,
                         i0 + 3 < w_hi && k[3] >= T0};
      append4(LL, warp, cnt, k, b_lo + i0, f);
    }
    // the CTA's list = the warp lists in warp order; its length, or kFList + 1 when it does not fit
    if (lane == 0) S.wgt[warp] = cnt;
    __syncthreads();
    uint32_t before = 0, total = 0;
    bool over = false;
    for (int w2 = 0; w2 < kFWarps; ++w2) {
      const uint32_t c2 = S.wgt[w2];
      if (w2 < warp) before += c2;
      total += c2;
      over |= c2 > (uint32_t)kFLocal;
    }
    over |= total > (uint32_t)kFList;
    if (!over) {
      for (uint32_t j = lane; j < cnt; j += 32) {
        st_cluster(&S.ckey[rank][before + j], 0u, LL.ckey[warp][j]);
        st_cluster(&S.cidx[rank][before + j], 0u, LL.cidx[warp][j]);
      }
    }
    if (tid == 0) st_cluster(&S.wcnt[rank], 0u, over ? (uint32_t)kFList + 1 : total);
  }
  cluster_barrier();  // 2: the leader holds every CTA's list; no shared memory is touched remotely after this
  // The next kernel may launch only once every cluster has reached its
  // selection (or left): launched earlier, its CTAs would take the shared
  // memory this grid's later clusters need and push them into a second wave.
  pdl_launch_dependents();
  if (!leader) return;

  // ---------------- B3. the exact select on the leader (warp w: the list of CTA w)
  uint32_t total = 0;
  bool overflow = false;
#pragma unroll
  for (int c = 0; c < kFC; ++c) {
    total += S.wcnt[c];
    overflow |= S.wcnt[c] > (uint32_t)kFList;
  }
  if (overflow || total < (uint32_t)K) {  // CTA-uniform
    topk_general<kFThreads>(a.scores + (size_t)q * a.ld, n, K, out, S.hist, S.wsum, S.wgt, S.weq, &S.bin, &S.above);
    return;
  }
  select_from_lists<kFThreads>(S, K, out);
}

bool aligned(const void* p, unsigned al) { return (reinterpret_cast<uintptr_t>(p) & (al - 1)) == 0; }

}  // namespace

extern "C" int qsa_index_topk_smem_bytes(const qsa_cache_t* cache, int64_t scores_ld) {
  if (!cache || scores_ld < 1 || cache->max_pages_per_seq < 1) return QSA_ERR_INVALID_ARG;
  int64_t max_blocks = (int64_t)cache->max_pages_per_seq * kBlocksPerPage;
  if (scores_ld < max_blocks) max_blocks = scores_ld;
  const int64_t pages = (max_blocks + kBlocksPerPage - 1) / kBlocksPerPage;
  const int64_t slice_pages = ((pages + kFC - 1) / kFC + 3) / 4 * 4;
  const int64_t bytes = (int64_t)kFOffIds + slice_pages * 4 + slice_pages * kBlocksPerPage * 4;
  return bytes > 0x7fffffff ? QSA_ERR_UNSUPPORTED : (int)bytes;
}

extern "C" int qsa_index_topk_resident_queries(const qsa_cache_t* cache, int64_t scores_ld) {
  const int smem = qsa_index_topk_smem_bytes(cache, scores_ld);
  if (smem < 0) return smem;
  int dev = 0, max_smem = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  if (smem > max_smem) return 0;
  if (cudaFuncSetAttribute(index_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kFC);
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kFC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  int clusters = 0;
  if (cudaOccupancyMaxActiveClusters(&clusters, index_topk_kernel, &cfg) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  return clusters;
}

extern "C" int qsa_index_topk(const qsa_cache_t* cache, const void* q_idx, const float* w, const int32_t* q_seq,
                              const int32_t* q_pos, int32_t nq, int32_t k, float* scores, int64_t scores_ld,
                              int32_t* sel, int32_t* count, int32_t* dev_status, void* stream) {
  if (!cache || nq < 0 || k < 0 || k > QSA_MAX_TOPK || scores_ld < 1) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!cache->kc_pages || !cache->block_table || !q_idx || !w || !q_seq || !q_pos || !scores || !count ||
      (k > 0 && !sel))
    return QSA_ERR_INVALID_ARG;
  if (cache->num_pages < 1 || cache->max_seqs < 1 || cache->max_pages_per_seq < 1) return QSA_ERR_INVALID_ARG;
  if (!aligned(cache->kc_pages, 16) || !aligned(q_idx, 16)) return QSA_ERR_INVALID_ARG;
  const int smem = qsa_index_topk_smem_bytes(cache, scores_ld);
  if (smem < 0) return smem;
  int dev = 0, max_smem = 0;
  if (cudaGetDevice(&dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  // a row longer than the cluster's shared memory holds: the two-kernel form
  if (smem > max_smem) {
    const int r = qsa_index_scores(cache, q_idx, w, q_seq, q_pos, nq, scores, scores_ld, dev_status, stream);
    if (r != QSA_OK) return r;
    return qsa_topk_blocks(scores, scores_ld, q_pos, nq, k, sel, count, dev_status, stream);
  }
  if ((int64_t)nq * kFC > 0x7fffffff) return QSA_ERR_UNSUPPORTED;
  if (cudaFuncSetAttribute(index_topk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  FusedArgs f;
  f.kc = static_cast<const __nv_bfloat16*>(cache->kc_pages);
  f.bt = cache->block_table;
  f.num_pages = cache->num_pages;
  f.max_seqs = cache->max_seqs;
  f.mpps = cache->max_pages_per_seq;
  f.q_idx = static_cast<const __nv_bfloat16*>(q_idx);
  f.w = w;
  f.q_seq = q_seq;
  f.q_pos = q_pos;
  f.scores = scores;
  f.ld = scores_ld;
  f.K = k;
  f.sel = sel;
  f.count = count;
  {
    int64_t max_blocks = (int64_t)cache->max_pages_per_seq * kBlocksPerPage;
    if (scores_ld < max_blocks) max_blocks = scores_ld;
    const int64_t pages = (max_blocks + kBlocksPerPage - 1) / kBlocksPerPage;
    f.slice_pages = (int32_t)(((pages + kFC - 1) / kFC + 3) / 4 * 4);
  }
  f.st = dev_status;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)(nq * kFC));
  cfg.blockDim = dim3(kFThreads);
  cfg.dynamicSmemBytes = (size_t)smem;
  cfg.stream = static_cast<cudaStream_t>(stream);
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kFC;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if (cudaLaunchKernelEx(&cfg, index_topk_kernel, f) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  return QSA_OK;
}
