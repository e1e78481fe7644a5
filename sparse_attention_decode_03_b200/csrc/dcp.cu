// Decode context parallelism (DCP): the main K/V of every sequence is sharded
// by context over N ranks, while the selector (indexer side cache, scores,
// top-K) is replicated, so every rank selects the same blocks and attends only
// to the selected blocks it holds; the ranks' partial results are merged by
// log-sum-exp afterwards.
//
// Source: [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section
// "Wat de pull request daadwerkelijk verandert": each rank reads its own slice
// of the main KV, the selector and main KV stay in one cache group, split
// results are combined across ranks, and a localisation step maps the globally
// selected blocks to the rank's own slots.  The shard rule is a fixed reading:
// logical page P of a sequence (64 tokens) lives on rank (P / I) mod N, at local
// page (P / (I N)) I + P mod I, I = interleave_pages (I = 1: round robin by
// page); a rank's local pages are numbered in context order, so its tokens sit
// at consecutive local positions.
#include "qsa_common.cuh"

namespace {

using namespace qsa;

struct Shard {
  int32_t n, r, I;  // ranks, this rank, interleave in pages
  __device__ __forceinline__ int owner(int P) const { return (P / I) % n; }
  __device__ __forceinline__ int local_page(int P) const { return (P / (I * n)) * I + P % I; }
  // pages in [0, P) held by this rank
  __device__ __forceinline__ int owned_before(int P) const {
    const int cyc = I * n;
    return (P / cyc) * I + max(0, min(P % cyc, (r + 1) * I) - r * I);
  }
};

__global__ void localize_tokens_kernel(const int32_t* seq_id, const int32_t* pos, int32_t n, Shard sh,
                                       int32_t* seq_local, int32_t* pos_local) {
  pdl_launch_dependents();
  pdl_wait_previous();
  const int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (i >= n) return;
  const int s = seq_id[i], p = pos[i];
  const bool mine = s >= 0 && p >= 0 && sh.owner(p / kPage) == sh.r;
  seq_local[i] = mine ? s : -1;
  pos_local[i] = mine ? sh.local_page(p / kPage) * kPage + p % kPage : 0;
}

constexpr int kLThreads = 256;

// One CTA per query: the owned entries of the selection, in order, as local
// block indices; the local count; and a local position whose (nb, t) make the
// rank attend to exactly those blocks plus the trailing tokens if it holds them.
__global__ void __launch_bounds__(kLThreads) localize_selection_kernel(const int32_t* sel, const int32_t* count,
                                                                         const int32_t* q_pos, int32_t K, Shard sh,
                                                                         int32_t* sel_local, int32_t* count_local,
                                                                         int32_t* q_pos_local, int32_t* st) {
  pdl_launch_dependents();
  pdl_wait_previous();
  __shared__ uint32_t wtot[kLThreads / 32];
  const int q = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int p = q_pos[q];
  if (p < 0) {  // passed through: the attention call flags it
    if (tid == 0) {
      count_local[q] = 0;
      q_pos_local[q] = p;
    }
    for (int i = tid; i < K; i += kLThreads) sel_local[(size_t)q * K + i] = -1;
    return;
  }
  const int nb = (p + 1) / kRatio, t = (p + 1) % kRatio;
  int cnt = count[q];
  const int cap = min(K, nb);
  if (cnt < 0 || cnt > cap) {
    if (tid == 0) flag(st, QSA_DEV_BAD_COUNT);
    cnt = cnt < 0 ? 0 : cap;
  }
  uint32_t base = 0;
  for (int i0 = 0; i0 < cnt; i0 += kLThreads) {
    const int i = i0 + tid;
    int j = -1;
    bool mine = false;
    if (i < cnt) {
      j = sel[(size_t)q * K + i];
      if (j < 0 || j >= nb) {
        flag(st, QSA_DEV_BAD_SEL);
      } else {
        mine = sh.owner(j / kBlocksPerPage) == sh.r;
      }
    }
    const uint32_t b = __ballot_sync(0xffffffffu, mine);
    if (lane == 0) wtot[warp] = __popc(b);
    __syncthreads();
    uint32_t before = base, all = 0;
#pragma unroll
    for (int w = 0; w < kLThreads / 32; ++w) {
      before += w < warp ? wtot[w] : 0u;
      all += wtot[w];
    }
    if (mine) {
      const int P = j / kBlocksPerPage;
      sel_local[(size_t)q * K + before + __popc(b & ((1u << lane) - 1u))] =
          sh.local_page(P) * kBlocksPerPage + j % kBlocksPerPage;
    }
    base += all;
    __syncthreads();  // wtot reused
  }
  for (int i = (int)base + tid; i < K; i += kLThreads) sel_local[(size_t)q * K + i] = -1;
  if (tid == 0) {
    const int Pt = nb / kBlocksPerPage;  // page of the trailing (incomplete) block
    const bool tail_page = sh.owner(Pt) == sh.r;
    const int nb_local = sh.owned_before(Pt) * kBlocksPerPage + (tail_page ? nb % kBlocksPerPage : 0);
    int pl;
    if (tail_page && t > 0) pl = kRatio * nb_local + t - 1;
    else if (nb_local > 0) pl = kRatio * nb_local - 1;
    else pl = kRatio - 1;  // holds nothing of this query: one (unread) block, no tail
    count_local[q] = (int32_t)base;
    q_pos_local[q] = pl;
  }
}

bool valid_shard(int32_t nranks, int32_t rank, int32_t interleave) {
  return nranks >= 1 && rank >= 0 && rank < nranks && interleave >= 1 && (int64_t)nranks * interleave <= (1 << 20);
}

}  // namespace

extern "C" int qsa_dcp_localize_tokens(const int32_t* seq_id, const int32_t* pos, int32_t n, int32_t nranks,
                                       int32_t rank, int32_t interleave_pages, int32_t* seq_id_local,
                                       int32_t* pos_local, void* stream) {
  if (n < 0 || !valid_shard(nranks, rank, interleave_pages)) return QSA_ERR_INVALID_ARG;
  if (n == 0) return QSA_OK;
  if (!seq_id || !pos || !seq_id_local || !pos_local) return QSA_ERR_INVALID_ARG;
  const Shard sh{nranks, rank, interleave_pages};
  return qsa_host::launch(localize_tokens_kernel, dim3((unsigned)((n + 255) / 256)), dim3(256), 0,
                          static_cast<cudaStream_t>(stream), seq_id, pos, n, sh, seq_id_local, pos_local);
}

extern "C" int qsa_dcp_localize_selection(const int32_t* sel, const int32_t* count, const int32_t* q_pos, int32_t nq,
                                          int32_t k, int32_t nranks, int32_t rank, int32_t interleave_pages,
                                          int32_t* sel_local, int32_t* count_local, int32_t* q_pos_local,
                                          int32_t* dev_status, void* stream) {
  if (nq < 0 || k < 0 || k > QSA_MAX_TOPK || !valid_shard(nranks, rank, interleave_pages)) return QSA_ERR_INVALID_ARG;
  if (nq == 0) return QSA_OK;
  if (!count || !q_pos || !count_local || !q_pos_local || (k > 0 && (!sel || !sel_local))) return QSA_ERR_INVALID_ARG;
  const Shard sh{nranks, rank, interleave_pages};
  return qsa_host::launch(localize_selection_kernel, dim3((unsigned)nq), dim3(kLThreads), 0,
                          static_cast<cudaStream_t>(stream), sel, count, q_pos, k, sh, sel_local, count_local,
                          q_pos_local, dev_status);
}
