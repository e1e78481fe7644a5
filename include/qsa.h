/*
 * qsa.h -- C ABI of libqsa: the Qwen Sparse Attention (QSA) decode hot path on
 * one NVIDIA B200 (sm_100a).
 *
 * What the path computes (sources: the pages
 *   [DCP]  "Qwen 4 QSA krijgt decode-contextparallellisme: in vLLM's concept-PR
 *          voor Qwen3.8-Flash-Next", section "Wat de pull request daadwerkelijk
 *          verandert";
 *   [CANN] "Qwen4-Exp QSA komt naar Huawei's Ascend: binnen SGLang's opt-in CANN
 *          prefill-PR", sections "Wat de pull request daadwerkelijk toevoegt",
 *          "Negen tests die geslaagd zijn ..." and "Waarom QSA het lastige
 *          onderdeel is, in cijfers";
 *   [BSS]  "Pengambilan sampel batch-sharded Qwen4Exp", section "Apa yang
 *          dikatakan oleh klaster patch di sekitarnya tentang Qwen4Exp"):
 *   a lightweight indexer compresses keys into micro-blocks of 4 tokens and
 *   scores every block against the query; the best 512 blocks (about 2,048
 *   token positions) are kept; softmax and value aggregation then run over the
 *   uncompressed K and V (BF16, or FP8 e4m3; head dim 256, GQA) at those
 *   positions only; the attention is split over KV chunks and merged with
 *   log-sum-exp (on one GPU the analogue of the cross-rank combine of [DCP];
 *   across GPUs the qsa_dcp_* calls shard the K/V by context and the same
 *   merge combines the ranks).
 * Fixed readings where the pages are silent: kc_j = sum of the 4 tokens'
 * indexer keys (fp32, token order, stored BF16 round-to-nearest-even);
 * s_j = sum_h w_h * ReLU(q_idx,h . kc_j) with 8 indexer heads of dim 128; ties
 * (equal scores, -0 and +0 included) go to the lower block index; a query at position p sees nb = (p+1)/4
 * complete blocks and always attends its t = (p+1)%4 trailing tokens.
 *
 * Conventions for every call
 *  - Pointers are DEVICE pointers owned and allocated by the caller, except
 *    the `cache` descriptor itself (host memory, read during the call only).
 *    The library allocates nothing and never synchronises the host.
 *  - `stream` is a cudaStream_t (NULL = the legacy default stream); calls only
 *    enqueue work on it.
 *  - Kernels are launched with programmatic dependent launch: a kernel may
 *    start before the preceding kernel of the stream has finished and waits
 *    for it before it reads anything that kernel may write.  The indexer
 *    calls (qsa_index_scores, qsa_index_topk) and qsa_topk_blocks read their
 *    query inputs (q_seq, q_pos, q_idx, w) and the block table BEFORE that
 *    wait.  They must therefore be complete by the time the preceding kernel
 *    of the stream starts; when that kernel is qsa_append_kv, by the end of
 *    the kernel before it (qsa_append_kv lets its dependents start only after
 *    its own predecessor has finished).  Inputs written by host copies, or by
 *    kernels that do not use programmatic dependent launch, earlier in the
 *    stream always are.
 *  - Return value: QSA_OK, or a negative qsa_status for a host-detected error
 *    (nothing is enqueued then).
 *  - `dev_status` (may be NULL) is a device int32 the kernels OR error bits
 *    into (QSA_DEV_*) when they meet bad data: an out-of-range page id,
 *    sequence id, position, selection index or count.  The offending read is
 *    skipped (masked); kernels never trap.  The caller clears and reads it.
 *  - All outputs are deterministic: no floating-point atomics.
 *  - Tensors are dense row-major with the shapes given; no strides (except
 *    qsa_combine_strided, which takes them explicitly).
 */
#ifndef QSA_H
#define QSA_H

#include <stdint.h>

#if defined(__GNUC__)
#define QSA_API __attribute__((visibility("default")))
#else
#define QSA_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* fixed geometry ([CANN] "Waarom QSA ...": head dim 256, indexer dim 128,
 * ratio 4; indexer heads 8 and 64-token pages are fixed readings) */
#define QSA_HEAD_DIM 256
#define QSA_IDX_HEADS 8
#define QSA_IDX_DIM 128
#define QSA_RATIO 4
#define QSA_PAGE_TOKENS 64
#define QSA_BLOCKS_PER_PAGE 16 /* micro-blocks per page */
#define QSA_MAX_TOPK 2048      /* largest K accepted by qsa_topk_blocks / qsa_sparse_decode */
#define QSA_MAX_GROUP 16       /* largest Hq / Hkv accepted by qsa_sparse_decode */

typedef enum {
  QSA_OK = 0,
  QSA_ERR_INVALID_ARG = -1, /* null pointer, negative size, Hq % Hkv != 0, K > QSA_MAX_TOPK, ... */
  QSA_ERR_UNSUPPORTED = -2, /* a shape the kernels do not implement (e.g. Hq / Hkv > 16) */
  QSA_ERR_CUDA = -3         /* a CUDA launch failed; cudaGetLastError() has been cleared */
} qsa_status;

/* bits OR-ed into *dev_status by the kernels */
#define QSA_DEV_BAD_PAGE 1    /* block-table entry outside [0, num_pages) */
#define QSA_DEV_BAD_SEQ 2     /* sequence id outside [0, max_seqs) */
#define QSA_DEV_BAD_POS 4     /* position < 0 or beyond the block-table capacity */
#define QSA_DEV_BAD_SEL 8     /* selected block index outside [0, nb_q) */
#define QSA_DEV_BAD_COUNT 16  /* selection count outside [0, min(K, nb_q)] */
#define QSA_DEV_BAD_ORDER 32  /* append tokens of one sequence not in consecutive positions */
#define QSA_DEV_TIMEOUT 64    /* a bounded pipeline wait expired; outputs of that call are invalid */
#define QSA_DEV_SCORES_LD 128 /* a query sees more blocks than the scores row holds */

/*
 * One cache group ([DCP]: the selector and the main KV cache are kept in one
 * cache group so they cannot drift apart).  The main K/V and the compressed
 * indexer side cache are paged by the SAME physical page ids.
 *   kv_pages    post-RoPE K and V of type kv_dtype: per page and KV head, its
 *               16 micro-blocks of 4 tokens (token t of a page: micro-block
 *               t / 4, row t % 4), each one contiguous run, so one selected
 *               micro-block of one KV head is one copy:
 *                 BF16: [num_pages][num_kv_heads][16] runs of 4 KiB, each
 *                   [4 dim atoms][8 rows][64 elements]: atom a holds dims
 *                   64a .. 64a+63 of rows 0-3 = K rows 0-3 and rows 4-7 =
 *                   V rows 0-3 (128 B per row), and the 16-byte chunk c
 *                   (elements 8c .. 8c+7) of row r sits at chunk position
 *                   c XOR r of that row (the tensor cores' 128-byte swizzled
 *                   operand layout, so a run is gathered into shared memory
 *                   as it is);
 *                 FP8: [num_pages][num_kv_heads][16][2][4][256] bytes: the 4 K
 *                   rows then the 4 V rows (2 KiB per run).
 *   kc_pages    bf16 [num_pages][16][128]  kc of the 16 micro-blocks of a page
 *   kc_partial  fp32 [max_seqs][128]       running fp32 sum of each sequence's
 *                                           open (incomplete) micro-block
 *   block_table int32 [max_seqs][max_pages_per_seq]  logical page -> physical page
 *   kv_dtype    QSA_KV_BF16, or QSA_KV_FP8_E4M3: the main K/V stored as FP8
 *               e4m3 (1 byte per element, the BF16 value rounded to nearest
 *               even and saturated to +-448, no scale; the FP8 e4m3 main KV
 *               cache of [BSS], section "Apa yang dikatakan oleh klaster patch
 *               di sekitarnya tentang Qwen4Exp"), which halves the bytes the
 *               sparse attention gathers.  The side cache stays BF16.
 * All buffers are caller-owned device memory; the library writes kv/kc pages
 * and kc_partial only in qsa_append_kv.
 * A group may leave out one part: kv_pages NULL (a selector-only group, e.g.
 * the replicated side cache of a DCP rank) or kc_pages and kc_partial NULL (a
 * main-K/V-only group, e.g. a DCP rank's K/V shard).  qsa_append_kv then
 * writes only the part that is there; qsa_index_scores needs kc_pages and
 * qsa_sparse_decode needs kv_pages.
 */
#define QSA_KV_BF16 0
#define QSA_KV_FP8_E4M3 1
typedef struct {
  void* kv_pages;
  void* kc_pages;
  float* kc_partial;
  const int32_t* block_table;
  int32_t num_pages;
  int32_t max_seqs;
  int32_t max_pages_per_seq;
  int32_t num_kv_heads;
  int32_t kv_dtype;
} qsa_cache_t;

/* Human-readable name of a qsa_status value (static string). */
QSA_API const char* qsa_status_string(int status);

/* ABI version of this header (bumped on any signature change). */
QSA_API int qsa_abi_version(void);
#define QSA_ABI_VERSION 7

/*
 * qsa_append_kv -- write n new tokens into the cache group.
 * [DCP] keeps the selector caches in step with the main cache; [CANN] marks
 * invalid slots with -1 padding and [DCP] stops synthetic batches from writing
 * the QSA side caches: a token with seq_id < 0 is skipped entirely.
 *   k_new, v_new  bf16 [n][Hkv][256];  kidx_new  bf16 [n][128] (indexer keys)
 *   seq_id, pos   int32 [n]  sequence and absolute position of each token
 * Effect: K/V rows written at page block_table[seq][pos/64], token pos%64 (as
 * e4m3, round to nearest even, saturated to +-448, when kv_dtype is FP8).  The
 * indexer keys of a micro-block are summed in fp32 in token order (continuing
 * kc_partial when the block began in an earlier call); when the token at
 * position 4j+3 arrives, kc_pages row j = BF16(sum) (round to nearest even).
 * A block left incomplete stores its running sum in kc_partial[seq].
 * Rules: the tokens of one sequence are contiguous in the arrays and at
 * consecutive increasing positions, and calls for a sequence arrive in
 * position order.  Detected (QSA_DEV_BAD_ORDER): a token whose predecessor
 * in the arrays belongs to the same sequence at a position other than its
 * own minus one.  NOT detected: a sequence whose tokens form several runs
 * within one call (other sequences' tokens between them), and calls that
 * skip or repeat positions across calls; every K/V row is still written, but
 * that sequence's kc_pages rows and kc_partial are then undefined (other
 * sequences are unaffected).  One kernel is
 * enqueued.  n = 0 is a no-op.
 */
QSA_API int qsa_append_kv(const qsa_cache_t* cache, const void* k_new, const void* v_new, const void* kidx_new,
                  const int32_t* seq_id, const int32_t* pos, int32_t n, int32_t* dev_status, void* stream);

/*
 * qsa_index_scores -- [DCP]/[CANN]/[BSS]: the indexer scores every complete
 * micro-block visible to each query:
 *   scores[q][j] = sum_{h<8} w[q][h] * max(0, sum_{d<128} q_idx[q][h][d] * kc[seq_q][j][d])
 * for j < nb_q = (q_pos[q] + 1) / 4 (entries j >= nb_q are not written).
 *   q_idx bf16 [nq][8][128]; w fp32 [nq][8]; q_seq, q_pos int32 [nq]
 *   scores fp32 [nq][scores_ld]; scores_ld >= the largest nb_q
 * Products are BF16 x BF16 accumulated in fp32 on the tensor cores; with
 * integer-valued indexer data and power-of-two weights every score is exact.
 * A page-table miss writes -inf for its 16 blocks and sets QSA_DEV_BAD_PAGE.
 */
QSA_API int qsa_index_scores(const qsa_cache_t* cache, const void* q_idx, const float* w, const int32_t* q_seq,
                     const int32_t* q_pos, int32_t nq, float* scores, int64_t scores_ld, int32_t* dev_status,
                     void* stream);

/*
 * qsa_topk_blocks -- per query, keep the best min(k, nb_q) blocks ([DCP]: "the
 * best 512 blocks") under the order (score descending, block index
 * ascending), written sorted by block index ascending:
 *   sel   int32 [nq][k]  selected block indices, then -1 padding
 *   count int32 [nq]     min(k, nb_q)
 * Deterministic radix select on the fp32 bit patterns; 0 <= k <= QSA_MAX_TOPK.
 */
QSA_API int qsa_topk_blocks(const float* scores, int64_t scores_ld, const int32_t* q_pos, int32_t nq, int32_t k,
                    int32_t* sel, int32_t* count, int32_t* dev_status, void* stream);

/*
 * qsa_index_topk -- qsa_index_scores followed by qsa_topk_blocks, in one
 * kernel ([DCP]: the indexer scores the micro-blocks and the best 512 are
 * kept): the same scores (bit for bit) and the same selections and counts.
 * The score row of a query stays in on-chip shared memory, spread over a
 * cluster of 8 CTAs, while it is selected from, instead of being read back
 * from global memory; scores[q][j < nb_q] is still written.
 * One cluster of 8 CTAs per query, so this form pays when the batch fills the
 * GPU (nq * 8 of at least about the SM count); with fewer queries the two
 * separate calls spread each query over more SMs.
 * Arguments and rules: those of qsa_index_scores and qsa_topk_blocks.  A query
 * whose q_seq or q_pos is out of range sets the status bit and gets count 0
 * and an all -1 selection.  When the longest possible row (min(scores_ld,
 * max_pages_per_seq * 16) blocks) needs more shared memory per CTA than the
 * device allows, the call enqueues the two separate kernels instead.
 */
QSA_API int qsa_index_topk(const qsa_cache_t* cache, const void* q_idx, const float* w, const int32_t* q_seq,
                   const int32_t* q_pos, int32_t nq, int32_t k, float* scores, int64_t scores_ld, int32_t* sel,
                   int32_t* count, int32_t* dev_status, void* stream);

/*
 * qsa_index_topk_smem_bytes -- host-only: the dynamic shared memory one CTA of
 * qsa_index_topk takes for this cache group and scores_ld (about 68 KiB plus
 * 68 B per page of the longest possible row / 8), or a negative qsa_status.
 */
QSA_API int qsa_index_topk_smem_bytes(const qsa_cache_t* cache, int64_t scores_ld);

/*
 * qsa_index_topk_resident_queries -- how many queries' clusters of
 * qsa_index_topk the current device holds at once for this cache group and
 * scores_ld (0 when a CTA's shared memory does not fit), or a negative
 * qsa_status.  A batch of at most this many queries runs in one wave.
 * Queries the CUDA runtime (needs a device; enqueues nothing).
 */
QSA_API int qsa_index_topk_resident_queries(const qsa_cache_t* cache, int64_t scores_ld);

/*
 * qsa_decode_plan -- host-only helper: choose the KV chunk size for
 * qsa_sparse_decode.  Every (query, KV head) pair owns k+1 unit slots (its k
 * selection slots, then its trailing micro-block); the slots of all pairs,
 * query-major, are cut into chunks of *chunk_units slots, one CTA per chunk.
 * The chunk size spreads the nq*hkv*(k+1) slots over about target_ctas CTAs
 * (pass the SM count).  *max_splits = the most chunks one pair can touch,
 * i.e. the split dimension S of part_o / part_lse.
 */
QSA_API int qsa_decode_plan(int32_t nq, int32_t hkv, int32_t k, int32_t target_ctas, int32_t* chunk_units,
                    int32_t* max_splits);

/*
 * qsa_sparse_decode -- sparse attention over the uncompressed K/V at the
 * selected positions ([DCP]: softmax and value aggregation run on the
 * uncompressed K and V), split over KV chunks ([DCP]: split read, results
 * combined afterwards).
 * For query q (position p, nb = (p+1)/4, t = (p+1)%4) and KV head g, unit slot
 * u < count[q] holds the 4 tokens of block sel[q][u]; slots count[q]..k-1 are
 * empty; slot k holds the t trailing tokens 4nb..p.  Chunk c covers the global
 * slots [c*chunk_units, (c+1)*chunk_units) of the order (q, g, u); the part of
 * pair (q, g) inside the s-th chunk it touches is split s.  For every Q head h
 * of group g (h / (hq/hkv) == g) and split s over token set T:
 *   z_t = scale * q[q][h] . K[t][g];  lse = log sum_t exp(z_t);
 *   o = sum_t exp(z_t - lse) V[t][g]
 * written to part_o[q][s][h][:] (fp32) and part_lse[q][s][h] (fp32, natural
 * log).  An empty split, and every slot s a pair does not reach, gets o = 0
 * and lse = -inf ([CANN]: fully masked rows keep the zero-output convention).
 *   q bf16 [nq][hq][256]; sel int32 [nq][k]; count int32 [nq]
 *   part_o fp32 [nq][max_splits][hq][256]; part_lse fp32 [nq][max_splits][hq]
 * Requirements: hq % Hkv == 0, hq / Hkv <= 16, 0 <= k <= QSA_MAX_TOPK,
 * chunk_units >= 1, max_splits >= the value qsa_decode_plan reports for
 * (k, chunk_units), scale > 0 (the pages keep the D256 scale 1/16).
 * The kernel gathers each selected micro-block (4 K rows + 4 V rows of one KV
 * head: one contiguous run) into shared memory as it is, with 16-byte async
 * copies, and runs QK^T and PV on the tensor cores with fp32 accumulation;
 * the softmax weights P enter PV as a BF16 hi + lo pair (about 17
 * significant bits), so short token sets keep full accuracy.
 */
QSA_API int qsa_sparse_decode(const qsa_cache_t* cache, const void* q, int32_t nq, int32_t hq, const int32_t* q_seq,
                      const int32_t* q_pos, const int32_t* sel, const int32_t* count, int32_t k, float scale,
                      int32_t chunk_units, int32_t max_splits, float* part_o, float* part_lse,
                      int32_t* dev_status, void* stream);

/*
 * qsa_sparse_attention -- qsa_sparse_decode followed by qsa_combine in one
 * kernel ([DCP]: the split results are combined afterwards; here the combine
 * runs inside the split kernel).  Every CTA writes its split partials exactly
 * as qsa_sparse_decode does; the CTA that writes the last split of a (query,
 * KV head) pair -- counted with a device-scope atomic in pair_done -- merges
 * that pair's splits into out / lse with qsa_combine's arithmetic, so out and
 * lse equal those of the two calls bit for bit.
 *   pair_done int32 [nq][Hkv], all zero on entry; the call leaves it all zero
 *             (after a QSA_DEV_TIMEOUT status the caller must zero it again);
 *             calls sharing one pair_done must not overlap on the GPU
 *   out bf16 [nq][hq][256] (8-byte aligned); lse fp32 [nq][hq]
 * Other arguments, rules and errors: those of qsa_sparse_decode.
 */
QSA_API int qsa_sparse_attention(const qsa_cache_t* cache, const void* q, int32_t nq, int32_t hq,
                         const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel, const int32_t* count,
                         int32_t k, float scale, int32_t chunk_units, int32_t max_splits, float* part_o,
                         float* part_lse, int32_t* pair_done, void* out, float* lse, int32_t* dev_status,
                         void* stream);

/*
 * qsa_combine -- log-sum-exp merge of the splits ([DCP]: attention results of
 * the split read are combined):
 *   lse[q][h] = log sum_s exp(part_lse[q][s][h]);
 *   out[q][h] = BF16( sum_s exp(part_lse[q][s][h] - lse[q][h]) * part_o[q][s][h] )
 * Splits with lse = -inf are skipped; if all are, out = 0 exactly and
 * lse = -inf ([CANN] zero-output convention).
 *   out bf16 [nq][hq][256]; lse fp32 [nq][hq]
 */
QSA_API int qsa_combine(const float* part_o, const float* part_lse, int32_t nq, int32_t max_splits, int32_t hq,
                void* out, float* lse, void* stream);

/*
 * qsa_combine_strided -- the same merge over nsplits splits laid out with
 * explicit element strides: split s of (query q, head h) is
 *   part_o[q * o_q_stride + s * o_split_stride + h * 256 + d],
 *   part_lse[q * lse_q_stride + s * lse_split_stride + h];
 * qsa_combine is the case o_split_stride = hq*256, o_q_stride = S*hq*256,
 * lse_split_stride = hq, lse_q_stride = S*hq.  With out_dtype QSA_OUT_F32 the
 * merged rows are written as fp32 (16-byte aligned out), so a merged result can
 * itself be one split of a later merge: a DCP rank merges its own splits, the
 * ranks' results are gathered rank-major ([rank][q][h][256], o_split_stride =
 * nq*hq*256) and merged again ([DCP]: split results combined across ranks).
 * o strides must be multiples of 4 elements.
 */
#define QSA_OUT_BF16 0
#define QSA_OUT_F32 1
QSA_API int qsa_combine_strided(const float* part_o, const float* part_lse, int32_t nq, int32_t nsplits, int32_t hq,
                        int64_t o_q_stride, int64_t o_split_stride, int64_t lse_q_stride,
                        int64_t lse_split_stride, void* out, int32_t out_dtype, float* lse, void* stream);

/*
 * Decode context parallelism ([DCP] "Qwen 4 QSA krijgt
 * decode-contextparallellisme ...", section "Wat de pull request daadwerkelijk
 * verandert"): the main K/V of each sequence is sharded by context over
 * nranks ranks while the selector (side cache, scores, top-K) is replicated;
 * each rank attends to the selected blocks it holds and the ranks' results are
 * merged by log-sum-exp.  Shard rule (a reading; the pages do not give one):
 * logical page P (64 tokens) of a sequence lives on rank (P / I) % nranks at
 * local page (P / (I*nranks)) * I + P % I, I = interleave_pages >= 1.  A
 * rank's K/V shard is a main-K/V-only cache group whose block table maps local
 * pages.
 *
 * qsa_dcp_localize_tokens -- the rank's view of a batch of appended tokens:
 *   seq_id_local[i] = seq_id[i] if the rank holds the token's page, else -1
 *   pos_local[i]    = its local position (local page * 64 + pos % 64), else 0
 * so qsa_append_kv on the shard writes exactly the rank's tokens.
 */
QSA_API int qsa_dcp_localize_tokens(const int32_t* seq_id, const int32_t* pos, int32_t n, int32_t nranks,
                            int32_t rank, int32_t interleave_pages, int32_t* seq_id_local, int32_t* pos_local,
                            void* stream);

/*
 * qsa_dcp_localize_selection -- the localisation step ([DCP] "the QSA
 * localization kernel"): for each query, the entries of the global selection
 * (sel/count from qsa_topk_blocks) that the rank holds, in order, as local block
 * indices (local page * 16 + j % 16), -1 padded to k; their number; and a
 * local position q_pos_local whose nb and tail make qsa_sparse_decode on the
 * shard attend to exactly those blocks, plus the trailing tokens when the rank
 * holds the page they are in (a rank holding nothing of a query gets count 0
 * and q_pos_local 3).  A query with q_pos < 0 is passed through with count 0.
 * Out-of-range entries set QSA_DEV_BAD_SEL and are dropped; a count outside
 * [0, min(k, nb)] sets QSA_DEV_BAD_COUNT and is clamped.
 *   sel, sel_local int32 [nq][k]; count, count_local, q_pos, q_pos_local int32 [nq]
 */
QSA_API int qsa_dcp_localize_selection(const int32_t* sel, const int32_t* count, const int32_t* q_pos, int32_t nq,
                               int32_t k, int32_t nranks, int32_t rank, int32_t interleave_pages,
                               int32_t* sel_local, int32_t* count_local, int32_t* q_pos_local,
                               int32_t* dev_status, void* stream);

/*
 * qsa_sparse_attention_noalloc -- qsa_sparse_decode then qsa_combine in one
 * call, for callers that cannot allocate device memory.  The pages have no
 * counterpart to this call; it is a convenience of this library.
 *
 * Some callers cannot call cudaMalloc: a serving engine that hands nearly all
 * device memory to its KV-cache pool at start-up, a plug-in whose host program
 * owns every device allocation, or a latency-critical loop that must not take
 * cudaMalloc's implicit device synchronisation.  This call needs no buffer
 * beyond its inputs and outputs: it keeps the split partials in a device array
 * of QSA_NOALLOC_SCRATCH_BYTES that libqsa reserves itself.  This is the one
 * exception to "the library allocates nothing": every GPU that loads the
 * library holds that array until the process exits.
 *
 * Arguments: as qsa_sparse_decode, with max_splits = the split bound that
 * qsa_decode_plan reports for (k, chunk_units); out and lse as qsa_combine
 * (bf16 [nq][hq][256] and fp32 [nq][hq]; out 8-byte aligned).
 * Limit: nq * S * hq * 1028 bytes of partials (S = that split bound) must fit
 * in QSA_NOALLOC_SCRATCH_BYTES; a larger call returns QSA_ERR_UNSUPPORTED and
 * enqueues nothing.
 * First call per device: it looks up the array's device address with that
 * device current and caches it.  Make the first call on each device before
 * any stream capture.
 * Sharing: all calls on a device use the same array, which keeps the last
 * call's contents (every partial the combine reads is rewritten by each call,
 * so nothing needs clearing).  Calls whose kernels can overlap on the GPU
 * (unordered streams, several host threads) race on the array: order them.
 */
#define QSA_NOALLOC_SCRATCH_BYTES (16u << 20)
QSA_API int qsa_sparse_attention_noalloc(const qsa_cache_t* cache, const void* q, int32_t nq, int32_t hq,
                                 const int32_t* q_seq, const int32_t* q_pos, const int32_t* sel,
                                 const int32_t* count, int32_t k, float scale, int32_t chunk_units, void* out,
                                 float* lse, int32_t* dev_status, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* QSA_H */
