// qsa_append_kv: scatter new tokens into the paged cache group and maintain the
// compressed indexer side cache (kc = fp32 sum of a micro-block's 4 indexer keys,
// stored BF16), continuing a block across calls through kc_partial.
//
// Source: [DCP] "Qwen 4 QSA krijgt decode-contextparallellisme ...", section
// "Wat de pull request daadwerkelijk verandert" (indexer compresses keys into
// micro-blocks of ratio 4; selector and main KV in one cache group; synthetic
// batches do not write the side caches) and [CANN] "Qwen4-Exp QSA komt naar
// Huawei's Ascend ...", section "Wat de pull request daadwerkelijk toevoegt"
// (-1 padding marks slots that must not be used).
//
// One kernel, one warp per token.  Every warp writes its token's K/V rows; a
// token at position 4j+3 whose whole block lies inside its run (the same
// sequence at consecutive positions in this call) writes kc row j.  The warp
// of a run's first token owns the run's open-block state: it finds the run's
// last token (warp-wide probes of 32 tokens, strides growing by 32), completes
// the run's first block when that block began in an earlier call (kc_partial
// + this call's tokens: kc row, or the new partial if the run ends inside it),
// and writes the running sum of the block left open at the run's end to
// kc_partial.  Only that warp reads or writes kc_partial[seq], so one launch
// orders every read of the old sum before its replacement.
#include "qsa_common.cuh"

namespace {

using namespace qsa;

constexpr int kWarps = 8;

struct AppendArgs {
  qsa_cache_t c;
  const __nv_bfloat16* k_new;
  const __nv_bfloat16* v_new;
  const __nv_bfloat16* kidx;
  const int32_t* seq_id;
  const int32_t* pos;
  int32_t n;
  int32_t* st;
};

// 8 BF16 values -> 8 FP8 e4m3 (round to nearest even, saturated to +-448), as 8 bytes
__device__ __forceinline__ uint2 bf16x8_to_e4m3x8(uint4 v) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
  uint32_t out[2];
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    uint16_t pr[2];
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const uint32_t x = w[2 * h + k];  // two BF16: low half = first element
      const float lo = __uint_as_float(x << 16), hi = __uint_as_float(x & 0xffff0000u);
      asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(pr[k]) : "f"(hi), "f"(lo));  // first element -> low byte
    }
    out[h] = (uint32_t)pr[0] | ((uint32_t)pr[1] << 16);
  }
  return make_uint2(out[0], out[1]);
}

// Number of this call's tokens directly before `tok` that belong to the same
// sequence at consecutive positions (at most `limit`).
__device__ __forceinline__ int run_before(const AppendArgs& a, int64_t tok, int seq, int p, int limit) {
  bool same[3];
#pragma unroll
  for (int k = 0; k < 3; ++k) {  // independent loads, then the prefix test
    const int64_t t = tok - k - 1;
    same[k] = k < limit && t >= 0 && a.seq_id[t] == seq && a.pos[t] == p - k - 1;
  }
  return same[0] ? (same[1] ? (same[2] ? 3 : 2) : 1) : 0;
}

// fp32 running sum (4 dims per lane) of tokens tok-m .. tok, starting from
// kc_partial[seq] when the block began before this call.
__device__ __forceinline__ float4 block_sum(const AppendArgs& a, int64_t tok, int seq, int m, bool from_partial,
                                            int lane) {
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (from_partial) acc = *reinterpret_cast<const float4*>(a.c.kc_partial + (size_t)seq * kIdxDim + lane * 4);
  for (int i = m; i >= 0; --i) {
    const uint2 raw = *reinterpret_cast<const uint2*>(a.kidx + (size_t)(tok - i) * kIdxDim + lane * 4);
    const float2 lo = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.x));
    const float2 hi = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&raw.y));
    acc.x = __fadd_rn(acc.x, lo.x);
    acc.y = __fadd_rn(acc.y, lo.y);
    acc.z = __fadd_rn(acc.z, hi.x);
    acc.w = __fadd_rn(acc.w, hi.y);
  }
  return acc;
}

// Is token t part of the run of sequence `seq` that starts at token `first`,
// position p0 (same sequence, consecutive positions)?
__device__ __forceinline__ bool in_run(const AppendArgs& a, int64_t t, int64_t first, int seq, int p0) {
  return t < a.n && a.seq_id[t] == seq && (int64_t)a.pos[t] == (int64_t)p0 + (t - first);
}

// Index of the last token of the run that starts at token `first` (warp-uniform).
// Runs are contiguous, so the probes that lie in the run form a prefix: grow the
// stride by 32 while all 32 probes are in, then narrow the first miss down.
__device__ __forceinline__ int64_t run_end(const AppendArgs& a, int64_t first, int seq, int p0, int lane) {
  int64_t base = first, stride = 1;
  for (;;) {
    const unsigned m = __ballot_sync(0xffffffffu, in_run(a, base + stride * (lane + 1), first, seq, p0));
    if (m != 0xffffffffu) {
      base += stride * (__ffs(~m) - 1);
      break;
    }
    base += stride * 32;
    stride *= 32;
  }
  while (stride > 1) {  // the probe at base + 32 * stride is outside the run
    stride /= 32;
    const unsigned m = __ballot_sync(0xffffffffu, in_run(a, base + stride * (lane + 1), first, seq, p0));
    base += stride * (__ffs(~m) - 1);
  }
  return base;
}

__global__ void __launch_bounds__(kWarps * 32) append_kernel(AppendArgs a) {
  // The dependents may launch once this kernel's predecessor has finished:
  // they read their query inputs before their own wait, and those may come
  // from the kernel before this one.
  pdl_wait_previous();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int64_t tok = (int64_t)blockIdx.x * kWarps + (threadIdx.x >> 5);
  if (tok >= a.n) return;
  const int seq = a.seq_id[tok];
  if (seq < 0) return;  // padding / synthetic token: writes nothing
  const int p = a.pos[tok];
  if (seq >= a.c.max_seqs) {
    if (lane == 0) flag(a.st, QSA_DEV_BAD_SEQ);
    return;
  }
  if (p < 0 || (int64_t)p >= (int64_t)a.c.max_pages_per_seq * kPage) {
    if (lane == 0) flag(a.st, QSA_DEV_BAD_POS);
    return;
  }
  const bool prev_same_seq = tok > 0 && a.seq_id[tok - 1] == seq;
  const bool run_start = !(prev_same_seq && a.pos[tok - 1] == p - 1);
  if (lane == 0 && prev_same_seq && a.pos[tok - 1] != p - 1) flag(a.st, QSA_DEV_BAD_ORDER);
  const int page = a.c.block_table[(int64_t)seq * a.c.max_pages_per_seq + p / kPage];
  if (page < 0 || page >= a.c.num_pages) {
    if (lane == 0) flag(a.st, QSA_DEV_BAD_PAGE);
    return;
  }
  const int slot = p % kPage;
  const int hkv = a.c.num_kv_heads;
  for (int h = 0; a.c.kv_pages && h < hkv; ++h) {  // no main K/V in a selector-only group
    const size_t unit = ((size_t)page * hkv + h) * kBlocksPerPage + slot / kRatio;  // micro-block of one KV head
    const int i = slot % kRatio;                                                     // its row
    const size_t src = ((size_t)tok * hkv + h) * kHeadDim + lane * 8;
    const uint4 kv8 = *reinterpret_cast<const uint4*>(a.k_new + src);
    const uint4 vv8 = *reinterpret_cast<const uint4*>(a.v_new + src);
    uint8_t* kv = static_cast<uint8_t*>(a.c.kv_pages);
    if (a.c.kv_dtype == QSA_KV_FP8_E4M3) {
      // [unit][K rows | V rows][256] bytes
      const size_t dst = unit * (2 * kRatio * kHeadDim) + (size_t)i * kHeadDim + lane * 8;
      *reinterpret_cast<uint2*>(kv + dst) = bf16x8_to_e4m3x8(kv8);
      *reinterpret_cast<uint2*>(kv + dst + kRatio * kHeadDim) = bf16x8_to_e4m3x8(vv8);
    } else {
      // [unit][4 dim atoms][8 rows: K 0-3, V 0-3][128 B]: the lane's 16 bytes are
      // chunk lane % 8 of atom lane / 8, stored at chunk position (lane % 8) ^ row
      const size_t base = unit * 4096 + (size_t)(lane >> 3) * 1024;
      const int kr = i, vr = kRatio + i;
      *reinterpret_cast<uint4*>(kv + base + kr * 128 + (((lane & 7) ^ kr) << 4)) = kv8;
      *reinterpret_cast<uint4*>(kv + base + vr * 128 + (((lane & 7) ^ vr) << 4)) = vv8;
    }
  }
  if (!a.c.kc_pages) return;
  __nv_bfloat16* kc_page = static_cast<__nv_bfloat16*>(a.c.kc_pages) + (size_t)page * kBlocksPerPage * kIdxDim;
  auto store_kc = [&](int blk_in_page, float4 acc) {
    uint2 out;
    out.x = pack_bf16(acc.x, acc.y);
    out.y = pack_bf16(acc.z, acc.w);
    *reinterpret_cast<uint2*>(kc_page + (size_t)blk_in_page * kIdxDim + lane * 4) = out;
  };
  // a block that lies wholly inside the run: its closing token writes kc
  if ((p & 3) == 3 && run_before(a, tok, seq, p, 3) == 3) store_kc(slot / kRatio, block_sum(a, tok, seq, 3, false, lane));
  if (!run_start) return;
  // ---- the run's open-block state (this warp only)
  const int64_t e = run_end(a, tok, seq, p, lane);
  const int pe = p + (int)(e - tok);  // position of the run's last token
  const int r0 = p & 3;
  const int closer = p + (3 - r0);    // position closing the run's first block
  if (r0 != 0) {  // the first block began in an earlier call: partial + this call's tokens
    const int last = min(pe, closer);
    const float4 acc = block_sum(a, tok + (last - p), seq, last - p, true, lane);
    if (pe >= closer)
      store_kc(slot / kRatio, acc);  // the block closes in this call (same page: blocks do not cross pages)
    else
      *reinterpret_cast<float4*>(a.c.kc_partial + (size_t)seq * kIdxDim + lane * 4) = acc;
  }
  if ((pe & 3) != 3 && (r0 == 0 || pe > closer)) {  // a block left open that began in this call
    const float4 acc = block_sum(a, e, seq, pe & 3, false, lane);
    *reinterpret_cast<float4*>(a.c.kc_partial + (size_t)seq * kIdxDim + lane * 4) = acc;
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" int qsa_append_kv(const qsa_cache_t* cache, const void* k_new, const void* v_new, const void* kidx_new,
                             const int32_t* seq_id, const int32_t* pos, int32_t n, int32_t* dev_status,
                             void* stream) {
  if (!cache || n < 0) return QSA_ERR_INVALID_ARG;
  if (n == 0) return QSA_OK;
  const qsa_cache_t& c = *cache;
  // a group may hold only the main K/V (kc_pages NULL) or only the side cache (kv_pages NULL)
  const bool has_kv = c.kv_pages != nullptr, has_kc = c.kc_pages != nullptr;
  if ((!has_kv && !has_kc) || !c.block_table || !seq_id || !pos) return QSA_ERR_INVALID_ARG;
  if (has_kv && (!k_new || !v_new)) return QSA_ERR_INVALID_ARG;
  if (has_kc && (!c.kc_partial || !kidx_new)) return QSA_ERR_INVALID_ARG;
  if (c.num_pages < 1 || c.max_seqs < 1 || c.max_pages_per_seq < 1 || c.num_kv_heads < 1) return QSA_ERR_INVALID_ARG;
  if (c.kv_dtype != QSA_KV_BF16 && c.kv_dtype != QSA_KV_FP8_E4M3) return QSA_ERR_UNSUPPORTED;
  if (has_kv && (!aligned16(c.kv_pages) || !aligned16(k_new) || !aligned16(v_new))) return QSA_ERR_INVALID_ARG;
  if (has_kc && (!aligned16(c.kc_partial) || (reinterpret_cast<uintptr_t>(c.kc_pages) & 7u) ||
                 (reinterpret_cast<uintptr_t>(kidx_new) & 7u)))
    return QSA_ERR_INVALID_ARG;
  AppendArgs a{c,
               static_cast<const __nv_bfloat16*>(k_new),
               static_cast<const __nv_bfloat16*>(v_new),
               static_cast<const __nv_bfloat16*>(kidx_new),
               seq_id,
               pos,
               n,
               dev_status};
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const unsigned grid = (unsigned)((n + kWarps - 1) / kWarps);
  return qsa_host::launch(append_kernel, dim3(grid), dim3(kWarps * 32), 0, s, a);
}
