// Shared device helpers for libqsa (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "../../include/qsa.h"

#define QSA_DEVINL __device__ __forceinline__

namespace qsa {

constexpr int kHeadDim = QSA_HEAD_DIM;   // 256
constexpr int kIdxHeads = QSA_IDX_HEADS; // 8
constexpr int kIdxDim = QSA_IDX_DIM;     // 128
constexpr int kRatio = QSA_RATIO;        // 4
constexpr int kPage = QSA_PAGE_TOKENS;   // 64
constexpr int kBlocksPerPage = QSA_BLOCKS_PER_PAGE;

// ---------------------------------------------------------------- status

QSA_DEVINL void flag(int32_t* st, int bits) {
  if (st) atomicOr(st, bits);
}

// ---------------------------------------------------------------- loads

// 16-byte streaming load: read-only path, no L1 allocation, 256-B L2 prefetch.
QSA_DEVINL uint4 ldg_stream(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}

QSA_DEVINL uint4 ldg_nc(const void* p) {
  uint4 r;
  asm volatile("ld.global.nc.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "l"(p));
  return r;
}

QSA_DEVINL uint4 lds128(uint32_t saddr) {
  uint4 r;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(saddr));
  return r;
}

QSA_DEVINL uint2 lds64(uint32_t saddr) {
  uint2 r;
  asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(saddr));
  return r;
}

QSA_DEVINL void sts128(uint32_t saddr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(saddr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w));
}

QSA_DEVINL uint32_t smem_u32(const void* p) { return static_cast<uint32_t>(__cvta_generic_to_shared(p)); }

// ---------------------------------------------------------------- tensor cores

// D(16x8 fp32) += A(16x16 bf16, row) * B(16x8 bf16, col)
QSA_DEVINL void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                               uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// D(16x8 fp32) += A(16x16 fp16, row) * B(16x8 fp16, col)
QSA_DEVINL void mma_f16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3, uint32_t b0,
                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Four FP8 e4m3 bytes (first element in the low byte) -> four FP16, exact
// (every e4m3 value is an FP16 value): .x = elements 0, 1 and .y = 2, 3, each
// with the lower-indexed element in the low half.
QSA_DEVINL uint2 e4m3x4_to_f16x4(uint32_t b) {
  uint2 r;
  asm("{\n\t.reg .b16 l, h;\n\tmov.b32 {l, h}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, l;\n\tcvt.rn.f16x2.e4m3x2 %1, h;\n\t}"
      : "=r"(r.x), "=r"(r.y)
      : "r"(b));
  return r;
}

// Eight e4m3 bytes -> eight FP16 laid out like eight BF16 loaded as a uint4.
QSA_DEVINL uint4 e4m3x8_to_f16x8(uint2 v) {
  const uint2 a = e4m3x4_to_f16x4(v.x), b = e4m3x4_to_f16x4(v.y);
  return make_uint4(a.x, a.y, b.x, b.y);
}

// FP16x2 of (lo, hi), rounded to nearest even, finite values clamped to +-65504.
QSA_DEVINL uint32_t pack_f16_sat(float lo, float hi) {
  lo = fminf(fmaxf(lo, -65504.f), 65504.f);
  hi = fminf(fmaxf(hi, -65504.f), 65504.f);
  __half2 v = __floats2half2_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&v);
}

QSA_DEVINL uint32_t pack_bf16(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // .x = lo (low half), .y = hi
  return *reinterpret_cast<uint32_t*>(&v);
}

// (a, b) -> hi = BF16x2(a, b) and lo = BF16x2 of the rounding residuals, so that
// hi + lo carries about 17 significant bits of each value.
QSA_DEVINL void split_bf16(float a, float b, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16(a, b);
  const float ah = __uint_as_float(hi << 16);
  const float bh = __uint_as_float(hi & 0xffff0000u);
  lo = pack_bf16(a - ah, b - bh);
}

// ---------------------------------------------------------------- split merge
// Log-sum-exp merge of split partials, in split order: with M = max lse,
// L += e_s and acc += e_s * x_s for e_s = exp(lse_s - M), empty splits
// (lse = -inf) skipped.  The separate combine and the attention kernel's
// in-kernel merge both call this, so the two forms give identical bits.
constexpr int kMergeBatch = 8;  // splits whose loads are issued together

QSA_DEVINL void merge_splits(const float* v, const float4* x, int n, float M, float& L, float4& acc) {
#pragma unroll
  for (int s = 0; s < n; ++s) {
    if (v[s] == -INFINITY) continue;
    const float e = expf(v[s] - M);
    L += e;
    acc.x += e * x[s].x;
    acc.y += e * x[s].y;
    acc.z += e * x[s].z;
    acc.w += e * x[s].w;
  }
}

// One thread's 4 dims of one (query, head): the merged output (zero when every
// split is empty) and the merged lse (-inf then).  Up to kMergeBatch splits,
// every lse value and partial row is requested at once; more take a loop.
// `lse_at(s)` / `row_at(s)` load split s.
template <class LseAt, class RowAt>
QSA_DEVINL float4 merge_row(int n, LseAt lse_at, RowAt row_at, float& lse_out) {
  float M = -INFINITY, L = 0.f;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (n <= kMergeBatch) {
    float v[kMergeBatch];
    float4 x[kMergeBatch];
#pragma unroll
    for (int s = 0; s < kMergeBatch; ++s) v[s] = s < n ? lse_at(s) : -INFINITY;
#pragma unroll
    for (int s = 0; s < kMergeBatch; ++s)  // rows of empty splits are loaded but not used
      x[s] = s < n ? row_at(s) : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int s = 0; s < kMergeBatch; ++s) M = fmaxf(M, v[s]);
    if (M != -INFINITY) merge_splits(v, x, kMergeBatch, M, L, acc);
  } else {
    for (int s = 0; s < n; ++s) M = fmaxf(M, lse_at(s));
    if (M != -INFINITY) {
      for (int s = 0; s < n; ++s) {
        const float v = lse_at(s);
        const float4 x = v == -INFINITY ? make_float4(0.f, 0.f, 0.f, 0.f) : row_at(s);
        merge_splits(&v, &x, 1, M, L, acc);
      }
    }
  }
  if (M == -INFINITY) {
    lse_out = -INFINITY;
    return make_float4(0.f, 0.f, 0.f, 0.f);
  }
  const float inv = 1.f / L;
  lse_out = M + logf(L);
  return make_float4(acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv);
}

// ---------------------------------------------------------------- mbarrier + bulk copy

QSA_DEVINL void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}

QSA_DEVINL void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory"); }

QSA_DEVINL void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}

QSA_DEVINL void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

QSA_DEVINL bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

QSA_DEVINL uint64_t global_timer_ns() {
  uint64_t t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait on an mbarrier phase.  Returns false when `limit_ns` of wall time
// passed without the phase completing.
QSA_DEVINL bool mbar_wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_timer_ns();
  for (uint32_t it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u && global_timer_ns() - t0 > limit_ns) return false;
  }
}

// 1-D bulk async copy global -> shared, completion signalled on `bar` as tx bytes.
// Addresses 16-byte aligned, bytes a multiple of 16.
QSA_DEVINL void bulk_g2s(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar, uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], "
      "%4;" ::"r"(dst),
      "l"(src), "r"(bytes), "r"(bar), "l"(policy)
      : "memory");
}

// 16-byte async copy global -> shared (L2 only, cache hint); 16-byte aligned.
QSA_DEVINL void cp_async16(uint32_t dst, const void* src, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "l"(policy)
               : "memory");
}

// Arrive on `bar` once every cp.async this thread issued so far has landed; the
// arrival counts toward the barrier's expected count (noinc).
QSA_DEVINL void cp_async_arrive_noinc(uint32_t bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(bar) : "memory");
}

QSA_DEVINL void cp_async_wait_all() { asm volatile("cp.async.wait_all;" ::: "memory"); }

// Fire-and-forget prefetch of [src, src+bytes) into L2 (16-byte aligned, multiple of 16).
QSA_DEVINL void prefetch_l2(const void* src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

QSA_DEVINL uint64_t l2_policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// Programmatic dependent launch.  Every library kernel is launched so that the
// next kernel on the stream may start while it runs: a kernel first lets its
// dependents be scheduled, then waits until the previous kernel on the stream
// has finished and its writes are visible, before it reads or writes any
// buffer that kernel touches.  Outside such a launch both are no-ops.
QSA_DEVINL void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
QSA_DEVINL void pdl_wait_previous() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

QSA_DEVINL void named_bar_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// order-preserving map fp32 -> uint32 (larger float -> larger key; equal
// floats -> equal keys: -0 and +0 are the same score and share +0's key, so
// they tie and the lower block index wins)
QSA_DEVINL uint32_t float_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// The float bound of a key threshold: float_key(x) >= T  <=>  x >= key_floor(T)
// for every non-NaN x, when T lies between the keys of -inf and +inf.  For T in
// the upper half (x >= +0) it is the float whose bits are T without the top
// bit; below, the negative float whose key is T.  -0 >= +0 holds for floats,
// as it does for the keys.
QSA_DEVINL float key_floor(uint32_t T) {
  return (T & 0x80000000u) ? __uint_as_float(T & 0x7fffffffu) : __uint_as_float(~T);
}

}  // namespace qsa

// host-side helpers
namespace qsa_host {
// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel on `stream` finishes (it waits for it on the device).
template <typename... KArgs, typename... Args>
inline int launch(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  if (cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) != cudaSuccess) {
    (void)cudaGetLastError();
    return QSA_ERR_CUDA;
  }
  return QSA_OK;
}

inline int launch_status() {
  cudaError_t e = cudaGetLastError();
  return e == cudaSuccess ? QSA_OK : QSA_ERR_CUDA;
}
}  // namespace qsa_host
