// device_common.cuh -- sm_100a building blocks shared by the gated-norm kernels:
// mbarrier pipeline waits with a time limit, 1-D TMA bulk copies (cp.async.bulk),
// programmatic dependent launch, BF16 packing and the logistic function.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "layout.h"

namespace gnorm {

// Bits of the device error word (see gnorm_device_error in include/gnorm.h).
constexpr unsigned kErrWaitFull = 1u;   // a consumer gave up waiting for copied rows
constexpr unsigned kErrWaitEmpty = 2u;  // the producer gave up waiting for a free stage
constexpr unsigned kErrSelfTest = 4u;   // the self-test's wait ran out, as it should

// A pipeline wait that has not completed after this long is abandoned.  A stage of a
// few tens of KB arrives in microseconds, so two seconds only trips on a real fault.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Makes barrier initialisation visible to the asynchronous (TMA) proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar_addr, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar_addr), "r"(parity)
      : "memory");
  return done != 0;
}

// The same test with a suspend-time hint: while the phase is incomplete the thread may sleep
// in hardware (woken when the phase completes, or after about `hint_ns`) instead of spinning,
// so waiting warps do not take issue slots from the warps that compute.
__device__ __forceinline__ bool mbar_try_wait_suspend(uint32_t bar_addr, uint32_t parity,
                                                      uint32_t hint_ns) {
  uint32_t done;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(done)
      : "r"(bar_addr), "r"(parity), "r"(hint_ns)
      : "memory");
  return done != 0;
}

// Suspend hint of the pipeline waits (ns): long against a stage's arrival, short against
// the waits' time limit, which is checked after every try.
constexpr uint32_t kWaitSuspendNs = 20000;

__device__ __forceinline__ unsigned long long globaltimer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Waits until the barrier phase with the given parity has completed, sleeping between tries
// (suspend hint).  Gives up after `limit_ns` (or 2^24 tries, whichever comes first), sets
// `err_bit` in the device error word and returns false; the caller then stops its loop and
// exits.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, unsigned* err_word,
                                          unsigned err_bit,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  const uint32_t a = smem_u32(bar);
  if (mbar_try_wait(a, parity)) return true;
  const unsigned long long t0 = globaltimer_ns();
  const uint32_t hint = limit_ns < 8ull * kWaitSuspendNs
                            ? static_cast<uint32_t>(limit_ns / 8) + 1u
                            : kWaitSuspendNs;
  for (uint32_t round = 0; round < (1u << 24); ++round) {
    if (mbar_try_wait_suspend(a, parity, hint)) return true;
    if (globaltimer_ns() - t0 > limit_ns) break;
  }
  atomicOr(err_word, err_bit);
  return false;
}

// 1-D bulk copy global -> shared through the TMA unit; completion is counted in bytes on
// `bar`.  Both addresses must be 16-byte aligned and `bytes` a multiple of 16.  One
// receiver: the source is always this GPU's memory and only this CTA receives it.
__device__ __forceinline__ void bulk_copy_g2s(void* smem_dst, const void* gmem_src,
                                              uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Tiled 2-D TMA load of the box at (c0, c1) of `map` into shared memory (128-byte aligned),
// completion counted in bytes on `bar`; only this CTA receives the box.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map, int c0, int c1,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
          "r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
      : "memory");
}

// Warms L2 with `bytes` of global memory (no shared memory, registers or barrier involved).
__device__ __forceinline__ void bulk_prefetch_l2(const void* gmem, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(gmem), "r"(bytes) : "memory");
}

// Programmatic dependent launch: wait for the previous grid on the stream to complete
// (and its memory to be visible) / allow the next grid to begin launching.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;" ::: "memory");
}
__device__ __forceinline__ void allow_dependent_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

__device__ __forceinline__ void named_barrier_sync(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Eight BF16 values in a 16-byte word -> FP32 (exact: BF16 is the high half of FP32).
__device__ __forceinline__ void bf16x8_to_f32(const uint4 v, float f[8]) {
  f[0] = __uint_as_float(v.x << 16);
  f[1] = __uint_as_float(v.x & 0xffff0000u);
  f[2] = __uint_as_float(v.y << 16);
  f[3] = __uint_as_float(v.y & 0xffff0000u);
  f[4] = __uint_as_float(v.z << 16);
  f[5] = __uint_as_float(v.z & 0xffff0000u);
  f[6] = __uint_as_float(v.w << 16);
  f[7] = __uint_as_float(v.w & 0xffff0000u);
}

// Two FP32 -> two BF16 (round to nearest even), `lo` at the lower address.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<uint32_t*>(&h);
}

__device__ __forceinline__ uint4 f32x8_to_bf16(const float f[8]) {
  uint4 v;
  v.x = pack_bf16x2(f[0], f[1]);
  v.y = pack_bf16x2(f[2], f[3]);
  v.z = pack_bf16x2(f[4], f[5]);
  v.w = pack_bf16x2(f[6], f[7]);
  return v;
}

// Posts the bytes a stage's bulk copies will deliver, without arriving.
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// 4-byte asynchronous copy global -> shared (LDGSTS), and an arrive on `bar` that fires
// once all of this thread's earlier asynchronous copies have landed (the arrival was
// counted in the barrier's initial count, hence .noinc).
__device__ __forceinline__ void async_copy_4(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void async_copies_arrive(uint64_t* bar) {
  asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// ---- packed FP32 pairs (sm_100 FFMA2 / FMUL2 / FADD2: two lanes of FP32 per instruction)
__device__ __forceinline__ float2 mul2(float2 a, float2 b) { return __fmul2_rn(a, b); }
__device__ __forceinline__ float2 add2(float2 a, float2 b) { return __fadd2_rn(a, b); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) { return __ffma2_rn(a, b, c); }
__device__ __forceinline__ float2 splat2(float v) { return make_float2(v, v); }

// Eight BF16 values in a 16-byte word -> four FP32 pairs (element 2i in .x, 2i+1 in .y).
__device__ __forceinline__ void bf16x8_to_pairs(const uint4 v, float2 p[4]) {
  p[0] = make_float2(__uint_as_float(v.x << 16), __uint_as_float(v.x & 0xffff0000u));
  p[1] = make_float2(__uint_as_float(v.y << 16), __uint_as_float(v.y & 0xffff0000u));
  p[2] = make_float2(__uint_as_float(v.z << 16), __uint_as_float(v.z & 0xffff0000u));
  p[3] = make_float2(__uint_as_float(v.w << 16), __uint_as_float(v.w & 0xffff0000u));
}

__device__ __forceinline__ uint4 pairs_to_bf16x8(const float2 p[4]) {
  uint4 v;
  v.x = pack_bf16x2(p[0].x, p[0].y);
  v.y = pack_bf16x2(p[1].x, p[1].y);
  v.z = pack_bf16x2(p[2].x, p[2].y);
  v.w = pack_bf16x2(p[3].x, p[3].y);
  return v;
}

__device__ __forceinline__ float ex2_approx(float v) {
  float r;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}
__device__ __forceinline__ float rcp_approx(float v) {
  float r;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r) : "f"(v));
  return r;
}

// Logistic function of a pair, sigma(t) = 1 / (1 + 2^(-t log2(e))): the MUFU exp2 and
// reciprocal approximations (each a few FP32 ulp) with the scaling and the +1 as packed
// pair instructions.  For t < -88 the sum overflows to +inf and sigma = 0 (true value
// below 2^-126); for large t, sigma = 1.
constexpr float kLog2e = 1.4426950408889634f;
__device__ __forceinline__ float2 sigmoid2(float2 t) {
  const float2 z = mul2(t, splat2(-kLog2e));
  float2 d = make_float2(ex2_approx(z.x), ex2_approx(z.y));
  d = add2(d, splat2(1.0f));
  return make_float2(rcp_approx(d.x), rcp_approx(d.y));
}

// The bracket of the gate's derivative, 1 + g (1 - sigmoid(g)), from the pair's sigmoid:
// 1 - sigmoid, then one fused multiply-add.  (Written as (1 + g) - g sigmoid(g) it would
// lose the 1 once g >= 2^24, where 1 + g rounds to g in FP32 and sigmoid(g) is exactly 1;
// this form keeps it, and gives NaN for g = +inf as the definition does.)
__device__ __forceinline__ float2 gate_grad_bracket(float2 g, float2 sgm) {
  const float2 one = splat2(1.0f);
  return fma2(g, fma2(sgm, splat2(-1.0f), one), one);
}

// Row reductions in an order that does not depend on the row geometry.  Each 16-byte chunk
// (8 values, 4 pairs) reduces to one partial in a fixed order; a thread's CPT chunks
// (chunk indices lr, lr + TPR, ..., lr + (CPT - 1) TPR) are then combined by halving, which
// is exactly what the first log2(CPT) levels of a butterfly over CPT x TPR one-chunk threads
// would add.  So a geometry with CPT chunks per thread and one with a single chunk per
// thread produce bitwise the same row sums, and the direct-load and staged kernels the
// same results.
__device__ __forceinline__ float chunk_dot(const float2 a[4], const float2 b[4]) {
  float2 s = mul2(a[0], b[0]);
#pragma unroll
  for (int i = 1; i < 4; ++i) s = fma2(a[i], b[i], s);
  return s.x + s.y;
}

template <int CPT>
__device__ __forceinline__ float combine_chunks(float part[CPT]) {
#pragma unroll
  for (int h = CPT / 2; h >= 1; h /= 2) {
#pragma unroll
    for (int k = 0; k < h; ++k) part[k] = part[k] + part[k + h];
  }
  return part[0];
}

// Sum over the `TPR` consecutive threads that share a row.  TPR <= 32: butterfly
// shuffles inside the warp (every lane of the warp must call).  TPR > 32: butterfly per
// warp, then the warps of the row exchange partials through shared-memory slots guarded
// by a named barrier; `slot` alternates between two buffers from row to row so a fast
// warp cannot overwrite slots a slow warp still reads.  The order of additions is fixed,
// and every thread of the row ends with the bitwise same value.
template <int TPR>
__device__ __forceinline__ float row_sum(float v, float* red_slots, int group, int lane_in_row,
                                         int slot) {
#pragma unroll
  for (int off = (TPR < 32 ? TPR : 32) / 2; off > 0; off >>= 1)
    v += __shfl_xor_sync(0xffffffffu, v, off);
  if constexpr (TPR > 32) {
    constexpr int kWarps = TPR / 32;
    const int wig = lane_in_row >> 5;  // warp index inside the row's thread group
    float* slots = red_slots + (group * 2 + slot) * kWarps;
    if ((lane_in_row & 31) == 0) slots[wig] = v;
    named_barrier_sync(1 + group, TPR);
    v = slots[0];
#pragma unroll
    for (int i = 1; i < kWarps; ++i) v += slots[i];
  }
  return v;
}

// Rows [r0, r0 + rows) of a tensor with row stride `ld` elements into shared memory as packed
// rows of N BF16 values.  Packed rows (ld == N) are one bulk copy issued by lane 0; strided
// rows are one bulk copy per row, spread over the warp's 32 lanes.  Every byte lands on
// `bar`, whose expected byte count the caller has already posted.
// A full block of a strided tensor that has a 2-D tiled tensor map (box N x R) is one tiled
// copy at coordinates (column 0, row r0): the innermost coordinate is 0, so 16-byte aligned.
__device__ __forceinline__ void copy_row_block(uint8_t* dst, const uint16_t* src, long long ld,
                                               int N, long long r0, int rows, int R,
                                               const CUtensorMap* map, uint64_t* bar,
                                               int lane) {
  const uint32_t row_bytes = static_cast<uint32_t>(N) * 2u;
  if (ld == N) {
    if (lane == 0) bulk_copy_g2s(dst, src + r0 * N, static_cast<uint32_t>(rows) * row_bytes, bar);
  } else if (map != nullptr && rows == R) {
    if (lane == 0) tma_load_2d(dst, map, 0, static_cast<int>(r0), bar);
  } else {
    for (int i = lane; i < rows; i += 32)
      bulk_copy_g2s(dst + static_cast<size_t>(i) * row_bytes, src + (r0 + i) * ld, row_bytes, bar);
  }
}

// This thread's 8 weights of chunk c as FP32 pairs, from a BF16 or (kWFp32) FP32 weight
// vector.  The weight type is a compile-time choice: a runtime branch here measurably slowed
// the wide-row backward.
template <bool kWFp32>
__device__ __forceinline__ void load_weight_pairs(const void* w, int c, float2 p[4]) {
  if constexpr (kWFp32) {
    const float4* w4 = reinterpret_cast<const float4*>(w) + 2 * c;
    const float4 a = w4[0], b = w4[1];
    p[0] = make_float2(a.x, a.y);
    p[1] = make_float2(a.z, a.w);
    p[2] = make_float2(b.x, b.y);
    p[3] = make_float2(b.z, b.w);
  } else {
    bf16x8_to_pairs(reinterpret_cast<const uint4*>(w)[c], p);
  }
}

}  // namespace gnorm
