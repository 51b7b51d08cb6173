// bwd_direct.cuh -- backward of the SiLU-gated RMSNorm for narrow rows, loading straight
// into registers (the dispatch rule's choice when each SM has very little data: measured on
// B200, 2048 x 128 backward 12.2 -> 10.4 us, 1024 x 128 12.3 -> 11.5 us, 16384 x 128
// checkpointed step 22.4 -> 20.9 us; equal at 65536 x 128, slower from ~1000 rows per SM).
//
// Rows of N <= 256: `TPR` threads per row, one 16-byte chunk (8 BF16 values) per thread.
// No shared-memory staging and no producer warp: every thread issues the 16-byte read-only
// loads of its chunks of dy, x and g (and the row's FP32 rstd) for kU rows before the first
// row sum, and CTAs walk the rows grid-stride with one trip count for every thread.  The
// per-row arithmetic and its order are those of gated_rmsnorm_bwd_kernel, so dx and dg are
// bitwise the same; each thread accumulates its dw columns over its rows in a fixed order,
// and at the end the CTA adds its row groups' accumulators in a fixed order into its FP32
// partial row, which the second pass sums like the staged kernel's.  Rows are assigned
// statically in both modes.
#pragma once

#include "args.h"
#include "device_common.cuh"

namespace gnorm {

template <int TPR, bool kWFp32>
__global__ void __launch_bounds__(kDirectThreads, kDirectBwdCtasPerSm)
    gated_rmsnorm_bwd_direct_kernel(const __grid_constant__ BwdArgs a) {
  static_assert(TPR <= 32, "rows must fit in a warp");
  constexpr int kU = kDirectBwdRows;
  constexpr int kGroups = kDirectThreads / TPR;
  // [kGroups, N] FP32 for the CTA's dw: N <= 8 TPR, so at most 8 KB.
  __shared__ __align__(16) float red[kDirectThreads * 8];
  const int group = threadIdx.x / TPR;
  const int lr = threadIdx.x % TPR;
  const int N = a.N;
  const int n8 = N >> 3;
  const bool cval = lr < n8;

  float2 wp[4], dwacc[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    wp[i] = splat2(0.f);
    dwacc[i] = splat2(0.f);
  }

  const long long groups = static_cast<long long>(gridDim.x) * kGroups;
  const long long gid = static_cast<long long>(blockIdx.x) * kGroups + group;
  const long long iters = (a.M + groups * kU - 1) / (groups * kU);

  long long row[kU];
  bool valid[kU];
  uint4 dyv[kU], xv[kU], gv[kU];
  float rv[kU];
  auto load_rows = [&](long long it) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      row[u] = (it * groups + gid) * kU + u;
      valid[u] = row[u] < a.M;
      dyv[u] = xv[u] = gv[u] = make_uint4(0u, 0u, 0u, 0u);
      if (valid[u] && cval) {
        dyv[u] = __ldg(reinterpret_cast<const uint4*>(a.dy + row[u] * a.lddy) + lr);
        xv[u] = __ldg(reinterpret_cast<const uint4*>(a.x + row[u] * a.ldx) + lr);
        gv[u] = __ldg(reinterpret_cast<const uint4*>(a.g + row[u] * a.ldg) + lr);
      }
    }
  };
  // The row's rstd is written by the previous kernel of a checkpointed step, so it is read
  // only after the dependency wait; dy, x and g are not, so with `prefetch` their first
  // loads may be issued before it.
  auto load_rstd = [&]() {
#pragma unroll
    for (int u = 0; u < kU; ++u) rv[u] = valid[u] ? a.rstd[row[u]] : 0.f;
  };
  if (a.prefetch && iters > 0) load_rows(0);
  grid_dependency_wait();
  allow_dependent_launch();
  if (cval) load_weight_pairs<kWFp32>(a.w, lr, wp);
  if (!a.prefetch && iters > 0) load_rows(0);
  if (iters > 0) load_rstd();

  for (long long it = 0; it < iters; ++it) {
    if (it > 0) {
      load_rows(it);
      load_rstd();
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const float r = rv[u];
      const float2 r2 = splat2(r);
      float2 dyp[4], xp[4], gp[4], dgp[4], ue[4], xh[4];
      bf16x8_to_pairs(dyv[u], dyp);
      bf16x8_to_pairs(xv[u], xp);
      bf16x8_to_pairs(gv[u], gp);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const float2 xhat = mul2(xp[i], r2);
        const float2 sgm = sigmoid2(gp[i]);
        const float2 silu = mul2(gp[i], sgm);
        const float2 t = mul2(dyp[i], xhat);                 // dy xhat
        ue[i] = mul2(dyp[i], mul2(wp[i], silu));              // dy (w s)
        xh[i] = xhat;
        if (valid[u]) dwacc[i] = fma2(t, silu, dwacc[i]);
        // sigmoid' = sigmoid (1 + g (1 - sigmoid))
        const float2 bracket = gate_grad_bracket(gp[i], sgm);
        dgp[i] = mul2(mul2(mul2(t, wp[i]), sgm), bracket);
      }
      if (valid[u] && cval)
        *(reinterpret_cast<uint4*>(a.dg + row[u] * a.lddg) + lr) = pairs_to_bf16x8(dgp);
      const float dot = row_sum<TPR>(chunk_dot(ue, xh), nullptr, group, lr, 0);
      const float2 nrc2 = splat2(-(r * (dot * a.inv_n)));
      float2 dxp[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) dxp[i] = fma2(nrc2, mul2(xp[i], r2), mul2(r2, ue[i]));
      if (valid[u] && cval)
        *(reinterpret_cast<uint4*>(a.dx + row[u] * a.lddx) + lr) = pairs_to_bf16x8(dxp);
    }
  }

  // This CTA's dw partial: its row groups' accumulators added in group order.
  if (cval) {
    float4* r4 = reinterpret_cast<float4*>(red + group * N + lr * 8);
    r4[0] = make_float4(dwacc[0].x, dwacc[0].y, dwacc[1].x, dwacc[1].y);
    r4[1] = make_float4(dwacc[2].x, dwacc[2].y, dwacc[3].x, dwacc[3].y);
  }
  __syncthreads();
  const int n4 = N >> 2;
  const float4* red4 = reinterpret_cast<const float4*>(red);
  float4* prow = reinterpret_cast<float4*>(a.partial + static_cast<size_t>(blockIdx.x) * N);
  for (int j4 = threadIdx.x; j4 < n4; j4 += kDirectThreads) {
    float4 acc = red4[j4];
#pragma unroll 4
    for (int gi = 1; gi < kGroups; ++gi) {
      const float4 v = red4[gi * n4 + j4];
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
    prow[j4] = acc;
  }
}

}  // namespace gnorm
