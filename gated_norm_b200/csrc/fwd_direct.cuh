// fwd_direct.cuh -- forward of the SiLU-gated RMSNorm for narrow rows, loading straight
// into registers (the dispatch rule's choice when each SM has little data).
//
// Rows of N <= 256: `TPR` threads per row, one 16-byte chunk (8 BF16 values) per thread.
// No shared-memory staging and no producer warp: every thread issues the 16-byte read-only
// loads of its chunks of x and g for kU rows before the first row sum, so with 32 warps per
// SM each SM has 64 rows in flight from the first cycles on; the row sums are shuffles
// inside the warp.  CTAs walk the rows grid-stride, the same trip count for every thread.
// With few rows per SM this starts streaming sooner and ends with a shorter tail than the
// staged pipeline of gated_rmsnorm_fwd_kernel (measured on B200: 65536 x 128 forward 17.8
// -> 17.0 us, checkpointed step 45.1 -> 43.8 us); with many rows per SM the staged pipeline
// is faster (368640 x 128 forward 54.6 vs 55.3 us), so the dispatch rule picks this kernel
// in the latency tier only.  The arithmetic and its order per row are those of
// gated_rmsnorm_fwd_kernel, so y and rstd are bitwise the same.
#pragma once

#include "args.h"
#include "device_common.cuh"

namespace gnorm {

template <int TPR, bool kWFp32>
__global__ void __launch_bounds__(kDirectThreads, kDirectCtasPerSm)
    gated_rmsnorm_fwd_direct_kernel(const __grid_constant__ FwdArgs a) {
  static_assert(TPR <= 32, "rows must fit in a warp");
  constexpr int kU = kDirectRows;
  constexpr int kGroups = kDirectThreads / TPR;
  const int group = threadIdx.x / TPR;
  const int lr = threadIdx.x % TPR;
  const int n8 = a.N >> 3;
  const bool cval = lr < n8;

  float2 wp[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) wp[i] = splat2(0.f);

  const long long groups = static_cast<long long>(gridDim.x) * kGroups;
  const long long gid = static_cast<long long>(blockIdx.x) * kGroups + group;
  const long long iters = (a.M + groups * kU - 1) / (groups * kU);

  long long row[kU];
  bool valid[kU];
  uint4 xv[kU], gv[kU];
  auto load_rows = [&](long long it) {
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      row[u] = (it * groups + gid) * kU + u;
      valid[u] = row[u] < a.M;
      xv[u] = make_uint4(0u, 0u, 0u, 0u);
      gv[u] = make_uint4(0u, 0u, 0u, 0u);
      if (valid[u] && cval) {
        xv[u] = __ldg(reinterpret_cast<const uint4*>(a.x + row[u] * a.ldx) + lr);
        gv[u] = __ldg(reinterpret_cast<const uint4*>(a.g + row[u] * a.ldg) + lr);
      }
    }
  };
  // x and g are not written by the previous kernel when `prefetch` is set: the first rows'
  // loads may start before the dependency wait.
  if (a.prefetch && iters > 0) load_rows(0);
  grid_dependency_wait();
  allow_dependent_launch();
  if (cval) load_weight_pairs<kWFp32>(a.w, lr, wp);
  if (!a.prefetch && iters > 0) load_rows(0);

  for (long long it = 0; it < iters; ++it) {
    if (it > 0) load_rows(it);
    float r[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      float2 xp[4];
      bf16x8_to_pairs(xv[u], xp);
      const float ss = row_sum<TPR>(chunk_dot(xp, xp), nullptr, group, lr, 0);
      r[u] = rsqrtf(fmaf(ss, a.inv_n, a.eps));
      if (valid[u] && lr == 0) a.rstd[row[u]] = r[u];
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      if (valid[u] && cval) {
        float2 xp[4], gp[4], yp[4];
        bf16x8_to_pairs(xv[u], xp);
        bf16x8_to_pairs(gv[u], gp);
        const float2 r2 = splat2(r[u]);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float2 silu = mul2(gp[i], sigmoid2(gp[i]));
          yp[i] = mul2(mul2(xp[i], r2), mul2(wp[i], silu));
        }
        *(reinterpret_cast<uint4*>(a.y + row[u] * a.ldy) + lr) = pairs_to_bf16x8(yp);
      }
    }
  }
}

}  // namespace gnorm
