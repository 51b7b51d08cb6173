// bwd.cu -- instantiations and launcher of the backward kernel and of the dw second pass.
#include "bwd_direct.cuh"
#include "bwd_kernel.cuh"
#include "launch.h"

namespace gnorm {

template <int TPR, int CPT, bool kWFp32, bool kFusedFwd>
static cudaError_t launch_bwd_variant(const gnorm_plan& p, const BwdArgs& a, cudaStream_t stream,
                                      bool pdl) {
  const void* k =
      reinterpret_cast<const void*>(&gated_rmsnorm_bwd_kernel<TPR, CPT, kWFp32, kFusedFwd>);
  cudaError_t e = ensure_smem_limit(k, p.smem_bytes);
  if (e != cudaSuccess) return e;
  return launch_kernel(gated_rmsnorm_bwd_kernel<TPR, CPT, kWFp32, kFusedFwd>, p.grid,
                       consumer_threads_for(1, TPR, CPT) + 32, p.smem_bytes, stream, pdl, a);
}

template <int TPR, int CPT>
static cudaError_t launch_bwd_geometry(const gnorm_plan& p, const BwdArgs& a,
                                       cudaStream_t stream, bool pdl) {
  if (a.fused_fwd)
    return a.w_fp32 ? launch_bwd_variant<TPR, CPT, true, true>(p, a, stream, pdl)
                    : launch_bwd_variant<TPR, CPT, false, true>(p, a, stream, pdl);
  return a.w_fp32 ? launch_bwd_variant<TPR, CPT, true, false>(p, a, stream, pdl)
                  : launch_bwd_variant<TPR, CPT, false, false>(p, a, stream, pdl);
}

template <int TPR>
static cudaError_t launch_bwd_direct(const gnorm_plan& p, const BwdArgs& a, cudaStream_t stream,
                                     bool pdl) {
  if (a.w_fp32)
    return launch_kernel(gated_rmsnorm_bwd_direct_kernel<TPR, true>, p.grid, kDirectThreads, 0,
                         stream, pdl, a);
  return launch_kernel(gated_rmsnorm_bwd_direct_kernel<TPR, false>, p.grid, kDirectThreads, 0,
                       stream, pdl, a);
}

cudaError_t launch_bwd(const gnorm_plan& p, const BwdArgs& a, cudaStream_t stream, bool pdl) {
  if (p.direct_loads) {
    if (a.fused_fwd) return cudaErrorInvalidConfiguration;  // staged kernels only
    if (p.chunks_per_thread != 1) return cudaErrorInvalidConfiguration;
    switch (p.threads_per_row) {
      case 4: return launch_bwd_direct<4>(p, a, stream, pdl);
      case 8: return launch_bwd_direct<8>(p, a, stream, pdl);
      case 16: return launch_bwd_direct<16>(p, a, stream, pdl);
      case 32: return launch_bwd_direct<32>(p, a, stream, pdl);
      default: return cudaErrorInvalidConfiguration;
    }
  }
  const int key = p.threads_per_row * 8 + p.chunks_per_thread;
  switch (key) {
    case 4 * 8 + 1: return launch_bwd_geometry<4, 1>(p, a, stream, pdl);
    case 8 * 8 + 1: return launch_bwd_geometry<8, 1>(p, a, stream, pdl);
    case 16 * 8 + 1: return launch_bwd_geometry<16, 1>(p, a, stream, pdl);
    case 4 * 8 + 4: return launch_bwd_geometry<4, 4>(p, a, stream, pdl);
    case 8 * 8 + 2: return launch_bwd_geometry<8, 2>(p, a, stream, pdl);
    case 8 * 8 + 4: return launch_bwd_geometry<8, 4>(p, a, stream, pdl);
    case 16 * 8 + 2: return launch_bwd_geometry<16, 2>(p, a, stream, pdl);
    case 16 * 8 + 4: return launch_bwd_geometry<16, 4>(p, a, stream, pdl);
    case 32 * 8 + 1: return launch_bwd_geometry<32, 1>(p, a, stream, pdl);
    case 32 * 8 + 2: return launch_bwd_geometry<32, 2>(p, a, stream, pdl);
    case 32 * 8 + 4: return launch_bwd_geometry<32, 4>(p, a, stream, pdl);
    case 64 * 8 + 2: return launch_bwd_geometry<64, 2>(p, a, stream, pdl);
    case 64 * 8 + 4: return launch_bwd_geometry<64, 4>(p, a, stream, pdl);
    case 128 * 8 + 2: return launch_bwd_geometry<128, 2>(p, a, stream, pdl);
    case 256 * 8 + 2: return launch_bwd_geometry<256, 2>(p, a, stream, pdl);
    case 128 * 8 + 4: return launch_bwd_geometry<128, 4>(p, a, stream, pdl);
    case 256 * 8 + 4: return launch_bwd_geometry<256, 4>(p, a, stream, pdl);
    case 512 * 8 + 4: return launch_bwd_geometry<512, 4>(p, a, stream, pdl);
    default: return cudaErrorInvalidConfiguration;
  }
}

cudaError_t launch_dw_reduce(const float* partial, int P, int N, void* dw, int dw_fp32,
                             unsigned long long* work_counter, cudaStream_t stream, bool pdl) {
  const int col_quads = N / 4;
  const int grid = (col_quads + kReduceQuads - 1) / kReduceQuads;
  return launch_kernel(dw_reduce_kernel, grid, kReduceThreads, 0, stream, pdl, partial, P, N, dw,
                       dw_fp32, work_counter);
}

}  // namespace gnorm
