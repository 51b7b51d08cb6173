// noalloc.cu -- gnorm_bwd_noalloc: the backward with its scratch in a static device array.
//
// The backward needs scratch for its FP32 dw partials and two counters.  gnorm_bwd takes
// that scratch from the caller.  Some callers cannot allocate device memory at all: a
// runtime whose memory is owned up front by another allocator, code that must not hit
// cudaMalloc's implicit device synchronisation in a latency-critical loop, or plug-ins
// that only receive tensors.  For them this file provides one more entry point whose
// scratch is a fixed array in the library's own device memory (every GPU that loads the
// library holds kStaticScratchBytes for as long as the process runs).
//
// In host code the array's name is only a host-side stand-in, not a device address, so
// its device address is looked up once per device with cudaGetSymbolAddress (with that
// device current) and passed to the kernels.  Every call shares the array; the counters
// that must start at zero are cleared on the stream before each launch.  A bounded wait that
// gives up reports through the library's device error word, read by gnorm_device_error.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "args.h"
#include "gnorm.h"
#include "layout.h"
#include "launch.h"
#include "plan.h"

namespace gnorm {
namespace {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;  // 4 MiB per device
constexpr int kMaxStaticDevices = 64;

static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

struct StaticScratch {
  bool ready = false;
  unsigned char* ptr = nullptr;
  int num_sms = 0;
  int smem_optin = 0;
};

std::mutex g_static_mu;
StaticScratch g_static[kMaxStaticDevices];

// Once per device, with that device current: the array's device address and the device's
// SM count and shared-memory limit.
int static_scratch(StaticScratch* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GNORM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxStaticDevices) return GNORM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_static_mu);
  StaticScratch& s = g_static[dev];
  if (!s.ready) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_static_scratch) != cudaSuccess) return GNORM_ERR_CUDA;
    if (cudaDeviceGetAttribute(&s.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return GNORM_ERR_CUDA;
    if (cudaDeviceGetAttribute(&s.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
        cudaSuccess)
      return GNORM_ERR_CUDA;
    s.ptr = static_cast<unsigned char*>(p);
    s.ready = true;
  }
  *out = s;
  return GNORM_OK;
}

bool na_aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

bool na_overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || !na || !nb) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

}  // namespace
}  // namespace gnorm

using namespace gnorm;

extern "C" int gnorm_bwd_noalloc(const void* dy, const void* x, const void* g, const void* w,
                                 const float* rstd, void* dx, void* dg, void* dw, int dw_fp32,
                                 int deterministic, int64_t M, int64_t N, void* stream) {
  if (M < 0 || M > (int64_t(1) << 40) || N < 8 || N > GNORM_N_MAX || (N % 8) != 0)
    return GNORM_ERR_SHAPE;
  if (!dw) return GNORM_ERR_NULL;
  if (!na_aligned(dw, 16)) return GNORM_ERR_ALIGN;
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t dw_bytes = static_cast<size_t>(N) * (dw_fp32 ? 4 : 2);
  if (M == 0) return cudaMemsetAsync(dw, 0, dw_bytes, s) == cudaSuccess ? GNORM_OK : GNORM_ERR_CUDA;
  if (!dy || !x || !g || !w || !rstd || !dx || !dg) return GNORM_ERR_NULL;
  if (!na_aligned(dy, 16) || !na_aligned(x, 16) || !na_aligned(g, 16) || !na_aligned(w, 16) ||
      !na_aligned(rstd, 4) || !na_aligned(dx, 16) || !na_aligned(dg, 16))
    return GNORM_ERR_ALIGN;
  const size_t mat = static_cast<size_t>(M) * N * 2;
  const void* in_p[] = {dy, x, g, w, rstd};
  const size_t in_n[] = {mat, mat, mat, static_cast<size_t>(N) * 2, static_cast<size_t>(M) * 4};
  const void* out_p[] = {dx, dg, dw};
  const size_t out_n[] = {mat, mat, dw_bytes};
  for (int i = 0; i < 3; ++i) {
    for (int j = 0; j < 5; ++j)
      if (na_overlap(out_p[i], out_n[i], in_p[j], in_n[j])) return GNORM_ERR_ALIAS;
    for (int j = i + 1; j < 3; ++j)
      if (na_overlap(out_p[i], out_n[i], out_p[j], out_n[j])) return GNORM_ERR_ALIAS;
  }

  StaticScratch sc;
  int st = static_scratch(&sc);
  if (st != GNORM_OK) return st;
  gnorm_plan plan;
  st = make_plan(1, M, N, deterministic, sc.num_sms, sc.smem_optin, &plan);
  if (st != GNORM_OK) return st;
  if (workspace_bytes_for(plan, N) > kStaticScratchBytes) return GNORM_ERR_UNSUPPORTED;

  // A bounded wait that gives up inside these kernels sets its bit in the library's device
  // error word (itself a static device symbol), so gnorm_device_error reports it as it does
  // for every other entry point.
  unsigned* err_word = nullptr;
  st = device_error_word(&err_word);
  if (st != GNORM_OK) return st;

  // The schedule counter and the completion ticket start at zero.
  if (cudaMemsetAsync(sc.ptr, 0, kWorkspaceHeader, s) != cudaSuccess) return GNORM_ERR_CUDA;

  BwdArgs a;
  a.dy = static_cast<const uint16_t*>(dy);
  a.x = static_cast<const uint16_t*>(x);
  a.g = static_cast<const uint16_t*>(g);
  a.w = static_cast<const uint16_t*>(w);
  a.rstd = rstd;
  a.dx = static_cast<uint16_t*>(dx);
  a.dg = static_cast<uint16_t*>(dg);
  a.lddy = a.ldx = a.ldg = a.lddx = a.lddg = N;  // packed rows, BF16 weight
  a.w_fp32 = 0;
  a.partial = reinterpret_cast<float*>(sc.ptr + kWorkspaceHeader);
  a.dw = dw;
  a.work_counter = reinterpret_cast<unsigned long long*>(sc.ptr);
  a.ticket = reinterpret_cast<unsigned*>(sc.ptr + 8);
  a.M = M;
  a.N = static_cast<int>(N);
  a.inv_n = static_cast<float>(1.0 / static_cast<double>(N));
  a.rows_per_stage = plan.rows_per_stage;
  a.stages = plan.stages;
  a.num_blocks = plan.num_blocks;
  a.dynamic_schedule = plan.dynamic_schedule;
  a.fused_reduce = plan.fused_reduce;
  a.dw_fp32 = dw_fp32 ? 1 : 0;
  a.prefetch = 0;
  a.l2_prefetch = plan.l2_prefetch;
  a.err = err_word;
  const bool pdl = get_tuning().disable_pdl == 0;
  if (launch_bwd(plan, a, s, pdl) != cudaSuccess) return GNORM_ERR_CUDA;
  if (!plan.fused_reduce &&
      launch_dw_reduce(a.partial, plan.partials, a.N, dw, a.dw_fp32,
                       plan.dynamic_schedule ? a.work_counter : nullptr, s, pdl) != cudaSuccess)
    return GNORM_ERR_CUDA;
  return GNORM_OK;
}
