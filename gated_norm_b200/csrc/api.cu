// api.cu -- the extern "C" entry points of libgnorm (declared in include/gnorm.h).
//
// Every argument is checked on the host before anything is enqueued; a bad argument
// returns a gnorm_status and launches nothing.  Entry points never synchronise and never
// allocate; they enqueue kernels on the caller's stream.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "args.h"
#include "gnorm.h"
#include "layout.h"
#include "launch.h"
#include "plan.h"

namespace gnorm {

// Bits set by kernels whose bounded pipeline waits gave up (see gnorm_device_error).
__device__ unsigned int g_device_error_word = 0u;

namespace {

constexpr int64_t kMaxRows = int64_t(1) << 40;
constexpr int kMaxDevices = 64;

struct DeviceInfo {
  bool ready = false;
  int num_sms = 0;
  int smem_optin = 0;
  unsigned* err_word = nullptr;
};

std::mutex g_dev_mu;
DeviceInfo g_dev[kMaxDevices];

int device_info(DeviceInfo* out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GNORM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxDevices) return GNORM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_dev_mu);
  DeviceInfo& d = g_dev[dev];
  if (!d.ready) {
    if (cudaDeviceGetAttribute(&d.num_sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
      return GNORM_ERR_CUDA;
    if (cudaDeviceGetAttribute(&d.smem_optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev) !=
        cudaSuccess)
      return GNORM_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_device_error_word) != cudaSuccess) return GNORM_ERR_CUDA;
    d.err_word = static_cast<unsigned*>(p);
    d.ready = true;
  }
  *out = d;
  return GNORM_OK;
}

struct Span {
  const void* p;
  size_t bytes;
};

bool overlaps(const Span& a, const Span& b) {
  if (a.p == nullptr || b.p == nullptr || a.bytes == 0 || b.bytes == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), a1 = a0 + a.bytes;
  const uintptr_t b0 = reinterpret_cast<uintptr_t>(b.p), b1 = b0 + b.bytes;
  return a0 < b1 && b0 < a1;
}

// Every output span against every input span and every other output span.
bool any_alias(const Span* in, int n_in, const Span* out, int n_out) {
  for (int i = 0; i < n_out; ++i) {
    for (int j = 0; j < n_in; ++j)
      if (overlaps(out[i], in[j])) return true;
    for (int j = i + 1; j < n_out; ++j)
      if (overlaps(out[i], out[j])) return true;
  }
  return false;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_shape(int64_t M, int64_t N) {
  if (M < 0 || M > kMaxRows) return GNORM_ERR_SHAPE;
  if (N < 8 || N > GNORM_N_MAX || (N % 8) != 0) return GNORM_ERR_SHAPE;
  return GNORM_OK;
}

bool use_pdl() { return get_tuning().disable_pdl == 0; }

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// `prefetch`: the previous kernel on the stream is known to write none of this call's
// inputs, so the kernel may start copying them before that kernel has finished.
int enqueue_fwd(const DeviceInfo& d, const void* x, const void* g, const void* w, float eps,
                void* y, float* rstd, int64_t M, int64_t N, cudaStream_t stream,
                bool prefetch = false) {
  gnorm_plan plan;
  int st = make_plan(0, M, N, 1, d.num_sms, d.smem_optin, &plan);
  if (st != GNORM_OK) return st;
  FwdArgs a;
  a.x = static_cast<const uint16_t*>(x);
  a.g = static_cast<const uint16_t*>(g);
  a.w = static_cast<const uint16_t*>(w);
  a.y = static_cast<uint16_t*>(y);
  a.rstd = rstd;
  a.M = M;
  a.N = static_cast<int>(N);
  a.eps = eps;
  a.inv_n = static_cast<float>(1.0 / static_cast<double>(N));
  a.rows_per_stage = plan.rows_per_stage;
  a.stages = plan.stages;
  a.num_blocks = plan.num_blocks;
  a.prefetch = prefetch ? 1 : 0;
  a.l2_prefetch = plan.l2_prefetch;
  a.err = d.err_word;
  if (launch_fwd(plan, a, stream, use_pdl()) != cudaSuccess) return GNORM_ERR_CUDA;
  return GNORM_OK;
}

int enqueue_bwd(const DeviceInfo& d, const void* dy, const void* x, const void* g,
                const void* w, const float* rstd, void* dx, void* dg, void* dw, int dw_fp32,
                int deterministic, int64_t M, int64_t N, void* ws, cudaStream_t stream,
                bool prefetch = false) {
  gnorm_plan plan;
  int st = make_plan(1, M, N, deterministic, d.num_sms, d.smem_optin, &plan);
  if (st != GNORM_OK) return st;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  BwdArgs a;
  a.dy = static_cast<const uint16_t*>(dy);
  a.x = static_cast<const uint16_t*>(x);
  a.g = static_cast<const uint16_t*>(g);
  a.w = static_cast<const uint16_t*>(w);
  a.rstd = rstd;
  a.dx = static_cast<uint16_t*>(dx);
  a.dg = static_cast<uint16_t*>(dg);
  a.partial = reinterpret_cast<float*>(wsb + kWorkspaceHeader);
  a.dw = dw;
  a.work_counter = reinterpret_cast<unsigned long long*>(wsb);
  a.ticket = reinterpret_cast<unsigned*>(wsb + 8);
  a.M = M;
  a.N = static_cast<int>(N);
  a.inv_n = static_cast<float>(1.0 / static_cast<double>(N));
  a.rows_per_stage = plan.rows_per_stage;
  a.stages = plan.stages;
  a.num_blocks = plan.num_blocks;
  a.dynamic_schedule = plan.dynamic_schedule;
  a.fused_reduce = plan.fused_reduce;
  a.dw_fp32 = dw_fp32 ? 1 : 0;
  a.prefetch = prefetch ? 1 : 0;
  a.l2_prefetch = plan.l2_prefetch;
  a.err = d.err_word;
  const bool pdl = use_pdl();
  if (launch_bwd(plan, a, stream, pdl) != cudaSuccess) return GNORM_ERR_CUDA;
  if (!plan.fused_reduce) {
    if (launch_dw_reduce(a.partial, plan.partials, a.N, dw, a.dw_fp32,
                         plan.dynamic_schedule ? a.work_counter : nullptr, stream,
                         pdl) != cudaSuccess)
      return GNORM_ERR_CUDA;
  }
  return GNORM_OK;
}

// Checks shared by gnorm_bwd and gnorm_ckpt_step once the shape is known to be valid.
int check_workspace(const DeviceInfo& d, int64_t M, int64_t N, int deterministic, void* ws,
                    size_t ws_bytes) {
  gnorm_plan plan;
  int st = make_plan(1, M, N, deterministic, d.num_sms, d.smem_optin, &plan);
  if (st != GNORM_OK) return st;
  if (ws == nullptr) return GNORM_ERR_WORKSPACE;
  if (!aligned(ws, GNORM_WORKSPACE_ALIGN)) return GNORM_ERR_WORKSPACE;
  if (ws_bytes < workspace_bytes_for(plan, N)) return GNORM_ERR_WORKSPACE;
  return GNORM_OK;
}

}  // namespace
}  // namespace gnorm

using namespace gnorm;

extern "C" {

int gnorm_fwd(const void* x, const void* g, const void* w, float eps, void* y, float* rstd,
              int64_t M, int64_t N, void* stream) {
  int st = check_shape(M, N);
  if (st != GNORM_OK) return st;
  if (!std::isfinite(eps) || eps < 0.f) return GNORM_ERR_ARG;
  if (M == 0) return GNORM_OK;
  if (!x || !g || !w || !y || !rstd) return GNORM_ERR_NULL;
  if (!aligned(x, 16) || !aligned(g, 16) || !aligned(w, 16) || !aligned(y, 16) ||
      !aligned(rstd, 4))
    return GNORM_ERR_ALIGN;
  const size_t mat = static_cast<size_t>(M) * N * 2;
  const Span in[] = {{x, mat}, {g, mat}, {w, static_cast<size_t>(N) * 2}};
  const Span out[] = {{y, mat}, {rstd, static_cast<size_t>(M) * 4}};
  if (any_alias(in, 3, out, 2)) return GNORM_ERR_ALIAS;
  DeviceInfo d;
  st = device_info(&d);
  if (st != GNORM_OK) return st;
  return enqueue_fwd(d, x, g, w, eps, y, rstd, M, N, as_stream(stream));
}

int gnorm_bwd(const void* dy, const void* x, const void* g, const void* w, const float* rstd,
              void* dx, void* dg, void* dw, int dw_fp32, int deterministic, int64_t M, int64_t N,
              void* workspace, size_t workspace_bytes, void* stream) {
  int st = check_shape(M, N);
  if (st != GNORM_OK) return st;
  if (!dw) return GNORM_ERR_NULL;
  if (!aligned(dw, 16)) return GNORM_ERR_ALIGN;
  const size_t dw_bytes = static_cast<size_t>(N) * (dw_fp32 ? 4 : 2);
  if (M == 0) {
    if (cudaMemsetAsync(dw, 0, dw_bytes, as_stream(stream)) != cudaSuccess) return GNORM_ERR_CUDA;
    return GNORM_OK;
  }
  if (!dy || !x || !g || !w || !rstd || !dx || !dg) return GNORM_ERR_NULL;
  if (!aligned(dy, 16) || !aligned(x, 16) || !aligned(g, 16) || !aligned(w, 16) ||
      !aligned(rstd, 4) || !aligned(dx, 16) || !aligned(dg, 16))
    return GNORM_ERR_ALIGN;
  const size_t mat = static_cast<size_t>(M) * N * 2;
  const Span in[] = {{dy, mat}, {x, mat}, {g, mat}, {w, static_cast<size_t>(N) * 2},
                     {rstd, static_cast<size_t>(M) * 4}};
  const Span out[] = {{dx, mat}, {dg, mat}, {dw, dw_bytes}, {workspace, workspace_bytes}};
  if (any_alias(in, 5, out, 4)) return GNORM_ERR_ALIAS;
  DeviceInfo d;
  st = device_info(&d);
  if (st != GNORM_OK) return st;
  st = check_workspace(d, M, N, deterministic, workspace, workspace_bytes);
  if (st != GNORM_OK) return st;
  return enqueue_bwd(d, dy, x, g, w, rstd, dx, dg, dw, dw_fp32, deterministic, M, N, workspace,
                     as_stream(stream));
}

int gnorm_ckpt_step(const void* x, const void* g, const void* w, float eps, const void* dy,
                    void* y, float* rstd, void* dx, void* dg, void* dw, int dw_fp32,
                    int deterministic, int64_t M, int64_t N, void* workspace,
                    size_t workspace_bytes, void* stream) {
  int st = check_shape(M, N);
  if (st != GNORM_OK) return st;
  if (!std::isfinite(eps) || eps < 0.f) return GNORM_ERR_ARG;
  if (!dw) return GNORM_ERR_NULL;
  if (!aligned(dw, 16)) return GNORM_ERR_ALIGN;
  const size_t dw_bytes = static_cast<size_t>(N) * (dw_fp32 ? 4 : 2);
  if (M == 0) {
    if (cudaMemsetAsync(dw, 0, dw_bytes, as_stream(stream)) != cudaSuccess) return GNORM_ERR_CUDA;
    return GNORM_OK;
  }
  if (!x || !g || !w || !dy || !y || !rstd || !dx || !dg) return GNORM_ERR_NULL;
  if (!aligned(x, 16) || !aligned(g, 16) || !aligned(w, 16) || !aligned(dy, 16) ||
      !aligned(y, 16) || !aligned(rstd, 4) || !aligned(dx, 16) || !aligned(dg, 16))
    return GNORM_ERR_ALIGN;
  const size_t mat = static_cast<size_t>(M) * N * 2;
  const Span in[] = {{x, mat}, {g, mat}, {w, static_cast<size_t>(N) * 2}, {dy, mat}};
  const Span out[] = {{y, mat},        {rstd, static_cast<size_t>(M) * 4},
                      {dx, mat},       {dg, mat},
                      {dw, dw_bytes}, {workspace, workspace_bytes}};
  if (any_alias(in, 4, out, 6)) return GNORM_ERR_ALIAS;
  DeviceInfo d;
  st = device_info(&d);
  if (st != GNORM_OK) return st;
  st = check_workspace(d, M, N, deterministic, workspace, workspace_bytes);
  if (st != GNORM_OK) return st;
  const cudaStream_t s = as_stream(stream);
  // The second forward (the recompute) follows the first, which writes only y and rstd;
  // the backward follows it and reads rstd only after it ends.  Neither predecessor writes
  // x, g or dy (outputs may not overlap inputs), so those copies may start early.
  const int cp = get_tuning().chain_prefetch;
  const bool chain = cp == 1 ? true : (cp == 2 ? false : kDefaultChainPrefetch != 0);
  st = enqueue_fwd(d, x, g, w, eps, y, rstd, M, N, s);
  if (st != GNORM_OK) return st;
  st = enqueue_fwd(d, x, g, w, eps, y, rstd, M, N, s, chain);
  if (st != GNORM_OK) return st;
  return enqueue_bwd(d, dy, x, g, w, rstd, dx, dg, dw, dw_fp32, deterministic, M, N, workspace, s,
                     chain);
}

int gnorm_dw_reduce(const float* partials, int64_t P, int64_t N, void* dw, int dw_fp32,
                    void* stream) {
  if (P < 0 || P > (int64_t(1) << 31) - 1 || N < 8 || N > GNORM_N_MAX || (N % 8) != 0)
    return GNORM_ERR_SHAPE;
  if (!dw) return GNORM_ERR_NULL;
  if (!aligned(dw, 16)) return GNORM_ERR_ALIGN;
  const size_t dw_bytes = static_cast<size_t>(N) * (dw_fp32 ? 4 : 2);
  const cudaStream_t s = as_stream(stream);
  if (P == 0) return cudaMemsetAsync(dw, 0, dw_bytes, s) == cudaSuccess ? GNORM_OK : GNORM_ERR_CUDA;
  if (!partials) return GNORM_ERR_NULL;
  if (!aligned(partials, 16)) return GNORM_ERR_ALIGN;
  const Span in[] = {{partials, static_cast<size_t>(P) * N * 4}};
  const Span out[] = {{dw, dw_bytes}};
  if (any_alias(in, 1, out, 1)) return GNORM_ERR_ALIAS;
  if (launch_dw_reduce(partials, static_cast<int>(P), static_cast<int>(N), dw, dw_fp32 ? 1 : 0,
                       nullptr, s, use_pdl()) != cudaSuccess)
    return GNORM_ERR_CUDA;
  return GNORM_OK;
}

size_t gnorm_bwd_workspace_bytes_for(int64_t M, int64_t N, int deterministic, int num_sms) {
  gnorm_plan plan;
  if (check_shape(M, N) != GNORM_OK) return 0;
  if (make_plan(1, M, N, deterministic, num_sms, 0, &plan) != GNORM_OK) return 0;
  return workspace_bytes_for(plan, N);
}

size_t gnorm_bwd_workspace_bytes(int64_t M, int64_t N, int deterministic) {
  DeviceInfo d;
  if (device_info(&d) != GNORM_OK) return 0;
  gnorm_plan plan;
  if (check_shape(M, N) != GNORM_OK) return 0;
  if (make_plan(1, M, N, deterministic, d.num_sms, d.smem_optin, &plan) != GNORM_OK) return 0;
  return workspace_bytes_for(plan, N);
}

const char* gnorm_status_string(int status) {
  switch (status) {
    case GNORM_OK: return "GNORM_OK";
    case GNORM_ERR_NULL: return "GNORM_ERR_NULL: a required pointer is NULL";
    case GNORM_ERR_SHAPE: return "GNORM_ERR_SHAPE: M < 0 or N not a multiple of 8 in [8, 16384]";
    case GNORM_ERR_ALIGN: return "GNORM_ERR_ALIGN: tensors need 16-byte (rstd 4-byte) alignment";
    case GNORM_ERR_ALIAS: return "GNORM_ERR_ALIAS: an output overlaps an input or another output";
    case GNORM_ERR_UNSUPPORTED: return "GNORM_ERR_UNSUPPORTED: no launch plan fits the device";
    case GNORM_ERR_WORKSPACE: return "GNORM_ERR_WORKSPACE: workspace NULL, misaligned or too small";
    case GNORM_ERR_CUDA: return "GNORM_ERR_CUDA: the CUDA runtime reported an error";
    case GNORM_ERR_ARG: return "GNORM_ERR_ARG: an argument is out of range";
    default: return "unknown gnorm status";
  }
}

int gnorm_plan_query(int kind, int64_t M, int64_t N, int deterministic, int num_sms,
                     int smem_per_block, gnorm_plan* out) {
  return make_plan(kind, M, N, deterministic, num_sms, smem_per_block, out);
}

int gnorm_device_error(int reset) {
  DeviceInfo d;
  if (device_info(&d) != GNORM_OK) return -1;
  if (cudaDeviceSynchronize() != cudaSuccess) return -1;
  unsigned v = 0;
  if (cudaMemcpy(&v, d.err_word, sizeof(v), cudaMemcpyDeviceToHost) != cudaSuccess) return -1;
  if (reset) {
    const unsigned zero = 0;
    if (cudaMemcpy(d.err_word, &zero, sizeof(zero), cudaMemcpyHostToDevice) != cudaSuccess)
      return -1;
  }
  return static_cast<int>(v);
}

void gnorm_set_tuning(const gnorm_tuning* tuning) {
  TuningKnobs k = {};
  if (tuning != nullptr) {
    k = *tuning;
    auto clamp0 = [](int v) { return v > 0 ? v : 0; };
    auto tri = [](int v) { return (v == 1 || v == 2) ? v : 0; };
    k.stage_bytes = clamp0(k.stage_bytes);
    k.max_stages = clamp0(k.max_stages);
    k.ctas_per_sm = clamp0(k.ctas_per_sm);
    k.disable_pdl = k.disable_pdl ? 1 : 0;
    k.threads_per_row = clamp0(k.threads_per_row);
    k.chunks_per_thread = clamp0(k.chunks_per_thread);
    k.l2_prefetch = tri(k.l2_prefetch);
    k.tail_reduce = tri(k.tail_reduce);
    k.chain_prefetch = tri(k.chain_prefetch);
  }
  set_tuning(k);
}

const char* gnorm_build_info(void) {
  static char buf[160];
  static std::once_flag once;
  std::call_once(once, [] {
    std::snprintf(buf, sizeof(buf), "libgnorm: nvcc %d.%d, target sm_100a, rows <= 2^40, N <= %d",
                  __CUDACC_VER_MAJOR__, __CUDACC_VER_MINOR__, GNORM_N_MAX);
  });
  return buf;
}

}  // extern "C"
