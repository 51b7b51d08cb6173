// api.cu -- the extern "C" entry points of libgnorm (declared in include/gnorm.h).
//
// Every argument is checked on the host before anything is enqueued; a bad argument
// returns a gnorm_status and launches nothing.  Entry points never synchronise and never
// allocate; they enqueue kernels on the caller's stream.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "args.h"
#include "device_common.cuh"
#include "gnorm.h"
#include "layout.h"
#include "launch.h"
#include "plan.h"

namespace gnorm {

// Bits set by kernels whose bounded pipeline waits gave up (see gnorm_device_error).
__device__ unsigned int g_device_error_word = 0u;

// Self-test of the bounded wait: one thread waits on a barrier nothing will arrive on; the
// wait gives up after `limit_ns`, sets kErrSelfTest in the error word and the kernel returns.
__global__ void wait_timeout_selftest_kernel(unsigned long long limit_ns, unsigned* err,
                                             unsigned long long* waited_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x != 0) return;
  mbar_init(&bar, 1);
  fence_barrier_init();
  const unsigned long long t0 = globaltimer_ns();
  const bool completed = mbar_wait(&bar, 0u, err, kErrSelfTest, limit_ns);
  *waited_ns = completed ? 0ull : globaltimer_ns() - t0;
}

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

}  // namespace

// The current device's error word (device address), for entry points in other files.
int device_error_word(unsigned** out) {
  DeviceInfo d;
  const int st = device_info(&d);
  if (st != GNORM_OK) return st;
  *out = d.err_word;
  return GNORM_OK;
}

namespace {

// A memory region an argument covers: a plain byte span, or a BF16 [rows, cols] matrix
// with row stride `ld` elements.
struct Region {
  const void* p;
  size_t bytes;     // whole extent
  bool is_mat;
  int64_t rows, cols, ld;
};

Region span(const void* p, size_t bytes) { return Region{p, bytes, false, 0, 0, 0}; }
Region mat(const void* p, int64_t rows, int64_t cols, int64_t ld) {
  const size_t bytes = rows > 0 ? static_cast<size_t>((rows - 1) * ld + cols) * 2 : 0;
  return Region{p, bytes, true, rows, cols, ld};
}

int64_t floor_div(int64_t a, int64_t b) { return a / b - ((a % b != 0) && ((a < 0) != (b < 0))); }

// Exact for two matrices with the same stride and width (their elements interleave
// row by row); whole-extent overlap otherwise.
bool overlaps(const Region& a, const Region& b) {
  if (a.p == nullptr || b.p == nullptr || a.bytes == 0 || b.bytes == 0) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a.p), a1 = a0 + a.bytes;
  const uintptr_t b0 = reinterpret_cast<uintptr_t>(b.p), b1 = b0 + b.bytes;
  if (!(a0 < b1 && b0 < a1)) return false;
  if (!(a.is_mat && b.is_mat && a.ld == b.ld && a.cols == b.cols)) return true;
  const int64_t diff = static_cast<int64_t>(b0 - a0);  // two's complement difference
  if (diff % 2 != 0) return true;
  const int64_t d = diff / 2, L = a.ld, n = a.cols;
  const int64_t q = floor_div(d, L), delta = d - q * L;  // b's row j starts in a's row q + j
  auto rows_meet = [&](int64_t off) { return off < a.rows && off + b.rows > 0; };
  if (delta < n && rows_meet(q)) return true;          // columns [delta, n) of the same row
  if (delta + n > L && rows_meet(q + 1)) return true;  // b's row runs into a's next row
  return false;
}

// Every output region against every input region and every other output region.
bool any_alias(const Region* in, int n_in, const Region* out, int n_out) {
  for (int i = 0; i < n_out; ++i) {
    for (int j = 0; j < n_in; ++j)
      if (overlaps(out[i], in[j])) return true;
    for (int j = i + 1; j < n_out; ++j)
      if (overlaps(out[i], out[j])) return true;
  }
  return false;
}

// Row stride in elements: 0 means packed (N); a stride must hold a row and keep rows
// 16-byte aligned.
int check_ld(int64_t* ld, int64_t N) {
  if (*ld == 0) *ld = N;
  if (*ld < N) return GNORM_ERR_SHAPE;
  if (*ld % 8 != 0) return GNORM_ERR_ALIGN;
  return GNORM_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

int check_shape(int64_t M, int64_t N) {
  if (M < 0 || M > kMaxRows) return GNORM_ERR_SHAPE;
  if (N < 8 || N > GNORM_N_MAX || (N % 8) != 0) return GNORM_ERR_SHAPE;
  return GNORM_OK;
}

bool use_pdl() { return get_tuning().disable_pdl == 0; }

// cuTensorMapEncodeTiled, fetched from the driver through the runtime (no libcuda link).
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q = cudaDriverEntryPointSymbolNotFound;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
            cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return static_cast<EncodeTiledFn>(nullptr);
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// A 2-D tiled map over a strided BF16 [M, N] tensor whose box is one whole row block
// (N columns x R rows), so a block lands packed in shared memory in one copy.  Used for
// narrow strided rows, where one bulk copy per row would be hundreds of small copies per
// stage.  Returns false (caller falls back to per-row copies) when the box does not fit the
// tiled-copy limits (256 per dimension) or the encoding fails.
bool rows_map(CUtensorMap* map, const void* base, int64_t M, int64_t N, int64_t ld, int R) {
  if (ld == N || N > 256 || R > 256 || M >= (int64_t(1) << 31)) return false;
  EncodeTiledFn fn = encode_tiled();
  if (fn == nullptr) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(N), static_cast<cuuint32_t>(R)};
  const cuuint32_t elem_strides[2] = {1, 1};
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
            box, elem_strides, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

cudaStream_t as_stream(void* s) { return static_cast<cudaStream_t>(s); }

// `prefetch`: the previous kernel on the stream is known to write none of this call's
// inputs, so the kernel may start copying them before that kernel has finished.
// Descriptors reaching here are validated and have every stride resolved.
int enqueue_fwd(const DeviceInfo& d, const gnorm_fwd_desc& f, cudaStream_t stream,
                bool prefetch = false) {
  gnorm_plan plan;
  int st = make_plan(0, f.M, f.N, 1, d.num_sms, d.smem_optin, &plan);
  if (st != GNORM_OK) return st;
  FwdArgs a;
  a.x = static_cast<const uint16_t*>(f.x);
  a.g = static_cast<const uint16_t*>(f.g);
  a.w = f.w;
  a.y = static_cast<uint16_t*>(f.y);
  a.rstd = f.rstd;
  a.ldx = f.ldx;
  a.ldg = f.ldg;
  a.ldy = f.ldy;
  a.w_fp32 = f.w_fp32 ? 1 : 0;
  a.M = f.M;
  a.N = static_cast<int>(f.N);
  a.eps = f.eps;
  a.inv_n = static_cast<float>(1.0 / static_cast<double>(f.N));
  a.rows_per_stage = plan.rows_per_stage;
  a.stages = plan.stages;
  a.num_blocks = plan.num_blocks;
  a.prefetch = prefetch ? 1 : 0;
  a.l2_prefetch = plan.l2_prefetch;
  a.err = d.err_word;
  const int R = plan.rows_per_stage;
  if (!plan.direct_loads && rows_map(&a.map_x, f.x, f.M, f.N, f.ldx, R)) a.map_bits |= 1;
  if (!plan.direct_loads && rows_map(&a.map_g, f.g, f.M, f.N, f.ldg, R)) a.map_bits |= 2;
  if (launch_fwd(plan, a, stream, use_pdl()) != cudaSuccess) return GNORM_ERR_CUDA;
  return GNORM_OK;
}

// `fused`: the forward of the same rows runs in the same kernel (gnorm_fwd_bwd); it writes
// fused->y and fused->rstd and reads no rstd.  Staged plans only (GNORM_ERR_UNSUPPORTED for a
// direct-load plan, which the caller then runs as two kernels).
int enqueue_bwd(const DeviceInfo& d, const gnorm_bwd_desc& b, cudaStream_t stream,
                bool prefetch = false, const gnorm_fwd_desc* fused = nullptr) {
  gnorm_plan plan;
  int st = make_plan(fused != nullptr ? 2 : 1, b.M, b.N, b.deterministic, d.num_sms,
                     d.smem_optin, &plan);
  if (st != GNORM_OK) return st;
  // The fused kernel is staged only, and its partial rows must fit the workspace sized for
  // the backward's plan.
  if (fused != nullptr &&
      (plan.direct_loads || workspace_bytes_for(plan, b.N) > b.workspace_bytes))
    return GNORM_ERR_UNSUPPORTED;
  uint8_t* wsb = static_cast<uint8_t*>(b.workspace);
  BwdArgs a;
  a.dy = static_cast<const uint16_t*>(b.dy);
  a.x = static_cast<const uint16_t*>(b.x);
  a.g = static_cast<const uint16_t*>(b.g);
  a.w = b.w;
  a.rstd = b.rstd;
  a.dx = static_cast<uint16_t*>(b.dx);
  a.dg = static_cast<uint16_t*>(b.dg);
  a.lddy = b.lddy;
  a.ldx = b.ldx;
  a.ldg = b.ldg;
  a.lddx = b.lddx;
  a.lddg = b.lddg;
  a.w_fp32 = b.w_fp32 ? 1 : 0;
  a.partial = reinterpret_cast<float*>(wsb + kWorkspaceHeader);
  a.dw = b.dw;
  a.work_counter = reinterpret_cast<unsigned long long*>(wsb);
  a.ticket = reinterpret_cast<unsigned*>(wsb + 8);
  a.M = b.M;
  a.N = static_cast<int>(b.N);
  a.inv_n = static_cast<float>(1.0 / static_cast<double>(b.N));
  a.rows_per_stage = plan.rows_per_stage;
  a.stages = plan.stages;
  a.num_blocks = plan.num_blocks;
  a.dynamic_schedule = plan.dynamic_schedule;
  a.fused_reduce = plan.fused_reduce;
  a.dw_fp32 = b.dw_fp32 ? 1 : 0;
  a.prefetch = prefetch ? 1 : 0;
  a.l2_prefetch = plan.l2_prefetch;
  a.err = d.err_word;
  if (fused != nullptr) {
    a.fused_fwd = 1;
    a.y = static_cast<uint16_t*>(fused->y);
    a.ldy = fused->ldy;
    a.rstd_out = fused->rstd;
    a.eps = fused->eps;
  }
  const int R = plan.rows_per_stage;
  if (!plan.direct_loads) {
    if (rows_map(&a.map_dy, b.dy, b.M, b.N, b.lddy, R)) a.map_bits |= 1;
    if (rows_map(&a.map_x, b.x, b.M, b.N, b.ldx, R)) a.map_bits |= 2;
    if (rows_map(&a.map_g, b.g, b.M, b.N, b.ldg, R)) a.map_bits |= 4;
  }
  const bool pdl = use_pdl();
  if (launch_bwd(plan, a, stream, pdl) != cudaSuccess) return GNORM_ERR_CUDA;
  if (!plan.fused_reduce) {
    if (launch_dw_reduce(a.partial, plan.partials, a.N, b.dw, a.dw_fp32,
                         plan.dynamic_schedule ? a.work_counter : nullptr, stream,
                         pdl) != cudaSuccess)
      return GNORM_ERR_CUDA;
  }
  return GNORM_OK;
}

// Validates a forward descriptor in place (resolving strides).  Returns GNORM_OK, or an
// error; *noop is set when M == 0.
int check_fwd(gnorm_fwd_desc* f, bool* noop) {
  *noop = false;
  int st = check_shape(f->M, f->N);
  if (st != GNORM_OK) return st;
  if (!std::isfinite(f->eps) || f->eps < 0.f) return GNORM_ERR_ARG;
  for (int64_t* ld : {&f->ldx, &f->ldg, &f->ldy})
    if ((st = check_ld(ld, f->N)) != GNORM_OK) return st;
  if (f->M == 0) {
    *noop = true;
    return GNORM_OK;
  }
  if (!f->x || !f->g || !f->w || !f->y || !f->rstd) return GNORM_ERR_NULL;
  if (!aligned(f->x, 16) || !aligned(f->g, 16) || !aligned(f->w, 16) || !aligned(f->y, 16) ||
      !aligned(f->rstd, 4))
    return GNORM_ERR_ALIGN;
  return GNORM_OK;
}

int check_bwd(gnorm_bwd_desc* b, bool* noop) {
  *noop = false;
  int st = check_shape(b->M, b->N);
  if (st != GNORM_OK) return st;
  for (int64_t* ld : {&b->lddy, &b->ldx, &b->ldg, &b->lddx, &b->lddg})
    if ((st = check_ld(ld, b->N)) != GNORM_OK) return st;
  if (!b->dw) return GNORM_ERR_NULL;
  if (!aligned(b->dw, 16)) return GNORM_ERR_ALIGN;
  if (b->M == 0) {
    *noop = true;
    return GNORM_OK;
  }
  if (!b->dy || !b->x || !b->g || !b->w || !b->rstd || !b->dx || !b->dg) return GNORM_ERR_NULL;
  if (!aligned(b->dy, 16) || !aligned(b->x, 16) || !aligned(b->g, 16) || !aligned(b->w, 16) ||
      !aligned(b->rstd, 4) || !aligned(b->dx, 16) || !aligned(b->dg, 16))
    return GNORM_ERR_ALIGN;
  return GNORM_OK;
}

size_t w_bytes(int64_t N, int w_fp32) { return static_cast<size_t>(N) * (w_fp32 ? 4 : 2); }

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

// Validates a forward/backward descriptor pair of one set of rows (gnorm_ckpt_step_ex,
// gnorm_fwd_bwd_ex): the backward's x, g, w, rstd must be NULL or the forward's, M and N
// equal.  Resolves strides, fills *f and *b, checks aliasing and the workspace.  *noop is set
// when M == 0 (dw has then been zeroed on `stream`).
int check_fwd_bwd(const gnorm_fwd_desc* fwd, const gnorm_bwd_desc* bwd, void* stream,
                  gnorm_fwd_desc* f_out, gnorm_bwd_desc* b_out, DeviceInfo* d, bool* noop) {
  *noop = false;
  if (fwd == nullptr || bwd == nullptr) return GNORM_ERR_NULL;
  gnorm_fwd_desc f = *fwd;
  gnorm_bwd_desc b = *bwd;
  if (b.M != f.M || b.N != f.N) return GNORM_ERR_ARG;
  // The backward reads the forward's x, g, w and the rstd it writes.
  if ((b.x && (b.x != f.x || (b.ldx ? b.ldx : f.N) != (f.ldx ? f.ldx : f.N))) ||
      (b.g && (b.g != f.g || (b.ldg ? b.ldg : f.N) != (f.ldg ? f.ldg : f.N))) ||
      (b.w && (b.w != f.w || b.w_fp32 != f.w_fp32)) || (b.rstd && b.rstd != f.rstd))
    return GNORM_ERR_ARG;
  b.x = f.x;
  b.ldx = f.ldx;
  b.g = f.g;
  b.ldg = f.ldg;
  b.w = f.w;
  b.w_fp32 = f.w_fp32;
  b.rstd = f.rstd;
  bool noop_f = false, noop_b = false;
  int st = check_fwd(&f, &noop_f);
  if (st != GNORM_OK) return st;
  st = check_bwd(&b, &noop_b);
  if (st != GNORM_OK) return st;
  const size_t dw_bytes = static_cast<size_t>(b.N) * (b.dw_fp32 ? 4 : 2);
  if (noop_b) {
    *noop = true;
    return cudaMemsetAsync(b.dw, 0, dw_bytes, as_stream(stream)) == cudaSuccess ? GNORM_OK
                                                                                 : GNORM_ERR_CUDA;
  }
  const Region in[] = {mat(f.x, f.M, f.N, f.ldx), mat(f.g, f.M, f.N, f.ldg),
                       span(f.w, w_bytes(f.N, f.w_fp32)), mat(b.dy, b.M, b.N, b.lddy)};
  const Region out[] = {mat(f.y, f.M, f.N, f.ldy),
                        span(f.rstd, static_cast<size_t>(f.M) * 4),
                        mat(b.dx, b.M, b.N, b.lddx),
                        mat(b.dg, b.M, b.N, b.lddg),
                        span(b.dw, dw_bytes),
                        span(b.workspace, b.workspace_bytes)};
  if (any_alias(in, 4, out, 6)) return GNORM_ERR_ALIAS;
  st = device_info(d);
  if (st != GNORM_OK) return st;
  st = check_workspace(*d, b.M, b.N, b.deterministic, b.workspace, b.workspace_bytes);
  if (st != GNORM_OK) return st;
  *f_out = f;
  *b_out = b;
  return GNORM_OK;
}

// The forward of a set of rows followed by its backward.  One fused kernel (the staged
// backward plan) or, for direct-load plans or when the fuse_fwd_bwd knob says so, the forward
// kernel then the backward kernel.  `chain`: the previous kernel on the stream writes none of
// x, g, dy (the first forward of a checkpointed step), so input copies may start early.
int enqueue_fwd_bwd(const DeviceInfo& d, const gnorm_fwd_desc& f, const gnorm_bwd_desc& b,
                    cudaStream_t s, bool chain) {
  const int fk = get_tuning().fuse_fwd_bwd;
  const bool fuse = fk == 1 ? true : (fk == 2 ? false : kDefaultFuseFwdBwd != 0);
  if (fuse) {
    const int st = enqueue_bwd(d, b, s, chain, &f);
    if (st != GNORM_ERR_UNSUPPORTED) return st;
  }
  // Two kernels: the forward, then the backward, which only reads rstd once the forward
  // has ended (neither writes x, g or dy, so the backward's input copies may start early).
  int st = enqueue_fwd(d, f, s, chain);
  if (st != GNORM_OK) return st;
  return enqueue_bwd(d, b, s, chain);
}

}  // namespace
}  // namespace gnorm

using namespace gnorm;

extern "C" {

int gnorm_fwd_ex(const gnorm_fwd_desc* desc, void* stream) {
  if (desc == nullptr) return GNORM_ERR_NULL;
  gnorm_fwd_desc f = *desc;
  bool noop = false;
  int st = check_fwd(&f, &noop);
  if (st != GNORM_OK || noop) return st;
  const Region in[] = {mat(f.x, f.M, f.N, f.ldx), mat(f.g, f.M, f.N, f.ldg),
                       span(f.w, w_bytes(f.N, f.w_fp32))};
  const Region out[] = {mat(f.y, f.M, f.N, f.ldy), span(f.rstd, static_cast<size_t>(f.M) * 4)};
  if (any_alias(in, 3, out, 2)) return GNORM_ERR_ALIAS;
  DeviceInfo d;
  st = device_info(&d);
  if (st != GNORM_OK) return st;
  return enqueue_fwd(d, f, as_stream(stream));
}

int gnorm_bwd_ex(const gnorm_bwd_desc* desc, void* stream) {
  if (desc == nullptr) return GNORM_ERR_NULL;
  gnorm_bwd_desc b = *desc;
  bool noop = false;
  int st = check_bwd(&b, &noop);
  if (st != GNORM_OK) return st;
  const size_t dw_bytes = static_cast<size_t>(b.N) * (b.dw_fp32 ? 4 : 2);
  if (noop)
    return cudaMemsetAsync(b.dw, 0, dw_bytes, as_stream(stream)) == cudaSuccess ? GNORM_OK
                                                                                 : GNORM_ERR_CUDA;
  const Region in[] = {mat(b.dy, b.M, b.N, b.lddy), mat(b.x, b.M, b.N, b.ldx),
                       mat(b.g, b.M, b.N, b.ldg), span(b.w, w_bytes(b.N, b.w_fp32)),
                       span(b.rstd, static_cast<size_t>(b.M) * 4)};
  const Region out[] = {mat(b.dx, b.M, b.N, b.lddx), mat(b.dg, b.M, b.N, b.lddg),
                        span(b.dw, dw_bytes), span(b.workspace, b.workspace_bytes)};
  if (any_alias(in, 5, out, 4)) return GNORM_ERR_ALIAS;
  DeviceInfo d;
  st = device_info(&d);
  if (st != GNORM_OK) return st;
  st = check_workspace(d, b.M, b.N, b.deterministic, b.workspace, b.workspace_bytes);
  if (st != GNORM_OK) return st;
  return enqueue_bwd(d, b, as_stream(stream));
}

int gnorm_ckpt_step_ex(const gnorm_fwd_desc* fwd, const gnorm_bwd_desc* bwd, void* stream) {
  gnorm_fwd_desc f;
  gnorm_bwd_desc b;
  DeviceInfo d;
  bool noop = false;
  int st = check_fwd_bwd(fwd, bwd, stream, &f, &b, &d, &noop);
  if (st != GNORM_OK || noop) return st;
  const cudaStream_t s = as_stream(stream);
  // The first forward, then the recompute forward fused with the backward (or the two as
  // separate kernels).  The first forward writes only y and rstd; the second forward and
  // the backward read x, g and dy, which it cannot overlap, so their copies may start early.
  const int cp = get_tuning().chain_prefetch;
  const bool chain = cp == 1 ? true : (cp == 2 ? false : kDefaultChainPrefetch != 0);
  st = enqueue_fwd(d, f, s);
  if (st != GNORM_OK) return st;
  return enqueue_fwd_bwd(d, f, b, s, chain);
}

int gnorm_fwd_bwd_ex(const gnorm_fwd_desc* fwd, const gnorm_bwd_desc* bwd, void* stream) {
  gnorm_fwd_desc f;
  gnorm_bwd_desc b;
  DeviceInfo d;
  bool noop = false;
  int st = check_fwd_bwd(fwd, bwd, stream, &f, &b, &d, &noop);
  if (st != GNORM_OK || noop) return st;
  return enqueue_fwd_bwd(d, f, b, as_stream(stream), false);
}

int gnorm_fwd(const void* x, const void* g, const void* w, float eps, void* y, float* rstd,
              int64_t M, int64_t N, void* stream) {
  gnorm_fwd_desc f = {};
  f.x = x;
  f.ldx = N;
  f.g = g;
  f.ldg = N;
  f.w = w;
  f.eps = eps;
  f.y = y;
  f.ldy = N;
  f.rstd = rstd;
  f.M = M;
  f.N = N;
  return gnorm_fwd_ex(&f, stream);
}

static gnorm_bwd_desc packed_bwd_desc(const void* dy, const void* x, const void* g,
                                      const void* w, const float* rstd, void* dx, void* dg,
                                      void* dw, int dw_fp32, int deterministic, int64_t M,
                                      int64_t N, void* workspace, size_t workspace_bytes) {
  gnorm_bwd_desc b = {};
  b.dy = dy;
  b.lddy = N;
  b.x = x;
  b.ldx = N;
  b.g = g;
  b.ldg = N;
  b.w = w;
  b.rstd = rstd;
  b.dx = dx;
  b.lddx = N;
  b.dg = dg;
  b.lddg = N;
  b.dw = dw;
  b.dw_fp32 = dw_fp32;
  b.deterministic = deterministic;
  b.M = M;
  b.N = N;
  b.workspace = workspace;
  b.workspace_bytes = workspace_bytes;
  return b;
}

int gnorm_bwd(const void* dy, const void* x, const void* g, const void* w, const float* rstd,
              void* dx, void* dg, void* dw, int dw_fp32, int deterministic, int64_t M, int64_t N,
              void* workspace, size_t workspace_bytes, void* stream) {
  const gnorm_bwd_desc b = packed_bwd_desc(dy, x, g, w, rstd, dx, dg, dw, dw_fp32, deterministic,
                                           M, N, workspace, workspace_bytes);
  return gnorm_bwd_ex(&b, stream);
}

int gnorm_ckpt_step(const void* x, const void* g, const void* w, float eps, const void* dy,
                    void* y, float* rstd, void* dx, void* dg, void* dw, int dw_fp32,
                    int deterministic, int64_t M, int64_t N, void* workspace,
                    size_t workspace_bytes, void* stream) {
  gnorm_fwd_desc f = {};
  f.x = x;
  f.ldx = N;
  f.g = g;
  f.ldg = N;
  f.w = w;
  f.eps = eps;
  f.y = y;
  f.ldy = N;
  f.rstd = rstd;
  f.M = M;
  f.N = N;
  const gnorm_bwd_desc b = packed_bwd_desc(dy, x, g, w, rstd, dx, dg, dw, dw_fp32, deterministic,
                                           M, N, workspace, workspace_bytes);
  return gnorm_ckpt_step_ex(&f, &b, stream);
}

int gnorm_fwd_bwd(const void* x, const void* g, const void* w, float eps, const void* dy,
                  void* y, float* rstd, void* dx, void* dg, void* dw, int dw_fp32,
                  int deterministic, int64_t M, int64_t N, void* workspace,
                  size_t workspace_bytes, void* stream) {
  gnorm_fwd_desc f = {};
  f.x = x;
  f.ldx = N;
  f.g = g;
  f.ldg = N;
  f.w = w;
  f.eps = eps;
  f.y = y;
  f.ldy = N;
  f.rstd = rstd;
  f.M = M;
  f.N = N;
  const gnorm_bwd_desc b = packed_bwd_desc(dy, x, g, w, rstd, dx, dg, dw, dw_fp32, deterministic,
                                           M, N, workspace, workspace_bytes);
  return gnorm_fwd_bwd_ex(&f, &b, stream);
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
  const Region in[] = {span(partials, static_cast<size_t>(P) * N * 4)};
  const Region out[] = {span(dw, dw_bytes)};
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
    k.host_chunk_bytes = clamp0(k.host_chunk_bytes);
    k.fwd_direct = tri(k.fwd_direct);
    k.bwd_direct = tri(k.bwd_direct);
    k.fuse_fwd_bwd = tri(k.fuse_fwd_bwd);
  }
  set_tuning(k);
}

int gnorm_selftest_wait_timeout(unsigned timeout_us, unsigned long long* waited_ns) {
  if (waited_ns == nullptr) return GNORM_ERR_NULL;
  if (timeout_us == 0 || timeout_us > 1000000u) return GNORM_ERR_ARG;
  DeviceInfo d;
  int st = device_info(&d);
  if (st != GNORM_OK) return st;
  unsigned long long* dev_ns = nullptr;
  // Test-only entry: this one allocates (8 bytes) and synchronises.
  if (cudaMalloc(&dev_ns, sizeof(*dev_ns)) != cudaSuccess) return GNORM_ERR_CUDA;
  wait_timeout_selftest_kernel<<<1, 32>>>(static_cast<unsigned long long>(timeout_us) * 1000ull,
                                          d.err_word, dev_ns);
  cudaError_t e = cudaGetLastError();
  if (e == cudaSuccess) e = cudaDeviceSynchronize();
  if (e == cudaSuccess)
    e = cudaMemcpy(waited_ns, dev_ns, sizeof(*waited_ns), cudaMemcpyDeviceToHost);
  cudaFree(dev_ns);
  return e == cudaSuccess ? GNORM_OK : GNORM_ERR_CUDA;
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
