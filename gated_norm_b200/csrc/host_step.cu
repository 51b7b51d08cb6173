// host_step.cu -- gnorm_ckpt_step_host: the checkpointed step on host buffers.
//
// A caller whose batch lives in host memory needs three things per step: the inputs
// copied in, the step, and the outputs copied back.  Done one after the other, the copies
// dominate (tens of MB over a host link of ~55 GB/s per direction against tens of us of
// kernels) and use one direction of the link at a time.  This entry point splits the rows
// into chunks (4 MiB of x, g and dy, or 32 MiB for batches above 64 MiB) and runs them as a
// pipeline over three streams:
//
//   copy-in stream   : w, then x, g, dy of chunk 0, 1, 2, ...            (host -> device)
//   caller's stream  : chunk k's checkpointed step once its inputs are in (fwd, fwd, bwd)
//   copy-out stream  : chunk k's y, rstd, dx, dg once its step is done    (device -> host)
//
// so the inputs of later chunks come in while the outputs of earlier ones go out (the link
// is full duplex).  Rows are independent, so y, rstd, dx and dg equal gnorm_ckpt_step's bit
// for bit.  dw is a sum over all rows: each chunk's step writes its own FP32 dw row, and a
// fixed-order sum over those rows (gnorm_dw_reduce) gives dw, deterministic run to run (in
// deterministic mode) but rounded differently from a single gnorm_ckpt_step over all rows
// unless there is one chunk.
//
// The two copy streams and the events that order them are created once per device (the
// first call on a device) and shared by every call on it; a mutex serialises enqueueing.
// The caller's stream is forked at the start (the copies in wait for all earlier work on
// it) and joined at the end (it waits for the last copy out), so the whole call is ordered
// on the caller's stream like any other entry point.
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <mutex>

#include "gnorm.h"
#include "plan.h"

namespace gnorm {
namespace {

constexpr int kMaxHostChunks = 256;
// x + g + dy bytes per chunk: 4 MiB for batches up to 64 MiB of x, g and dy, 32 MiB above
// (measured on B200, GB/s of the step's algorithmic bytes with 4 / 16 / 32 MiB chunks:
// 65536 x 128 126 / 122 / 113; 368640 x 128 140 / 143 / 149; 16384 x 4096 128 / 146 / 150;
// 262144 x 256 138 / 143 / 149 -- larger chunks pay once the batch is large; 8 MiB chunks
// were the slowest size at every workload tried).
constexpr int64_t kSmallHostChunkBytes = int64_t(4) << 20;
constexpr int64_t kLargeHostChunkBytes = int64_t(32) << 20;
constexpr int64_t kLargeHostBatchBytes = int64_t(64) << 20;
constexpr int kMaxHostDevices = 64;

struct HostPipe {
  bool ready = false;
  cudaStream_t in = nullptr, out = nullptr;
  cudaEvent_t start = nullptr, dw_done = nullptr, end = nullptr;
  cudaEvent_t in_done[kMaxHostChunks] = {};
  cudaEvent_t step_done[kMaxHostChunks] = {};
};

std::mutex g_pipe_mu[kMaxHostDevices];
HostPipe g_pipe[kMaxHostDevices];

int pipe_for_device(int dev, HostPipe** out) {
  HostPipe& p = g_pipe[dev];
  if (!p.ready) {
    const unsigned sf = cudaStreamNonBlocking;
    const unsigned ef = cudaEventDisableTiming;
    if (cudaStreamCreateWithFlags(&p.in, sf) != cudaSuccess ||
        cudaStreamCreateWithFlags(&p.out, sf) != cudaSuccess ||
        cudaEventCreateWithFlags(&p.start, ef) != cudaSuccess ||
        cudaEventCreateWithFlags(&p.dw_done, ef) != cudaSuccess ||
        cudaEventCreateWithFlags(&p.end, ef) != cudaSuccess)
      return GNORM_ERR_CUDA;
    for (int k = 0; k < kMaxHostChunks; ++k)
      if (cudaEventCreateWithFlags(&p.in_done[k], ef) != cudaSuccess ||
          cudaEventCreateWithFlags(&p.step_done[k], ef) != cudaSuccess)
        return GNORM_ERR_CUDA;
    p.ready = true;
  }
  *out = &p;
  return GNORM_OK;
}

size_t round256(size_t v) { return (v + 255) / 256 * 256; }

// The chunking and the layout of the device buffer, a pure function of the shape, the
// SM count (through the workspace size) and the chunk-size knob.
struct HostLayout {
  int64_t rows_per_chunk = 0;
  int chunks = 0;
  size_t mat = 0;  // bytes of one [M, N] BF16 matrix slot
  size_t off_x = 0, off_g = 0, off_dy = 0, off_y = 0, off_dx = 0, off_dg = 0;
  size_t off_rstd = 0, off_w = 0, off_dwc = 0, off_dw = 0, off_ws = 0;
  size_t ws_bytes = 0;
  size_t total = 0;
};

int host_layout(int64_t M, int64_t N, int deterministic, HostLayout* L) {
  if (M < 0 || N < 8 || N > GNORM_N_MAX || (N % 8) != 0 || M > (int64_t(1) << 40))
    return GNORM_ERR_SHAPE;
  const int knob = get_tuning().host_chunk_bytes;
  const int64_t batch_bytes = 6 * M * N;
  const int64_t chunk_bytes = knob > 0 ? knob
                              : (batch_bytes > kLargeHostBatchBytes ? kLargeHostChunkBytes
                                                                    : kSmallHostChunkBytes);
  int64_t rows = chunk_bytes / (6 * N);
  if (rows < 1) rows = 1;
  if (M > 0 && (M + rows - 1) / rows > kMaxHostChunks) rows = (M + kMaxHostChunks - 1) / kMaxHostChunks;
  if (M > 0 && rows > M) rows = M;
  L->rows_per_chunk = rows;
  L->chunks = M > 0 ? static_cast<int>((M + rows - 1) / rows) : 0;
  if (M > 0) {
    // The last chunk may be shorter, and a shorter chunk can plan more CTAs (fewer rows
    // each), so the workspace covers both chunk sizes.
    const int64_t last = M - (L->chunks - 1) * rows;
    const size_t a = gnorm_bwd_workspace_bytes(rows, N, deterministic);
    const size_t b = gnorm_bwd_workspace_bytes(last, N, deterministic);
    if (a == 0 || b == 0) return GNORM_ERR_CUDA;  // no device, or no plan
    L->ws_bytes = a > b ? a : b;
  }
  L->mat = round256(static_cast<size_t>(M) * N * 2);
  size_t o = 0;
  for (size_t* off : {&L->off_x, &L->off_g, &L->off_dy, &L->off_y, &L->off_dx, &L->off_dg}) {
    *off = o;
    o += L->mat;
  }
  L->off_rstd = o;
  o += round256(static_cast<size_t>(M) * 4);
  L->off_w = o;
  o += round256(static_cast<size_t>(N) * 2);
  L->off_dwc = o;
  o += round256(static_cast<size_t>(L->chunks) * N * 4);
  L->off_dw = o;
  o += round256(static_cast<size_t>(N) * 4);
  L->off_ws = o;
  o += L->ws_bytes;
  L->total = o;
  return GNORM_OK;
}

bool spans_overlap(const void* a, size_t na, const void* b, size_t nb) {
  if (!a || !b || !na || !nb) return false;
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + nb && b0 < a0 + na;
}

}  // namespace
}  // namespace gnorm

using namespace gnorm;

extern "C" size_t gnorm_ckpt_step_host_bytes(int64_t M, int64_t N, int deterministic) {
  HostLayout L;
  if (host_layout(M, N, deterministic, &L) != GNORM_OK) return 0;
  return L.total;
}

extern "C" int gnorm_ckpt_step_host(const void* x, const void* g, const void* w, float eps,
                                    const void* dy, void* y, float* rstd, void* dx, void* dg,
                                    void* dw, int dw_fp32, int deterministic, int64_t M,
                                    int64_t N, void* dev_buf, size_t dev_bytes, void* stream) {
  // Argument checks first, before any CUDA call.
  if (M < 0 || N < 8 || N > GNORM_N_MAX || (N % 8) != 0 || M > (int64_t(1) << 40))
    return GNORM_ERR_SHAPE;
  if (!std::isfinite(eps) || eps < 0.f) return GNORM_ERR_ARG;
  if (!dw) return GNORM_ERR_NULL;
  if (M > 0 && (!x || !g || !w || !dy || !y || !rstd || !dx || !dg)) return GNORM_ERR_NULL;
  if (!dev_buf || reinterpret_cast<uintptr_t>(dev_buf) % GNORM_WORKSPACE_ALIGN != 0)
    return GNORM_ERR_WORKSPACE;
  // Host outputs may overlap neither a host input nor each other.
  const size_t mat = static_cast<size_t>(M) * N * 2;
  const size_t dwb = static_cast<size_t>(N) * (dw_fp32 ? 4 : 2);
  const void* in_p[] = {x, g, w, dy};
  const size_t in_n[] = {mat, mat, static_cast<size_t>(N) * 2, mat};
  const void* out_p[] = {y, rstd, dx, dg, dw};
  const size_t out_n[] = {mat, static_cast<size_t>(M) * 4, mat, mat, dwb};
  for (int i = 0; i < 5; ++i) {
    for (int j = 0; j < 4; ++j)
      if (spans_overlap(out_p[i], out_n[i], in_p[j], in_n[j])) return GNORM_ERR_ALIAS;
    for (int j = i + 1; j < 5; ++j)
      if (spans_overlap(out_p[i], out_n[i], out_p[j], out_n[j])) return GNORM_ERR_ALIAS;
  }
  HostLayout L;
  int st = host_layout(M, N, deterministic, &L);  // queries the device
  if (st != GNORM_OK) return st;
  if (dev_bytes < L.total) return GNORM_ERR_WORKSPACE;

  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return GNORM_ERR_CUDA;
  if (dev < 0 || dev >= kMaxHostDevices) return GNORM_ERR_UNSUPPORTED;
  std::lock_guard<std::mutex> lock(g_pipe_mu[dev]);
  HostPipe* p = nullptr;
  st = pipe_for_device(dev, &p);
  if (st != GNORM_OK) return st;

  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* base = static_cast<uint8_t*>(dev_buf);
  uint8_t* x_dev = base + L.off_x;
  uint8_t* g_dev = base + L.off_g;
  uint8_t* dy_dev = base + L.off_dy;
  uint8_t* y_dev = base + L.off_y;
  uint8_t* dx_dev = base + L.off_dx;
  uint8_t* dg_dev = base + L.off_dg;
  float* rstd_dev = reinterpret_cast<float*>(base + L.off_rstd);
  uint8_t* w_dev = base + L.off_w;
  float* dwc_dev = reinterpret_cast<float*>(base + L.off_dwc);
  uint8_t* dw_dev = base + L.off_dw;
  uint8_t* ws_dev = base + L.off_ws;
  auto ok = [](cudaError_t e) { return e == cudaSuccess; };

  if (M == 0) {  // dw = 0, copied out in stream order
    if (!ok(cudaMemsetAsync(dw_dev, 0, dwb, s)) ||
        !ok(cudaMemcpyAsync(dw, dw_dev, dwb, cudaMemcpyDeviceToHost, s)))
      return GNORM_ERR_CUDA;
    return GNORM_OK;
  }

  // Fork: the copies in wait for everything already on the caller's stream.  The
  // workspace's counters start at zero.  From here on every return joins the copy streams
  // back into the caller's stream (best effort on a failing runtime), so even a call that
  // fails part way stays ordered on `stream`; its outputs are then undefined.
  auto fail = [&](int status) {
    if (cudaEventRecord(p->dw_done, p->in) == cudaSuccess)
      (void)cudaStreamWaitEvent(p->out, p->dw_done, 0);
    if (cudaEventRecord(p->end, p->out) == cudaSuccess) (void)cudaStreamWaitEvent(s, p->end, 0);
    return status;
  };
  if (!ok(cudaMemsetAsync(ws_dev, 0, GNORM_WORKSPACE_ALIGN, s)) || !ok(cudaEventRecord(p->start, s)))
    return GNORM_ERR_CUDA;  // nothing forked yet
  if (!ok(cudaStreamWaitEvent(p->in, p->start, 0)) || !ok(cudaStreamWaitEvent(p->out, p->start, 0)))
    return fail(GNORM_ERR_CUDA);
  if (!ok(cudaMemcpyAsync(w_dev, w, static_cast<size_t>(N) * 2, cudaMemcpyHostToDevice, p->in)))
    return fail(GNORM_ERR_CUDA);
  const size_t row_b = static_cast<size_t>(N) * 2;
  for (int k = 0; k < L.chunks; ++k) {
    const int64_t r0 = k * L.rows_per_chunk;
    const int64_t rows = (M - r0 < L.rows_per_chunk) ? M - r0 : L.rows_per_chunk;
    const size_t o = static_cast<size_t>(r0) * row_b, n = static_cast<size_t>(rows) * row_b;
    if (!ok(cudaMemcpyAsync(x_dev + o, static_cast<const uint8_t*>(x) + o, n, cudaMemcpyHostToDevice, p->in)) ||
        !ok(cudaMemcpyAsync(g_dev + o, static_cast<const uint8_t*>(g) + o, n, cudaMemcpyHostToDevice, p->in)) ||
        !ok(cudaMemcpyAsync(dy_dev + o, static_cast<const uint8_t*>(dy) + o, n, cudaMemcpyHostToDevice, p->in)) ||
        !ok(cudaEventRecord(p->in_done[k], p->in)))
      return fail(GNORM_ERR_CUDA);
  }
  for (int k = 0; k < L.chunks; ++k) {
    const int64_t r0 = k * L.rows_per_chunk;
    const int64_t rows = (M - r0 < L.rows_per_chunk) ? M - r0 : L.rows_per_chunk;
    const size_t o = static_cast<size_t>(r0) * row_b, n = static_cast<size_t>(rows) * row_b;
    if (!ok(cudaStreamWaitEvent(s, p->in_done[k], 0))) return fail(GNORM_ERR_CUDA);
    st = gnorm_ckpt_step(x_dev + o, g_dev + o, w_dev, eps, dy_dev + o, y_dev + o, rstd_dev + r0,
                         dx_dev + o, dg_dev + o, dwc_dev + static_cast<size_t>(k) * N, 1,
                         deterministic, rows, N, ws_dev, L.ws_bytes, s);
    if (st != GNORM_OK) return fail(st);
    if (!ok(cudaEventRecord(p->step_done[k], s)) || !ok(cudaStreamWaitEvent(p->out, p->step_done[k], 0)))
      return fail(GNORM_ERR_CUDA);
    if (!ok(cudaMemcpyAsync(static_cast<uint8_t*>(y) + o, y_dev + o, n, cudaMemcpyDeviceToHost, p->out)) ||
        !ok(cudaMemcpyAsync(rstd + r0, rstd_dev + r0, static_cast<size_t>(rows) * 4,
                            cudaMemcpyDeviceToHost, p->out)) ||
        !ok(cudaMemcpyAsync(static_cast<uint8_t*>(dx) + o, dx_dev + o, n, cudaMemcpyDeviceToHost, p->out)) ||
        !ok(cudaMemcpyAsync(static_cast<uint8_t*>(dg) + o, dg_dev + o, n, cudaMemcpyDeviceToHost, p->out)))
      return fail(GNORM_ERR_CUDA);
  }
  // dw: the chunks' FP32 rows summed in chunk order, then copied out; join.
  st = gnorm_dw_reduce(dwc_dev, L.chunks, N, dw_dev, dw_fp32, s);
  if (st != GNORM_OK) return fail(st);
  if (!ok(cudaEventRecord(p->dw_done, s)) || !ok(cudaStreamWaitEvent(p->out, p->dw_done, 0)) ||
      !ok(cudaMemcpyAsync(dw, dw_dev, dwb, cudaMemcpyDeviceToHost, p->out)) ||
      !ok(cudaEventRecord(p->end, p->out)) || !ok(cudaStreamWaitEvent(s, p->end, 0)))
    return fail(GNORM_ERR_CUDA);
  return GNORM_OK;
}
