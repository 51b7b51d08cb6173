/*
 * gnorm.h -- C ABI of libgnorm: SiLU-gated RMSNorm training kernels for B200 (sm_100a).
 *
 * The operation is "Cake's SiLU-gated RMSNorm training kernel" of flashinfer PR #8701
 * ("perf(cake_rmsnorm_silu_gate_train): L2-prefetching extra-long forward on SM107",
 * PR description), with the semantics of the comparator kernels listed in that page's
 * section "How the tables were measured" (FLA rms_norm_gated, mamba_ssm rmsnorm_fn):
 * normalise each row, scale by the weight, gate by silu(g).  For a row x of length N,
 * gate g, weight w and upstream gradient dy:
 *
 *     r   = 1 / sqrt(mean_j(x_j^2) + eps)                      (rstd, FP32, saved)
 *     y_j = x_j * r * w_j * g_j * sigmoid(g_j)                 (BF16)
 *     xhat = x r,  s = g sigmoid(g),  u = dy w s,  c = mean_j(u_j xhat_j)
 *     dx  = r (u - xhat c)                                     (BF16)
 *     dg  = dy xhat w sigmoid(g) (1 + g (1 - sigmoid(g)))      (BF16)
 *     dw  = sum over rows of dy xhat s                         (BF16 or FP32)
 *
 * Conventions for every entry point:
 *   - Tensors are row-major and contiguous ("packed" rows): element (m, j) of an [M, N]
 *     tensor sits at index m*N + j.  x, g, w, y, dy, dx, dg are BF16 (IEEE bfloat16 bit
 *     patterns, 2 bytes); rstd is FP32; dw is BF16 or FP32 (dw_fp32).
 *   - All tensor pointers are DEVICE pointers of the current CUDA device (except for
 *     gnorm_ckpt_step_host, which takes host buffers).  Every pointer except rstd must be
 *     16-byte aligned; rstd must be 4-byte aligned.
 *   - N must be a multiple of 8 with 8 <= N <= GNORM_N_MAX.  M >= 0; M == 0 is a no-op
 *     for the forward, and the backward then writes dw = 0.  When M == 0 the per-row
 *     tensors may be NULL.
 *   - eps must be finite and >= 0.
 *   - `stream` is a cudaStream_t (NULL = the legacy default stream).  Calls only enqueue
 *     work: they never synchronise, never allocate and are safe to capture in a CUDA
 *     graph (gnorm_ckpt_step_host excepted; see there).  Each kernel is launched with
 *     programmatic dependent launch, so it may start its prologue while the previous
 *     kernel on the stream drains; it reads and writes global memory only after that
 *     kernel has completed -- except that inside gnorm_ckpt_step the second forward and
 *     the backward may start reading x, g and dy early, which their predecessors in the
 *     same call never write.
 *   - The caller owns every buffer; the library keeps no pointer after a call returns.
 *   - Outputs must not overlap any input or each other (GNORM_ERR_ALIAS).
 *   - Errors are detected on the host before any launch and returned as a gnorm_status;
 *     no kernel traps.  A CUDA error at launch returns GNORM_ERR_CUDA.
 */
#ifndef GNORM_H_
#define GNORM_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GNORM_API __attribute__((visibility("default")))
#else
#define GNORM_API
#endif

#define GNORM_N_MAX 16384
#define GNORM_WORKSPACE_ALIGN 256

typedef enum gnorm_status {
  GNORM_OK = 0,
  GNORM_ERR_NULL = -1,        /* a required pointer is NULL */
  GNORM_ERR_SHAPE = -2,       /* M < 0, N not a multiple of 8, N < 8 or N > GNORM_N_MAX */
  GNORM_ERR_ALIGN = -3,       /* a pointer breaks the alignment rule above */
  GNORM_ERR_ALIAS = -4,       /* an output overlaps an input or another output */
  GNORM_ERR_UNSUPPORTED = -5, /* no kernel plan fits the device (e.g. too little shared memory) */
  GNORM_ERR_WORKSPACE = -6,   /* workspace NULL, misaligned or smaller than required */
  GNORM_ERR_CUDA = -7,        /* the CUDA runtime reported an error */
  GNORM_ERR_ARG = -8          /* another argument is out of range (eps, flags, kind) */
} gnorm_status;

/*
 * Forward.  Reads x[M,N], g[M,N], w[N]; writes y[M,N] (BF16) and rstd[M] (FP32).
 * Flashinfer PR #8701, section "How the tables were measured": "fwd" is one forward call.
 * The result does not depend on any mode flag: the deterministic and non-deterministic
 * packages of that page produce bitwise-equal y (commit message of the PR).
 */
GNORM_API int gnorm_fwd(const void* x, const void* g, const void* w, float eps,
              void* y, float* rstd, int64_t M, int64_t N, void* stream);

/*
 * Backward.  Reads dy, x, g [M,N], w[N] and the forward's rstd[M]; writes dx, dg [M,N]
 * (BF16) and dw[N] (BF16 if dw_fp32 == 0, else FP32).  dw is overwritten, not accumulated.
 * Flashinfer PR #8701, section "How the tables were measured": "bwdg" (BF16 dw) and
 * "bwdg_f32" (FP32 dw); the deterministic package is the same API with deterministic=True.
 *
 * Each CTA sums its rows' dw terms in FP32 into one partial row; a second pass sums the
 * partials in a fixed order in a second launch (or, when the tail_reduce knob asks and
 * partials x N <= 65536, in the backward's last CTA to finish).
 * deterministic != 0: rows are assigned to CTAs by a fixed rule, so dx, dg and dw are
 *   bitwise identical from run to run on the same device model with the same arguments.
 * deterministic == 0: CTAs take row blocks from a shared counter, so dw's FP32 summation
 *   order can change between runs (dx and dg do not); dw is never accumulated with float
 *   atomics.
 *
 * workspace: device scratch of at least gnorm_bwd_workspace_bytes(M, N, deterministic)
 *   bytes, GNORM_WORKSPACE_ALIGN-aligned.  Its first GNORM_WORKSPACE_ALIGN bytes must be
 *   zero before the first call (e.g. cudaMemset once after allocation); every call that
 *   completes normally leaves them zero again.  A call whose bounded wait gave up (a nonzero
 *   gnorm_device_error) may return before it restores them, and its outputs are then
 *   undefined: zero the first GNORM_WORKSPACE_ALIGN bytes again before reusing the
 *   workspace.  Concurrent calls must not share a workspace.
 */
GNORM_API int gnorm_bwd(const void* dy, const void* x, const void* g, const void* w, const float* rstd,
              void* dx, void* dg, void* dw, int dw_fp32, int deterministic,
              int64_t M, int64_t N, void* workspace, size_t workspace_bytes, void* stream);

/*
 * Backward without any caller-provided scratch (the pages have no counterpart to this entry
 * point).  For callers that cannot allocate device memory -- a runtime whose device memory
 * is owned up front by another allocator, a latency-critical loop that must not hit
 * cudaMalloc's implicit synchronisation, a plug-in that only receives tensors -- and so
 * cannot provide gnorm_bwd's workspace.  Same arguments and results as gnorm_bwd, minus the
 * workspace; it allocates nothing and calls no allocating routine.
 *
 * Its scratch is a file-scope static device array of 4 MiB in the library, held on every
 * GPU that loads the library until the process exits.  Calls whose FP32 dw partials need
 * more (about partials x N x 4 bytes + 256; e.g. N > 7000 on a 148-SM B200) return
 * GNORM_ERR_UNSUPPORTED.  The first call on a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current); make that first call before any stream
 * capture.  Every call clears the array's 256-byte counter header on `stream` before its
 * kernels start; all calls share the array, so calls that overlap on the GPU (other
 * streams, other threads) race and must be serialised by the caller.  A wait timeout inside
 * these kernels sets its bit in the device error word that gnorm_device_error reads, as for
 * every other entry point; the next call clears the array's header again in any case.
 */
GNORM_API int gnorm_bwd_noalloc(const void* dy, const void* x, const void* g, const void* w,
                                const float* rstd, void* dx, void* dg, void* dw, int dw_fp32,
                                int deterministic, int64_t M, int64_t N, void* stream);

/*
 * Strided rows and an FP32 weight.  Flashinfer PR #8701's commit message specialises its
 * forward for inputs "where x and z hold their rows packed", so its API also takes rows
 * that are not packed; these descriptors carry a row stride per tensor.  ld* = elements
 * between the starts of consecutive rows (0 means N, i.e. packed); a stride must be >= N
 * and a multiple of 8 (rows start 16-byte aligned).  w is FP32 [N] if w_fp32 != 0, else
 * BF16.  rstd and dw are always packed vectors.  Outputs may share a buffer with other
 * tensors as long as no element is shared (e.g. dx and dg as the two column halves of one
 * [M, 2N] gradient): the alias check is exact for tensors with the same stride and
 * conservative (whole byte extents) otherwise.  All other rules are those of gnorm_fwd /
 * gnorm_bwd; the packed entry points are these with every stride N and a BF16 weight.
 */
typedef struct gnorm_fwd_desc {
  const void* x;
  int64_t ldx;
  const void* g;
  int64_t ldg;
  const void* w;
  int w_fp32;
  float eps;
  void* y;
  int64_t ldy;
  float* rstd;
  int64_t M;
  int64_t N;
} gnorm_fwd_desc;

typedef struct gnorm_bwd_desc {
  const void* dy;
  int64_t lddy;
  const void* x;
  int64_t ldx;
  const void* g;
  int64_t ldg;
  const void* w;
  int w_fp32;
  const float* rstd;
  void* dx;
  int64_t lddx;
  void* dg;
  int64_t lddg;
  void* dw;
  int dw_fp32;
  int deterministic;
  int64_t M;
  int64_t N;
  void* workspace;
  size_t workspace_bytes;
} gnorm_bwd_desc;

GNORM_API int gnorm_fwd_ex(const gnorm_fwd_desc* desc, void* stream);
GNORM_API int gnorm_bwd_ex(const gnorm_bwd_desc* desc, void* stream);

/*
 * Checkpointed step with descriptors: x, g, w, eps, y, rstd, M, N come from `fwd`; dy, dx,
 * dg, dw, dw_fp32, deterministic and the workspace from `bwd`, whose x, g, w, rstd fields
 * must be NULL or equal to the forward's (same pointers, strides and weight type), and whose
 * M and N must equal the forward's.
 */
GNORM_API int gnorm_ckpt_step_ex(const gnorm_fwd_desc* fwd, const gnorm_bwd_desc* bwd,
                                 void* stream);

/*
 * Checkpointed training step: forward, forward again (activation recomputation), backward,
 * all enqueued on `stream`.  Flashinfer PR #8701, section "How the tables were measured":
 * "ckptg" is the checkpointed step (2 x forward + backward), "stepg_f32" the same with an
 * FP32 dw.  y and rstd hold the second forward's outputs (bitwise equal to the first's);
 * the backward consumes that rstd.  The recompute forward and the backward run as
 * gnorm_fwd_bwd (one kernel that reads x, g and dy once for both).  Arguments as for
 * gnorm_fwd and gnorm_bwd.
 */
GNORM_API int gnorm_ckpt_step(const void* x, const void* g, const void* w, float eps, const void* dy,
                    void* y, float* rstd, void* dx, void* dg, void* dw,
                    int dw_fp32, int deterministic, int64_t M, int64_t N,
                    void* workspace, size_t workspace_bytes, void* stream);

/*
 * Forward and backward of the same rows in one pass: the recompute forward of an
 * activation-checkpointed layer followed by its backward (the last two calls of the pages'
 * "ckptg", flashinfer PR #8701, section "How the tables were measured", which times them as
 * separate calls; fusing them is this library's own).  Reads x, g, w and dy; writes the
 * forward's outputs y and rstd and the backward's dx, dg and dw -- bitwise the values of
 * gnorm_fwd followed by gnorm_bwd with the same arguments (dw too in deterministic mode) --
 * while reading x and g once instead of twice and never reading rstd back: per row 12N + 4
 * bytes of DRAM traffic instead of 16N + 8.  Where the backward's plan loads rows straight
 * into registers (few rows per SM) it runs as those two kernels.  Arguments and workspace
 * as for gnorm_ckpt_step (and gnorm_fwd_bwd_ex as for gnorm_ckpt_step_ex).
 */
GNORM_API int gnorm_fwd_bwd(const void* x, const void* g, const void* w, float eps, const void* dy,
                            void* y, float* rstd, void* dx, void* dg, void* dw, int dw_fp32,
                            int deterministic, int64_t M, int64_t N, void* workspace,
                            size_t workspace_bytes, void* stream);
GNORM_API int gnorm_fwd_bwd_ex(const gnorm_fwd_desc* fwd, const gnorm_bwd_desc* bwd, void* stream);

/*
 * Checkpointed step on HOST buffers (no counterpart in the pages: an entry point for callers
 * whose batch lives in host memory).  x, g, dy [M, N] BF16 and w [N] BF16 are read from host
 * memory; y, dx, dg [M, N] BF16, rstd [M] FP32 and dw [N] (FP32 if dw_fp32, else BF16) are
 * written to host memory; all rows packed.  The rows are processed in chunks (about 4 MiB of
 * x, g and dy each; 32 MiB when x, g and dy exceed 64 MiB) as a pipeline over the caller's
 * stream and two copy streams the library creates once per device: chunk k's inputs are
 * copied in while chunk k-1's step runs and earlier chunks' outputs are copied out, so both
 * directions of the host link work at once.
 * Each chunk runs gnorm_ckpt_step with an FP32 dw of its own rows; dw is the fixed-order sum
 * of those rows (gnorm_dw_reduce).  y, rstd, dx and dg are bitwise equal to gnorm_ckpt_step's;
 * dw is too when there is one chunk (M x N x 6 bytes <= 4 MiB), and otherwise is rounded
 * differently but is still bitwise stable run to run in deterministic mode.
 *
 * dev_buf: device scratch of at least gnorm_ckpt_step_host_bytes(M, N, deterministic) bytes,
 *   GNORM_WORKSPACE_ALIGN-aligned, owned by the caller; it holds device copies of every
 *   tensor, so it must not be shared by calls that may overlap on the GPU.  No state is kept
 *   between calls.
 * Host buffers: pinned memory (cudaHostAlloc / cudaHostRegister) makes the copies
 *   asynchronous and lets them overlap; pageable memory works but serialises them and blocks
 *   the calling thread.  Outputs may overlap neither an input nor each other
 *   (GNORM_ERR_ALIAS).  The buffers must stay valid until `stream` has reached the end of
 *   the call: it returns once everything is enqueued; the caller's stream waits for the
 *   last copy out, so synchronising the stream (or an event recorded on it afterwards)
 *   means every host output is written.  Errors: as gnorm_ckpt_step, and GNORM_ERR_WORKSPACE
 *   for a missing, misaligned or small dev_buf.  A call that fails after it has started
 *   enqueueing still joins its copy streams back into `stream` before it returns, so the
 *   copies already queued are ordered on `stream` as well; its outputs are then undefined.
 *   Not meant for CUDA graph capture.
 */
GNORM_API int gnorm_ckpt_step_host(const void* x, const void* g, const void* w, float eps,
                                   const void* dy, void* y, float* rstd, void* dx, void* dg,
                                   void* dw, int dw_fp32, int deterministic, int64_t M, int64_t N,
                                   void* dev_buf, size_t dev_bytes, void* stream);

/*
 * Device bytes gnorm_ckpt_step_host needs on the CURRENT device for this shape (0 if the
 * arguments are invalid or no device is present).
 */
GNORM_API size_t gnorm_ckpt_step_host_bytes(int64_t M, int64_t N, int deterministic);

/*
 * Fixed-order sum of P rows of FP32 partials [P, N] (device memory, row-major) into dw[N]
 * (BF16 if dw_fp32 == 0, else FP32), with the same kernel and summation order as the
 * backward's deterministic second pass (the fixed-order FP32 partial reduction of flashinfer
 * PR #8878's commit message).  Data-parallel training uses it to combine per-rank FP32 dw
 * gathered in rank order: every rank then holds bitwise the same dw, independent of the
 * collective's own reduction order.  P == 0 writes dw = 0.  partials and dw 16-byte aligned,
 * not overlapping; N a multiple of 8 up to GNORM_N_MAX.
 */
GNORM_API int gnorm_dw_reduce(const float* partials, int64_t P, int64_t N, void* dw, int dw_fp32,
                              void* stream);

/*
 * Workspace bytes gnorm_bwd / gnorm_ckpt_step need on the CURRENT device (reads its SM count).
 * Returns 0 if the arguments are invalid or no device is present.
 */
GNORM_API size_t gnorm_bwd_workspace_bytes(int64_t M, int64_t N, int deterministic);

/* The same for a device with `num_sms` SMs.  Pure host function; needs no GPU. */
GNORM_API size_t gnorm_bwd_workspace_bytes_for(int64_t M, int64_t N, int deterministic, int num_sms);

/* Human-readable name of a gnorm_status value (static storage). */
GNORM_API const char* gnorm_status_string(int status);

/*
 * Launch plan chosen by the rows-per-SM dispatch rule.  Flashinfer PR #8701 (PR description
 * and commit message) routes its forward by architecture and by rows per SM
 * (M / number of SMs) into tiers; this library's rule is its own, tuned for B200.
 */
typedef struct gnorm_plan {
  int kind;              /* 0 forward, 1 backward, 2 forward fused into the backward */
  int threads_per_row;   /* threads that share one row */
  int chunks_per_thread; /* 16-byte chunks (8 BF16 values) per thread and tensor */
  int consumer_threads;  /* computing threads per CTA (one extra warp issues the copies) */
  int rows_per_stage;    /* rows copied into shared memory per pipeline stage */
  int stages;            /* pipeline depth */
  int ctas_per_sm;       /* resident CTAs per SM */
  int grid;              /* persistent CTAs launched */
  int64_t num_blocks;    /* row blocks: ceil(M / rows_per_stage) */
  int smem_bytes;        /* dynamic shared memory per CTA */
  int dynamic_schedule;  /* 1: CTAs take row blocks from an atomic counter */
  int fused_reduce;      /* 1: the last CTA to finish reduces the dw partials */
  int partials;          /* rows of the FP32 dw partial buffer (backward), else 0 */
  int l2_prefetch;       /* 1: warm L2 with the block each CTA loads after its ring's */
  int direct_loads;      /* 1 = rows loaded straight into registers, no staging
                            (rows_per_stage = rows per CTA and iteration, stages = 0) */
} gnorm_plan;

/*
 * The dispatch rule as a pure host function: plan for `kind` (0 fwd, 1 bwd, 2 the fused
 * forward + backward of gnorm_fwd_bwd, which falls back to kinds 0 and 1 when its plan loads
 * rows straight into registers) on a device with
 * `num_sms` SMs and `smem_per_block` bytes of opt-in shared memory per CTA (0 = 232448, the
 * B200 value).  Needs no GPU.  Returns GNORM_OK or an error status.
 */
GNORM_API int gnorm_plan_query(int kind, int64_t M, int64_t N, int deterministic, int num_sms,
                     int smem_per_block, gnorm_plan* out);

/*
 * Device-side error word: kernels set a bit here if a bounded wait inside them gave up
 * (1 = a wait for copied data, 2 = a wait for a free pipeline stage, 4 = the self-test's
 * wait, see gnorm_selftest_wait_timeout).  Synchronises the
 * current device, returns the word and clears it if `reset` != 0.  Returns -1 (as an int)
 * if the word cannot be read.
 */
GNORM_API int gnorm_device_error(int reset);

/*
 * Process-wide tuning knobs for experiments.  Every field 0 keeps the built-in choice.
 * Affects plans and launches made after the call (including gnorm_plan_query and
 * gnorm_bwd_workspace_bytes); not thread-safe with concurrent calls.  NULL resets all.
 */
typedef struct gnorm_tuning {
  int stage_bytes;       /* target bytes per pipeline stage */
  int max_stages;        /* maximum pipeline depth */
  int ctas_per_sm;       /* resident CTAs per SM (capped by the kernel's compiled residency) */
  int disable_pdl;       /* 1: launch without programmatic dependent launch */
  int threads_per_row;   /* with chunks_per_thread: force a compiled row geometry covering N, */
  int chunks_per_thread; /*   else plans fail with GNORM_ERR_UNSUPPORTED */
  int l2_prefetch;       /* 1: warm L2 with the block after each CTA's ring, 2: do not */
  int tail_reduce;       /* 1: dw second pass in the backward's last CTA when small, 2: never */
  int chain_prefetch;    /* 1: in gnorm_ckpt_step, copy inputs before the previous kernel ends, 2: do not */
  int host_chunk_bytes;  /* gnorm_ckpt_step_host: bytes of x, g and dy per chunk */
  int fwd_direct;        /* forward of rows of N <= 256: 1 load straight into registers at any
                            size, 2 always stage rows in shared memory (0: by rows per SM) */
  int bwd_direct;        /* backward of rows of N <= 256: 1 load straight into registers at any
                            size, 2 always stage rows in shared memory (0: by rows per SM) */
  int fuse_fwd_bwd;      /* gnorm_fwd_bwd and the checkpointed step's recompute: 1 the forward
                            and the backward in one kernel where the backward plan stages its
                            rows, 2 always two kernels (0: built-in, fused) */
} gnorm_tuning;

GNORM_API void gnorm_set_tuning(const gnorm_tuning* tuning);

/*
 * Self-test of the bounded waits every kernel uses: launches one thread that waits on a
 * barrier nothing arrives on, with a limit of `timeout_us` microseconds (1 .. 1000000).
 * The wait gives up, sets bit 4 in the device error word (see gnorm_device_error) and the
 * kernel returns; no fault, trap or hang.  Writes the time the wait took before giving up
 * to *waited_ns (0 would mean the wait completed, which it cannot).  Synchronises the
 * device and allocates 8 bytes: a diagnostic, not for use inside graphs.
 */
GNORM_API int gnorm_selftest_wait_timeout(unsigned timeout_us, unsigned long long* waited_ns);

/* Build description: compiler version, target architecture (static storage). */
GNORM_API const char* gnorm_build_info(void);

#ifdef __cplusplus
}
#endif

#endif /* GNORM_H_ */
