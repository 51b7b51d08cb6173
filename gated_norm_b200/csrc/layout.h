// layout.h -- constants shared by the host-side plan and the kernels.
#pragma once

#ifdef __CUDACC__
#define GNORM_HD __host__ __device__
#else
#define GNORM_HD
#endif

namespace gnorm {

constexpr int kMaxStages = 16;       // mbarrier pairs reserved in the shared-memory header
constexpr int kHeaderBytes = 1024;   // barriers, block ids, flags and reduction slots
constexpr int kRedSlotOffset = 512;  // float slots for cross-warp row reductions
constexpr int kWorkspaceHeader = 256;  // workspace bytes before the dw partials
// dw second pass: a CTA owns kReduceQuads column quads, with kReduceLanes row lanes each
constexpr int kReduceThreads = 256;
constexpr int kReduceQuads = 8;
constexpr int kReduceLanes = kReduceThreads / kReduceQuads;

// Computing threads per CTA for a row geometry: 8 warps; one 16-warp row group for the
// widest rows; and 16 warps for the backward of narrow rows (<= 16 threads per row, one
// chunk per thread), which is latency-bound with 8 (measured on B200: the 368640 x 128
// checkpointed step 181 -> 176 us).  One more warp (the producer) issues the copies.
GNORM_HD constexpr int consumer_threads_for(int kind, int threads_per_row, int chunks_per_thread) {
  return threads_per_row > 256 ? threads_per_row
         : (kind == 1 && threads_per_row <= 16 && chunks_per_thread == 1) ? 512
                                                                           : 256;
}

// Resident CTAs per SM a kernel is compiled for (its __launch_bounds__ minimum), which caps
// its registers: 3 CTAs of 288 threads leave 75 registers per thread, 2 leave 113.  The
// dispatch rule never plans more CTAs per SM than this.
GNORM_HD constexpr int max_ctas_per_sm(int kind, int threads_per_row, int chunks_per_thread) {
  return consumer_threads_for(kind, threads_per_row, chunks_per_thread) > 256 ? 1
         : kind == 0 ? (chunks_per_thread == 1 ? 3 : (chunks_per_thread <= 4 ? 2 : 1))
                     : (chunks_per_thread == 1 ? 2 : 1);
}

// The forward for narrow rows in the latency tier loads its rows straight into registers
// (gated_rmsnorm_fwd_direct_kernel): 256 threads per CTA, all computing; each row group
// takes kDirectRows rows per iteration; kDirectCtasPerSm CTAs per SM (its
// __launch_bounds__ minimum: 64 registers per thread).
constexpr int kDirectThreads = 256;
constexpr int kDirectRows = 2;
constexpr int kDirectCtasPerSm = 4;
// The backward's counterpart (gated_rmsnorm_bwd_direct_kernel) for very few rows per SM:
// two rows per row group per iteration, 2 CTAs per SM (up to 128 registers per thread).
constexpr int kDirectBwdRows = 2;
constexpr int kDirectBwdCtasPerSm = 2;

// Bytes one tensor of a pipeline stage occupies: R rows of N BF16 values, rounded up to
// 128 bytes so every tensor of a stage starts 128-byte aligned (as tiled TMA copies require).
GNORM_HD constexpr long long stage_tensor_bytes(long long rows, long long n) {
  return (rows * n * 2 + 127) / 128 * 128;
}

}  // namespace gnorm
