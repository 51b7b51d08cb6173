// plan.h -- host-side launch planning (pure functions, no CUDA calls).
#pragma once

#include <cstddef>
#include <cstdint>

#include "gnorm.h"

namespace gnorm {

constexpr int kB200SmemPerBlock = 232448;  // opt-in dynamic shared memory per CTA (227 KB)
constexpr int kB200SmemPerSm = 233472;     // shared memory per SM (228 KB)
constexpr int kSmemPerCtaReserve = 1024;   // the driver's per-CTA reservation
// Defaults chosen by measurement on B200 (sweeps of stage size x CTAs per SM x row geometry
// over the five workloads):
//  * forward, streaming tier: 2 CTAs per SM, ~48 KB stages;
//  * forward, latency tier (under kFwdLatencyTierBytes of staged rows per SM): 3 CTAs per SM
//    (where the geometry's registers allow), ~16 KB stages -- more, smaller CTAs start
//    streaming sooner when each SM has little data;
//  * backward: 1 CTA per SM, stages of ~48 KB or at least three rows.
constexpr int64_t kFwdStageBytes = 49152;
constexpr int64_t kFwdLatencyStageBytes = 16384;
constexpr int64_t kFwdLatencyTierBytes = 512 * 1024;
constexpr int64_t kBwdStageBytes = 49152;
constexpr int kBwdMinStageRows = 3;
// Backward of rows of N <= 256 loaded straight into registers under this many bytes of dy,
// x and g per SM (measured on B200: faster or equal up to ~220 rows per SM at N = 128, equal
// at ~440, slower beyond).
constexpr int64_t kBwdDirectTierBytes = 256 * 1024;
// At most 3 backward stages in flight per SM: measured best or equal on every workload
// (368640x128 backward 89.2 -> 83.1 us with 3 instead of 4 stages of ~48 KB).
constexpr int kBwdMaxStages = 3;
// Measured on B200 in same-box A/B runs (graph replays, cold L2):
//  * an L2 bulk prefetch of the block after each CTA's ring slows every workload (e.g.
//    368640x128 forward 55 -> 68 us, backward 86 -> 113 us): off;
//  * the dw second pass as a second (programmatic-dependent) launch is as fast as or faster
//    than running it in the backward's last CTA (e.g. 262144x256 backward 118.8 vs 121 us):
//    second launch by default;
//  * letting gnorm_ckpt_step's recompute forward and backward copy their inputs before the
//    previous kernel ends saves 3-6 us per step (e.g. 16384x4096 241 -> 235.5 us): on.
constexpr int kDefaultL2Prefetch = 0;
constexpr int kDefaultTailReduce = 0;
constexpr int kDefaultChainPrefetch = 1;
// gnorm_fwd_bwd / gnorm_ckpt_step: the (recompute) forward and the backward in one kernel,
// which reads x, g and dy once for both.
constexpr int kDefaultFuseFwdBwd = 1;
constexpr int64_t kFusedReduceMaxFloats = 65536;

struct RowGeometry {
  int threads_per_row;
  int chunks_per_thread;
};

// Experiment knobs (gnorm_tuning of include/gnorm.h; 0 = built-in value).  Process-wide.
using TuningKnobs = gnorm_tuning;

void set_tuning(const TuningKnobs& k);
TuningKnobs get_tuning();

// Row geometries with compiled kernels, per kind (0 forward, 1 backward).
bool geometry_compiled(int kind, int threads_per_row, int chunks_per_thread);

RowGeometry geometry_for(int kind, int64_t N);
int make_plan(int kind, int64_t M, int64_t N, int deterministic, int num_sms,
              int smem_per_block, gnorm_plan* out);
size_t workspace_bytes_for(const gnorm_plan& p, int64_t N);

}  // namespace gnorm
