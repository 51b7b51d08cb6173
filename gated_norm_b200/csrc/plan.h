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
constexpr int64_t kFusedReduceMaxFloats = 65536;

struct RowGeometry {
  int threads_per_row;
  int chunks_per_thread;
};

// Experiment knobs (0 = built-in value).  Process-wide; not used unless set.
struct TuningKnobs {
  int stage_bytes;
  int max_stages;
  int ctas_per_sm;
  int disable_pdl;
  int threads_per_row;    // with chunks_per_thread: force a compiled row geometry
  int chunks_per_thread;
};

// Row geometries with compiled kernels, per kind (0 forward, 1 backward).
bool geometry_compiled(int kind, int threads_per_row, int chunks_per_thread);

void set_tuning(const TuningKnobs& k);
TuningKnobs get_tuning();

RowGeometry geometry_for(int64_t N);
int make_plan(int kind, int64_t M, int64_t N, int deterministic, int num_sms,
              int smem_per_block, gnorm_plan* out);
size_t workspace_bytes_for(const gnorm_plan& p, int64_t N);

}  // namespace gnorm
