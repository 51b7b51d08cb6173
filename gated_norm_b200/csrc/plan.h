// plan.h -- host-side launch planning (pure functions, no CUDA calls).
#pragma once

#include <cstddef>
#include <cstdint>

#include "gnorm.h"

namespace gnorm {

constexpr int kB200SmemPerBlock = 232448;  // opt-in dynamic shared memory per CTA (227 KB)
constexpr int kB200SmemPerSm = 233472;     // shared memory per SM (228 KB)
constexpr int kSmemPerCtaReserve = 1024;   // the driver's per-CTA reservation
constexpr int64_t kStageTargetBytes = 24576;
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
};

void set_tuning(const TuningKnobs& k);
TuningKnobs get_tuning();

RowGeometry geometry_for(int64_t N);
int make_plan(int kind, int64_t M, int64_t N, int deterministic, int num_sms,
              int smem_per_block, gnorm_plan* out);
size_t workspace_bytes_for(const gnorm_plan& p, int64_t N);

}  // namespace gnorm
