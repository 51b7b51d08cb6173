// args.h -- kernel argument blocks (plain structs shared by host and device code).
#pragma once

#include <stdint.h>

namespace gnorm {

struct FwdArgs {
  const uint16_t* x;
  const uint16_t* g;
  const uint16_t* w;
  uint16_t* y;
  float* rstd;
  long long M;
  int N;
  float eps;
  float inv_n;
  int rows_per_stage;
  int stages;
  long long num_blocks;
  int prefetch = 0;  // 1: the first stages' inputs may be copied before the previous grid ends
  int l2_prefetch = 0;  // 1: also warm L2 with the block the CTA loads after the ring's
  unsigned* err;
};

struct BwdArgs {
  const uint16_t* dy;
  const uint16_t* x;
  const uint16_t* g;
  const uint16_t* w;
  const float* rstd;
  uint16_t* dx;
  uint16_t* dg;
  float* partial;                    // [gridDim.x, N] FP32 dw partials (workspace)
  void* dw;                          // written by the fused tail only
  unsigned long long* work_counter;  // dynamic schedule (workspace header)
  unsigned* ticket;                  // fused tail (workspace header)
  long long M;
  int N;
  float inv_n;
  int rows_per_stage;
  int stages;
  long long num_blocks;
  int dynamic_schedule;
  int fused_reduce;
  int dw_fp32;
  int prefetch = 0;  // 1: the first stages' dy, x, g may be copied before the previous grid ends
  int l2_prefetch = 0;  // 1: also warm L2 with the block the CTA loads after the ring's
  unsigned* err;
};

}  // namespace gnorm
