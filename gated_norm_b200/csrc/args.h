// args.h -- kernel argument blocks (plain structs shared by host and device code).
#pragma once

#include <cuda.h>  // CUtensorMap
#include <stdint.h>

namespace gnorm {

// Row strides (ld*) are in elements; a tensor with ld == N is packed.  A strided tensor may
// also come with a 2-D tiled tensor map (box = N columns x rows_per_stage rows) that loads a
// whole row block in one copy; map_bits says which maps are valid.
struct FwdArgs {
  CUtensorMap map_x, map_g;
  int map_bits = 0;  // bit 0: map_x, bit 1: map_g
  const uint16_t* x;
  const uint16_t* g;
  const void* w;  // BF16 or FP32 [N] (w_fp32)
  uint16_t* y;
  float* rstd;
  long long ldx = 0, ldg = 0, ldy = 0;
  int w_fp32 = 0;
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
  CUtensorMap map_dy, map_x, map_g;
  int map_bits = 0;  // bit 0: map_dy, bit 1: map_x, bit 2: map_g
  const uint16_t* dy;
  const uint16_t* x;
  const uint16_t* g;
  const void* w;  // BF16 or FP32 [N] (w_fp32)
  const float* rstd;
  uint16_t* dx;
  uint16_t* dg;
  long long lddy = 0, ldx = 0, ldg = 0, lddx = 0, lddg = 0;
  int w_fp32 = 0;
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
  // Fused forward (gnorm_fwd_bwd): the kernel computes each row's rstd itself from the
  // staged x, writes it to rstd_out and y = x r w silu(g) to y, and reads no rstd.
  int fused_fwd = 0;
  uint16_t* y = nullptr;
  long long ldy = 0;
  float* rstd_out = nullptr;
  float eps = 0.f;
};

}  // namespace gnorm
