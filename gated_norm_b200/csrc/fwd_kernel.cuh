// fwd_kernel.cuh -- forward of the SiLU-gated RMSNorm on sm_100a.
//
// y = x * rsqrt(mean(x^2) + eps) * w * g * sigmoid(g) over packed BF16 rows [M, N]; the
// FP32 rstd of every row is saved for the backward.  (flashinfer PR #8701, "perf(
// cake_rmsnorm_silu_gate_train): L2-prefetching extra-long forward on SM107": the forward
// of "Cake's SiLU-gated RMSNorm training kernel"; the pages print no kernel, so the design
// below is this library's own.)
//
// Design: a persistent, warp-specialised CTA.  Warp 0 streams row blocks of x and g from
// HBM into a ring of shared-memory stages with 1-D TMA bulk copies and mbarrier transaction
// counts (packed rows: a block of R rows of one tensor is one contiguous copy; strided rows:
// one copy per row, spread over the warp's lanes).  The consumer warps own `TPR` threads per row and `CPT`
// 16-byte chunks per thread: pass 1 reads x from shared memory and reduces the sum of
// squares (shuffles, plus named-barrier slots when a row spans several warps); pass 2
// reads g and writes y straight to HBM with 16-byte stores.  Row blocks are assigned
// round-robin (block b, b + grid, ...), a pure function of the launch plan.
#pragma once

#include "args.h"
#include "device_common.cuh"

namespace gnorm {


template <int TPR, int CPT, bool kWFp32>
__global__ void __launch_bounds__(consumer_threads_for(0, TPR, CPT) + 32, max_ctas_per_sm(0, TPR, CPT))
    gated_rmsnorm_fwd_kernel(const __grid_constant__ FwdArgs a) {
  constexpr int kNCT = consumer_threads_for(0, TPR, CPT);
  constexpr int kGroups = kNCT / TPR;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  long long* blk_id = reinterpret_cast<long long*>(smem + 256);
  float* red_slots = reinterpret_cast<float*>(smem + kRedSlotOffset);
  uint8_t* stage0 = smem + kHeaderBytes;

  const int S = a.stages;
  const int R = a.rows_per_stage;
  const int N = a.N;
  const uint32_t tensor_bytes = static_cast<uint32_t>(stage_tensor_bytes(R, N));  // one tensor of a stage
  const uint32_t stage_bytes = (2u * tensor_bytes + 127u) & ~127u;
  constexpr int num_consumer_warps = kNCT / 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], num_consumer_warps);
    }
    fence_barrier_init();
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Copies of stage s's block `blk` (x and g) by the producer warp's lanes, counted on the
  // stage's full barrier (lane 0 posts the byte count first).
  auto issue_copies = [&](int s, long long blk) {
    const long long r0 = blk * R;
    const long long left = a.M - r0;
    const int rows = static_cast<int>(left < R ? left : R);
    uint8_t* st = stage0 + static_cast<size_t>(s) * stage_bytes;
    if (lane == 0) mbar_expect_tx(&full[s], 2u * static_cast<uint32_t>(rows) * N * 2u);
    __syncwarp();
    copy_row_block(st, a.x, a.ldx, N, r0, rows, R, (a.map_bits & 1) ? &a.map_x : nullptr,
                   &full[s], lane);
    copy_row_block(st + tensor_bytes, a.g, a.ldg, N, r0, rows, R,
                   (a.map_bits & 2) ? &a.map_g : nullptr, &full[s], lane);
  };

  // When the host knows the previous kernel on the stream does not write x or g (the
  // recompute forward of a checkpointed step), the first stages' copies start before that
  // kernel has finished; nothing is written, and no stage is released to the consumers,
  // before the dependency wait below.
  int prefetched = 0;
  if (a.prefetch && warp == 0) {
    for (long long blk = blockIdx.x; prefetched < S && blk < a.num_blocks; blk += gridDim.x)
      issue_copies(prefetched++, blk);
  }
  grid_dependency_wait();     // inputs may come from the previous kernel on the stream
  allow_dependent_launch();   // the next kernel may start its prologue on free SMs

  if (warp == 0) {
    // ---------------- producer warp ----------------
    // Lane 0 waits for a free stage and publishes the block; the lanes issue its copies.
    int s = 0;
    uint32_t phase = 0;
    int it = 0;
    for (long long blk = blockIdx.x;; blk += gridDim.x, ++it) {
      if (it >= prefetched) {
        bool ok = true;
        if (lane == 0) ok = mbar_wait(&empty[s], phase ^ 1u, a.err, kErrWaitEmpty);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        __syncwarp();
        if (!ok) break;
        if (blk >= a.num_blocks) {
          if (lane == 0) {
            blk_id[s] = -1;
            mbar_arrive(&full[s]);
          }
          break;
        }
        issue_copies(s, blk);
        if (a.l2_prefetch && a.ldx == N && a.ldg == N && lane == 0) {
          // the block this stage will hold next time round the ring
          const long long ahead = blk + static_cast<long long>(S) * gridDim.x;
          if (ahead < a.num_blocks) {
            const long long left = a.M - ahead * R;
            const uint32_t rows = static_cast<uint32_t>(left < R ? left : R);
            const uint32_t bytes = rows * static_cast<uint32_t>(N) * 2u;
            bulk_prefetch_l2(a.x + ahead * R * N, bytes);
            bulk_prefetch_l2(a.g + ahead * R * N, bytes);
          }
        }
      }
      if (lane == 0) {  // publish the block (its copies are in flight)
        blk_id[s] = blk;
        mbar_arrive(&full[s]);
      }
      if (++s == S) {
        s = 0;
        phase ^= 1u;
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int ctid = threadIdx.x - 32;
  const int group = ctid / TPR;         // row slot inside a pass over the stage
  const int lr = ctid - group * TPR;    // thread index inside the row
  const int warp_group0 = (ctid & ~31) / TPR;  // first row slot of this warp
  const int n8 = N >> 3;                // 16-byte chunks per row

  float2 wp[CPT][4];  // this thread's weights, as FP32 pairs
  bool cval[CPT];
#pragma unroll
  for (int k = 0; k < CPT; ++k) {
    const int c = k * TPR + lr;
    cval[k] = c < n8;
#pragma unroll
    for (int i = 0; i < 4; ++i) wp[k][i] = splat2(0.f);
    if (cval[k]) load_weight_pairs<kWFp32>(a.w, c, wp[k]);
  }

  int s = 0;
  uint32_t phase = 0;
  int slot = 0;
  while (true) {
    if (!mbar_wait(&full[s], phase, a.err, kErrWaitFull)) break;
    const long long blk = blk_id[s];
    if (blk < 0) break;
    const long long r0 = blk * R;
    const long long left = a.M - r0;
    const int rows = static_cast<int>(left < R ? left : R);
    const uint8_t* sx = stage0 + static_cast<size_t>(s) * stage_bytes;
    const uint8_t* sg = sx + tensor_bytes;

    for (int rb = 0; rb < rows; rb += kGroups) {
      // A warp whose rows are all past the block's end skips the pass (a warp never spans
      // two row groups' barriers, so this is uniform per warp and per row group).
      if (rb + warp_group0 >= rows) break;
      const int row = rb + group;
      const bool valid = row < rows;
      const int srow = valid ? row : 0;  // keep shared-memory reads inside the stage
      const size_t roff = static_cast<size_t>(srow) * N * 2;

      // pass 1: sum of squares of the row (one partial per chunk, combined in the order
      // every row geometry shares)
      uint4 xv[CPT];
      float part[CPT];
#pragma unroll
      for (int k = 0; k < CPT; ++k) {
        part[k] = 0.f;
        if (cval[k]) {
          xv[k] = *reinterpret_cast<const uint4*>(sx + roff + (k * TPR + lr) * 16);
          float2 xp[4];
          bf16x8_to_pairs(xv[k], xp);
          part[k] = chunk_dot(xp, xp);
        }
      }
      const float ss = row_sum<TPR>(combine_chunks<CPT>(part), red_slots, group, lr, slot);
      slot ^= 1;
      const float r = rsqrtf(fmaf(ss, a.inv_n, a.eps));
      const long long grow = r0 + row;
      if (valid && lr == 0) a.rstd[grow] = r;

      // pass 2: y = (x r) (w (g sigmoid(g)))
      const float2 r2 = splat2(r);
#pragma unroll
      for (int k = 0; k < CPT; ++k) {
        if (cval[k]) {
          const int c = k * TPR + lr;
          const uint4 gv = *reinterpret_cast<const uint4*>(sg + roff + c * 16);
          float2 xp[4], gp[4], yp[4];
          bf16x8_to_pairs(xv[k], xp);
          bf16x8_to_pairs(gv, gp);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 silu = mul2(gp[i], sigmoid2(gp[i]));
            yp[i] = mul2(mul2(xp[i], r2), mul2(wp[k][i], silu));
          }
          if (valid)
            *reinterpret_cast<uint4*>(a.y + grow * a.ldy + c * 8) = pairs_to_bf16x8(yp);
        }
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&empty[s]);
    if (++s == S) {
      s = 0;
      phase ^= 1u;
    }
  }
}

}  // namespace gnorm
