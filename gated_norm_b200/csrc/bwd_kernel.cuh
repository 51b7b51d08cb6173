// bwd_kernel.cuh -- backward of the SiLU-gated RMSNorm on sm_100a, and the dw reduction.
//
// Per row, with the forward's FP32 rstd r:  xhat = x r,  s = g sigmoid(g),  u = dy w s,
// c = mean(u xhat),  dx = r (u - xhat c),  dg = dy xhat w sigmoid(g) (1 + g (1 - sigmoid(g))),
// and dw = sum over rows of dy xhat s.  (flashinfer PR #8701, "perf(cake_rmsnorm_silu_gate_
// train): L2-prefetching extra-long forward on SM107", section "How the tables were
// measured": "bwdg" / "bwdg_f32" -- the backward with a BF16 / FP32 dw; the deterministic
// package gives run-to-run bitwise results.  The fixed-order FP32 partial reduction follows
// the pattern described in flashinfer PR #8878's commit message: per-CTA FP32 accumulators
// reduced in a fixed order.)
//
// Design: the same persistent, warp-specialised TMA pipeline as the forward, with three
// tensors (dy, x, g) per stage (packed or strided rows).  Pass 1 recomputes xhat and the gate from shared memory,
// writes dg, accumulates the row dot product sum(u xhat) and this thread's dw columns in
// FP32 registers (arithmetic on packed FP32 pairs), and keeps u and xhat in registers; after
// the row reduction pass 2 writes dx.  The producer warp also stages the rows' rstd
// with 4-byte asynchronous copies tracked by the same stage barrier.  At the end each CTA adds its row groups' dw accumulators in a fixed order into one
// FP32 partial row [P, N] in the workspace.  A second pass sums the P partials in a fixed
// order and writes dw once, rounded to BF16 or kept in FP32: by default a second launch whose
// CTAs each own a few column quads; optionally (small partials) the backward's last CTA to finish,
// found with an integer ticket, never a wait.
#pragma once

#include "args.h"
#include "device_common.cuh"

namespace gnorm {


// Sums P rows of FP32 partials [P, N] into dw[N] in a fixed order: thread (bl, q) adds
// rows bl, bl + BL, bl + 2 BL, ... of column quad q, then the BL lanes are combined by a
// binary tree (BL = nthreads / 32, a power of two).  `scratch` holds nthreads float4.
template <bool kNamedBarrier>
__device__ __forceinline__ void reduce_partials(const float* __restrict__ partial, int P, int N,
                                                void* dw, int dw_fp32, int col_tile0,
                                                int col_tile_step, int tid, int nthreads,
                                                float4* scratch) {
  const int BL = nthreads >> 5;
  const int bl = tid >> 5;
  const int q = tid & 31;
  const int n4 = N >> 2;
  auto sync = [&]() {
    if constexpr (kNamedBarrier)
      named_barrier_sync(15, nthreads);
    else
      __syncthreads();
  };
  for (int t0 = col_tile0; t0 < n4; t0 += col_tile_step) {
    const int j4 = t0 + q;
    const bool valid = j4 < n4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    if (valid) {
      // Rows bl, bl + BL, ... in increasing order.  Loads are issued kBatch at a time
      // before the (sequential, fixed-order) adds, so a thread waits for one memory round
      // trip per batch instead of one per row.
      constexpr int kBatch = 8;
      const float4* p4 = reinterpret_cast<const float4*>(partial) + j4;
      for (int b0 = bl; b0 < P; b0 += kBatch * BL) {
        float4 v[kBatch];
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
          const int b = b0 + i * BL;
          v[i] = b < P ? __ldcg(p4 + static_cast<size_t>(b) * n4) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
#pragma unroll
        for (int i = 0; i < kBatch; ++i) {
          if (b0 + i * BL < P) {
            acc.x += v[i].x;
            acc.y += v[i].y;
            acc.z += v[i].z;
            acc.w += v[i].w;
          }
        }
      }
    }
    scratch[tid] = acc;
    sync();
    for (int st = BL >> 1; st > 0; st >>= 1) {
      if (bl < st) {
        const float4 o = scratch[tid + st * 32];
        float4 m = scratch[tid];
        m.x += o.x;
        m.y += o.y;
        m.z += o.z;
        m.w += o.w;
        scratch[tid] = m;
      }
      sync();
    }
    if (bl == 0 && valid) {
      const float4 m = scratch[q];
      if (dw_fp32) {
        reinterpret_cast<float4*>(dw)[j4] = m;
      } else {
        uint2 h;
        h.x = pack_bf16x2(m.x, m.y);
        h.y = pack_bf16x2(m.z, m.w);
        reinterpret_cast<uint2*>(dw)[j4] = h;
      }
    }
    sync();
  }
}

// Second pass over the dw partials (both modes).  A CTA of kReduceThreads threads owns
// kReduceQuads column quads (4 columns each); thread t takes quad t % kReduceQuads and row lane
// t / kReduceQuads (kReduceLanes lanes).  A lane adds partial rows lane, lane + kReduceLanes,
// ... of its quad in increasing order, all its loads in one batch for P <= 8 kReduceLanes; the
// lanes of a quad are then combined by a fixed tree: inside the warp by shuffles over its 4 row
// lanes (xor 8, then xor 16), then across the warps through shared memory, pairwise (offsets
// 4, 2, 1).  The order depends only on P.  A warp's loads are 4 rows x 128 contiguous bytes.
// Also clears the dynamic-schedule counter of the workspace (the backward grid has finished
// by now).
__global__ void __launch_bounds__(kReduceThreads)
    dw_reduce_kernel(const float* __restrict__ partial, int P, int N, void* dw, int dw_fp32,
                     unsigned long long* work_counter) {
  constexpr int kWarps = kReduceThreads / 32;
  constexpr int kBatch = 8;
  __shared__ float4 red[kWarps][kReduceQuads];
  grid_dependency_wait();
  allow_dependent_launch();
  const int q = threadIdx.x % kReduceQuads;
  const int rl = threadIdx.x / kReduceQuads;
  const int warp = threadIdx.x >> 5;
  const int n4 = N >> 2;
  const int j4 = blockIdx.x * kReduceQuads + q;
  const bool valid = j4 < n4;
  const float4* p4 = reinterpret_cast<const float4*>(partial);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int b0 = rl; b0 < P; b0 += kReduceLanes * kBatch) {
    float4 v[kBatch];
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      const int b = b0 + kReduceLanes * i;
      v[i] = (valid && b < P) ? __ldcg(p4 + static_cast<size_t>(b) * n4 + j4)
                              : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int i = 0; i < kBatch; ++i) {
      if (b0 + kReduceLanes * i < P) {
        acc.x += v[i].x;
        acc.y += v[i].y;
        acc.z += v[i].z;
        acc.w += v[i].w;
      }
    }
  }
  // the warp's 4 row lanes (lane bits 3 and 4)
#pragma unroll
  for (int off = kReduceQuads; off < 32; off <<= 1) {
    acc.x += __shfl_xor_sync(0xffffffffu, acc.x, off);
    acc.y += __shfl_xor_sync(0xffffffffu, acc.y, off);
    acc.z += __shfl_xor_sync(0xffffffffu, acc.z, off);
    acc.w += __shfl_xor_sync(0xffffffffu, acc.w, off);
  }
  if ((threadIdx.x & 31) < kReduceQuads) red[warp][q] = acc;
  __syncthreads();
#pragma unroll
  for (int st = kWarps / 2; st > 0; st >>= 1) {
    if (threadIdx.x < st * kReduceQuads) {
      const int w = threadIdx.x / kReduceQuads;
      float4 m = red[w][q];
      const float4 o = red[w + st][q];
      m.x += o.x;
      m.y += o.y;
      m.z += o.z;
      m.w += o.w;
      red[w][q] = m;
    }
    __syncthreads();
  }
  if (threadIdx.x < kReduceQuads && valid) {
    const float4 m = red[0][q];
    if (dw_fp32) {
      reinterpret_cast<float4*>(dw)[j4] = m;
    } else {
      uint2 h;
      h.x = pack_bf16x2(m.x, m.y);
      h.y = pack_bf16x2(m.z, m.w);
      reinterpret_cast<uint2*>(dw)[j4] = h;
    }
  }
  if (work_counter != nullptr && blockIdx.x == 0 && threadIdx.x == 0) *work_counter = 0ull;
}

// kFusedFwd: the forward of the same rows in the same pass (gnorm_fwd_bwd) -- each row's
// rstd is computed from the staged x (the forward's arithmetic and order, so the same bits),
// written out with y, and used for the backward; no rstd is read.
template <int TPR, int CPT, bool kWFp32, bool kFusedFwd>
__global__ void __launch_bounds__(consumer_threads_for(1, TPR, CPT) + 32, max_ctas_per_sm(1, TPR, CPT))
    gated_rmsnorm_bwd_kernel(const __grid_constant__ BwdArgs a) {
  constexpr int kNCT = consumer_threads_for(1, TPR, CPT);
  constexpr int kGroups = kNCT / TPR;
  // xhat stays in registers from pass 1 to pass 2 with one or two chunks per thread; with
  // four (rows wider than 4096) it is recomputed from the staged x, since keeping it spilled
  // registers, and spills are slow next to ~200 KB of stages (8192 x 8192 backward 132 ->
  // 113 us, fused forward + backward 226 -> 137 us without them)
  constexpr bool kKeepXhat = (kNCT <= 256 && CPT <= 2) || CPT == 1;
  // u = dy (w s) and the weights stay in registers too, except with 544 threads per CTA and
  // four chunks per thread (rows wider than 8192), where the registers are capped at 96:
  // each pass then reloads its chunk's weights and pass 2 recomputes u from the staged dy
  // and g (the same operations, so the same bits)
  constexpr bool kKeepU = kNCT <= 256 || CPT <= 2;
  // the fused forward's staged x, kept in registers from its row sum for pass 1.  Measured
  // together with y and u sharing w s (against neither): faster with 16 or more threads per
  // row (262144 x 256: 133.5 -> 129.9 us; 16384 x 4096: 145.6 -> 139.3 us), slower with 8
  // (368640 x 128: 93.8 -> 97.9 us); not with four chunks per thread (register spills)
  constexpr bool kKeepX = kFusedFwd && kKeepXhat && CPT <= 2 && TPR >= 16;
  extern __shared__ __align__(128) uint8_t smem[];
  uint64_t* full = reinterpret_cast<uint64_t*>(smem);
  uint64_t* empty = full + kMaxStages;
  long long* blk_id = reinterpret_cast<long long*>(smem + 256);
  int* last_flag = reinterpret_cast<int*>(smem + 384);
  float* red_slots = reinterpret_cast<float*>(smem + kRedSlotOffset);
  uint8_t* stage0 = smem + kHeaderBytes;

  const int S = a.stages;
  const int R = a.rows_per_stage;
  const int N = a.N;
  const uint32_t tensor_bytes = static_cast<uint32_t>(stage_tensor_bytes(R, N));
  const uint32_t stage_bytes = (3u * tensor_bytes + static_cast<uint32_t>(R) * 4u + 127u) & ~127u;

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      // 32 producer lanes' asynchronous rstd copies + the producer's own arrival
      mbar_init(&full[s], 33);
      mbar_init(&empty[s], kNCT / 32);
    }
    fence_barrier_init();
  }
  __syncthreads();

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  // Bulk copies of stage s's block `blk` (dy, x, g) by the producer warp's lanes, counted on
  // the stage's full barrier (lane 0 posts the byte count first).
  auto issue_copies = [&](int s, long long blk) {
    const long long r0 = blk * R;
    const long long left = a.M - r0;
    const int rows = static_cast<int>(left < R ? left : R);
    uint8_t* st = stage0 + static_cast<size_t>(s) * stage_bytes;
    if (lane == 0) mbar_expect_tx(&full[s], 3u * static_cast<uint32_t>(rows) * N * 2u);
    __syncwarp();
    copy_row_block(st, a.dy, a.lddy, N, r0, rows, R, (a.map_bits & 1) ? &a.map_dy : nullptr,
                   &full[s], lane);
    copy_row_block(st + tensor_bytes, a.x, a.ldx, N, r0, rows, R,
                   (a.map_bits & 2) ? &a.map_x : nullptr, &full[s], lane);
    copy_row_block(st + 2u * tensor_bytes, a.g, a.ldg, N, r0, rows, R,
                   (a.map_bits & 4) ? &a.map_g : nullptr, &full[s], lane);
  };

  // When the host knows the previous kernel on the stream writes none of dy, x, g (the
  // forward of a checkpointed step), the first stages' copies of those start before it has
  // finished.  rstd, which that forward writes, is copied only after the wait below.
  int prefetched = 0;
  long long pre_blk[kMaxStages];
  if (a.prefetch && warp == 0) {
    long long next = blockIdx.x;
    while (prefetched < S) {
      long long blk = 0;
      if (lane == 0)
        blk = a.dynamic_schedule ? static_cast<long long>(atomicAdd(a.work_counter, 1ull)) : next;
      blk = __shfl_sync(0xffffffffu, blk, 0);
      next += gridDim.x;
      pre_blk[prefetched] = blk;
      if (blk >= a.num_blocks) break;
      issue_copies(prefetched++, blk);
    }
  }
  grid_dependency_wait();
  allow_dependent_launch();

  if (warp == 0) {
    // ---------------- producer warp ----------------
    // Lane 0 takes the next row block and waits for a free stage; the lanes issue the bulk
    // copies of dy, x and g and copy the block's rstd values with 4-byte asynchronous copies
    // whose completion the stage's barrier also tracks.
    int s = 0;
    uint32_t phase = 0;
    const int pre = prefetched;  // the same in every lane of this warp
    // A prefetch that ran into the end of the rows already took its terminating block.
    const bool pre_ended = a.prefetch && prefetched < S;
    long long next = blockIdx.x + static_cast<long long>(pre) * gridDim.x;
    for (int it = 0;; ++it) {
      long long blk = 0;
      bool ok = true;
      const bool was_prefetched = it < pre;
      if (lane == 0) {
        if (was_prefetched || (it == pre && pre_ended)) {
          blk = pre_blk[it];
        } else {
          blk = a.dynamic_schedule ? static_cast<long long>(atomicAdd(a.work_counter, 1ull))
                                   : next;
          next += gridDim.x;
        }
        if (!was_prefetched) ok = mbar_wait(&empty[s], phase ^ 1u, a.err, kErrWaitEmpty);
      }
      blk = __shfl_sync(0xffffffffu, blk, 0);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      __syncwarp();
      if (!ok) break;
      if (blk >= a.num_blocks) {
        if (lane == 0) blk_id[s] = -1;
        async_copies_arrive(&full[s]);
        if (lane == 0) mbar_arrive(&full[s]);
        break;
      }
      const long long r0 = blk * R;
      const long long left = a.M - r0;
      const int rows = static_cast<int>(left < R ? left : R);
      uint8_t* st = stage0 + static_cast<size_t>(s) * stage_bytes;
      if (!was_prefetched) issue_copies(s, blk);
      if (lane == 0) {
        blk_id[s] = blk;
        if (a.l2_prefetch && !a.dynamic_schedule && a.lddy == N && a.ldx == N && a.ldg == N) {
          // the block this stage will hold next time round the ring
          const long long ahead = blk + static_cast<long long>(S) * gridDim.x;
          if (ahead < a.num_blocks) {
            const long long aleft = a.M - ahead * R;
            const uint32_t arows = static_cast<uint32_t>(aleft < R ? aleft : R);
            const uint32_t abytes = arows * static_cast<uint32_t>(N) * 2u;
            bulk_prefetch_l2(a.dy + ahead * R * N, abytes);
            bulk_prefetch_l2(a.x + ahead * R * N, abytes);
            bulk_prefetch_l2(a.g + ahead * R * N, abytes);
          }
        }
      }
      if constexpr (!kFusedFwd) {
        float* srs = reinterpret_cast<float*>(st + 3u * tensor_bytes);
        for (int i = lane; i < rows; i += 32) async_copy_4(srs + i, a.rstd + r0 + i);
      }
      async_copies_arrive(&full[s]);
      if (lane == 0) mbar_arrive(&full[s]);
      if (++s == S) {
        s = 0;
        phase ^= 1u;
      }
    }
    return;
  }

  // ---------------- consumers ----------------
  const int ctid = threadIdx.x - 32;
  const int group = ctid / TPR;
  const int lr = ctid - group * TPR;
  const int warp_group0 = (ctid & ~31) / TPR;  // first row slot of this warp
  const int n8 = N >> 3;

  float2 wp[CPT][4];     // this thread's weights, as FP32 pairs
  float2 dwacc[CPT][4];  // this thread's dw columns, accumulated over its rows
  bool cval[CPT];
#pragma unroll
  for (int k = 0; k < CPT; ++k) {
    const int c = k * TPR + lr;
    cval[k] = c < n8;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      wp[k][i] = splat2(0.f);
      dwacc[k][i] = splat2(0.f);
    }
    if constexpr (kKeepU)  // else each pass reloads its chunk's weights (L1-resident)
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
    const uint8_t* sdy = stage0 + static_cast<size_t>(s) * stage_bytes;
    const uint8_t* sx = sdy + tensor_bytes;
    const uint8_t* sg = sx + tensor_bytes;
    const float* srs = reinterpret_cast<const float*>(sg + tensor_bytes);

    for (int rb = 0; rb < rows; rb += kGroups) {
      // A warp whose rows are all past the block's end skips the pass (a warp never spans
      // two row groups' barriers, so this is uniform per warp and per row group).
      if (rb + warp_group0 >= rows) break;
      const int row = rb + group;
      const bool valid = row < rows;
      const int srow = valid ? row : 0;
      const size_t roff = static_cast<size_t>(srow) * N * 2;
      const long long grow = r0 + row;
      float r;
      float2 xs[CPT][4];  // the staged x as pairs (kKeepX)
      if constexpr (kFusedFwd) {
        // the forward's row sum: sum of squares of the staged x, one partial per chunk
        float sq[CPT];
#pragma unroll
        for (int k = 0; k < CPT; ++k) {
          sq[k] = 0.f;
          if (cval[k]) {
            bf16x8_to_pairs(
                *reinterpret_cast<const uint4*>(sx + roff + static_cast<size_t>(k * TPR + lr) * 16),
                xs[k]);
            sq[k] = chunk_dot(xs[k], xs[k]);
          }
        }
        const float ss = row_sum<TPR>(combine_chunks<CPT>(sq), red_slots, group, lr, slot);
        slot ^= 1;
        r = rsqrtf(fmaf(ss, a.inv_n, a.eps));
        if (valid && lr == 0) a.rstd_out[grow] = r;
      } else {
        r = srs[srow];
      }
      const float2 r2 = splat2(r);

      // pass 1: recompute xhat and the gate; dg; row dot product; dw accumulators
      float2 u[CPT][4];   // u, kept for pass 2 where the registers allow it (kKeepU)
      float2 xh[CPT][4];  // xhat, likewise (kKeepXhat)
      float part[CPT];
#pragma unroll
      for (int k = 0; k < CPT; ++k) {
        part[k] = 0.f;
        if (cval[k]) {
          const int c = k * TPR + lr;
          const size_t off = roff + static_cast<size_t>(c) * 16;
          float2 dyp[4], xp[4], gp[4], dgp[4], yp[4], ul[4], xl[4], wk[4];
          if constexpr (kKeepU) {
#pragma unroll
            for (int i = 0; i < 4; ++i) wk[i] = wp[k][i];
          } else {
            load_weight_pairs<kWFp32>(a.w, c, wk);
          }
          bf16x8_to_pairs(*reinterpret_cast<const uint4*>(sdy + off), dyp);
          if constexpr (kKeepX) {
#pragma unroll
            for (int i = 0; i < 4; ++i) xp[i] = xs[k][i];
          } else {
            bf16x8_to_pairs(*reinterpret_cast<const uint4*>(sx + off), xp);
          }
          bf16x8_to_pairs(*reinterpret_cast<const uint4*>(sg + off), gp);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 xhat = mul2(xp[i], r2);
            const float2 sgm = sigmoid2(gp[i]);
            const float2 silu = mul2(gp[i], sgm);
            const float2 ws = mul2(wk[i], silu);                    // w s
            if constexpr (kFusedFwd) yp[i] = mul2(xhat, ws);        // the forward's y
            const float2 t = mul2(dyp[i], xhat);                    // dy xhat
            const float2 ue = mul2(dyp[i], ws);                     // dy (w s)
            ul[i] = ue;
            xl[i] = xhat;
            if (valid) dwacc[k][i] = fma2(t, silu, dwacc[k][i]);
            // sigmoid' = sigmoid (1 + g (1 - sigmoid))
            const float2 bracket = gate_grad_bracket(gp[i], sgm);
            dgp[i] = mul2(mul2(mul2(t, wk[i]), sgm), bracket);
          }
          part[k] = chunk_dot(ul, xl);  // this chunk's share of sum(u xhat)
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            if constexpr (kKeepU) u[k][i] = ul[i];
            if constexpr (kKeepXhat) xh[k][i] = xl[i];
          }
          if (valid) {
            *reinterpret_cast<uint4*>(a.dg + grow * a.lddg + c * 8) = pairs_to_bf16x8(dgp);
            if constexpr (kFusedFwd)
              *reinterpret_cast<uint4*>(a.y + grow * a.ldy + c * 8) = pairs_to_bf16x8(yp);
          }
        }
      }
      const float dot = row_sum<TPR>(combine_chunks<CPT>(part), red_slots, group, lr, slot);
      slot ^= 1;
      const float2 nrc2 = splat2(-(r * (dot * a.inv_n)));

      // pass 2: dx = r u - (r c) xhat.  xhat comes from pass 1's registers, except for rows
      // of four chunks per thread (kKeepXhat), which recompute it from the staged x -- the
      // same product, so the same bits.
#pragma unroll
      for (int k = 0; k < CPT; ++k) {
        if (cval[k]) {
          const int c = k * TPR + lr;
          float2 dxp[4];
          if constexpr (kKeepXhat && kKeepU) {
#pragma unroll
            for (int i = 0; i < 4; ++i) dxp[i] = fma2(nrc2, xh[k][i], mul2(r2, u[k][i]));
          } else if constexpr (kKeepU) {
            float2 xp[4];
            bf16x8_to_pairs(
                *reinterpret_cast<const uint4*>(sx + roff + static_cast<size_t>(c) * 16), xp);
#pragma unroll
            for (int i = 0; i < 4; ++i) dxp[i] = fma2(nrc2, mul2(xp[i], r2), mul2(r2, u[k][i]));
          } else {
            const size_t off = roff + static_cast<size_t>(c) * 16;
            float2 dyp[4], xp[4], gp[4], wk[4];
            load_weight_pairs<kWFp32>(a.w, c, wk);
            bf16x8_to_pairs(*reinterpret_cast<const uint4*>(sdy + off), dyp);
            bf16x8_to_pairs(*reinterpret_cast<const uint4*>(sx + off), xp);
            bf16x8_to_pairs(*reinterpret_cast<const uint4*>(sg + off), gp);
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              const float2 ue = mul2(dyp[i], mul2(wk[i], mul2(gp[i], sigmoid2(gp[i]))));
              dxp[i] = fma2(nrc2, mul2(xp[i], r2), mul2(r2, ue));
            }
          }
          if (valid)
            *reinterpret_cast<uint4*>(a.dx + grow * a.lddx + c * 8) = pairs_to_bf16x8(dxp);
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

  // ---------------- this CTA's dw partial: row groups added in a fixed order ----------------
  named_barrier_sync(15, kNCT);  // every consumer is done with the stage buffers
  float* prow = a.partial + static_cast<size_t>(blockIdx.x) * N;
  if constexpr (kGroups == 1) {
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
      if (cval[k]) {
        float4* p4 = reinterpret_cast<float4*>(prow + (k * TPR + lr) * 8);
        p4[0] = make_float4(dwacc[k][0].x, dwacc[k][0].y, dwacc[k][1].x, dwacc[k][1].y);
        p4[1] = make_float4(dwacc[k][2].x, dwacc[k][2].y, dwacc[k][3].x, dwacc[k][3].y);
      }
    }
  } else {
    float* red = reinterpret_cast<float*>(stage0);  // [kGroups, N]
#pragma unroll
    for (int k = 0; k < CPT; ++k) {
      if (cval[k]) {
        float4* r4 = reinterpret_cast<float4*>(red + group * N + (k * TPR + lr) * 8);
        r4[0] = make_float4(dwacc[k][0].x, dwacc[k][0].y, dwacc[k][1].x, dwacc[k][1].y);
        r4[1] = make_float4(dwacc[k][2].x, dwacc[k][2].y, dwacc[k][3].x, dwacc[k][3].y);
      }
    }
    named_barrier_sync(15, kNCT);
    const int n4 = N >> 2;
    const float4* red4 = reinterpret_cast<const float4*>(red);
    for (int j4 = ctid; j4 < n4; j4 += kNCT) {
      float4 acc = red4[j4];
#pragma unroll
      for (int gi = 1; gi < kGroups; ++gi) {
        const float4 v = red4[gi * n4 + j4];
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      reinterpret_cast<float4*>(prow)[j4] = acc;
    }
  }

  if (!a.fused_reduce) return;

  // ---------------- fused tail: the last CTA to finish sums all partials ----------------
  __threadfence();
  named_barrier_sync(15, kNCT);
  if (ctid == 0) {
    const unsigned done = atomicAdd(a.ticket, 1u);
    *last_flag = (done == gridDim.x - 1) ? 1 : 0;
  }
  named_barrier_sync(15, kNCT);
  if (*last_flag) {
    __threadfence();
    float4* scratch = reinterpret_cast<float4*>(stage0 + static_cast<size_t>(kGroups) * N * 4);
    reduce_partials<true>(a.partial, gridDim.x, N, a.dw, a.dw_fp32, 0, 32, ctid, kNCT, scratch);
    if (ctid == 0) {
      *a.work_counter = 0ull;
      *a.ticket = 0u;
    }
  }
}

}  // namespace gnorm
