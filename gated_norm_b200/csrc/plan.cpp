// plan.cpp -- the rows-per-SM dispatch rule (pure host code; needs no GPU).
//
// flashinfer PR #8701 ("perf(cake_rmsnorm_silu_gate_train): L2-prefetching extra-long
// forward on SM107", PR description and commit message) routes its forward by architecture
// and by rows per SM (M / #SMs) into "long" and "extra-long" tiers with per-architecture
// thresholds.  This rule is this library's own for B200: it picks a row geometry from N
// (about two 16-byte chunks per thread), sets CTAs per SM and the stage size by a rows-per-SM
// tier, and splits the rows evenly over the persistent CTAs:
//   forward with < 512 KB of staged rows per SM : 3 CTAs per SM, ~16 KB stages (latency tier);
//   other forwards                              : 2 CTAs per SM, ~48 KB stages;
//   backward                                    : 1 CTA per SM, <= 3 stages of ~48 KB
//                                                 (at least 3 rows);
// and within a tier: if the rows per CTA fit in one stage, one block per CTA; otherwise k
// equal blocks per CTA, block size chosen so all CTAs get the same number of rows.  In the
// forward's latency tier, rows of N <= 256 skip the staging altogether: 4 CTAs of 256
// threads per SM load them straight into registers (gated_rmsnorm_fwd_direct_kernel); so
// does the backward of such rows under 256 KB of dy, x and g per SM (2 CTAs per SM).
#include <algorithm>
#include <cstdint>
#include <cstring>

#include "gnorm.h"
#include "layout.h"
#include "plan.h"

namespace gnorm {

static TuningKnobs g_knobs = {};  // all zero: built-in values

void set_tuning(const TuningKnobs& k) { g_knobs = k; }
TuningKnobs get_tuning() { return g_knobs; }

bool geometry_compiled(int kind, int tpr, int cpt) {
  static const int kBoth[][2] = {{4, 1},   {8, 1},   {16, 1},  {32, 1},  {32, 2},
                                 {32, 4},  {64, 2},  {64, 4},  {128, 2}, {128, 4},
                                 {256, 2}, {256, 4}, {512, 4}, {4, 4},   {8, 2},
                                 {8, 4},   {16, 2},  {16, 4}};
  static const int kFwdOnly[][2] = {{64, 8}};
  for (const auto& g : kBoth)
    if (g[0] == tpr && g[1] == cpt) return true;
  if (kind == 0)
    for (const auto& g : kFwdOnly)
      if (g[0] == tpr && g[1] == cpt) return true;
  return false;
}

// Staged kernels: two 16-byte chunks per thread for 128 < N <= 256, and for the forward from
// N > 64 on (measured on B200, same box, back-to-back graph replays: 262144 x 256 forward
// 69.8 -> 66.0 us and backward 116.9 -> 106.9 us with 16 x 2 instead of 32 x 1; 368640 x 128
// forward 48.7 -> 47.8 us with 8 x 2 instead of 16 x 1; the backward of rows of 128 keeps 16 x 1
// with 16 computing warps: equal at 368640 x 128, 19.8 against 20.5 us at 65536 x 128).
RowGeometry geometry_for(int kind, int64_t N) {
  const int64_t n8 = N / 8;  // 16-byte chunks per row
  if (n8 <= 4) return {4, 1};
  if (n8 <= 8) return {8, 1};
  if (n8 <= 16) return kind == 1 ? RowGeometry{16, 1} : RowGeometry{8, 2};
  if (n8 <= 32) return {16, 2};
  if (n8 <= 64) return {32, 2};
  if (n8 <= 128) return {64, 2};
  if (n8 <= 256) return {128, 2};
  if (n8 <= 512) return {256, 2};
  if (n8 <= 1024) return {256, 4};
  return {512, 4};
}

// Direct-load kernels (rows of N <= 256): one 16-byte chunk per thread, so a row is at most
// one warp; {0, 0} for wider rows.
RowGeometry direct_geometry_for(int64_t N) {
  const int64_t n8 = N / 8;
  if (n8 <= 4) return {4, 1};
  if (n8 <= 8) return {8, 1};
  if (n8 <= 16) return {16, 1};
  if (n8 <= 32) return {32, 1};
  return {0, 0};
}

static int64_t ceil_div(int64_t a, int64_t b) { return (a + b - 1) / b; }

int make_plan(int kind, int64_t M, int64_t N, int deterministic, int num_sms,
              int smem_per_block, gnorm_plan* out) {
  if (out == nullptr) return GNORM_ERR_NULL;
  std::memset(out, 0, sizeof(*out));
  if (kind != 0 && kind != 1 && kind != 2) return GNORM_ERR_ARG;
  // kind 2, the forward fused into the backward (gnorm_fwd_bwd), is the backward kernel with
  // its own row geometry for rows of N <= 128 (geometry_for); everything else as kind 1.
  const int plan_kind = kind;
  if (kind == 2) kind = 1;
  if (M < 0 || N < 8 || N > GNORM_N_MAX || (N % 8) != 0) return GNORM_ERR_SHAPE;
  if (num_sms <= 0) return GNORM_ERR_ARG;
  if (smem_per_block <= 0) smem_per_block = kB200SmemPerBlock;

  RowGeometry geo = geometry_for(plan_kind, N);
  RowGeometry dgeo = direct_geometry_for(N);
  if (g_knobs.threads_per_row > 0 && g_knobs.chunks_per_thread > 0) {
    geo = {g_knobs.threads_per_row, g_knobs.chunks_per_thread};
    if (!geometry_compiled(kind, geo.threads_per_row, geo.chunks_per_thread) ||
        static_cast<int64_t>(geo.threads_per_row) * geo.chunks_per_thread * 8 < N)
      return GNORM_ERR_UNSUPPORTED;
    // a forced geometry applies to the direct-load kernels too, where they can run it
    dgeo = (geo.chunks_per_thread == 1 && geo.threads_per_row <= 32) ? geo : RowGeometry{0, 0};
  }
  const int nct = consumer_threads_for(kind, geo.threads_per_row, geo.chunks_per_thread);
  const int groups = nct / geo.threads_per_row;
  const int tensors = kind == 0 ? 2 : 3;
  const int64_t row_bytes = static_cast<int64_t>(tensors) * N * 2;

  // Rows-per-SM tiers (bytes of staged rows per SM decide, so wide and narrow rows compare).
  const int64_t rows_per_sm = (M + num_sms - 1) / num_sms;
  const bool latency_tier = kind == 0 && rows_per_sm * row_bytes < kFwdLatencyTierBytes;
  // Forward of narrow rows in the latency tier (or always / never, by knob): rows loaded
  // straight into registers, no shared-memory stages.
  const bool direct_capable = kind == 0 && dgeo.threads_per_row > 0;
  const bool direct = direct_capable && (g_knobs.fwd_direct == 1 ||
                                         (g_knobs.fwd_direct == 0 && latency_tier));
  if (direct) {
    geo = dgeo;
    const int64_t rows_per_iter =
        static_cast<int64_t>(kDirectThreads / geo.threads_per_row) * kDirectRows;
    const int ctas = std::min(kDirectCtasPerSm,
                              g_knobs.ctas_per_sm > 0 ? g_knobs.ctas_per_sm : kDirectCtasPerSm);
    const int64_t blocks = ceil_div(M, rows_per_iter);
    out->kind = 0;
    out->threads_per_row = geo.threads_per_row;
    out->chunks_per_thread = 1;
    out->consumer_threads = kDirectThreads;
    out->rows_per_stage = static_cast<int>(rows_per_iter);
    out->stages = 0;
    out->ctas_per_sm = ctas;
    out->grid = static_cast<int>(std::min<int64_t>(blocks, static_cast<int64_t>(num_sms) * ctas));
    out->num_blocks = blocks;
    out->smem_bytes = 0;
    out->direct_loads = 1;
    return GNORM_OK;
  }

  // Backward of narrow rows with very few rows per SM: straight into registers as well.
  const bool bwd_capable = kind == 1 && dgeo.threads_per_row > 0;
  const bool bwd_tier = rows_per_sm * (3 * N * 2) < kBwdDirectTierBytes;
  if (bwd_capable && (g_knobs.bwd_direct == 1 || (g_knobs.bwd_direct == 0 && bwd_tier))) {
    geo = dgeo;
    const int64_t rows_per_iter =
        static_cast<int64_t>(kDirectThreads / geo.threads_per_row) * kDirectBwdRows;
    const int ctas = std::min(kDirectBwdCtasPerSm, g_knobs.ctas_per_sm > 0
                                                       ? g_knobs.ctas_per_sm
                                                       : kDirectBwdCtasPerSm);
    const int64_t blocks = ceil_div(M, rows_per_iter);
    out->kind = plan_kind;
    out->threads_per_row = geo.threads_per_row;
    out->chunks_per_thread = 1;
    out->consumer_threads = kDirectThreads;
    out->rows_per_stage = static_cast<int>(rows_per_iter);
    out->stages = 0;
    out->ctas_per_sm = ctas;
    out->grid = static_cast<int>(std::min<int64_t>(blocks, static_cast<int64_t>(num_sms) * ctas));
    out->num_blocks = blocks;
    out->smem_bytes = 0;
    out->dynamic_schedule = 0;  // rows are assigned statically in both modes
    out->fused_reduce = 0;
    out->partials = out->grid;
    out->direct_loads = 1;
    return GNORM_OK;
  }

  const int fit = max_ctas_per_sm(kind, geo.threads_per_row, geo.chunks_per_thread);
  const int default_ctas = kind == 1 ? 1 : (latency_tier ? 3 : 2);
  int64_t default_stage = kind == 1 ? std::max<int64_t>(kBwdStageBytes, kBwdMinStageRows * (row_bytes + 4))
                                    : (latency_tier ? kFwdLatencyStageBytes : kFwdStageBytes);
  const int ctas_per_sm =
      std::min(fit, g_knobs.ctas_per_sm > 0 ? g_knobs.ctas_per_sm : default_ctas);
  const int64_t stage_target = g_knobs.stage_bytes > 0 ? g_knobs.stage_bytes : default_stage;
  const int max_stages = std::min(
      kMaxStages, g_knobs.max_stages > 0 ? g_knobs.max_stages
                                         : (kind == 1 ? kBwdMaxStages : kMaxStages));

  // Shared memory available to one CTA when `ctas_per_sm` share an SM.
  int64_t smem_cta = smem_per_block;
  if (ctas_per_sm > 1)
    smem_cta = std::min<int64_t>(smem_cta, kB200SmemPerSm / ctas_per_sm - kSmemPerCtaReserve);
  const int64_t budget = smem_cta - kHeaderBytes;

  // Rows per stage: about `stage_target` bytes, at least one row per row group.
  const int64_t row_stage_bytes = row_bytes + (kind == 1 ? 4 : 0);
  int64_t target_rows = std::max<int64_t>(groups, stage_target / row_stage_bytes);
  while (target_rows > 1 && 2 * (target_rows * row_stage_bytes + 127) > budget) --target_rows;
  if (2 * (row_stage_bytes + 127) > budget) return GNORM_ERR_UNSUPPORTED;  // two stages of one row

  const int64_t grid_max = static_cast<int64_t>(num_sms) * ctas_per_sm;
  int64_t R, blocks, grid;
  if (M == 0) {
    R = target_rows;
    blocks = 0;
    grid = 0;
  } else {
    const int64_t rows_per_cta = ceil_div(M, grid_max);
    if (rows_per_cta <= target_rows) {
      R = rows_per_cta;  // latency tier: one block per CTA
    } else {
      const int64_t k = ceil_div(rows_per_cta, target_rows);
      R = ceil_div(rows_per_cta, k);  // streaming tier: k equal blocks per CTA
    }
    blocks = ceil_div(M, R);
    grid = std::min(blocks, grid_max);
  }

  // A stage holds R rows of each tensor; the backward's also holds their R FP32 rstd values.
  const int64_t stage_raw = static_cast<int64_t>(tensors) * stage_tensor_bytes(R, N) +
                            (kind == 1 ? R * 4 : 0);
  const int64_t stage_bytes = (stage_raw + 127) / 128 * 128;
  int64_t stages = std::min<int64_t>(max_stages, budget / stage_bytes);
  if (stages < 2) return GNORM_ERR_UNSUPPORTED;

  // The backward reuses the stage buffers at the end for the per-group dw rows and, in the
  // fused tail, for the reduction scratch.
  int64_t body = stages * stage_bytes;
  if (kind == 1) body = std::max<int64_t>(body, static_cast<int64_t>(groups) * N * 4 + nct * 16);
  const int64_t smem = kHeaderBytes + body;
  if (smem > smem_cta) return GNORM_ERR_UNSUPPORTED;

  out->kind = plan_kind;
  out->threads_per_row = geo.threads_per_row;
  out->chunks_per_thread = geo.chunks_per_thread;
  out->consumer_threads = nct;
  out->rows_per_stage = static_cast<int>(R);
  out->stages = static_cast<int>(stages);
  out->ctas_per_sm = ctas_per_sm;
  out->grid = static_cast<int>(grid);
  out->num_blocks = blocks;
  out->smem_bytes = static_cast<int>(smem);
  out->l2_prefetch = g_knobs.l2_prefetch == 1 ? 1 : (g_knobs.l2_prefetch == 2 ? 0 : kDefaultL2Prefetch);
  if (kind == 1) {
    out->dynamic_schedule = deterministic ? 0 : 1;
    out->partials = static_cast<int>(grid);
    // The fixed-order second pass over the partials runs in the last CTA to finish when the
    // partials are small (one launch; the result does not depend on which CTA is last),
    // and as a second launch whose CTAs read them in parallel for wide rows.
    const int tail = g_knobs.tail_reduce == 1 ? 1 : (g_knobs.tail_reduce == 2 ? 0 : kDefaultTailReduce);
    out->fused_reduce =
        (tail && grid > 0 && static_cast<int64_t>(grid) * N <= kFusedReduceMaxFloats) ? 1 : 0;
  }
  return GNORM_OK;
}

size_t workspace_bytes_for(const gnorm_plan& p, int64_t N) {
  const size_t raw = kWorkspaceHeader + static_cast<size_t>(p.partials) * N * 4;
  return (raw + GNORM_WORKSPACE_ALIGN - 1) / GNORM_WORKSPACE_ALIGN * GNORM_WORKSPACE_ALIGN;
}

}  // namespace gnorm
