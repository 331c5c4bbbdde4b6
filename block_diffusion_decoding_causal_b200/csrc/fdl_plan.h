// Host-side launch plan and workspace layout of one step configuration.
#pragma once

#include <cmath>
#include <cstddef>
#include <string>

#include "fdl.h"

namespace fdl {

constexpr int kAttnRowTile = 16;   // query rows per attention CTA
constexpr int kPlanCTAs = 148;     // grid sizing unit: one B200's SM count
constexpr int kLmMaxCTAs = 4 * kPlanCTAs;
#ifndef FDL_ATTN_ALONE_CTAS_PER_SM
#define FDL_ATTN_ALONE_CTAS_PER_SM 2
#endif
// tensor-core attention alone on the GPU: two CTAs per SM
constexpr int kAttnTcCTAs = FDL_ATTN_ALONE_CTAS_PER_SM * kPlanCTAs;
constexpr int kLmPassRows = 256;   // LM-head rows per pass over the weight
constexpr long kMaxStepRows = 4096;  // batch * q_len of one step
constexpr int kMaxAttnRows = 4096;   // block_size / q_len of the attention entry points

struct AttnSplit {
  int split_keys;  // keys per split, multiple of 64
  int n_split;
};

struct Plan {
  bool step_ok;    // within the fused step's limits (LM head, commit sized)
  int R;           // LM-head rows = batch * q_len
  int lm_pass_rows;  // rows per LM-head pass: whole sequences, at most 256
  int lm_part_regions;  // LM-head partial regions of kLmMaxCTAs x lm_pass_rows
  int elem;        // bytes per floating element
  int n_row_tiles;
  AttnSplit attn_plain, attn_dual;
  int lm_cta, lm_rows_per_cta;        // CUDA-core LM head (fp32)
  int lm_tc_cta, lm_tc_rows_per_cta;  // tensor-core LM head (bf16): one CTA per SM
  bool attn_tc;     // tensor-core attention (bf16, d 128)
  size_t off_tc_tickets;  // tensor-core attention: one ticket per (item, tile row)
  size_t off_ctrl, off_tickets, off_part_o, off_part_ml, off_rows, off_lm_part,
      off_attn, off_tc_part_o, off_tc_part_ml, total;
};

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Vocabulary rows per CTA of the tensor-core LM head: V over one CTA per SM,
// rounded up to 16 rows.  Depends on V alone, so it also fixes the tiled
// weight layout (FDL_W_PACKED) whatever the number of rows of a call.
inline long lm_tc_rows_per_cta(long vocab) {
  long per = (vocab + kPlanCTAs - 1) / kPlanCTAs;
  return (per + 15) / 16 * 16;
}

// Split the (b, kv head, row tile) key sequences so that about two CTAs per
// SM are in flight.
inline AttnSplit plan_split(long keys_cap, long items) {
  AttnSplit s;
  long want = (2L * kPlanCTAs + items - 1) / items;
  long max_split = (keys_cap + 63) / 64;
  if (want < 1) want = 1;
  if (want > max_split) want = max_split;
  long per = (keys_cap + want - 1) / want;
  per = (per + 63) / 64 * 64;
  s.split_keys = (int)per;
  s.n_split = (int)((keys_cap + per - 1) / per);
  return s;
}

// step: the limits of the fused step, LM head and commit entry points
// (block <= 64, unit <= 32 positions, batch * q_len <= 4096); otherwise the
// wider limits of the attention entry points (block and query rows up to
// 4096, beyond 64 / 32 on the tensor-core kernel only).
inline bool make_plan(const fdl_step_cfg* c, Plan* p, std::string* why, bool step = true) {
  if (c == nullptr) { *why = "cfg is NULL"; return false; }
  if (c->dtype != FDL_F32 && c->dtype != FDL_BF16) { *why = "dtype must be FDL_F32 or FDL_BF16"; return false; }
  if (c->w_layout != FDL_W_ROW_MAJOR && c->w_layout != FDL_W_PACKED) {
    *why = "w_layout must be FDL_W_ROW_MAJOR or FDL_W_PACKED"; return false;
  }
  if (c->batch < 1) { *why = "batch must be >= 1"; return false; }
  if (c->n_q_heads < 1 || c->n_kv_heads < 1 || c->n_q_heads % c->n_kv_heads != 0) {
    *why = "n_q_heads must be a positive multiple of n_kv_heads"; return false;
  }
  if (c->head_dim != 32 && c->head_dim != 64 && c->head_dim != 128) {
    *why = "head_dim must be 32, 64 or 128"; return false;
  }
  const bool step_shape = c->block_size >= 1 && c->block_size <= 64 && c->q_len >= 1 &&
                          c->q_len <= 32;
  if (step) {
    if (c->block_size < 1 || c->block_size > 64) { *why = "block_size must be in [1, 64]"; return false; }
    if (c->q_len < 1 || c->q_len > 32) { *why = "q_len must be in [1, 32]"; return false; }
  } else {
    if (c->block_size < 1 || c->block_size > kMaxAttnRows) {
      *why = "block_size must be in [1, 4096]"; return false;
    }
    if (c->q_len < 1 || c->q_len > kMaxAttnRows) { *why = "q_len must be in [1, 4096]"; return false; }
    if (!step_shape && !(c->dtype == FDL_BF16 && c->head_dim == 128 && c->batch <= 256 &&
                         c->n_q_heads / c->n_kv_heads <= 128)) {
      *why = "block_size > 64 or q_len > 32 needs bf16, head_dim 128, batch <= 256";
      return false;
    }
  }
  if (c->q_off < 0 || c->q_off + c->q_len > c->block_size) {
    *why = "the unit [q_off, q_off+q_len) must lie inside the block"; return false;
  }
  if (c->cap_prefix < 0 || c->cap_suffix < 0) { *why = "cache capacities must be >= 0"; return false; }
  if (c->hidden < 8 || c->hidden % 8 != 0) { *why = "hidden must be a positive multiple of 8"; return false; }
  if (c->vocab < 2) { *why = "vocab must be >= 2"; return false; }
  if (c->mask_id < 0 || c->mask_id >= c->vocab) { *why = "mask_id must be in [0, vocab)"; return false; }
  if (c->shift != 0 && c->shift != 1) { *why = "shift must be 0 or 1"; return false; }
  if (!std::isfinite(c->tau)) { *why = "tau must be finite"; return false; }
  const long R = (long)c->batch * c->q_len;
  p->step_ok = step_shape && R <= kMaxStepRows;
  if (step && !p->step_ok) { *why = "batch * q_len must be <= 4096"; return false; }

  p->R = p->step_ok ? (int)R : 0;
  p->lm_pass_rows = p->step_ok ? (R <= kLmPassRows ? (int)R : kLmPassRows / c->q_len * c->q_len)
                               : 0;
  p->elem = c->dtype == FDL_BF16 ? 2 : 4;
  const int group = c->n_q_heads / c->n_kv_heads;
  const int rows = c->q_len * group;
  p->n_row_tiles = (rows + kAttnRowTile - 1) / kAttnRowTile;
  const long items = (long)c->batch * c->n_kv_heads * p->n_row_tiles;
  const long keys_plain = (long)c->cap_prefix + c->block_size;
  const long keys_dual = keys_plain + c->cap_suffix;
  p->attn_plain = plan_split(keys_plain, items);
  p->attn_dual = plan_split(keys_dual, items);
  const long max_split = p->attn_plain.n_split > p->attn_dual.n_split
                             ? p->attn_plain.n_split : p->attn_dual.n_split;

  // LM head: contiguous vocabulary ranges (multiples of 16 rows) over about
  // two CTAs per SM.
  long per = ((long)c->vocab + 2 * kPlanCTAs - 1) / (2 * kPlanCTAs);
  per = (per + 15) / 16 * 16;
  p->lm_rows_per_cta = (int)per;
  p->lm_cta = (int)(((long)c->vocab + per - 1) / per);
  const long per_tc = lm_tc_rows_per_cta(c->vocab);
  p->lm_tc_rows_per_cta = (int)per_tc;
  p->lm_tc_cta = (int)(((long)c->vocab + per_tc - 1) / per_tc);

  size_t off = 0;
  p->off_ctrl = off;
  off = align256(off + 256);
  // CUDA-core attention (fp32, head_dim 32 / 64): step shapes only.
  const size_t simt_items = step_shape ? (size_t)items : 0;
  p->off_tickets = off;
  off = align256(off + sizeof(unsigned int) * simt_items);
  p->off_part_o = off;
  off = align256(off + sizeof(float) * simt_items * max_split * kAttnRowTile * c->head_dim);
  p->off_part_ml = off;
  off = align256(off + 8 * simt_items * max_split * kAttnRowTile);
  // LM-head rows, per-CTA partials (one pass) and the attention output of
  // the fused step: sized only for configurations the step accepts.
  p->off_rows = off;
  off = align256(off + (size_t)p->elem * p->R * c->hidden);
  // LM-head partials: one region per pass of a launch (two when the rows
  // take more than one pass: the CTA-pair form runs two passes a launch).
  p->off_lm_part = off;
  p->lm_part_regions = p->R > p->lm_pass_rows ? 2 : 1;
  off = align256(off + 16 * (size_t)kLmMaxCTAs * p->lm_pass_rows * p->lm_part_regions);
  p->off_attn = off;
  off = align256(off + (size_t)p->elem * p->R * c->n_q_heads * c->head_dim);
  // Tensor-core attention: at most two partials (first and last item) per CTA.
  p->attn_tc = c->dtype == FDL_BF16 && c->head_dim == 128 && group <= 128 && c->batch <= 256;
  p->off_tc_part_o = off;
  p->off_tc_part_ml = off;
  p->off_tc_tickets = off;
  if (p->attn_tc) {
    off = align256(off + sizeof(float) * 2 * (size_t)kAttnTcCTAs * 128 * 128);
    p->off_tc_part_ml = off;
    off = align256(off + 8 * 2 * (size_t)kAttnTcCTAs * 128);
    // 128-row tiles: the GQA group x as many positions as fit.
    const int qpt = 128 / group < c->q_len ? 128 / group : c->q_len;
    const long tc_items = (long)c->batch * c->n_kv_heads * ((c->q_len + qpt - 1) / qpt);
    p->off_tc_tickets = off;
    off = align256(off + sizeof(unsigned int) * 128 * (size_t)tc_items);
  }
  p->total = off;
  return true;
}

}  // namespace fdl
