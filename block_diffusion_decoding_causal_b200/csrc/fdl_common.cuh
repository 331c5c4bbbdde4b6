// Shared device helpers and launch parameter blocks of libfdl.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "fdl.h"

namespace fdl {

constexpr int kPlanSMs = 148;          // B200: 148 SMs (2 dies x 74)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kEmptyMax = -1.0e30f;  // running max of an empty set
constexpr int kMaxRows = 256;          // LM-head rows (B * q_len) per call

typedef __nv_bfloat16 bf16;

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(bf16 x) { return __bfloat162float(x); }
template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ bf16 from_f32<bf16>(float x) {
  return __float2bfloat16_rn(x);
}

// Running (max logit, sum of exp(l - max), argmax) of a softmax reduction.
// m is kept in natural (logit) units; exponentials are taken as exp2 of a
// scaled difference.  Empty = {kEmptyMax, 0, INT_MAX}; merging with an empty
// state is exact because exp2(kEmptyMax - m) underflows to 0.
struct MSI {
  float m;
  float s;
  int i;
};

__device__ __forceinline__ MSI msi_empty() { return {kEmptyMax, 0.f, 0x7fffffff}; }

__device__ __forceinline__ MSI msi_merge(MSI a, MSI b) {
  MSI r;
  r.m = fmaxf(a.m, b.m);
  r.s = a.s * exp2f((a.m - r.m) * kLog2e) + b.s * exp2f((b.m - r.m) * kLog2e);
  r.i = (b.m > a.m || (b.m == a.m && b.i < a.i)) ? b.i : a.i;
  return r;
}

__device__ __forceinline__ MSI msi_shfl_xor(MSI a, int mask) {
  MSI r;
  r.m = __shfl_xor_sync(0xffffffffu, a.m, mask);
  r.s = __shfl_xor_sync(0xffffffffu, a.s, mask);
  r.i = __shfl_xor_sync(0xffffffffu, a.i, mask);
  return r;
}

__device__ __forceinline__ MSI msi_warp_allmerge(MSI a) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) a = msi_merge(a, msi_shfl_xor(a, o));
  return a;
}

// Per-CTA partial of the LM-head reduction for one row, 16 bytes.
struct alignas(16) Partial {
  float m;
  float s;
  int i;
  int pad;
};

// Workspace control words (first 256 bytes of the workspace).
constexpr int kLmTeam = 16;      // LM-head CTAs per first-level merge
constexpr int kLmMaxTeams = 16;  // teams the control words count for
// The LM head's tickets come in two sets (LmArgs::slot): one launch of the
// CTA-pair form can run two passes, whose merges overlap.
struct Control {
  unsigned int status;                   // FDL_DEV_* bits
  unsigned int lm_ticket[2];             // LM-head last-CTA (or last-team) tickets
  unsigned int lm_team[2][kLmMaxTeams];  // LM-head per-team tickets
};

// ----------------------------------------------------------------- attention

struct AttnArgs {
  const void* q;
  const void* k_pre;
  const void* v_pre;
  const int32_t* len_pre;
  const void* k_blk;
  const void* v_blk;
  const void* k_suf;   // NULL unless DualCache
  const void* v_suf;
  const int32_t* len_suf;
  void* out;
  Control* ctrl;
  unsigned int* tickets;  // one per (b, kvh, row tile)
  float* part_o;          // [item][row_tile_rows][d]
  float2* part_ml;        // [item][row_tile_rows]  (m, l)
  int B, Hq, Hkv, d, D, q_len, cap_p, cap_s;
  int group;       // Hq / Hkv
  int rows;        // q_len * group
  int split_keys;  // keys per split (multiple of 64)
  int n_split;
  float scale_log2;  // log2(e) / sqrt(d)
};

// ------------------------------------------------------------------ LM head

struct LmArgs {
  const void* rows;          // [R, H]
  const void* w;             // [V, H]
  const uint8_t* row_active; // [R] or NULL
  const int32_t* block_tokens_in;  // fused: activity from the block tokens
  float* conf;               // [R]
  int32_t* tok;              // [R]
  Control* ctrl;
  Partial* part;             // [n_cta][R]
  int R, H, V;
  int n_cta;
  int rows_per_cta;          // vocab rows per CTA (multiple of 16)
  int w_packed;              // w in the tiled layout of fdl_lmhead_pack_weight
  int rows_ready;            // tensor-core LM head: the rows were in place before
                             // its programmatic predecessor began, so it reads
                             // them without waiting for that grid
  int slot;                  // ticket set in Control (0, or 1 for a launch's second pass)
  // fused commit (when commit != 0)
  int commit;
  int32_t* block_tokens;
  uint8_t* committed;
  int32_t* n_committed;
  int32_t* n_masked_left;
  int B, D, q_off, q_len, mask_id;
  float tau;
};

// --------------------------------------------------------------- commit

// One warp commits sequence b (technical review, section 4, Algorithm 2).
// conf_of(i) / tok_of(i) give the unit row i's confidence and token.
template <typename ConfF, typename TokF>
__device__ __forceinline__ void commit_sequence_warp(
    int b, int lane, int D, int q_off, int q_len, int mask_id, float tau,
    ConfF conf_of, TokF tok_of, int32_t* block_tokens, uint8_t* committed,
    int32_t* n_committed, int32_t* n_masked_left) {
  int32_t* bt = block_tokens + (size_t)b * D;
  const bool in_unit = lane < q_len;
  const int p = q_off + lane;
  const int cur = in_unit ? bt[p] : 0;
  const bool cand = in_unit && cur == mask_id;
  const float c = cand ? conf_of(lane) : -__int_as_float(0x7f800000);
  const bool above = cand && c >= tau;
  const unsigned any_cand = __ballot_sync(0xffffffffu, cand);
  unsigned sel = __ballot_sync(0xffffffffu, above);
  if (sel == 0u && any_cand != 0u) {
    // fallback: the most confident candidate, lowest position on a tie
    float bc = c;
    int bl = cand ? lane : 64;
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      float oc = __shfl_xor_sync(0xffffffffu, bc, o);
      int ol = __shfl_xor_sync(0xffffffffu, bl, o);
      if (oc > bc || (oc == bc && ol < bl)) {
        bc = oc;
        bl = ol;
      }
    }
    sel = 1u << bl;
  }
  const bool mine = (sel >> lane) & 1u;
  int now = cur;
  if (mine) {
    now = tok_of(lane);
    bt[p] = now;
  }
  const unsigned left = __ballot_sync(0xffffffffu, in_unit && now == mask_id);
  for (int j = lane; j < D; j += 32) {
    const int jl = j - q_off;
    const bool s = jl >= 0 && jl < 32 && ((sel >> jl) & 1u);
    committed[(size_t)b * D + j] = s ? 1 : 0;
  }
  if (lane == 0) {
    n_committed[b] = __popc(sel);
    n_masked_left[b] = __popc(left);
  }
}

// Write the selection `sel` (bit i = unit position q_off + i) of sequence b:
// tokens, the committed bitmap over the whole block, and the two counts.
template <typename TokF>
__device__ __forceinline__ void apply_selection_warp(
    int b, int lane, int D, int q_off, int q_len, int mask_id, unsigned sel,
    TokF tok_of, int32_t* block_tokens, uint8_t* committed, int32_t* n_committed,
    int32_t* n_masked_left) {
  int32_t* bt = block_tokens + (size_t)b * D;
  const bool in_unit = lane < q_len;
  const int p = q_off + lane;
  int now = in_unit ? bt[p] : 0;
  __syncwarp();
  if (in_unit && ((sel >> lane) & 1u)) {
    now = tok_of(lane);
    bt[p] = now;
  }
  const unsigned left = __ballot_sync(0xffffffffu, in_unit && now == mask_id);
  for (int j = lane; j < D; j += 32) {
    const int jl = j - q_off;
    const bool s = jl >= 0 && jl < 32 && ((sel >> jl) & 1u);
    committed[(size_t)b * D + j] = s ? 1 : 0;
  }
  if (lane == 0) {
    n_committed[b] = __popc(sel);
    n_masked_left[b] = __popc(left);
  }
}

// Factor rule (technical review, section 6, eq. 13 and Algorithm 3) and
// heterogeneous-budget rule (section 5.1, eq. 9) for sequence b.  The unit's
// still-masked positions are sorted by decreasing confidence (lower
// position first on ties) with a 32-lane bitonic network; lane n-1 then
// holds the n-th best.  The largest admissible n is taken (the first
// position alone if none is admissible).
constexpr int kSelectFactor = 1;
constexpr int kSelectBudget = 2;

template <typename ConfF>
__device__ __forceinline__ unsigned ranked_selection_warp(int b, int lane, int D, int q_off,
                                                          int q_len, int mask_id, int policy,
                                                          float param, const int32_t* block_tokens,
                                                          ConfF conf_of) {
  const bool in_unit = lane < q_len;
  const bool cand = in_unit && block_tokens[(size_t)b * D + q_off + lane] == mask_id;
  float c = cand ? conf_of(lane) : -__int_as_float(0x7f800000);
  int idx = lane;
#pragma unroll
  for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
    for (int j = k >> 1; j > 0; j >>= 1) {
      const float c2 = __shfl_xor_sync(0xffffffffu, c, j);
      const int i2 = __shfl_xor_sync(0xffffffffu, idx, j);
      const bool self_first = c > c2 || (c == c2 && idx < i2);
      const bool up = (lane & k) == 0, lower = (lane & j) == 0;
      const bool keep = (lower == up) ? self_first : !self_first;
      if (!keep) {
        c = c2;
        idx = i2;
      }
    }
  }
  const unsigned n_cand = __popc(__ballot_sync(0xffffffffu, cand));
  const bool valid = (unsigned)lane < n_cand;
  const int n = lane + 1;
  const float eps = 1.0f - c;
  bool adm;
  if (policy == kSelectFactor) {
    adm = valid && (float)(n + 1) * eps < param;
  } else {
    float incl = valid ? eps : 0.f;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const float v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    adm = valid && incl + eps < 1.0f;
  }
  const unsigned am = __ballot_sync(0xffffffffu, adm);
  int n_sel = am ? 32 - __clz(am) : 0;
  if (n_sel == 0 && n_cand > 0) n_sel = 1;
  unsigned contrib = (lane < n_sel) ? (1u << idx) : 0u;
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) contrib |= __shfl_xor_sync(0xffffffffu, contrib, o);
  return contrib;
}

// Host-side launchers (one .cu file each).
cudaError_t launch_attn_simt(const AttnArgs& a, fdl_dtype dt, int row_tile,
                             cudaStream_t s);
// beside_prior: launched as a programmatic dependent of the kernel before it
// (the step's LM head), so its CTAs start beside that kernel's; it reads
// nothing that kernel writes and, before it completes, waits for it.
cudaError_t launch_attn_tc(const AttnArgs& a, float* part_o, float2* part_ml,
                           unsigned int* tickets, int n_cta, cudaStream_t s,
                           bool beside_prior = false);
cudaError_t launch_lmhead_simt(const LmArgs& a, fdl_dtype dt, cudaStream_t s);
// beside_smem > 0: the shared form, leaving room on every SM for one
// attention CTA of that many bytes of shared memory (see lmhead_tc.cu).
// after_producer: a programmatic dependent of the kernel before it (the
// token-shift gather that writes its rows), which it waits for only before
// its first read of the rows.
cudaError_t launch_lmhead_tc(const LmArgs& a, cudaStream_t s, size_t beside_smem = 0,
                             bool after_producer = false);
bool lmhead_tc_shared_ok(const LmArgs& a, size_t beside_smem);
// Two consecutive passes (129..256 rows each, full form) in one launch of
// the CTA-pair form: b's partials in their own region and b.slot = 1, so
// the first pass's merges run under the second pass's stream.  False: not
// applicable (the caller launches the passes one by one).
bool lmhead_tc_two_pass_ok(const LmArgs& a, const LmArgs& b);
cudaError_t launch_lmhead_tc_two_pass(const LmArgs& a, const LmArgs& b, cudaStream_t s,
                                      bool after_producer = false);
// Rewrites the bf16 weight [V, H] into the tiled layout the LM head reads
// when LmArgs::w_packed is set (see lmhead_tc.cu).
cudaError_t launch_pack_weight(const void* w, void* out, int V, int H, int rows_per_cta,
                               cudaStream_t s);
// Shared memory of one tensor-core attention CTA for these shapes.
size_t attn_tc_smem_for(int q_len, int group, int B, bool beside);
cudaError_t launch_commit(const float* conf, const int32_t* tok,
                          int32_t* block_tokens, uint8_t* committed,
                          int32_t* n_committed, int32_t* n_masked_left, int B,
                          int D, int q_off, int q_len, int mask_id, float tau,
                          cudaStream_t s);
cudaError_t launch_select_commit(int policy, float param, const float* conf,
                                 const int32_t* tok, int32_t* block_tokens,
                                 uint8_t* committed, int32_t* n_committed,
                                 int32_t* n_masked_left, int B, int D, int q_off,
                                 int q_len, int mask_id, cudaStream_t s);
cudaError_t launch_unit_status(const int32_t* n_masked_left, int B, int32_t* any_out,
                               int32_t* steps, unsigned long long handle, int limit,
                               cudaStream_t s);
cudaError_t launch_append_block(const void* k_blk, const void* v_blk, void* k_pre, void* v_pre,
                                int32_t* len_pre, unsigned int* status, int B, int Hkv, int D,
                                int cap, int row_bytes, cudaStream_t s);
cudaError_t launch_gather_rows(const void* src, const void* h_prev, void* rows,
                               int B, int q_len, int H, int shift, int elem,
                               cudaStream_t s);

}  // namespace fdl
