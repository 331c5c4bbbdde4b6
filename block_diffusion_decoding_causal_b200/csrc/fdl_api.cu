// C ABI of libfdl: argument checks, workspace layout, launches.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "fdl_common.cuh"
#include "fdl_plan.h"

namespace fdl {
namespace {

thread_local std::string g_err;

int fail(int code, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_err = buf;
  return code;
}

int ok() {
  g_err.clear();
  return FDL_OK;
}

int cuda_fail(cudaError_t e, const char* what) {
  return fail(FDL_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define FDL_CHECK_PTR(p)                                                    \
  do {                                                                      \
    if ((p) == nullptr) return fail(FDL_ERR_INVALID_ARG, #p " is NULL");     \
    if (!aligned16(p))                                                      \
      return fail(FDL_ERR_INVALID_ARG, #p " is not 16-byte aligned");       \
  } while (0)

int check_ws(const Plan& p, const void* ws, size_t ws_bytes) {
  if (ws == nullptr) return fail(FDL_ERR_WORKSPACE, "workspace is NULL");
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(FDL_ERR_WORKSPACE, "workspace is not 256-byte aligned");
  if (ws_bytes < p.total)
    return fail(FDL_ERR_WORKSPACE, "workspace has %zu bytes, needs %zu", ws_bytes,
                p.total);
  return FDL_OK;
}

template <typename T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(static_cast<char*>(ws) + off);
}

AttnArgs attn_args(const fdl_step_cfg& c, const Plan& p, bool dual, const void* q,
                   const void* k_pre, const void* v_pre, const int32_t* len_pre,
                   const void* k_blk, const void* v_blk, const void* k_suf,
                   const void* v_suf, const int32_t* len_suf, void* out, void* ws) {
  AttnArgs a;
  a.q = q;
  a.k_pre = k_pre;
  a.v_pre = v_pre;
  a.len_pre = len_pre;
  a.k_blk = k_blk;
  a.v_blk = v_blk;
  a.k_suf = dual ? k_suf : nullptr;
  a.v_suf = dual ? v_suf : nullptr;
  a.len_suf = dual ? len_suf : nullptr;
  a.out = out;
  a.ctrl = at<Control>(ws, p.off_ctrl);
  a.tickets = at<unsigned int>(ws, p.off_tickets);
  a.part_o = at<float>(ws, p.off_part_o);
  a.part_ml = at<float2>(ws, p.off_part_ml);
  a.B = c.batch;
  a.Hq = c.n_q_heads;
  a.Hkv = c.n_kv_heads;
  a.d = c.head_dim;
  a.D = c.block_size;
  a.q_len = c.q_len;
  a.cap_p = c.cap_prefix;
  a.cap_s = c.cap_suffix;
  a.group = c.n_q_heads / c.n_kv_heads;
  a.rows = c.q_len * a.group;
  const AttnSplit& s = dual ? p.attn_dual : p.attn_plain;
  a.split_keys = s.split_keys;
  a.n_split = s.n_split;
  a.scale_log2 = kLog2e / std::sqrt((float)c.head_dim);
  return a;
}

LmArgs lm_args(const fdl_step_cfg& c, const Plan& p, const void* rows,
               const void* w, const uint8_t* row_active, float* conf,
               int32_t* tok, void* ws) {
  LmArgs a;
  memset(&a, 0, sizeof(a));
  a.rows = rows;
  a.w = w;
  a.row_active = row_active;
  a.block_tokens_in = nullptr;
  a.conf = conf;
  a.tok = tok;
  a.ctrl = at<Control>(ws, p.off_ctrl);
  a.part = at<Partial>(ws, p.off_lm_part);
  a.R = p.R;
  a.H = c.hidden;
  a.V = c.vocab;
  const bool tc = c.dtype == FDL_BF16;
  a.n_cta = tc ? p.lm_tc_cta : p.lm_cta;
  a.rows_per_cta = tc ? p.lm_tc_rows_per_cta : p.lm_rows_per_cta;
  a.w_packed = c.w_layout == FDL_W_PACKED;
  a.commit = 0;
  a.B = c.batch;
  a.D = c.block_size;
  a.q_off = c.q_off;
  a.q_len = c.q_len;
  a.mask_id = c.mask_id;
  a.tau = c.tau;
  return a;
}

// CTAs for the attention beside the LM head: the largest possible chunk
// count (lengths at capacity) over about 32 chunks per CTA, between 1 and one
// per SM.
int attn_ctas_beside(const fdl_step_cfg& c, bool dual) {
  const long group = c.n_q_heads / c.n_kv_heads;
  const long qpt = 128 / group < c.q_len ? 128 / group : c.q_len;
  const long items = (long)c.batch * c.n_kv_heads * ((c.q_len + qpt - 1) / qpt);
  const long per_item = (c.cap_prefix + 63) / 64 + 1 + (dual ? (c.cap_suffix + 63) / 64 : 0);
  const long want = (items * per_item + 31) / 32;
  return (int)(want < 1 ? 1 : (want > kPlanCTAs ? kPlanCTAs : want));
}

int run_attention(const fdl_step_cfg& c, const Plan& p, bool dual, const void* q,
                  const void* k_pre, const void* v_pre, const int32_t* len_pre,
                  const void* k_blk, const void* v_blk, const void* k_suf,
                  const void* v_suf, const int32_t* len_suf, void* out, void* ws,
                  cudaStream_t s, bool beside_lmhead = false) {
  AttnArgs a = attn_args(c, p, dual, q, k_pre, v_pre, len_pre, k_blk, v_blk,
                         k_suf, v_suf, len_suf, out, ws);
  // bf16 with d = 128: tensor-core kernel (two CTAs per SM; beside the LM
  // head, at most one per SM and only as many as keep about 32 chunks each,
  // so that few partials need merging); otherwise the CUDA-core kernel.
  cudaError_t e = p.attn_tc
                      ? launch_attn_tc(a, at<float>(ws, p.off_tc_part_o),
                                       at<float2>(ws, p.off_tc_part_ml),
                                       at<unsigned int>(ws, p.off_tc_tickets),
                                       beside_lmhead ? attn_ctas_beside(c, dual) : kAttnTcCTAs,
                                       s, beside_lmhead)
                      : launch_attn_simt(a, (fdl_dtype)c.dtype, kAttnRowTile, s);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return FDL_OK;
}

// bf16: tensor-core kernel (TMA + tcgen05, K in chunks of 64); fp32: the
// CUDA-core kernel.
int check_lmhead_supported(const fdl_step_cfg& c) {
  if (c.dtype == FDL_BF16 && c.hidden % 64 != 0)
    return fail(FDL_ERR_UNSUPPORTED, "bf16 LM head needs hidden %% 64 == 0 (got %d)", c.hidden);
  if (c.w_layout == FDL_W_PACKED && c.dtype != FDL_BF16)
    return fail(FDL_ERR_UNSUPPORTED, "the tiled weight layout is bf16 only");
  return FDL_OK;
}

int run_lmhead(const LmArgs& a, const fdl_step_cfg& c, cudaStream_t s, size_t beside_smem = 0,
               bool after_gather = false) {
  cudaError_t e = c.dtype == FDL_BF16 ? launch_lmhead_tc(a, s, beside_smem, after_gather)
                                      : launch_lmhead_simt(a, (fdl_dtype)c.dtype, s);
  if (e != cudaSuccess) return cuda_fail(e, "lm-head launch");
  return FDL_OK;
}

// More rows than one pass holds (batch * q_len > 256): one pass per group of
// whole sequences, each a full read of the weight.  At 256 rows a pass sits
// at the ridge (as many FLOPs per weight byte as the tensor cores have per
// HBM byte), so beyond it the passes cost what the arithmetic does.
int run_lmhead_passes(const LmArgs& a, const fdl_step_cfg& c, const Plan& p, cudaStream_t s,
                      bool after_gather = false) {
  if (a.R <= p.lm_pass_rows) return run_lmhead(a, c, s, 0, after_gather);
  const size_t row_bytes = (size_t)c.hidden * p.elem;
  auto pass_args = [&](int r0) {
    LmArgs pa = a;
    const int b0 = r0 / c.q_len;
    pa.R = a.R - r0 < p.lm_pass_rows ? a.R - r0 : p.lm_pass_rows;
    pa.B = pa.R / c.q_len;
    pa.rows = static_cast<const uint8_t*>(a.rows) + (size_t)r0 * row_bytes;
    if (a.row_active != nullptr) pa.row_active = a.row_active + r0;
    pa.conf = a.conf + r0;
    pa.tok = a.tok + r0;
    if (a.block_tokens_in != nullptr) pa.block_tokens_in = a.block_tokens_in + (size_t)b0 * c.block_size;
    if (a.commit) {
      pa.block_tokens = a.block_tokens + (size_t)b0 * c.block_size;
      pa.committed = a.committed + (size_t)b0 * c.block_size;
      pa.n_committed = a.n_committed + b0;
      pa.n_masked_left = a.n_masked_left + b0;
    }
    return pa;
  };
  bool first = true;
  for (int r0 = 0; r0 < a.R;) {
    const LmArgs pa = pass_args(r0);
    const int r1 = r0 + pa.R;
    if (c.dtype == FDL_BF16 && r1 < a.R && p.lm_part_regions >= 2) {
      // Two passes of the CTA-pair form in one launch, the second with its
      // own partial region and ticket set.
      LmArgs pb = pass_args(r1);
      pb.part = a.part + (size_t)kLmMaxCTAs * p.lm_pass_rows;
      pb.slot = 1;
      if (lmhead_tc_two_pass_ok(pa, pb)) {
        const cudaError_t e = launch_lmhead_tc_two_pass(pa, pb, s, after_gather && first);
        if (e != cudaSuccess) return cuda_fail(e, "lm-head launch");
        first = false;
        r0 = r1 + pb.R;
        continue;
      }
    }
    const int rc = run_lmhead(pa, c, s, 0, after_gather && first);
    if (rc != FDL_OK) return rc;
    first = false;
    r0 = r1;
  }
  return FDL_OK;
}

// An NVTX range around an entry point (visible to profilers; no cost when
// none is attached).
struct NvtxRange {
  explicit NvtxRange(const char* name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

}  // namespace

// Error reporting for entry points defined in other files.
int record_error(int code, const std::string& msg) { return fail(code, "%s", msg.c_str()); }
int record_ok() { return ok(); }

}  // namespace fdl

using namespace fdl;

extern "C" {

int fdl_version(void) { return FDL_VERSION; }

const char* fdl_last_error(void) { return g_err.c_str(); }

size_t fdl_workspace_size(const fdl_step_cfg* cfg) {
  Plan p;
  std::string why;
  if (!make_plan(cfg, &p, &why, false)) {
    fail(FDL_ERR_INVALID_ARG, "%s", why.c_str());
    return 0;
  }
  ok();
  return p.total;
}

int fdl_reset_workspace(void* ws, size_t ws_bytes, void* stream) {
  if (ws == nullptr) return fail(FDL_ERR_WORKSPACE, "workspace is NULL");
  cudaError_t e = cudaMemsetAsync(ws, 0, ws_bytes, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync");
  return ok();
}

static int attn_common(const fdl_step_cfg* cfg, bool dual, const void* q,
                       const void* k_pre, const void* v_pre, const int32_t* len_pre,
                       const void* k_blk, const void* v_blk, const void* k_suf,
                       const void* v_suf, const int32_t* len_suf, void* out,
                       void* ws, size_t ws_bytes, void* stream) {
  Plan p;
  std::string why;
  if (!make_plan(cfg, &p, &why, false)) return fail(FDL_ERR_INVALID_ARG, "%s", why.c_str());
  FDL_CHECK_PTR(q);
  FDL_CHECK_PTR(k_blk);
  FDL_CHECK_PTR(v_blk);
  FDL_CHECK_PTR(len_pre);
  FDL_CHECK_PTR(out);
  if (cfg->cap_prefix > 0) {
    FDL_CHECK_PTR(k_pre);
    FDL_CHECK_PTR(v_pre);
  }
  if (dual) {
    if (cfg->cap_suffix <= 0)
      return fail(FDL_ERR_INVALID_ARG, "DualCache needs cap_suffix > 0");
    FDL_CHECK_PTR(k_suf);
    FDL_CHECK_PTR(v_suf);
    FDL_CHECK_PTR(len_suf);
  }
  int rc = check_ws(p, ws, ws_bytes);
  if (rc != FDL_OK) return rc;
  rc = run_attention(*cfg, p, dual, q, k_pre, v_pre, len_pre, k_blk, v_blk, k_suf,
                     v_suf, len_suf, out, ws, (cudaStream_t)stream);
  return rc != FDL_OK ? rc : ok();
}

int fdl_block_attn(const fdl_step_cfg* cfg, const void* q, const void* k_pre,
                   const void* v_pre, const int32_t* len_pre, const void* k_blk,
                   const void* v_blk, void* out, void* ws, size_t ws_bytes,
                   void* stream) {
  NvtxRange nvtx_range("fdl_block_attn");
  return attn_common(cfg, false, q, k_pre, v_pre, len_pre, k_blk, v_blk, nullptr,
                     nullptr, nullptr, out, ws, ws_bytes, stream);
}

int fdl_dualcache_attn(const fdl_step_cfg* cfg, const void* q, const void* k_pre,
                       const void* v_pre, const int32_t* len_pre,
                       const void* k_blk, const void* v_blk, const void* k_suf,
                       const void* v_suf, const int32_t* len_suf, void* out,
                       void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("fdl_dualcache_attn");
  return attn_common(cfg, true, q, k_pre, v_pre, len_pre, k_blk, v_blk, k_suf,
                     v_suf, len_suf, out, ws, ws_bytes, stream);
}

int fdl_prefixcache_attn(const fdl_step_cfg* cfg, const void* q, const void* k_pre,
                         const void* v_pre, const int32_t* len_pre, const void* k_fresh,
                         const void* v_fresh, void* out, void* ws, size_t ws_bytes,
                         void* stream) {
  NvtxRange nvtx_range("fdl_prefixcache_attn");
  if (cfg != nullptr && (cfg->q_off != 0 || cfg->q_len != cfg->block_size))
    return fail(FDL_ERR_INVALID_ARG,
                "PrefixCache queries are all recomputed rows: need q_off = 0 and "
                "q_len = block_size (got %d, %d, %d)", cfg->q_off, cfg->q_len, cfg->block_size);
  // The recomputed rows take the block's place: every key of
  // [prefix | recomputed rows] is visible to every query.
  return attn_common(cfg, false, q, k_pre, v_pre, len_pre, k_fresh, v_fresh, nullptr, nullptr,
                     nullptr, out, ws, ws_bytes, stream);
}

int fdl_lmhead_confidence(const fdl_step_cfg* cfg, const void* rows,
                          const void* w_lm, const uint8_t* row_active,
                          float* conf, int32_t* tok, void* ws, size_t ws_bytes,
                          void* stream) {
  NvtxRange nvtx_range("fdl_lmhead_confidence");
  Plan p;
  std::string why;
  if (!make_plan(cfg, &p, &why)) return fail(FDL_ERR_INVALID_ARG, "%s", why.c_str());
  FDL_CHECK_PTR(rows);
  FDL_CHECK_PTR(w_lm);
  FDL_CHECK_PTR(conf);
  FDL_CHECK_PTR(tok);
  int rc = check_lmhead_supported(*cfg);
  if (rc != FDL_OK) return rc;
  rc = check_ws(p, ws, ws_bytes);
  if (rc != FDL_OK) return rc;
  LmArgs a = lm_args(*cfg, p, rows, w_lm, row_active, conf, tok, ws);
  rc = run_lmhead_passes(a, *cfg, p, (cudaStream_t)stream);
  return rc != FDL_OK ? rc : ok();
}

int fdl_lmhead_pack_weight(const fdl_step_cfg* cfg, const void* w_lm, void* w_packed,
                           void* stream) {
  NvtxRange nvtx_range("fdl_lmhead_pack_weight");
  if (cfg == nullptr) return fail(FDL_ERR_INVALID_ARG, "cfg is NULL");
  if (cfg->dtype != FDL_BF16)
    return fail(FDL_ERR_UNSUPPORTED, "the tiled weight layout is bf16 only");
  if (cfg->vocab < 1 || cfg->hidden < 64)
    return fail(FDL_ERR_INVALID_ARG, "need vocab >= 1 and hidden >= 64 (got %d, %d)", cfg->vocab,
                cfg->hidden);
  if (cfg->hidden % 64 != 0)
    return fail(FDL_ERR_UNSUPPORTED, "the tiled weight layout needs hidden %% 64 == 0 (got %d)",
                cfg->hidden);
  if ((long)cfg->vocab * (cfg->hidden / 64) > 0x7fffffffL)
    return fail(FDL_ERR_INVALID_ARG, "vocab * hidden / 64 exceeds 2^31 - 1");
  FDL_CHECK_PTR(w_lm);
  FDL_CHECK_PTR(w_packed);
  const uintptr_t src = reinterpret_cast<uintptr_t>(w_lm);
  const uintptr_t dst = reinterpret_cast<uintptr_t>(w_packed);
  const uintptr_t bytes = (uintptr_t)cfg->vocab * (uintptr_t)cfg->hidden * 2u;
  if (src < dst + bytes && dst < src + bytes)
    return fail(FDL_ERR_INVALID_ARG, "w_lm and w_packed overlap");
  const cudaError_t e =
      launch_pack_weight(w_lm, w_packed, cfg->vocab, cfg->hidden,
                         (int)lm_tc_rows_per_cta(cfg->vocab), (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "weight pack launch");
  return ok();
}

int fdl_threshold_commit(const fdl_step_cfg* cfg, const float* conf,
                         const int32_t* tok, int32_t* block_tokens,
                         uint8_t* committed, int32_t* n_committed,
                         int32_t* n_masked_left, void* stream) {
  NvtxRange nvtx_range("fdl_threshold_commit");
  Plan p;
  std::string why;
  if (!make_plan(cfg, &p, &why)) return fail(FDL_ERR_INVALID_ARG, "%s", why.c_str());
  FDL_CHECK_PTR(conf);
  FDL_CHECK_PTR(tok);
  FDL_CHECK_PTR(block_tokens);
  FDL_CHECK_PTR(committed);
  FDL_CHECK_PTR(n_committed);
  FDL_CHECK_PTR(n_masked_left);
  cudaError_t e = launch_commit(conf, tok, block_tokens, committed, n_committed,
                                n_masked_left, cfg->batch, cfg->block_size,
                                cfg->q_off, cfg->q_len, cfg->mask_id, cfg->tau,
                                (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "commit launch");
  return ok();
}

int fdl_select_commit(const fdl_step_cfg* cfg, int policy, float param, const float* conf,
                      const int32_t* tok, int32_t* block_tokens, uint8_t* committed,
                      int32_t* n_committed, int32_t* n_masked_left, void* stream) {
  NvtxRange nvtx_range("fdl_select_commit");
  Plan p;
  std::string why;
  if (!make_plan(cfg, &p, &why)) return fail(FDL_ERR_INVALID_ARG, "%s", why.c_str());
  if (policy != FDL_SELECT_THRESHOLD && policy != FDL_SELECT_FACTOR &&
      policy != FDL_SELECT_BUDGET)
    return fail(FDL_ERR_INVALID_ARG, "unknown selection policy %d", policy);
  if (!std::isfinite(param)) return fail(FDL_ERR_INVALID_ARG, "param must be finite");
  FDL_CHECK_PTR(conf);
  FDL_CHECK_PTR(tok);
  FDL_CHECK_PTR(block_tokens);
  FDL_CHECK_PTR(committed);
  FDL_CHECK_PTR(n_committed);
  FDL_CHECK_PTR(n_masked_left);
  cudaError_t e =
      policy == FDL_SELECT_THRESHOLD
          ? launch_commit(conf, tok, block_tokens, committed, n_committed, n_masked_left,
                          cfg->batch, cfg->block_size, cfg->q_off, cfg->q_len, cfg->mask_id,
                          param, (cudaStream_t)stream)
          : launch_select_commit(policy, param, conf, tok, block_tokens, committed, n_committed,
                                 n_masked_left, cfg->batch, cfg->block_size, cfg->q_off,
                                 cfg->q_len, cfg->mask_id, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "select-commit launch");
  return ok();
}

int fdl_unit_status(const fdl_step_cfg* cfg, const int32_t* n_masked_left,
                    int32_t* any_masked, int32_t* step_count,
                    unsigned long long while_handle, void* stream) {
  NvtxRange nvtx_range("fdl_unit_status");
  Plan p;
  std::string why;
  if (!make_plan(cfg, &p, &why)) return fail(FDL_ERR_INVALID_ARG, "%s", why.c_str());
  if (n_masked_left == nullptr) return fail(FDL_ERR_INVALID_ARG, "n_masked_left is NULL");
  if (while_handle != 0ull && step_count == nullptr)
    return fail(FDL_ERR_INVALID_ARG, "a WHILE handle needs step_count (the loop bound)");
  cudaError_t e = launch_unit_status(n_masked_left, cfg->batch, any_masked, step_count,
                                     while_handle, cfg->q_len, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "unit-status launch");
  return ok();
}

int fdl_append_block(const fdl_step_cfg* cfg, const void* k_blk, const void* v_blk, void* k_pre,
                     void* v_pre, int32_t* len_pre, void* ws, size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("fdl_append_block");
  Plan p;
  std::string why;
  if (!make_plan(cfg, &p, &why, false)) return fail(FDL_ERR_INVALID_ARG, "%s", why.c_str());
  FDL_CHECK_PTR(k_blk);
  FDL_CHECK_PTR(v_blk);
  FDL_CHECK_PTR(k_pre);
  FDL_CHECK_PTR(v_pre);
  FDL_CHECK_PTR(len_pre);
  if (cfg->cap_prefix < cfg->block_size)
    return fail(FDL_ERR_INVALID_ARG, "cap_prefix is smaller than one block");
  int rc = check_ws(p, ws, ws_bytes);
  if (rc != FDL_OK) return rc;
  cudaError_t e = launch_append_block(k_blk, v_blk, k_pre, v_pre, len_pre,
                                      &at<Control>(ws, p.off_ctrl)->status, cfg->batch,
                                      cfg->n_kv_heads, cfg->block_size, cfg->cap_prefix,
                                      cfg->head_dim * p.elem, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "append-block launch");
  return ok();
}

int fdl_denoise_step(const fdl_step_cfg* cfg, const void* q, const void* k_pre,
                     const void* v_pre, const int32_t* len_pre, const void* k_blk,
                     const void* v_blk, const void* k_suf, const void* v_suf,
                     const int32_t* len_suf, const void* hidden,
                     const void* h_prev, const void* w_lm, int32_t* block_tokens,
                     void* attn_out, float* conf, int32_t* tok, uint8_t* committed,
                     int32_t* n_committed, int32_t* n_masked_left, void* ws,
                     size_t ws_bytes, void* stream) {
  NvtxRange nvtx_range("fdl_denoise_step");
  Plan p;
  std::string why;
  if (!make_plan(cfg, &p, &why)) return fail(FDL_ERR_INVALID_ARG, "%s", why.c_str());
  const fdl_step_cfg& c = *cfg;
  const bool dual = k_suf != nullptr || v_suf != nullptr || len_suf != nullptr;
  if (dual && (k_suf == nullptr || v_suf == nullptr || len_suf == nullptr))
    return fail(FDL_ERR_INVALID_ARG, "k_suf, v_suf and len_suf must all be set or all NULL");
  FDL_CHECK_PTR(q);
  FDL_CHECK_PTR(k_blk);
  FDL_CHECK_PTR(v_blk);
  FDL_CHECK_PTR(len_pre);
  FDL_CHECK_PTR(w_lm);
  FDL_CHECK_PTR(block_tokens);
  FDL_CHECK_PTR(conf);
  FDL_CHECK_PTR(tok);
  FDL_CHECK_PTR(committed);
  FDL_CHECK_PTR(n_committed);
  FDL_CHECK_PTR(n_masked_left);
  if (c.cap_prefix > 0) {
    FDL_CHECK_PTR(k_pre);
    FDL_CHECK_PTR(v_pre);
  }
  if (dual) {
    if (c.cap_suffix <= 0) return fail(FDL_ERR_INVALID_ARG, "DualCache needs cap_suffix > 0");
    FDL_CHECK_PTR(k_suf);
    FDL_CHECK_PTR(v_suf);
    FDL_CHECK_PTR(len_suf);
  }
  if (hidden != nullptr) FDL_CHECK_PTR(hidden);
  if (hidden == nullptr && c.hidden != c.n_q_heads * c.head_dim)
    return fail(FDL_ERR_INVALID_ARG,
                "hidden is NULL (attention output feeds the LM head) but hidden=%d != Hq*d=%d",
                c.hidden, c.n_q_heads * c.head_dim);
  if (c.shift) FDL_CHECK_PTR(h_prev);
  if (attn_out != nullptr) FDL_CHECK_PTR(attn_out);
  int rc = check_lmhead_supported(c);
  if (rc != FDL_OK) return rc;
  rc = check_ws(p, ws, ws_bytes);
  if (rc != FDL_OK) return rc;
  cudaStream_t s = (cudaStream_t)stream;
  void* out = attn_out != nullptr ? attn_out : at<void>(ws, p.off_attn);

  auto lm_rows = [&](const void* src, const void** rows) -> int {
    *rows = src;
    if (c.shift) {
      void* g = at<void>(ws, p.off_rows);
      cudaError_t e = launch_gather_rows(src, h_prev, g, c.batch, c.q_len, c.hidden,
                                         1, p.elem, s);
      if (e != cudaSuccess) return cuda_fail(e, "gather launch");
      *rows = g;
    }
    return FDL_OK;
  };
  auto lm_fused = [&](const void* rows) {
    LmArgs a = lm_args(c, p, rows, w_lm, nullptr, conf, tok, ws);
    a.block_tokens_in = block_tokens;
    a.commit = 1;
    a.block_tokens = block_tokens;
    a.committed = committed;
    a.n_committed = n_committed;
    a.n_masked_left = n_masked_left;
    return a;
  };

  if (hidden != nullptr && p.attn_tc && c.dtype == FDL_BF16) {
    // The LM-head rows are an input, so attention and the LM head are
    // independent: the LM head goes first in its shared-SM form and the
    // attention grid starts beside it, one CTA per SM, both streaming HBM.
    const void* rows = nullptr;
    rc = lm_rows(hidden, &rows);
    if (rc != FDL_OK) return rc;
    LmArgs a = lm_fused(rows);
    const size_t attn_smem =
        attn_tc_smem_for(c.q_len, c.n_q_heads / c.n_kv_heads, c.batch, true);
    if (lmhead_tc_shared_ok(a, attn_smem)) {
      rc = run_lmhead(a, c, s, attn_smem, c.shift != 0);
      if (rc != FDL_OK) return rc;
      rc = run_attention(c, p, dual, q, k_pre, v_pre, len_pre, k_blk, v_blk, k_suf, v_suf,
                         len_suf, out, ws, s, true);
      return rc != FDL_OK ? rc : ok();
    }
    // Too many rows for the shared form: the gather (already launched), the
    // attention and its merge, then the LM head as a programmatic dependent
    // of the merge, streaming the weight from the rows gathered before the
    // attention began while the merge still runs.
    rc = run_attention(c, p, dual, q, k_pre, v_pre, len_pre, k_blk, v_blk, k_suf, v_suf,
                       len_suf, out, ws, s);
    if (rc != FDL_OK) return rc;
    a.rows_ready = 1;
    rc = run_lmhead_passes(a, c, p, s, true);
    return rc != FDL_OK ? rc : ok();
  }

  rc = run_attention(c, p, dual, q, k_pre, v_pre, len_pre, k_blk, v_blk, k_suf,
                     v_suf, len_suf, out, ws, s);
  if (rc != FDL_OK) return rc;
  const void* rows = nullptr;
  rc = lm_rows(hidden != nullptr ? hidden : out, &rows);
  if (rc != FDL_OK) return rc;
  rc = run_lmhead_passes(lm_fused(rows), c, p, s, c.shift != 0);
  return rc != FDL_OK ? rc : ok();
}

int fdl_get_status(void* ws, void* stream, uint32_t* status) {
  if (ws == nullptr || status == nullptr)
    return fail(FDL_ERR_INVALID_ARG, "ws and status must be non-NULL");
  cudaStream_t s = (cudaStream_t)stream;
  uint32_t host = 0;
  cudaError_t e = cudaMemcpyAsync(&host, ws, sizeof(host), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(ws, 0, sizeof(uint32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word");
  *status = host;
  if (host != 0) return fail(FDL_ERR_DEVICE_STATUS, "device status 0x%x", host);
  return ok();
}

}  // extern "C"
