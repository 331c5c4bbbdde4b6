// C ABI of libfdl: argument checks, workspace layout, launches.
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

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
  a.commit = 0;
  a.B = c.batch;
  a.D = c.block_size;
  a.q_off = c.q_off;
  a.q_len = c.q_len;
  a.mask_id = c.mask_id;
  a.tau = c.tau;
  return a;
}

int run_attention(const fdl_step_cfg& c, const Plan& p, bool dual, const void* q,
                  const void* k_pre, const void* v_pre, const int32_t* len_pre,
                  const void* k_blk, const void* v_blk, const void* k_suf,
                  const void* v_suf, const int32_t* len_suf, void* out, void* ws,
                  cudaStream_t s) {
  AttnArgs a = attn_args(c, p, dual, q, k_pre, v_pre, len_pre, k_blk, v_blk,
                         k_suf, v_suf, len_suf, out, ws);
  // bf16 with d = 128: tensor-core kernel; otherwise the CUDA-core kernel.
  cudaError_t e = p.attn_tc
                      ? launch_attn_tc(a, at<float>(ws, p.off_tc_part_o),
                                       at<float2>(ws, p.off_tc_part_ml), a.tickets,
                                       kAttnTcCTAs, s)
                      : launch_attn_simt(a, (fdl_dtype)c.dtype, kAttnRowTile, s);
  if (e != cudaSuccess) return cuda_fail(e, "attention launch");
  return FDL_OK;
}

// bf16: tensor-core kernel (TMA + tcgen05, K in chunks of 64); fp32: the
// CUDA-core kernel.
int check_lmhead_supported(const fdl_step_cfg& c) {
  if (c.dtype == FDL_BF16 && c.hidden % 64 != 0)
    return fail(FDL_ERR_UNSUPPORTED, "bf16 LM head needs hidden %% 64 == 0 (got %d)", c.hidden);
  return FDL_OK;
}

int run_lmhead(const LmArgs& a, const fdl_step_cfg& c, cudaStream_t s) {
  cudaError_t e = c.dtype == FDL_BF16 ? launch_lmhead_tc(a, s)
                                      : launch_lmhead_simt(a, (fdl_dtype)c.dtype, s);
  if (e != cudaSuccess) return cuda_fail(e, "lm-head launch");
  return FDL_OK;
}

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
  if (!make_plan(cfg, &p, &why)) {
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
  if (!make_plan(cfg, &p, &why)) return fail(FDL_ERR_INVALID_ARG, "%s", why.c_str());
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
  return attn_common(cfg, false, q, k_pre, v_pre, len_pre, k_blk, v_blk, nullptr,
                     nullptr, nullptr, out, ws, ws_bytes, stream);
}

int fdl_dualcache_attn(const fdl_step_cfg* cfg, const void* q, const void* k_pre,
                       const void* v_pre, const int32_t* len_pre,
                       const void* k_blk, const void* v_blk, const void* k_suf,
                       const void* v_suf, const int32_t* len_suf, void* out,
                       void* ws, size_t ws_bytes, void* stream) {
  return attn_common(cfg, true, q, k_pre, v_pre, len_pre, k_blk, v_blk, k_suf,
                     v_suf, len_suf, out, ws, ws_bytes, stream);
}

int fdl_lmhead_confidence(const fdl_step_cfg* cfg, const void* rows,
                          const void* w_lm, const uint8_t* row_active,
                          float* conf, int32_t* tok, void* ws, size_t ws_bytes,
                          void* stream) {
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
  rc = run_lmhead(a, *cfg, (cudaStream_t)stream);
  return rc != FDL_OK ? rc : ok();
}

int fdl_threshold_commit(const fdl_step_cfg* cfg, const float* conf,
                         const int32_t* tok, int32_t* block_tokens,
                         uint8_t* committed, int32_t* n_committed,
                         int32_t* n_masked_left, void* stream) {
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

int fdl_denoise_step(const fdl_step_cfg* cfg, const void* q, const void* k_pre,
                     const void* v_pre, const int32_t* len_pre, const void* k_blk,
                     const void* v_blk, const void* k_suf, const void* v_suf,
                     const int32_t* len_suf, const void* hidden,
                     const void* h_prev, const void* w_lm, int32_t* block_tokens,
                     void* attn_out, float* conf, int32_t* tok, uint8_t* committed,
                     int32_t* n_committed, int32_t* n_masked_left, void* ws,
                     size_t ws_bytes, void* stream) {
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
  rc = run_attention(c, p, dual, q, k_pre, v_pre, len_pre, k_blk, v_blk, k_suf,
                     v_suf, len_suf, out, ws, s);
  if (rc != FDL_OK) return rc;

  const void* src = hidden != nullptr ? hidden : out;
  const void* rows = src;
  if (c.shift) {
    void* g = at<void>(ws, p.off_rows);
    cudaError_t e = launch_gather_rows(src, h_prev, g, c.batch, c.q_len, c.hidden,
                                       1, p.elem, s);
    if (e != cudaSuccess) return cuda_fail(e, "gather launch");
    rows = g;
  }
  LmArgs a = lm_args(c, p, rows, w_lm, nullptr, conf, tok, ws);
  a.block_tokens_in = block_tokens;
  a.commit = 1;
  a.block_tokens = block_tokens;
  a.committed = committed;
  a.n_committed = n_committed;
  a.n_masked_left = n_masked_left;
  rc = run_lmhead(a, c, s);
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
