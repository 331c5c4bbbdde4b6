// LM head + confidence for callers that cannot allocate device memory.
//
// Some callers cannot call cudaMalloc or hand the library a workspace: a
// plugin running inside another engine that owns every device allocation, a
// real-time loop where allocation is forbidden after start-up, or a host
// framework whose allocator cannot be reached from the code that calls us.
// For them this file keeps the LM head's scratch (the control words and the
// per-CTA partial results) in a fixed array in the library itself, which
// every GPU that loads the library holds until the process exits.
#include <cstring>
#include <mutex>
#include <string>

#include "fdl_common.cuh"
#include "fdl_plan.h"

namespace fdl {
namespace {

constexpr int kStaticMaxRows = 128;           // B * q_len
constexpr int kStaticMaxCtas = 2 * kPlanCTAs;  // CUDA-core plan uses up to 296
constexpr size_t kStaticControl = 256;
constexpr size_t kStaticBytes =
    kStaticControl + sizeof(Partial) * (size_t)kStaticMaxCtas * kStaticMaxRows;  // 606,464 B

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, never a device address: the address is looked up per device below.
static __device__ __align__(256) unsigned char g_lm_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};

// Device address of the scratch on the current device; the first call on a
// device looks it up and zeroes the control words (synchronously).
cudaError_t static_scratch(void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_lm_scratch);
    if (e != cudaSuccess) return e;
    e = cudaMemset(p, 0, kStaticControl);
    if (e != cudaSuccess) return e;
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return cudaSuccess;
}

}  // namespace

// Sizes the static scratch can serve; fills `why` otherwise.
int lmhead_static_check(const Plan& p, const fdl_step_cfg& c, std::string* why) {
  const int n_cta = c.dtype == FDL_BF16 ? p.lm_tc_cta : p.lm_cta;
  if (p.R > kStaticMaxRows) {
    *why = "allocation-free LM head handles at most " + std::to_string(kStaticMaxRows) +
           " rows (batch * q_len); got " + std::to_string(p.R);
    return FDL_ERR_UNSUPPORTED;
  }
  if (n_cta > kStaticMaxCtas) {
    *why = "allocation-free LM head: vocabulary split needs more CTAs than its scratch holds";
    return FDL_ERR_UNSUPPORTED;
  }
  return FDL_OK;
}

cudaError_t lmhead_static_workspace(Control** ctrl, Partial** part) {
  void* p = nullptr;
  cudaError_t e = static_scratch(&p);
  if (e != cudaSuccess) return e;
  *ctrl = static_cast<Control*>(p);
  *part = reinterpret_cast<Partial*>(static_cast<unsigned char*>(p) + kStaticControl);
  return cudaSuccess;
}

}  // namespace fdl

namespace fdl {
int record_error(int code, const std::string& msg);
int record_ok();
}  // namespace fdl

extern "C" int fdl_lmhead_confidence_noalloc(const fdl_step_cfg* cfg, const void* rows,
                                             const void* w_lm, const uint8_t* row_active,
                                             float* conf, int32_t* tok, void* stream) {
  using namespace fdl;
  Plan p;
  std::string why;
  if (!make_plan(cfg, &p, &why)) return record_error(FDL_ERR_INVALID_ARG, why);
  const void* need[4] = {rows, w_lm, conf, tok};
  const char* names[4] = {"rows", "w_lm", "conf", "tok"};
  for (int i = 0; i < 4; ++i) {
    if (need[i] == nullptr) return record_error(FDL_ERR_INVALID_ARG, std::string(names[i]) + " is NULL");
    if ((reinterpret_cast<uintptr_t>(need[i]) & 15u) != 0)
      return record_error(FDL_ERR_INVALID_ARG, std::string(names[i]) + " is not 16-byte aligned");
  }
  if (cfg->dtype == FDL_BF16 && cfg->hidden % 64 != 0)
    return record_error(FDL_ERR_UNSUPPORTED, "bf16 LM head needs hidden % 64 == 0");
  if (cfg->w_layout == FDL_W_PACKED && cfg->dtype != FDL_BF16)
    return record_error(FDL_ERR_UNSUPPORTED, "the tiled weight layout is bf16 only");
  const int rc = lmhead_static_check(p, *cfg, &why);
  if (rc != FDL_OK) return record_error(rc, why);
  LmArgs a;
  memset(&a, 0, sizeof(a));
  cudaError_t e = lmhead_static_workspace(&a.ctrl, &a.part);
  if (e != cudaSuccess)
    return record_error(FDL_ERR_CUDA, std::string("static scratch: ") + cudaGetErrorString(e));
  const bool tc = cfg->dtype == FDL_BF16;
  a.rows = rows;
  a.w = w_lm;
  a.row_active = row_active;
  a.conf = conf;
  a.tok = tok;
  a.R = p.R;
  a.H = cfg->hidden;
  a.V = cfg->vocab;
  a.n_cta = tc ? p.lm_tc_cta : p.lm_cta;
  a.rows_per_cta = tc ? p.lm_tc_rows_per_cta : p.lm_rows_per_cta;
  a.w_packed = cfg->w_layout == FDL_W_PACKED;
  a.B = cfg->batch;
  a.D = cfg->block_size;
  a.q_off = cfg->q_off;
  a.q_len = cfg->q_len;
  a.mask_id = cfg->mask_id;
  a.tau = cfg->tau;
  e = tc ? launch_lmhead_tc(a, (cudaStream_t)stream)
         : launch_lmhead_simt(a, (fdl_dtype)cfg->dtype, (cudaStream_t)stream);
  if (e != cudaSuccess)
    return record_error(FDL_ERR_CUDA, std::string("lm-head launch: ") + cudaGetErrorString(e));
  return record_ok();
}
