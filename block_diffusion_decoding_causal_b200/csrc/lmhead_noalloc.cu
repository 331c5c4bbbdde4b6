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

constexpr int kStaticMaxRows = FDL_NOALLOC_MAX_ROWS;  // B * q_len
constexpr int kStaticMaxCtas = 2 * kPlanCTAs;         // CUDA-core plan uses up to 296
constexpr size_t kStaticControl = 256;
constexpr size_t kStaticBytes =
    kStaticControl + sizeof(Partial) * (size_t)kStaticMaxCtas * kStaticMaxRows;
// The header states both limits as numbers; keep them tied to the code.
static_assert(kStaticBytes == FDL_NOALLOC_SCRATCH_BYTES,
              "FDL_NOALLOC_SCRATCH_BYTES in fdl.h must match the static scratch");
static_assert(sizeof(Control) <= kStaticControl, "control words exceed their slot");

// The scratch itself.  In host code this name is only a stand-in for the
// symbol, never a device address: the address is looked up per device below.
static __device__ __align__(256) unsigned char g_lm_scratch[kStaticBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch[kMaxDevices] = {};

// Device address of the scratch on the current device.  The first call on a
// device looks it up and queues the zeroing of the control words on `stream`,
// ahead of whatever the caller launches next on that stream.
cudaError_t static_scratch(cudaStream_t stream, void** out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_scratch[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_lm_scratch);
    if (e != cudaSuccess) return e;
    e = cudaMemsetAsync(p, 0, kStaticControl, stream);
    if (e != cudaSuccess) return e;
    g_scratch[dev] = p;
  }
  *out = g_scratch[dev];
  return cudaSuccess;
}

}  // namespace

constexpr size_t kStaticControlSize = kStaticControl;

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

cudaError_t lmhead_static_workspace(cudaStream_t stream, Control** ctrl, Partial** part) {
  void* p = nullptr;
  cudaError_t e = static_scratch(stream, &p);
  if (e != cudaSuccess) return e;
  *ctrl = static_cast<Control*>(p);
  *part = reinterpret_cast<Partial*>(static_cast<unsigned char*>(p) + kStaticControl);
  return cudaSuccess;
}

}  // namespace fdl

namespace fdl {
int record_error(int code, const std::string& msg);
int record_ok();
int launch_wait_timeout(unsigned int* status, long long limit_cycles, cudaStream_t stream);
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
  cudaError_t e = lmhead_static_workspace((cudaStream_t)stream, &a.ctrl, &a.part);
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

// Status of the allocation-free LM head: synchronise `stream`, read the static
// scratch's status word into *status and clear it.
extern "C" int fdl_lmhead_noalloc_status(void* stream, uint32_t* status) {
  using namespace fdl;
  if (status == nullptr) return record_error(FDL_ERR_INVALID_ARG, "status is NULL");
  cudaStream_t s = (cudaStream_t)stream;
  Control* ctrl = nullptr;
  Partial* part = nullptr;
  uint32_t host = 0;
  cudaError_t e = lmhead_static_workspace(s, &ctrl, &part);
  if (e == cudaSuccess)
    e = cudaMemcpyAsync(&host, &ctrl->status, sizeof(host), cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess) e = cudaMemsetAsync(&ctrl->status, 0, sizeof(uint32_t), s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess)
    return record_error(FDL_ERR_CUDA, std::string("static status word: ") + cudaGetErrorString(e));
  *status = host;
  if (host != 0)
    return record_error(FDL_ERR_DEVICE_STATUS, "device status " + std::to_string(host));
  return record_ok();
}

// Zero every control word of the static scratch (status and counters), on
// `stream`.
extern "C" int fdl_lmhead_noalloc_reset(void* stream) {
  using namespace fdl;
  cudaStream_t s = (cudaStream_t)stream;
  Control* ctrl = nullptr;
  Partial* part = nullptr;
  cudaError_t e = lmhead_static_workspace(s, &ctrl, &part);
  if (e == cudaSuccess) e = cudaMemsetAsync(ctrl, 0, fdl::kStaticControlSize, s);
  if (e != cudaSuccess)
    return record_error(FDL_ERR_CUDA, std::string("static scratch reset: ") + cudaGetErrorString(e));
  return record_ok();
}

// The failure self-check of fdl_check_wait_timeout, aimed at the static
// scratch's status word.
extern "C" int fdl_lmhead_noalloc_check_wait_timeout(long long limit_cycles, void* stream) {
  using namespace fdl;
  if (limit_cycles < 1000 || limit_cycles > 2000000000LL)
    return record_error(FDL_ERR_INVALID_ARG, "limit_cycles must be in [1e3, 2e9]");
  cudaStream_t s = (cudaStream_t)stream;
  Control* ctrl = nullptr;
  Partial* part = nullptr;
  cudaError_t e = lmhead_static_workspace(s, &ctrl, &part);
  if (e != cudaSuccess)
    return record_error(FDL_ERR_CUDA, std::string("static scratch: ") + cudaGetErrorString(e));
  return launch_wait_timeout(&ctrl->status, limit_cycles, s);
}
