// LM head + confidence on CUDA cores (fp32 arithmetic), any dtype.
//
// For each row: logits over the full vocabulary, reduced on the fly to the
// running (max, sum exp, argmax) triple, so logits never reach global
// memory ("Fast-dLLM v2" Level 2; technical review, section 4, Algorithm 2).
// Each CTA owns a contiguous vocabulary range; a warp computes one vocab row
// against 32 input rows per pass (lane-strided 16-byte loads, warp
// all-reduce), lane r keeps row r's running triple.  The last CTA merges the
// per-CTA partials (and commits, in the fused step).  This is the fp32 path
// and the reference for the tensor-core kernel.
#include "lm_merge.cuh"

namespace fdl {
namespace {

constexpr int kWarps = 8;

template <typename T>
struct Vec;
template <>
struct Vec<float> {
  static constexpr int N = 4;
  __device__ static void load(const float* p, float* x) {
    const float4 v = *reinterpret_cast<const float4*>(p);
    x[0] = v.x; x[1] = v.y; x[2] = v.z; x[3] = v.w;
  }
};
template <>
struct Vec<bf16> {
  static constexpr int N = 8;
  __device__ static void load(const bf16* p, float* x) {
    const uint4 v = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      x[2 * j] = __uint_as_float(w[j] << 16);
      x[2 * j + 1] = __uint_as_float(w[j] & 0xffff0000u);
    }
  }
};

template <typename T>
__global__ void __launch_bounds__(kWarps * 32)
lmhead_simt_kernel(const LmArgs a) {
  constexpr int VN = Vec<T>::N;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int v0 = blockIdx.x * a.rows_per_cta;
  const int v1 = min(a.V, v0 + a.rows_per_cta);
  const T* w = static_cast<const T*>(a.w);
  const T* x = static_cast<const T*>(a.rows);
  __shared__ MSI s_st[kWarps][32];

  for (int r0 = 0; r0 < a.R; r0 += 32) {
    const int nr = min(32, a.R - r0);
    MSI st = msi_empty();  // lane's row r0 + lane
    for (int v = v0 + warp; v < v1; v += kWarps) {
      float acc[32];
#pragma unroll
      for (int r = 0; r < 32; ++r) acc[r] = 0.f;
      const T* wr = w + (size_t)v * a.H;
      for (int k = lane * VN; k < a.H; k += 32 * VN) {
        float wv[VN];
        Vec<T>::load(wr + k, wv);
#pragma unroll
        for (int r = 0; r < 32; ++r) {
          if (r < nr) {
            float xv[VN];
            Vec<T>::load(x + (size_t)(r0 + r) * a.H + k, xv);
#pragma unroll
            for (int j = 0; j < VN; ++j) acc[r] = fmaf(wv[j], xv[j], acc[r]);
          }
        }
      }
      float mine = 0.f;
#pragma unroll
      for (int r = 0; r < 32; ++r) {
        float s = acc[r];
#pragma unroll
        for (int o = 16; o >= 1; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
        if (r == lane) mine = s;
      }
      if (lane < nr) st = msi_merge(st, MSI{mine, 1.f, v});
    }
    s_st[warp][lane] = st;
    __syncthreads();
    if (warp == 0) {
      MSI t = s_st[0][lane];
      for (int j = 1; j < kWarps; ++j) t = msi_merge(t, s_st[j][lane]);
      if (lane < nr) {
        Partial p;
        p.m = t.m;
        p.s = t.s;
        p.i = t.i;
        p.pad = 0;
        a.part[(size_t)blockIdx.x * a.R + r0 + lane] = p;
      }
    }
    __syncthreads();
  }
  if (!last_cta_arrives(&a.ctrl->lm_ticket[a.slot], a.n_cta)) return;
  lm_final_merge(a);
  if (threadIdx.x == 0) a.ctrl->lm_ticket[a.slot] = 0u;
}

}  // namespace

cudaError_t launch_lmhead_simt(const LmArgs& a, fdl_dtype dt, cudaStream_t s) {
  if (dt == FDL_BF16)
    lmhead_simt_kernel<bf16><<<a.n_cta, kWarps * 32, 0, s>>>(a);
  else
    lmhead_simt_kernel<float><<<a.n_cta, kWarps * 32, 0, s>>>(a);
  return cudaGetLastError();
}

}  // namespace fdl
