// Split-KV attention on CUDA cores (fp32 arithmetic), any dtype.
//
// Attention of the active unit's queries over [prefix cache | block rows |
// suffix cache] ("Fast-dLLM v2" section 3.4, Figure 7b; technical review
// eq. (3) and section 3).  The key sequence of (b, kv head) is cut into
// splits; each CTA runs an online softmax over one split for one tile of
// query rows, and the last CTA of a (b, kv head, row tile) to finish merges
// the splits' (m, l, o) partials (flash-decoding), so one launch produces the
// final output.  This is the fp32 path and the reference for the tensor-core
// kernel.
#include "fdl_common.cuh"

namespace fdl {
namespace {

constexpr int kChunk = 32;      // keys per shared-memory chunk
constexpr int kWarps = 4;
constexpr int kRowsPerWarp = 4;
constexpr int kRowTile = kWarps * kRowsPerWarp;  // 16 query rows per CTA

template <typename T>
__device__ __forceinline__ const T* key_row(const AttnArgs& a, const T* pre,
                                            const T* blk, const T* suf, int b,
                                            int kvh, int k, int Lp) {
  if (k < Lp) return pre + (((size_t)b * a.Hkv + kvh) * a.cap_p + k) * a.d;
  k -= Lp;
  if (k < a.D) return blk + (((size_t)b * a.Hkv + kvh) * a.D + k) * a.d;
  k -= a.D;
  return suf + (((size_t)b * a.Hkv + kvh) * a.cap_s + k) * a.d;
}

template <typename T, int DH>
__global__ void __launch_bounds__(kWarps * 32)
attn_simt_kernel(const AttnArgs a) {
  constexpr int DPL = DH / 32;  // head dims per lane
  const int split = blockIdx.x;
  const int n_tiles = (a.rows + kRowTile - 1) / kRowTile;
  const int kvh = blockIdx.y / n_tiles;
  const int tile = blockIdx.y % n_tiles;
  const int b = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  __shared__ float sq[kRowTile][DH];
  __shared__ float sk[kChunk][DH + 1];
  __shared__ float sv[kChunk][DH + 1];
  __shared__ float sp[kWarps][kChunk];
  __shared__ int s_last;

  // Device-side length checks: a bad length is treated as 0 and flagged.
  int Lp = a.len_pre[b];
  if (Lp < 0 || Lp > a.cap_p) {
    if (threadIdx.x == 0) atomicOr(&a.ctrl->status, FDL_DEV_BAD_PREFIX_LEN);
    Lp = 0;
  }
  int Ls = 0;
  if (a.k_suf != nullptr) {
    Ls = a.len_suf[b];
    if (Ls < 0 || Ls > a.cap_s) {
      if (threadIdx.x == 0) atomicOr(&a.ctrl->status, FDL_DEV_BAD_SUFFIX_LEN);
      Ls = 0;
    }
  }
  const int n_keys = Lp + a.D + Ls;
  const int k_begin = split * a.split_keys;
  const int k_end = min(n_keys, k_begin + a.split_keys);

  const T* q = static_cast<const T*>(a.q);
  const T* kp = static_cast<const T*>(a.k_pre);
  const T* vp = static_cast<const T*>(a.v_pre);
  const T* kb = static_cast<const T*>(a.k_blk);
  const T* vb = static_cast<const T*>(a.v_blk);
  const T* ks = static_cast<const T*>(a.k_suf);
  const T* vs = static_cast<const T*>(a.v_suf);

  // Query rows of this tile: row r = qi * group + j -> head kvh*group + j.
  for (int t = threadIdx.x; t < kRowTile * DH; t += blockDim.x) {
    const int rr = t / DH, i = t % DH;
    const int r = tile * kRowTile + rr;
    float x = 0.f;
    if (r < a.rows) {
      const int qi = r / a.group, h = kvh * a.group + r % a.group;
      x = to_f32(q[(((size_t)b * a.q_len + qi) * a.Hq + h) * DH + i]);
    }
    sq[rr][i] = x;
  }

  float m[kRowsPerWarp], l[kRowsPerWarp], o[kRowsPerWarp][DPL];
#pragma unroll
  for (int j = 0; j < kRowsPerWarp; ++j) {
    m[j] = kEmptyMax;
    l[j] = 0.f;
#pragma unroll
    for (int u = 0; u < DPL; ++u) o[j][u] = 0.f;
  }

  for (int c0 = k_begin; c0 < k_end; c0 += kChunk) {
    const int nk = min(kChunk, k_end - c0);
    __syncthreads();
    for (int t = threadIdx.x; t < kChunk * DH; t += blockDim.x) {
      const int kk = t / DH, i = t % DH;
      float kx = 0.f, vx = 0.f;
      if (kk < nk) {
        kx = to_f32(key_row(a, kp, kb, ks, b, kvh, c0 + kk, Lp)[i]);
        vx = to_f32(key_row(a, vp, vb, vs, b, kvh, c0 + kk, Lp)[i]);
      }
      sk[kk][i] = kx;
      sv[kk][i] = vx;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kRowsPerWarp; ++j) {
      const int rr = warp * kRowsPerWarp + j;
      // lane = key within the chunk
      float s = 0.f;
#pragma unroll 8
      for (int i = 0; i < DH; ++i) s = fmaf(sq[rr][i], sk[lane][i], s);
      s = lane < nk ? s * a.scale_log2 : kEmptyMax;  // log2 units
      float cm = s;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1)
        cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, off));
      const float m_new = fmaxf(m[j], cm);
      const float p = lane < nk ? exp2f(s - m_new) : 0.f;
      const float alpha = exp2f(m[j] - m_new);
      float ps = p;
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1)
        ps += __shfl_xor_sync(0xffffffffu, ps, off);
      l[j] = l[j] * alpha + ps;
      m[j] = m_new;
      sp[warp][lane] = p;
      __syncwarp();
#pragma unroll
      for (int u = 0; u < DPL; ++u) {
        float acc = o[j][u] * alpha;
        const int i = lane + 32 * u;
        for (int kk = 0; kk < nk; ++kk) acc = fmaf(sp[warp][kk], sv[kk][i], acc);
        o[j][u] = acc;
      }
      __syncwarp();
    }
  }

  const int item = ((b * a.Hkv + kvh) * n_tiles + tile);
  T* out = static_cast<T*>(a.out);
  if (a.n_split == 1) {
#pragma unroll
    for (int j = 0; j < kRowsPerWarp; ++j) {
      const int r = tile * kRowTile + warp * kRowsPerWarp + j;
      if (r >= a.rows) continue;
      const int qi = r / a.group, h = kvh * a.group + r % a.group;
      const float inv = l[j] > 0.f ? 1.f / l[j] : 0.f;
#pragma unroll
      for (int u = 0; u < DPL; ++u)
        out[(((size_t)b * a.q_len + qi) * a.Hq + h) * DH + lane + 32 * u] =
            from_f32<T>(o[j][u] * inv);
    }
    return;
  }

  // Partial of this split, then the last CTA of the item merges all splits.
  const size_t pbase = ((size_t)item * a.n_split + split) * kRowTile;
#pragma unroll
  for (int j = 0; j < kRowsPerWarp; ++j) {
    const int rr = warp * kRowsPerWarp + j;
#pragma unroll
    for (int u = 0; u < DPL; ++u)
      a.part_o[(pbase + rr) * DH + lane + 32 * u] = o[j][u];
    if (lane == 0) a.part_ml[pbase + rr] = make_float2(m[j], l[j]);
  }
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned prev = atomicAdd(&a.tickets[item], 1u);
    s_last = prev == (unsigned)(a.n_split - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int t = threadIdx.x; t < kRowTile * DH; t += blockDim.x) {
    const int rr = t / DH, i = t % DH;
    const int r = tile * kRowTile + rr;
    if (r >= a.rows) continue;
    const size_t base = (size_t)item * a.n_split * kRowTile + rr;
    float M = kEmptyMax;
    for (int sp_ = 0; sp_ < a.n_split; ++sp_)
      M = fmaxf(M, __ldcg(&a.part_ml[base + (size_t)sp_ * kRowTile]).x);
    float L = 0.f, O = 0.f;
    for (int sp_ = 0; sp_ < a.n_split; ++sp_) {
      const float2 ml = __ldcg(&a.part_ml[base + (size_t)sp_ * kRowTile]);
      const float w = exp2f(ml.x - M);
      L += ml.y * w;
      O += __ldcg(&a.part_o[(base + (size_t)sp_ * kRowTile) * DH + i]) * w;
    }
    const int qi = r / a.group, h = kvh * a.group + r % a.group;
    out[(((size_t)b * a.q_len + qi) * a.Hq + h) * DH + i] =
        from_f32<T>(L > 0.f ? O / L : 0.f);
  }
  if (threadIdx.x == 0) a.tickets[item] = 0u;  // ready for the next call
}

template <typename T>
cudaError_t launch_t(const AttnArgs& a, cudaStream_t s) {
  const int n_tiles = (a.rows + kRowTile - 1) / kRowTile;
  dim3 grid(a.n_split, a.Hkv * n_tiles, a.B);
  switch (a.d) {
    case 32: attn_simt_kernel<T, 32><<<grid, kWarps * 32, 0, s>>>(a); break;
    case 64: attn_simt_kernel<T, 64><<<grid, kWarps * 32, 0, s>>>(a); break;
    case 128: attn_simt_kernel<T, 128><<<grid, kWarps * 32, 0, s>>>(a); break;
    default: return cudaErrorInvalidValue;
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_attn_simt(const AttnArgs& a, fdl_dtype dt, int row_tile,
                             cudaStream_t s) {
  if (row_tile != kRowTile) return cudaErrorInvalidValue;
  return dt == FDL_BF16 ? launch_t<bf16>(a, s) : launch_t<float>(a, s);
}

}  // namespace fdl
