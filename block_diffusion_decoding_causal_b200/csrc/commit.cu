// Threshold commit (standalone) and the token-shift row gather.
#include "fdl_common.cuh"

namespace fdl {
namespace {

// One warp per sequence (technical review, section 4, Algorithm 2).
__global__ void commit_kernel(const float* conf, const int32_t* tok,
                              int32_t* block_tokens, uint8_t* committed,
                              int32_t* n_committed, int32_t* n_masked_left,
                              int B, int D, int q_off, int q_len, int mask_id,
                              float tau) {
  const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  const float* cb = conf + (size_t)b * q_len;
  const int32_t* tb = tok + (size_t)b * q_len;
  commit_sequence_warp(
      b, lane, D, q_off, q_len, mask_id, tau, [&](int i) { return cb[i]; },
      [&](int i) { return tb[i]; }, block_tokens, committed, n_committed,
      n_masked_left);
}

// Factor / budget selection and commit, one warp per sequence.
__global__ void select_commit_kernel(int policy, float param, const float* conf,
                                     const int32_t* tok, int32_t* block_tokens,
                                     uint8_t* committed, int32_t* n_committed,
                                     int32_t* n_masked_left, int B, int D, int q_off,
                                     int q_len, int mask_id) {
  const int b = blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (b >= B) return;
  const float* cb = conf + (size_t)b * q_len;
  const int32_t* tb = tok + (size_t)b * q_len;
  const unsigned sel = ranked_selection_warp(b, lane, D, q_off, q_len, mask_id, policy, param,
                                             block_tokens, [&](int i) { return cb[i]; });
  apply_selection_warp(b, lane, D, q_off, q_len, mask_id, sel, [&](int i) { return tb[i]; },
                       block_tokens, committed, n_committed, n_masked_left);
}

// LM-head input rows with the token shift ("Fast-dLLM v2" section 3.4,
// Step 5): rows[b, i] = src[b, i - shift], and rows[b, 0] = h_prev[b] when
// shifting.  16-byte vectors; H * elem is a multiple of 16.
__global__ void gather_rows_kernel(const uint4* src, const uint4* h_prev,
                                   uint4* rows, int B, int q_len, int vec_per_row,
                                   int shift) {
  // The LM head launched behind this kernel may start its weight stream now;
  // it waits for this grid before reading the rows.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // Launched as a programmatic dependent of the previous step (whose last
  // grid, the attention, completes only after that step's LM head, the
  // reader of `rows`): its launch overlapped that step; wait for it before
  // reading the inputs or overwriting the rows.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const size_t n = (size_t)B * q_len * vec_per_row;
  for (size_t t = blockIdx.x * (size_t)blockDim.x + threadIdx.x; t < n;
       t += (size_t)gridDim.x * blockDim.x) {
    const int k = (int)(t % vec_per_row);
    const size_t row = t / vec_per_row;
    const int i = (int)(row % q_len);
    const int b = (int)(row / q_len);
    uint4 v;
    if (shift && i == 0)
      v = h_prev[(size_t)b * vec_per_row + k];
    else
      v = src[((size_t)b * q_len + i - shift) * vec_per_row + k];
    rows[t] = v;
  }
}

}  // namespace

cudaError_t launch_commit(const float* conf, const int32_t* tok,
                          int32_t* block_tokens, uint8_t* committed,
                          int32_t* n_committed, int32_t* n_masked_left, int B,
                          int D, int q_off, int q_len, int mask_id, float tau,
                          cudaStream_t s) {
  const int warps = 4;
  commit_kernel<<<(B + warps - 1) / warps, warps * 32, 0, s>>>(
      conf, tok, block_tokens, committed, n_committed, n_masked_left, B, D,
      q_off, q_len, mask_id, tau);
  return cudaGetLastError();
}

cudaError_t launch_select_commit(int policy, float param, const float* conf,
                                 const int32_t* tok, int32_t* block_tokens,
                                 uint8_t* committed, int32_t* n_committed,
                                 int32_t* n_masked_left, int B, int D, int q_off,
                                 int q_len, int mask_id, cudaStream_t s) {
  const int warps = 4;
  select_commit_kernel<<<(B + warps - 1) / warps, warps * 32, 0, s>>>(
      policy, param, conf, tok, block_tokens, committed, n_committed, n_masked_left, B, D,
      q_off, q_len, mask_id);
  return cudaGetLastError();
}

cudaError_t launch_gather_rows(const void* src, const void* h_prev, void* rows,
                               int B, int q_len, int H, int shift, int elem,
                               cudaStream_t s) {
  const int vec_per_row = H * elem / 16;
  const size_t n = (size_t)B * q_len * vec_per_row;
  const int threads = 256;
  const int blocks = (int)((n + threads - 1) / threads);
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(blocks, 1, 1);
  lc.blockDim = dim3(threads, 1, 1);
  lc.dynamicSmemBytes = 0;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&lc, gather_rows_kernel,
                                           static_cast<const uint4*>(src),
                                           static_cast<const uint4*>(h_prev),
                                           static_cast<uint4*>(rows), B, q_len, vec_per_row, shift);
  return e != cudaSuccess ? e : cudaGetLastError();
}

}  // namespace fdl

namespace fdl {
namespace {

// Loop control of the sub-block iteration (technical review Algorithm 1:
// steps repeat while masked positions remain): any[0] = 1 if any sequence still
// has a masked position in the unit; optionally sets a CUDA-graph conditional
// (the WHILE node around one denoising step) and counts steps.
// The WHILE condition also stops after `limit` steps (the unit length: every
// step commits at least one masked position), so a graph loop is bounded.
__global__ void unit_status_kernel(const int32_t* n_masked_left, int B, int32_t* any_out,
                                   int32_t* steps, unsigned long long handle, int limit) {
  const int lane = threadIdx.x;
  int any = 0;
  for (int b = lane; b < B; b += 32) any |= n_masked_left[b] > 0;
  any = __any_sync(0xffffffffu, any);
  if (lane == 0) {
    if (any_out != nullptr) *any_out = any;
    int n = 0;
    if (steps != nullptr) {
      n = *steps + 1;
      *steps = n;
    }
    if (handle != 0ull)
      cudaGraphSetConditional((cudaGraphConditionalHandle)handle,
                              (any && n < limit) ? 1u : 0u);
  }
}

// Block-level KV cache (v2 digest, Level 3): once a block is fully decoded
// its D rows of K and V are appended to the prefix cache of every (sequence,
// KV head) and the prefix length grows by D, all on the device.
__global__ void append_block_kernel(const uint4* k_blk, const uint4* v_blk, uint4* k_pre,
                                    uint4* v_pre, int32_t* len_pre, unsigned int* status,
                                    int B, int Hkv, int D, int cap, int vec_per_row) {
  const int b = blockIdx.y;
  const int Lp = len_pre[b];
  const bool ok = Lp >= 0 && Lp + D <= cap;
  if (!ok) {
    if (blockIdx.x == 0 && threadIdx.x == 0) atomicOr(status, FDL_DEV_BAD_PREFIX_LEN);
    return;
  }
  const size_t per_b = (size_t)Hkv * D * vec_per_row;
  for (size_t t = blockIdx.x * (size_t)blockDim.x + threadIdx.x; t < per_b;
       t += (size_t)gridDim.x * blockDim.x) {
    const int k = (int)(t % vec_per_row);
    const size_t row = t / vec_per_row;
    const int j = (int)(row % D), h = (int)(row / D);
    const size_t src = (((size_t)b * Hkv + h) * D + j) * vec_per_row + k;
    const size_t dst = (((size_t)b * Hkv + h) * cap + Lp + j) * vec_per_row + k;
    k_pre[dst] = k_blk[src];
    v_pre[dst] = v_blk[src];
  }
}

// The length grows after every CTA copied (a separate launch keeps it simple).
__global__ void grow_len_kernel(int32_t* len_pre, int B, int D, int cap) {
  const int b = blockIdx.x * blockDim.x + threadIdx.x;
  if (b < B) {
    const int Lp = len_pre[b];
    if (Lp >= 0 && Lp + D <= cap) len_pre[b] = Lp + D;
  }
}

}  // namespace

cudaError_t launch_unit_status(const int32_t* n_masked_left, int B, int32_t* any_out,
                               int32_t* steps, unsigned long long handle, int limit,
                               cudaStream_t s) {
  unit_status_kernel<<<1, 32, 0, s>>>(n_masked_left, B, any_out, steps, handle, limit);
  return cudaGetLastError();
}

cudaError_t launch_append_block(const void* k_blk, const void* v_blk, void* k_pre, void* v_pre,
                                int32_t* len_pre, unsigned int* status, int B, int Hkv, int D,
                                int cap, int row_bytes, cudaStream_t s) {
  const int vec = row_bytes / 16;
  dim3 grid((unsigned)((Hkv * D * vec + 255) / 256 < 64 ? (Hkv * D * vec + 255) / 256 : 64),
            (unsigned)B);
  append_block_kernel<<<grid, 256, 0, s>>>(
      static_cast<const uint4*>(k_blk), static_cast<const uint4*>(v_blk),
      static_cast<uint4*>(k_pre), static_cast<uint4*>(v_pre), len_pre, status, B, Hkv, D, cap,
      vec);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  grow_len_kernel<<<(B + 127) / 128, 128, 0, s>>>(len_pre, B, D, cap);
  return cudaGetLastError();
}

}  // namespace fdl
