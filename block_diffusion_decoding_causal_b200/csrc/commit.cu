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

// LM-head input rows with the token shift ("Fast-dLLM v2" section 3.4,
// Step 5): rows[b, i] = src[b, i - shift], and rows[b, 0] = h_prev[b] when
// shifting.  16-byte vectors; H * elem is a multiple of 16.
__global__ void gather_rows_kernel(const uint4* src, const uint4* h_prev,
                                   uint4* rows, int B, int q_len, int vec_per_row,
                                   int shift) {
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

cudaError_t launch_gather_rows(const void* src, const void* h_prev, void* rows,
                               int B, int q_len, int H, int shift, int elem,
                               cudaStream_t s) {
  const int vec_per_row = H * elem / 16;
  const size_t n = (size_t)B * q_len * vec_per_row;
  const int threads = 256;
  const int blocks = (int)((n + threads - 1) / threads);
  gather_rows_kernel<<<blocks, threads, 0, s>>>(
      static_cast<const uint4*>(src), static_cast<const uint4*>(h_prev),
      static_cast<uint4*>(rows), B, q_len, vec_per_row, shift);
  return cudaGetLastError();
}

}  // namespace fdl
