// Last-CTA merge of the LM-head partials, confidence/token output and the
// fused commit.  Shared by the CUDA-core and the tensor-core LM-head kernels.
#pragma once

#include "fdl_common.cuh"

namespace fdl {

// "Last CTA to arrive" ticket: every CTA has written its partials; returns
// true in exactly one CTA, after all other CTAs' writes are visible.  No
// thread ever waits on another CTA.
__device__ __forceinline__ bool last_cta_arrives(unsigned int* ticket,
                                                 unsigned int n_cta) {
  __shared__ int s_last;
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) s_last = atomicAdd(ticket, 1u) == n_cta - 1u;
  __syncthreads();
  if (s_last) __threadfence();
  return s_last != 0;
}

// Merge the n_cta partials of each row into (conf, tok); then, when the call
// is the fused step, commit (technical review, section 4, Algorithm 2).
// conf = 1 / sum_v exp(l_v - l_max) is the max softmax probability; the
// token is the argmax with the lowest vocabulary index on a tie.
// If a CTA's bounded wait ran out (FDL_DEV_TIMEOUT in the status word, set
// before its ticket), its partials are stale: every row then reports
// conf = -1 and tok = -1 and the commit selects nothing (block tokens kept,
// counts written), until the caller reads and clears the status word.
__device__ __forceinline__ void lm_final_merge(const LmArgs& a) {
  __shared__ float s_conf[kMaxRows];
  __shared__ int s_tok[kMaxRows];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nw = blockDim.x >> 5;
  const bool timed_out =
      (*reinterpret_cast<volatile unsigned int*>(&a.ctrl->status) & FDL_DEV_TIMEOUT) != 0u;
  for (int r = warp; r < a.R; r += nw) {
    MSI st = msi_empty();
    for (int c = lane; c < a.n_cta; c += 32) {
      const float4 p = __ldcg(reinterpret_cast<const float4*>(a.part + (size_t)c * a.R + r));
      st = msi_merge(st, MSI{p.x, p.y, __float_as_int(p.z)});
    }
    st = msi_warp_allmerge(st);
    if (lane == 0) {
      bool act = true;
      if (a.row_active != nullptr) act = a.row_active[r] != 0;
      if (a.block_tokens_in != nullptr) {
        const int b = r / a.q_len, i = r % a.q_len;
        act = a.block_tokens_in[(size_t)b * a.D + a.q_off + i] == a.mask_id;
      }
      act = act && !timed_out;
      const float c = act ? 1.0f / st.s : -1.0f;
      const int t = act ? st.i : -1;
      a.conf[r] = c;
      a.tok[r] = t;
      s_conf[r] = c;
      s_tok[r] = t;
    }
  }
  if (!a.commit) return;
  __syncthreads();
  for (int b = warp; b < a.B; b += nw) {
    const int base = b * a.q_len;
    if (timed_out) {
      apply_selection_warp(b, lane, a.D, a.q_off, a.q_len, a.mask_id, 0u,
                           [&](int i) { return s_tok[base + i]; }, a.block_tokens,
                           a.committed, a.n_committed, a.n_masked_left);
      continue;
    }
    commit_sequence_warp(
        b, lane, a.D, a.q_off, a.q_len, a.mask_id, a.tau,
        [&](int i) { return s_conf[base + i]; },
        [&](int i) { return s_tok[base + i]; }, a.block_tokens, a.committed,
        a.n_committed, a.n_masked_left);
  }
}

}  // namespace fdl
