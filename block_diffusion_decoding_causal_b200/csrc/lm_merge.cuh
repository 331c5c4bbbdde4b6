// Merge of the LM-head partials (by the last CTA to arrive, or in two levels
// by teams of CTAs), confidence/token output and the fused commit.  Shared
// by the CUDA-core and the tensor-core LM-head kernels.
#pragma once

#include "fdl_common.cuh"

namespace fdl {

// The threads of a CTA that run a merge: all of them, or the tensor-core LM
// head's four epilogue warps (threads 64..191, named barrier 1) while its
// other warps already stream the next pass.
struct CtaThreads {
  __device__ static int rank() { return threadIdx.x; }
  __device__ static int size() { return blockDim.x; }
  __device__ static void sync() { __syncthreads(); }
};
struct EpilogueThreads {
  __device__ static int rank() { return threadIdx.x - 64; }
  __device__ static int size() { return 128; }
  __device__ static void sync() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
};

// "Last CTA to arrive" ticket: every CTA has written its partials; returns
// true in exactly one CTA, after all other CTAs' writes are visible.  No
// thread ever waits on another CTA.
template <class G = CtaThreads>
__device__ __forceinline__ bool last_cta_arrives(unsigned int* ticket,
                                                 unsigned int n_cta) {
  __shared__ int s_last;
  __threadfence();
  G::sync();
  if (G::rank() == 0) s_last = atomicAdd(ticket, 1u) == n_cta - 1u;
  G::sync();
  const bool last = s_last != 0;
  if (last) __threadfence();
  return last;
}

// Row r's merge of n partials part[(first + j * stride) * R + r], j < n, in
// increasing j: one thread per row, sixteen reads in flight at a time (the
// partials of one source are consecutive rows, so a warp's reads coalesce).
__device__ __forceinline__ MSI lm_merge_sources(const Partial* part, int R, int r, int first,
                                                int stride, int n) {
  MSI st = msi_empty();
  for (int j0 = 0; j0 < n; j0 += 16) {
    float4 p[16];
#pragma unroll
    for (int u = 0; u < 16; ++u)
      if (j0 + u < n)
        p[u] = __ldcg(reinterpret_cast<const float4*>(
            part + (size_t)(first + (j0 + u) * stride) * R + r));
#pragma unroll
    for (int u = 0; u < 16; ++u)
      if (j0 + u < n) st = msi_merge(st, MSI{p[u].x, p[u].y, __float_as_int(p[u].z)});
  }
  return st;
}

// Two-level arrival of the tensor-core LM head's CTAs, after each wrote its
// partials.  CTAs come in teams of kLmTeam (by index); the last of a team to
// arrive merges the team's partials row by row, in CTA order, into the slot
// of the team's first CTA, and then arrives on the grid-wide ticket over the
// teams.  Returns true in exactly one CTA, the last team's merger, with every
// team's merged partial visible: it finishes with lm_final_merge(a, kLmTeam).
// The merges run one thread per row with all of a team's reads in flight, so
// the tail after the last CTA is two short merges instead of one over every
// CTA.  Each merger rearms its ticket.  No thread waits on another CTA.
template <class G = CtaThreads>
__device__ __forceinline__ bool lm_team_arrives(const LmArgs& a) {
  const int team = blockIdx.x / kLmTeam;
  const int first = team * kLmTeam;
  const int size = min(kLmTeam, a.n_cta - first);
  const int n_teams = (a.n_cta + kLmTeam - 1) / kLmTeam;
  unsigned int* team_ticket = &a.ctrl->lm_team[a.slot][team];
  unsigned int* ticket = &a.ctrl->lm_ticket[a.slot];
  if (!last_cta_arrives<G>(team_ticket, (unsigned int)size)) return false;
  if (G::rank() == 0) *team_ticket = 0u;
  for (int r = G::rank(); r < a.R; r += G::size()) {
    const MSI st = lm_merge_sources(a.part, a.R, r, first, 1, size);
    Partial p;
    p.m = st.m;
    p.s = st.s;
    p.i = st.i;
    p.pad = 0;
    a.part[(size_t)first * a.R + r] = p;  // read above by this thread only
  }
  if (!last_cta_arrives<G>(ticket, (unsigned int)n_teams)) return false;
  if (G::rank() == 0) *ticket = 0u;
  return true;
}

// Merge the partials of each row into (conf, tok); then, when the call is
// the fused step, commit (technical review, section 4, Algorithm 2).  The
// sources are part[(j * stride) * R + r] for the n_src = ceil(n_cta / stride)
// values of j: every CTA's own partials (stride 1), or the teams' merged
// ones (stride kLmTeam, after lm_team_arrives).
// conf = 1 / sum_v exp(l_v - l_max) is the max softmax probability; the
// token is the argmax with the lowest vocabulary index on a tie.
// If a CTA's bounded wait ran out (FDL_DEV_TIMEOUT in the status word, set
// before its ticket), its partials are stale: every row then reports
// conf = -1 and tok = -1 and the commit selects nothing (block tokens kept,
// counts written), until the caller reads and clears the status word.
template <class G = CtaThreads>
__device__ __forceinline__ void lm_final_merge(const LmArgs& a, int stride = 1) {
  __shared__ float s_conf[kMaxRows];
  __shared__ int s_tok[kMaxRows];
  const int warp = G::rank() >> 5, lane = threadIdx.x & 31;
  const int nw = G::size() >> 5;
  const int n_src = (a.n_cta + stride - 1) / stride;
  const bool timed_out =
      (*reinterpret_cast<volatile unsigned int*>(&a.ctrl->status) & FDL_DEV_TIMEOUT) != 0u;
  for (int r = G::rank(); r < a.R; r += G::size()) {
    const MSI st = lm_merge_sources(a.part, a.R, r, 0, stride, n_src);
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
  if (!a.commit) return;
  G::sync();
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
