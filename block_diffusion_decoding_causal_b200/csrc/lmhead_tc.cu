// LM head + confidence on the 5th-generation tensor cores (bf16, sm_100a).
//
// logits[v, r] = W[v, :] . X[r, :] over the full vocabulary, reduced on the
// chip to each row's running (max logit, sum exp(l - max), argmax)
// ("Fast-dLLM v2" Level 2: the greedy token and its probability; technical
// review, section 4, Algorithm 2).  Logits never reach global memory.
//
// Swap-AB: the weight is the M = 128 operand (a tile of 128 vocabulary rows),
// the <= 256 input rows are N.  Each CTA (one per SM) owns a contiguous
// vocabulary range of ~V/148 rows and streams it once:
//   warp 0   TMA producer: W tiles [128 x 64*KSUB] (KSUB boxes of 128-byte
//            swizzled rows, so each weight row is read 512 contiguous bytes at
//            a time; with the tiled weight layout each box is one contiguous
//            16 KB block) through an A ring, X chunks [N x 64*KSUB] through a
//            B ring;
//   warp 1   MMA issuer: tcgen05.mma kind::f16, accumulators in TMEM; tiles
//            are processed in groups of G, K-outer inside a group so each X
//            chunk is reused by G tiles; two TMEM buffers let the epilogue
//            of group g overlap the MMAs of group g+1 (at N = 256, one
//            buffer of two tiles instead: half the X traffic);
//   warps 2-5  epilogue: tcgen05.ld 32 lanes x 32 columns, a warp
//            reduce-scatter of (max, sum-exp, argmax) over the 32 vocab rows
//            leaves column j's triple in lane j, merged into a running state.
//            From N = 128 on, where the epilogue and not the weight stream
//            bounds the kernel, the 32 x 32 block is transposed through
//            shared memory instead and lane j folds column j's 32 logits into
//            its running state one at a time (one exponential per logit).
// The per-CTA triples go to the workspace; the last CTA of each team of 16
// merges its team's, the last team's merger merges the teams' (and, in the
// fused step, commits).  No thread waits on another CTA.
#include "lm_merge.cuh"
#include "sm100.cuh"

#include <cudaTypedefs.h>

#include <cstring>
#include <mutex>

namespace fdl {
namespace {

using namespace sm100;

constexpr int kTileM = 128;                 // vocab rows per MMA tile
constexpr int kKChunk = 64;                 // bf16 per 128-byte row
constexpr int kStageA = kTileM * kKChunk * 2;  // 16 KB
constexpr int kBoxPart = 16;                // rows per box of a partial tile
constexpr int kTail = 16;                   // short last tile of the CTA-pair form
constexpr int kThreads = 192;
constexpr unsigned kDevTimeout = FDL_DEV_TIMEOUT;

struct TcParams {
  int npad;        // MMA N: 32, 64, 128 or 256
  int ksub;        // 64-wide K boxes per pipeline stage
  int group;       // tiles per TMEM buffer
  int nbuf;        // TMEM buffers: 2 (epilogue overlaps the next group) or 1
  int stages_a;
  int stages_b;
  uint32_t tmem_cols;
};

constexpr int kTrStride = 33;  // transpose rows: 32 floats + 1 (no bank conflicts)
constexpr int kTrBytes = 4 * 32 * kTrStride * 4;  // one 32 x 33 buffer per epilogue warp

// Shared bytes of the epilogue's cross-warp region: the per-quarter states
// of every column, which from N = 128 on also hold the transpose buffers.
__host__ __device__ constexpr size_t red_bytes(int npad) {
  return npad >= 128 && (size_t)kTrBytes > 4 * (size_t)npad * sizeof(MSI)
             ? (size_t)kTrBytes : 4 * (size_t)npad * sizeof(MSI);
}

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// Fold one logit v of vocabulary entry idx into a running state; entries
// arrive in increasing idx, so an equal logit keeps the earlier index.  The
// larger of the two maxima scales the other side: one exponential.
__device__ __forceinline__ void msi_push(MSI& st, float v, int idx) {
  const float d = v - st.m;
  const bool up = d > 0.f;
  const float e = ex2_approx(-fabsf(d) * kLog2e);
  st.s = up ? fmaf(st.s, e, 1.f) : st.s + e;
  st.m = up ? v : st.m;
  st.i = up ? idx : st.i;
}

__device__ __forceinline__ void named_barrier_epilogue() {
  asm volatile("bar.sync 1, 128;" ::: "memory");
}

// Reduce-scatter of 32 columns over the 32 lanes of a warp: on return,
// lane j holds column j's (max, sum-exp, argmax) over all 32 lanes' rows.
__device__ __forceinline__ MSI reduce_scatter32(MSI (&s)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool upper = (lane & w) != 0;
#pragma unroll
    for (int j = 0; j < w; ++j) {
      const MSI keep = upper ? s[j + w] : s[j];
      const MSI send = upper ? s[j] : s[j + w];
      s[j] = msi_merge(keep, msi_shfl_xor(send, w));
    }
  }
  return s[0];
}

template <int NCH, int KSUB>
__global__ void __launch_bounds__(kThreads, 1)
lmhead_tc_kernel(const __grid_constant__ CUtensorMap tm_w_full,
                 const __grid_constant__ CUtensorMap tm_w_part,
                 const __grid_constant__ CUtensorMap tm_x, const LmArgs a,
                 const TcParams tp) {
  constexpr int NPAD = NCH * 32;
  constexpr int SA_BYTES = kStageA * KSUB;        // one A stage: 128 rows x 64*KSUB
  constexpr int SB_BYTES = NPAD * 128 * KSUB;     // one B stage: NPAD rows x 64*KSUB
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int SA = tp.stages_a, SB = tp.stages_b;
  uint8_t* sa = smem;
  uint8_t* sb = sa + SA * SA_BYTES;
  uint64_t* full_a = reinterpret_cast<uint64_t*>(sb + SB * SB_BYTES);
  uint64_t* empty_a = full_a + SA;
  uint64_t* full_b = empty_a + SA;
  uint64_t* empty_b = full_b + SB;
  uint64_t* acc_full = empty_b + SB;   // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint64_t* drain = acc_empty + 2;     // [1]
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 1);
  MSI* s_red = reinterpret_cast<MSI*>(tmem_holder + 4);  // [4][NPAD]

  // A kernel queued behind this one with programmatic serialisation (the
  // attention of the same step, which reads nothing this kernel writes) may
  // start on the SM room this CTA leaves.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int v0 = blockIdx.x * a.rows_per_cta;
  const int v1 = min(a.V, v0 + a.rows_per_cta);
  const int n_rows = max(0, v1 - v0);
  const int n_tiles = (n_rows + kTileM - 1) / kTileM;
  const int G = tp.group;
  const int n_groups = (n_tiles + G - 1) / G;
  const int KC = a.H / (kKChunk * KSUB);
  const int KCT = a.H / kKChunk;  // 64-wide chunks of one weight row

  if (threadIdx.x == 0) {
    for (int i = 0; i < SA; ++i) {
      mbar_init(&full_a[i], 1);
      mbar_init(&empty_a[i], 1);
    }
    for (int i = 0; i < SB; ++i) {
      mbar_init(&full_b[i], 1);
      mbar_init(&empty_b[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 128);
    }
    mbar_init(drain, 1);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc(tmem_holder, tp.tmem_cols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  bool failed = false;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tm_w_full);
      tma_prefetch_desc(&tm_w_part);
      tma_prefetch_desc(&tm_x);
      const uint64_t pol_w = policy_evict_first();
      int ia = 0, ib = 0;
      // The kernel before this one (the gather) finished, or the rows were
      // in place before that kernel began.
      bool x_ready = a.rows_ready != 0;
      auto load_x = [&](int kc) {
        if (!x_ready) {
          asm volatile("griddepcontrol.wait;" ::: "memory");
          x_ready = true;
        }
        const int slot_b = ib % SB;
        if (!mbar_wait(&empty_b[slot_b], ((ib / SB) & 1) ^ 1)) { failed = true; return; }
        mbar_arrive_expect_tx(&full_b[slot_b], SB_BYTES);
#pragma unroll
        for (int u = 0; u < KSUB; ++u)
          tma_load_2d(sb + slot_b * SB_BYTES + u * NPAD * 128, &tm_x,
                      (kc * KSUB + u) * kKChunk, 0, &full_b[slot_b]);
        ++ib;
      };
      for (int g = 0; g < n_groups && !failed; ++g) {
        const int t0 = g * G, t1 = min(n_tiles, t0 + G);
        for (int kc = 0; kc < KC && !failed; ++kc) {
          // The rows may come from the kernel launched just before this one
          // (the token-shift gather, programmatic launch): the first chunk's
          // weight tiles stream before waiting for it when they all fit in
          // the empty ring; later chunks load the rows first.
          const bool x_after = !x_ready && (t1 - t0) <= SA;
          if (!x_after) {
            load_x(kc);
            if (failed) break;
          }
          for (int t = t0; t < t1; ++t) {
            const int slot_a = ia % SA;
            if (!mbar_wait(&empty_a[slot_a], ((ia / SA) & 1) ^ 1)) { failed = true; break; }
            const int row0 = v0 + t * kTileM;
            const int rows = min(kTileM, v1 - row0);
            uint8_t* dst = sa + slot_a * SA_BYTES;
            if (rows == kTileM) {
              mbar_arrive_expect_tx(&full_a[slot_a], SA_BYTES);
#pragma unroll
              for (int u = 0; u < KSUB; ++u) {
                const int kk = kc * KSUB + u;
                if (a.w_packed)
                  tma_load_2d_hint(dst + u * kStageA, &tm_w_full, 0, row0 * KCT + kk * kTileM,
                                   &full_a[slot_a], pol_w);
                else
                  tma_load_2d_hint(dst + u * kStageA, &tm_w_full, kk * kKChunk, row0,
                                   &full_a[slot_a], pol_w);
              }
            } else {
              const int nbox = (rows + kBoxPart - 1) / kBoxPart;
              mbar_arrive_expect_tx(&full_a[slot_a], KSUB * nbox * kBoxPart * 128);
              for (int u = 0; u < KSUB; ++u) {
                const int kk = kc * KSUB + u;
                for (int j = 0; j < nbox; ++j) {
                  // Box rows past the tile's last row read neighbouring
                  // weight rows (or the zero fill past the end); the
                  // epilogue masks their logits.
                  if (a.w_packed)
                    tma_load_2d_hint(dst + u * kStageA + j * kBoxPart * 128, &tm_w_part, 0,
                                     row0 * KCT + kk * rows + j * kBoxPart, &full_a[slot_a],
                                     pol_w);
                  else
                    tma_load_2d_hint(dst + u * kStageA + j * kBoxPart * 128, &tm_w_part,
                                     kk * kKChunk, row0 + j * kBoxPart, &full_a[slot_a], pol_w);
                }
              }
            }
            ++ia;
          }
          if (x_after && !failed) load_x(kc);
        }
      }
      // Drain: every load issued has landed before this CTA can exit.
      for (int n = max(0, ia - SA); n < ia; ++n)
        if (!mbar_wait(&full_a[n % SA], (n / SA) & 1)) failed = true;
      for (int n = max(0, ib - SB); n < ib; ++n)
        if (!mbar_wait(&full_b[n % SB], (n / SB) & 1)) failed = true;
    }
  } else if (warp == 1) {
    // -------------------------------------------------------- MMA issuer
    if (lane == 0 && n_tiles > 0) {
      const uint32_t idesc = idesc_bf16_f32(kTileM, NPAD);
      int ia = 0, ib = 0;
      for (int g = 0; g < n_groups && !failed; ++g) {
        const int buf = tp.nbuf == 2 ? (g & 1) : 0;
        const uint32_t ph = tp.nbuf == 2 ? ((g >> 1) & 1) : (g & 1);
        if (!mbar_wait(&acc_empty[buf], ph ^ 1)) { failed = true; break; }
        tc_fence_after();
        const int t0 = g * G, t1 = min(n_tiles, t0 + G);
        for (int kc = 0; kc < KC && !failed; ++kc) {
          const int slot_b = ib % SB;
          if (!mbar_wait(&full_b[slot_b], (ib / SB) & 1)) { failed = true; break; }
          tc_fence_after();
          const uint32_t b_base = smem_u32(sb + slot_b * SB_BYTES);
          for (int t = t0; t < t1; ++t) {
            const int slot_a = ia % SA;
            if (!mbar_wait(&full_a[slot_a], (ia / SA) & 1)) { failed = true; break; }
            tc_fence_after();
            const uint32_t a_base = smem_u32(sa + slot_a * SA_BYTES);
            const uint32_t d = tmem + (uint32_t)((buf * G + (t - t0)) * NPAD);
#pragma unroll
            for (int u = 0; u < KSUB; ++u)
#pragma unroll
              for (int k = 0; k < kKChunk / 16; ++k)
                mma_bf16(d, desc_k_sw128(a_base + u * kStageA + k * 32),
                         desc_k_sw128(b_base + u * NPAD * 128 + k * 32), idesc,
                         (kc | u | k) != 0 ? 1u : 0u);
            mma_commit(&empty_a[slot_a]);
            ++ia;
          }
          mma_commit(&empty_b[slot_b]);
          ++ib;
        }
        mma_commit(&acc_full[buf]);
      }
      // Drain: all MMAs this thread issued have completed.
      mma_commit(drain);
      if (!mbar_wait(drain, 0)) failed = true;
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    float* tr = reinterpret_cast<float*>(s_red) + (warp - 2) * (32 * kTrStride);
    MSI st[NCH];
#pragma unroll
    for (int c = 0; c < NCH; ++c) st[c] = msi_empty();
    for (int g = 0; g < n_groups; ++g) {
      const int buf = tp.nbuf == 2 ? (g & 1) : 0;
      const uint32_t ph = tp.nbuf == 2 ? ((g >> 1) & 1) : (g & 1);
      if (!mbar_wait(&acc_full[buf], ph)) { failed = true; break; }
      tc_fence_after();
      const int t0 = g * G, t1 = min(n_tiles, t0 + G);
      for (int t = t0; t < t1; ++t) {
        const int vbase = v0 + t * kTileM + q * 32;
        const int vocab = vbase + lane;
        const bool valid = vocab < v1;
        const int n_valid = min(32, v1 - vbase);  // same for the whole warp
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) +
                                 (uint32_t)((buf * G + (t - t0)) * NPAD + c * 32),
                             r);
          tmem_ld_wait();
          if constexpr (NCH >= 4) {
            // Lane = vocabulary row in r; after the transpose lane j reads
            // column j, rows in increasing vocabulary order.
#pragma unroll
            for (int j = 0; j < 32; ++j) tr[lane * kTrStride + j] = __uint_as_float(r[j]);
            __syncwarp();
            MSI m = st[c];
            for (int k = 0; k < n_valid; ++k) msi_push(m, tr[k * kTrStride + lane], vbase + k);
            st[c] = m;
            __syncwarp();
          } else {
            MSI s[32];
#pragma unroll
            for (int j = 0; j < 32; ++j)
              s[j] = valid ? MSI{__uint_as_float(r[j]), 1.f, vocab} : msi_empty();
            st[c] = msi_merge(st[c], reduce_scatter32(s, lane));
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
    // From N = 128 on the transpose buffers share this region: every warp
    // is done with its buffer before the states are written.
    if constexpr (NCH >= 4) named_barrier_epilogue();
#pragma unroll
    for (int c = 0; c < NCH; ++c) s_red[q * NPAD + c * 32 + lane] = st[c];
    named_barrier_epilogue();
    for (int col = threadIdx.x - 64; col < NPAD; col += 128) {
      MSI m = s_red[col];
#pragma unroll
      for (int j = 1; j < 4; ++j) m = msi_merge(m, s_red[j * NPAD + col]);
      if (col < a.R) {
        Partial p;
        p.m = m.m;
        p.s = m.s;
        p.i = m.i;
        p.pad = 0;
        a.part[(size_t)blockIdx.x * a.R + col] = p;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, tp.tmem_cols);
  }
  if (failed) atomicOr(&a.ctrl->status, kDevTimeout);
  if (!lm_team_arrives(a)) return;
  lm_final_merge(a, kLmTeam);
}

// The LM head over CTA pairs (from 129 rows on, full form).  The two CTAs of
// a cluster keep their own vocabulary ranges and tiles, and each stages its
// own weight tile, but they share every X chunk: CTA r stages rows
// [r N/2, (r+1) N/2) of it, and the even CTA issues tcgen05.mma.cta_group::2
// (M = 256: its tile over the odd CTA's tile), whose result lands in each
// CTA's own TMEM.  Per SM that halves the X bytes, which past 64 rows are
// what the shared-memory stream carries besides the weight.  Weight tiles
// are always loaded as full 128-row boxes (rows past a range are masked in
// the epilogue, rows past the tensor read zeros), so the two CTAs expect the
// same bytes at every step.  Barriers:
//   full_a / full_b   on the even CTA only: the even CTA arms them for both
//                     CTAs' bytes, both CTAs' loads complete on them;
//   empty_a / empty_b in each CTA: the MMA commits to both;
//   acc_full          in each CTA: the MMA commits to both;
//   acc_empty         on the even CTA: both CTAs' epilogue threads arrive.
// Short last tile.  A range of 128 k + t rows with 0 < t <= kTail (t = 16
// at the Qwen2.5 vocabulary over 148 CTAs) would spend a whole M = 256 tile
// of MMAs on t rows.  Instead the t rows of each CTA ride along with the
// first tile with the operands swapped: A = the X chunk already staged (this
// CTA's 128 X rows), B = the two CTAs' t-row weight pieces (kTail rows each,
// N = 2 kTail), D in the first 2 kTail columns of the second TMEM buffer,
// which the first tile leaves free.  Lane = X row there, so the epilogue
// folds those 2 kTail vocabulary entries into its own X rows' states, the
// even CTA's entries before the odd CTA's; every (X row, vocabulary row)
// pair is still counted once.  The MMA waits for those columns (tail_empty)
// before the second tile.
// Two passes in one launch (ps.n == 2: 257..512 rows as two groups of whole
// sequences): the producer and the MMA go on from the first pass's last tile
// to the second pass's first, with one count of TMEM buffers across both,
// while the epilogue warps write the first pass's partials and run its
// merges (its own ticket set) by themselves.  The last tile's epilogue and
// the two merges of the first pass, about 25 us, then hide under the second
// pass's MMAs, and one launch gap goes.
struct XMaps {
  CUtensorMap m[2];  // the X rows of each pass
};
struct LmPasses {
  LmArgs p[2];  // outputs, partials and ticket set of each pass
  int n;        // 1 or 2
};
template <int NCH, int KSUB>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
lmhead_tc2_kernel(const __grid_constant__ CUtensorMap tm_w_full,
                  const __grid_constant__ CUtensorMap tm_w_tail,
                  const __grid_constant__ XMaps tm_x, const __grid_constant__ LmPasses ps,
                  const TcParams tp) {
  const LmArgs& a = ps.p[0];  // vocabulary, weight and control: the same in every pass
  constexpr int NPAD = NCH * 32;
  constexpr int NH = NPAD / 2;                    // X rows this CTA stages
  constexpr int SA_BYTES = kStageA * KSUB;        // one A stage: 128 rows x 64*KSUB
  constexpr int TAIL_BYTES = kTail * 128 * KSUB;  // short-tile rows of one A stage
  constexpr int SA_STRIDE = SA_BYTES + TAIL_BYTES;
  constexpr int SB_BYTES = NH * 128 * KSUB;       // one B stage: NH rows x 64*KSUB
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const int SA = tp.stages_a, SB = tp.stages_b;
  uint8_t* sa = smem;
  uint8_t* sb = sa + SA * SA_STRIDE;
  uint64_t* full_a = reinterpret_cast<uint64_t*>(sb + SB * SB_BYTES);
  uint64_t* empty_a = full_a + SA;
  uint64_t* full_b = empty_a + SA;
  uint64_t* empty_b = full_b + SB;
  uint64_t* acc_full = empty_b + SB;   // [2]
  uint64_t* acc_empty = acc_full + 2;  // [2]
  uint64_t* drain = acc_empty + 2;     // [1]
  uint64_t* tail_empty = drain + 1;    // [1]
  uint64_t* tail_free = tail_empty + 1;  // [1] next pass's short-tile columns read out
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tail_free + 1);
  MSI* s_red = reinterpret_cast<MSI*>(tmem_holder + 4);  // [4][NPAD], then [NH] short tile
  static_assert((4 * NPAD + NH) * sizeof(MSI) <= red_bytes(NPAD), "epilogue states fit");

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int v0 = blockIdx.x * a.rows_per_cta;
  const int v1 = min(a.V, v0 + a.rows_per_cta);
  // The pair steps through the same number of tiles: the larger range's.
  const int pair0 = (blockIdx.x & ~1) * a.rows_per_cta;
  const int pair_rows = max(0, min(a.V, pair0 + a.rows_per_cta) - pair0);
  // Short last tile folded into the first one (same decision in both CTAs).
  const int t_rows = pair_rows % kTileM;
  const bool fold = pair_rows > kTileM && t_rows > 0 && t_rows <= kTail;
  const int n_tiles = fold ? pair_rows / kTileM : (pair_rows + kTileM - 1) / kTileM;
  const int G = tp.group;
  const int n_groups = (n_tiles + G - 1) / G;
  const int KC = a.H / (kKChunk * KSUB);
  const int KCT = a.H / kKChunk;

  if (threadIdx.x == 0) {
    for (int i = 0; i < SA; ++i) {
      mbar_init(&full_a[i], 1);
      mbar_init(&empty_a[i], 1);
    }
    for (int i = 0; i < SB; ++i) {
      mbar_init(&full_b[i], 1);
      mbar_init(&empty_b[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 256);
    }
    mbar_init(drain, 1);
    mbar_init(tail_empty, 256);
    mbar_init(tail_free, 256);
    fence_barrier_init();
  }
  if (warp == 1) tmem_alloc_pair(tmem_holder, tp.tmem_cols);
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers exist before either signals the other
  tc_fence_after();
  const uint32_t tmem = *tmem_holder;
  bool failed = false;

  if (warp == 0) {
    // ------------------------------------------------------ TMA producer
    if (lane == 0 && n_tiles > 0) {
      tma_prefetch_desc(&tm_w_full);
      tma_prefetch_desc(&tm_w_tail);
      for (int pass = 0; pass < ps.n; ++pass) tma_prefetch_desc(&tm_x.m[pass]);
      const uint64_t pol_w = policy_evict_first();
      const uint64_t pol_x = policy_evict_last();
      // The rows may come from the kernel launched just before this one (the
      // token-shift gather, programmatic launch); without one this returns.
      if (!a.rows_ready) asm volatile("griddepcontrol.wait;" ::: "memory");
      int ia = 0, ib = 0;
      for (int pass = 0; pass < ps.n && !failed; ++pass) {
      const CUtensorMap* xm = &tm_x.m[pass];
      for (int g = 0; g < n_groups && !failed; ++g) {
        const int t0 = g * G, t1 = min(n_tiles, t0 + G);
        for (int kc = 0; kc < KC && !failed; ++kc) {
          {
            const int slot_b = ib % SB;
            if (!mbar_wait(&empty_b[slot_b], ((ib / SB) & 1) ^ 1)) { failed = true; break; }
            if (leader) mbar_arrive_expect_tx(&full_b[slot_b], 2 * SB_BYTES);
            const uint32_t bar = mapa_shared(smem_u32(&full_b[slot_b]), 0u);
#pragma unroll
            for (int u = 0; u < KSUB; ++u)
              tma_load_2d_pair(sb + slot_b * SB_BYTES + u * NH * 128, xm,
                               (kc * KSUB + u) * kKChunk, (int)rank * NH, bar, pol_x);
            ++ib;
          }
          for (int t = t0; t < t1; ++t) {
            const int slot_a = ia % SA;
            const bool with_tail = fold && t == 0;
            if (!mbar_wait(&empty_a[slot_a], ((ia / SA) & 1) ^ 1)) { failed = true; break; }
            if (leader)
              mbar_arrive_expect_tx(&full_a[slot_a],
                                    2 * (SA_BYTES + (with_tail ? TAIL_BYTES : 0)));
            const uint32_t bar = mapa_shared(smem_u32(&full_a[slot_a]), 0u);
            const int row0 = v0 + t * kTileM;
            const int rt = max(0, min(kTileM, v1 - row0));  // rows of the tile (packed layout)
            uint8_t* dst = sa + slot_a * SA_STRIDE;
            if (with_tail) {
              // This CTA's short-tile rows (a full kTail box; rows past its
              // range read the next chunk's pieces or zeros, masked later).
              const int trow0 = v0 + n_tiles * kTileM;
              const int trt = max(0, min(kTileM, v1 - trow0));
#pragma unroll
              for (int u = 0; u < KSUB; ++u) {
                const int kk = kc * KSUB + u;
                if (a.w_packed)
                  tma_load_2d_pair(dst + SA_BYTES + u * kTail * 128, &tm_w_tail, 0,
                                   trow0 * KCT + kk * trt, bar, pol_w);
                else
                  tma_load_2d_pair(dst + SA_BYTES + u * kTail * 128, &tm_w_tail, kk * kKChunk,
                                   trow0, bar, pol_w);
              }
            }
#pragma unroll
            for (int u = 0; u < KSUB; ++u) {
              const int kk = kc * KSUB + u;
              if (a.w_packed)
                tma_load_2d_pair(dst + u * kStageA, &tm_w_full, 0, row0 * KCT + kk * rt, bar,
                                 pol_w);
              else
                tma_load_2d_pair(dst + u * kStageA, &tm_w_full, kk * kKChunk, row0, bar, pol_w);
            }
            ++ia;
          }
        }
      }
      }
      // Drain: every load of this CTA has landed before it can exit (the
      // even CTA's full barriers count both CTAs' bytes; the odd CTA waits
      // on its empty barriers, which the MMA releases only after the loads
      // they followed).
      if (leader) {
        for (int n = max(0, ia - SA); n < ia; ++n)
          if (!mbar_wait(&full_a[n % SA], (n / SA) & 1)) failed = true;
        for (int n = max(0, ib - SB); n < ib; ++n)
          if (!mbar_wait(&full_b[n % SB], (n / SB) & 1)) failed = true;
      } else {
        for (int n = max(0, ia - SA); n < ia; ++n)
          if (!mbar_wait(&empty_a[n % SA], (n / SA) & 1)) failed = true;
        for (int n = max(0, ib - SB); n < ib; ++n)
          if (!mbar_wait(&empty_b[n % SB], (n / SB) & 1)) failed = true;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------- MMA issuer (even CTA)
    if (leader && lane == 0 && n_tiles > 0) {
      const uint32_t idesc = idesc_bf16_f32(2 * kTileM, NPAD);
      const uint32_t idesc_tail = idesc_bf16_f32(2 * kTileM, 2 * kTail);
      int ia = 0, ib = 0;
      int gg = 0;                        // groups over all passes: TMEM buffer gg & 1
      int tail_buf = -1, tail_pass = 0;  // short-tile columns the epilogue still reads
      for (int pass = 0; pass < ps.n && !failed; ++pass) {
      for (int g = 0; g < n_groups && !failed; ++g, ++gg) {
        const int buf = gg & 1;
        const uint32_t ph = (gg >> 1) & 1;
        if (!mbar_wait(&acc_empty[buf], ph ^ 1)) { failed = true; break; }
        if (buf == tail_buf) {
          if (!mbar_wait(tail_empty, (uint32_t)(tail_pass & 1))) { failed = true; break; }
          tail_buf = -1;
        }
        const int tb = buf ^ 1;  // the short tile's columns: the start of the other buffer
        if (fold && g == 0) {
          // After the first pass that buffer holds the previous pass's last
          // tile: the epilogue reads its first 32 columns first and says so.
          if (pass > 0 && !mbar_wait(tail_free, (uint32_t)((pass - 1) & 1))) { failed = true; break; }
          tail_buf = tb;
          tail_pass = pass;
        }
        tc_fence_after();
        const int t0 = g * G, t1 = min(n_tiles, t0 + G);
        for (int kc = 0; kc < KC && !failed; ++kc) {
          const int slot_b = ib % SB;
          if (!mbar_wait(&full_b[slot_b], (ib / SB) & 1)) { failed = true; break; }
          tc_fence_after();
          const uint32_t b_base = smem_u32(sb + slot_b * SB_BYTES);
          for (int t = t0; t < t1; ++t) {
            const int slot_a = ia % SA;
            if (!mbar_wait(&full_a[slot_a], (ia / SA) & 1)) { failed = true; break; }
            tc_fence_after();
            const uint32_t a_base = smem_u32(sa + slot_a * SA_STRIDE);
            const uint32_t d = tmem + (uint32_t)((buf * G + (t - t0)) * NPAD);
            if (fold && t == 0) {
              // Short tile, operands swapped: X rows x (kTail + kTail) rows.
#pragma unroll
              for (int u = 0; u < KSUB; ++u)
#pragma unroll
                for (int k = 0; k < kKChunk / 16; ++k)
                  mma_bf16_pair(tmem + (uint32_t)(tb * NPAD),
                                desc_k_sw128(b_base + u * NH * 128 + k * 32),
                                desc_k_sw128(a_base + SA_BYTES + u * kTail * 128 + k * 32),
                                idesc_tail, (kc | u | k) != 0 ? 1u : 0u);
            }
#pragma unroll
            for (int u = 0; u < KSUB; ++u)
#pragma unroll
              for (int k = 0; k < kKChunk / 16; ++k)
                mma_bf16_pair(d, desc_k_sw128(a_base + u * kStageA + k * 32),
                              desc_k_sw128(b_base + u * NH * 128 + k * 32), idesc,
                              (kc | u | k) != 0 ? 1u : 0u);
            mma_commit_pair(&empty_a[slot_a]);
            ++ia;
          }
          mma_commit_pair(&empty_b[slot_b]);
          ++ib;
        }
        mma_commit_pair(&acc_full[buf]);
      }
      }
      mma_commit_pair_local(drain);
      if (!mbar_wait(drain, 0)) failed = true;
    }
  } else {
    // ---------------------------------------------------------- epilogue
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    float* tr = reinterpret_cast<float*>(s_red) + (warp - 2) * (32 * kTrStride);
    const uint32_t acc_empty_lead0 = mapa_shared(smem_u32(&acc_empty[0]), 0u);
    const uint32_t acc_empty_lead1 = mapa_shared(smem_u32(&acc_empty[1]), 0u);
    const uint32_t tail_free_lead = mapa_shared(smem_u32(tail_free), 0u);
    int gg = 0;
    for (int pass = 0; pass < ps.n; ++pass) {
    const LmArgs& ap = ps.p[pass];
    MSI st[NCH];
#pragma unroll
    for (int c = 0; c < NCH; ++c) st[c] = msi_empty();
    MSI st_tail = msi_empty();  // X row rank * NH + q * 32 + lane, short-tile entries
    for (int g = 0; g < n_groups && !failed; ++g, ++gg) {
      const int buf = gg & 1;
      const uint32_t ph = (gg >> 1) & 1;
      if (!mbar_wait(&acc_full[buf], ph)) { failed = true; break; }
      tc_fence_after();
      if (fold && g == 0) {
        // Columns j < kTail: the even CTA's short-tile rows, j >= kTail the
        // odd CTA's, each in increasing vocabulary order.
        uint32_t r[32];
        static_assert(2 * kTail == 32, "one 32-column load holds the short tile");
        tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)((buf ^ 1) * NPAD), r);
        tmem_ld_wait();
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int c0 = (blockIdx.x & ~1) + h;
          const int tv0 = c0 * a.rows_per_cta + n_tiles * kTileM;
          const int tv1 = min(a.V, c0 * a.rows_per_cta + a.rows_per_cta);
#pragma unroll
          for (int j = 0; j < kTail; ++j)
            if (tv0 + j < tv1) msi_push(st_tail, __uint_as_float(r[h * kTail + j]), tv0 + j);
        }
        tc_fence_before();
        mbar_arrive_cluster(mapa_shared(smem_u32(tail_empty), 0u));
      }
      const int t0 = g * G, t1 = min(n_tiles, t0 + G);
      // The last group of a pass before a folding one: its first 32 columns
      // are the next pass's short-tile columns.
      const bool free_head = fold && g == n_groups - 1 && pass + 1 < ps.n;
      for (int t = t0; t < t1; ++t) {
        const int vbase = v0 + t * kTileM + q * 32;
        const int n_valid = min(32, v1 - vbase);  // same for the whole warp; may be <= 0
#pragma unroll
        for (int c = 0; c < NCH; ++c) {
          uint32_t r[32];
          tmem_ld_32x32b_x32(tmem + ((uint32_t)(q * 32) << 16) +
                                 (uint32_t)((buf * G + (t - t0)) * NPAD + c * 32),
                             r);
          tmem_ld_wait();
          if (c == 0 && free_head) {
            tc_fence_before();
            mbar_arrive_cluster(tail_free_lead);
          }
          // Lane = vocabulary row in r; after the transpose lane j reads
          // column j, rows in increasing vocabulary order.
#pragma unroll
          for (int j = 0; j < 32; ++j) tr[lane * kTrStride + j] = __uint_as_float(r[j]);
          __syncwarp();
          MSI m = st[c];
          for (int k = 0; k < n_valid; ++k) msi_push(m, tr[k * kTrStride + lane], vbase + k);
          st[c] = m;
          __syncwarp();
        }
      }
      tc_fence_before();
      mbar_arrive_cluster(buf == 0 ? acc_empty_lead0 : acc_empty_lead1);
    }
    named_barrier_epilogue();
#pragma unroll
    for (int c = 0; c < NCH; ++c) s_red[q * NPAD + c * 32 + lane] = st[c];
    MSI* s_tail = s_red + 4 * NPAD;  // [NH], this CTA's X rows
    s_tail[q * 32 + lane] = st_tail;
    named_barrier_epilogue();
    for (int col = threadIdx.x - 64; col < NPAD; col += 128) {
      MSI m = s_red[col];
#pragma unroll
      for (int j = 1; j < 4; ++j) m = msi_merge(m, s_red[j * NPAD + col]);
      const int xl = col - (int)rank * NH;
      if (xl >= 0 && xl < NH) m = msi_merge(m, s_tail[xl]);
      if (col < ap.R) {
        Partial p;
        p.m = m.m;
        p.s = m.s;
        p.i = m.i;
        p.pad = 0;
        ap.part[(size_t)blockIdx.x * ap.R + col] = p;
      }
    }
    // A pass before the last merges now, by the four epilogue warps alone
    // while the others stream the next pass (their barriers also keep the
    // transpose buffers, which share s_red, from being rewritten before
    // every warp has read it); the last pass merges below with every
    // thread.  Every CTA arrives on every pass, failed or not, so the
    // tickets always complete and rearm.
    if (pass + 1 < ps.n) {
      if (failed) atomicOr(&a.ctrl->status, kDevTimeout);
      if (lm_team_arrives<EpilogueThreads>(ap)) lm_final_merge<EpilogueThreads>(ap, kLmTeam);
    }
    }
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while the pair's MMAs or arrivals may touch it
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, tp.tmem_cols);
  }
  if (failed) atomicOr(&a.ctrl->status, kDevTimeout);
  if (!lm_team_arrives(ps.p[ps.n - 1])) return;
  lm_final_merge(ps.p[ps.n - 1], kLmTeam);
}

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// 2D bf16 tensor map [outer, inner] (inner contiguous), 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
              uint32_t box_inner, uint32_t box_outer, CUtensorMapL2promotion promo) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides,
            box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, promo,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Tiled weight layout.  The vocabulary is cut into the CTA ranges of the LM
// head (per rows each) and each range into tiles of up to 128 rows; tile
// (first row row0, rt rows) occupies rt * KCT consecutive 128-byte rows
// starting at row0 * KCT, chunk kk's rt rows (columns 64 kk .. 64 kk + 63 of
// every row of the tile) at row0 * KCT + kk * rt.  A weight row's 128-byte
// piece (v, kk) thus moves from v * KCT + kk to the row computed here.
// One thread per 16 bytes; reads are coalesced, writes 128 bytes per eight
// threads.
__global__ void pack_weight_kernel(const uint4* __restrict__ w, uint4* __restrict__ out,
                                   int V, int KCT, int per) {
  const long n = (long)V * KCT * 8;
  for (long i = blockIdx.x * (long)blockDim.x + threadIdx.x; i < n;
       i += (long)gridDim.x * blockDim.x) {
    const long seg = i >> 3;
    const int v = (int)(seg / KCT), kk = (int)(seg % KCT);
    const int v_lo = v / per * per;
    const int v_hi = min(V, v_lo + per);
    const int row0 = v_lo + (v - v_lo) / kTileM * kTileM;
    const int rt = min(kTileM, v_hi - row0);
    out[((long)row0 * KCT + (long)kk * rt + (v - row0)) * 8 + (i & 7)] = w[i];
  }
}

template <int NCH, int KSUB>
cudaError_t launch_nch(const CUtensorMap& wf, const CUtensorMap& wp, const CUtensorMap& x,
                       const LmArgs& a, const TcParams& tp, size_t smem, cudaStream_t s,
                       bool after_producer) {
  auto k = lmhead_tc_kernel<NCH, KSUB>;
  // Opened up once per device and size: the driver calls cost more than the
  // launch itself.
  static std::mutex mu;
  static size_t smem_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (smem_set[dev] < smem) {
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      // The whole unified L1/shared array as shared memory, so an SM running
      // one of these CTAs still has room for an attention CTA of the same step.
      e = cudaFuncSetAttribute(k, cudaFuncAttributePreferredSharedMemoryCarveout,
                               cudaSharedmemCarveoutMaxShared);
      if (e != cudaSuccess) return e;
      smem_set[dev] = smem;
    }
  }
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(a.n_cta, 1, 1);
  lc.blockDim = dim3(kThreads, 1, 1);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = after_producer ? 1 : 0;
  return cudaLaunchKernelEx(&lc, k, wf, wp, x, a, tp);
}

template <int NCH, int KSUB>
cudaError_t launch_pair(const CUtensorMap& wf, const CUtensorMap& wt, const XMaps& x,
                        const LmPasses& ps, const TcParams& tp, size_t smem, cudaStream_t s,
                        bool after_producer) {
  const LmArgs& a = ps.p[0];
  auto k = lmhead_tc2_kernel<NCH, KSUB>;
  static std::mutex mu;
  static size_t smem_set[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (smem_set[dev] < smem) {
      e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
      smem_set[dev] = smem;
    }
  }
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3(a.n_cta, 1, 1);  // even: whole pairs
  lc.blockDim = dim3(kThreads, 1, 1);
  lc.dynamicSmemBytes = smem;
  lc.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  lc.attrs = attr;
  lc.numAttrs = after_producer ? 1 : 0;
  return cudaLaunchKernelEx(&lc, k, wf, wt, x, ps, tp);
}

// Ring shapes of the CTA-pair form (256 padded rows, full form): two-box K
// stages (32 KB weight stages, each with room for the short tile's 2 x 2 KB;
// X stages of half the rows), one tile per TMEM buffer, two buffers, about
// 204 KB of rings.  With the short tile folded into the first one the 7B
// vocabulary takes eight tiles per CTA instead of nine: 287 -> 275 us a pass
// at 256 rows on one box.  (Other shapes measured at 256 rows, before the
// fold: 3 + 3 stages 327 us; 4 weight + 2 X stages 350 us; 4 + 3 stages with
// the epilogue reducing in registers to make room, no faster than 3 + 3;
// two tiles per buffer sharing each X chunk 334 us; a single X stage
// 490-560 us.)
bool lmhead_tc2_params(int npad, int H, TcParams* tp, size_t* smem) {
  if (npad != 256) return false;
  if ((H / kKChunk) % 2 != 0) return false;
  tp->npad = npad;
  tp->ksub = 2;
  tp->nbuf = 2;
  tp->group = 1;
  tp->tmem_cols = 512;
  const size_t a_stage = (size_t)kStageA * 2 + (size_t)kTail * 128 * 2;  // + short-tile rows
  const size_t b_stage = (size_t)(npad / 2) * 128 * 2;
  tp->stages_b = 3;
  tp->stages_a = 3;
  const size_t bars = 8 * (size_t)(2 * tp->stages_a + 2 * tp->stages_b + 7) + 16;
  *smem = 1024 + (size_t)tp->stages_a * a_stage + (size_t)tp->stages_b * b_stage + bars +
          red_bytes(npad);
  // Dynamic plus static (the row scratch of the two final-merge forms, all
  // threads and epilogue warps only) within 227 KB.
  return *smem + 2 * kMaxRows * 8 + 64 <= 227 * 1024;
}

}  // namespace

// Tiles per CTA, group size, ring depths and TMEM columns for a call.
//
// Shared mode (beside_smem > 0): the CTA leaves room on its SM for one
// attention CTA of the same step that needs beside_smem bytes of shared
// memory, 256 TMEM columns and 192 threads of 168 registers, so the two
// kernels stream HBM side by side.  Its shared memory is what is left of
// the SM's 228 KB after that CTA and the two per-CTA reservations, and must
// exceed half the SM (so two LM-head CTAs never share one); TMEM stays within
// 256 columns and registers within 168 per thread (R <= 64: at 128 rows the
// attention beside the LM head cost more than running it before, 339 against
// 270 us a batch-16 step at prefix 2048).  The widest K stage (4, 2 or 1
// boxes of 64) that still fits two weight stages is taken.
bool lmhead_tc_params(int R, int H, int rows_per_cta, size_t beside_smem, TcParams* tp,
                      size_t* smem);

namespace {
constexpr size_t kSmPerSM = 228 * 1024;  // unified shared memory of one SM
constexpr size_t kSmReserve = 1024;      // reserved by the system per CTA
}  // namespace

bool lmhead_tc_params(int R, int H, int rows_per_cta, size_t beside_smem, TcParams* tp,
                      size_t* smem) {
  const bool shared = beside_smem > 0;
  int nch = 1;
  while (nch * 32 < R) nch *= 2;
  if (nch > (shared ? 2 : 8)) return false;
  tp->npad = nch * 32;
  // Tiles per TMEM buffer: about half a CTA's range, so each X chunk serves
  // several weight tiles and the epilogue of one group hides under the next
  // group's stream (both buffers together stay within TMEM's 512 columns, or
  // 256 when shared, in groups of equal size).
  const int n_tiles = (rows_per_cta + kTileM - 1) / kTileM;
  int G = (n_tiles + 1) / 2;
  const int gmax = (shared ? 128 : 256) / tp->npad;
  if (G > gmax) {
    const int n_groups = (n_tiles + gmax - 1) / gmax;
    G = (n_tiles + n_groups - 1) / n_groups;
  }
  if (G < 1) G = 1;
  tp->nbuf = 2;
  // N = 256 (full form): one tile per TMEM buffer, two buffers (so the
  // epilogue of one tile overlaps the next tile's MMAs), and two-box K
  // stages: 64 KB X chunks and 32 KB weight stages, two of each.  Measured
  // at the Qwen2.5-7B vocabulary, 256 rows: 348 us, against 385 us for one
  // buffer of two tiles sharing each 32 KB X chunk with 16 KB weight stages
  // (wide stages cost fewer barrier round trips than the shared X saves).
  if (!shared && tp->npad == 256 && (H / kKChunk) % 2 == 0) {
    tp->group = 1;
    tp->nbuf = 2;
    tp->tmem_cols = 512;
    tp->ksub = 2;
    tp->stages_b = 2;
    tp->stages_a = 2;
    const size_t a_stage = (size_t)kStageA * 2, b_stage = (size_t)256 * 128 * 2;
    const size_t bars = 8 * (size_t)(2 * 2 + 2 * 2 + 5) + 16;
    *smem = 1024 + 2 * a_stage + 2 * b_stage + bars + red_bytes(256);
    return *smem <= 227 * 1024;
  }
  if (!shared && tp->npad == 256 && n_tiles > 1) {
    G = 2;
    tp->nbuf = 1;
  }
  tp->group = G;
  const int col_limit = shared ? 256 : 512;
  if (tp->nbuf * tp->group * tp->npad > col_limit) return false;
  uint32_t cols = 32;
  while (cols < (uint32_t)(tp->nbuf * tp->group * tp->npad)) cols *= 2;
  tp->tmem_cols = cols;
  // Shared memory: the full form keeps 200 KB of rings; the shared form
  // what the SM has left.
  const size_t cap = shared ? (beside_smem + 2 * kSmReserve < kSmPerSM
                                   ? kSmPerSM - beside_smem - 2 * kSmReserve : 0)
                            : 227 * 1024;
  const int kchunks = H / kKChunk;
  for (int ksub = 4; ksub >= 1; ksub >>= 1) {
    if (kchunks % ksub != 0) continue;
    const size_t b_stage = (size_t)tp->npad * 128 * ksub;
    if (b_stage > 32768 && ksub > 1) continue;  // X stage within 32 KB when possible
    const size_t a_stage = (size_t)kStageA * ksub;
    // Stages as wide as the X chunk allows: every stage costs a barrier round
    // trip between the TMA, MMA and (for X) epilogue-paced threads, and at
    // 128 rows 32 KB stages stream the weight 1.36x faster than 16 KB ones
    // (310 -> 228 us at the Qwen2.5-7B vocabulary).  Four X stages of up to
    // 16 KB in the full form, two of 32 KB (two when shared).
    int sb = shared ? 2 : (b_stage > 16384 ? 2 : 4);
    int sa = 0;
    if (tp->nbuf == 1) {
      // Balanced rings: as many K steps in flight for the X chunks as for
      // the G weight boxes that use each one.
      const size_t per_step = b_stage + (size_t)G * a_stage;
      int n = (int)((200 * 1024) / per_step);
      if (n * G > 12) n = 12 / G;
      if (n < 2) continue;
      sb = n;
      sa = n * G;
    } else {
      const size_t fixed = 1024 + 8 * (size_t)(2 * 12 + 2 * sb + 5) + 16 + red_bytes(tp->npad);
      const size_t ring_cap = shared ? cap : fixed + 200 * 1024;
      if (ring_cap < fixed + (size_t)sb * b_stage + 2 * a_stage) continue;
      sa = (int)((ring_cap - fixed - (size_t)sb * b_stage) / a_stage);
      if (sa > 12) sa = 12;
    }
    const size_t b_bytes = (size_t)sb * b_stage;
    tp->ksub = ksub;
    tp->stages_b = sb;
    tp->stages_a = sa;
    const size_t bars = 8 * (size_t)(2 * sa + 2 * sb + 5) + 16;
    *smem = 1024 + (size_t)sa * a_stage + b_bytes + bars + red_bytes(tp->npad);
    if (shared && 2 * (*smem + kSmReserve) <= kSmPerSM) *smem = kSmPerSM / 2;  // one per SM
    if (*smem > cap) return false;
    return true;
  }
  return false;
}

bool lmhead_tc_shared_ok(const LmArgs& a, size_t beside_smem) {
  TcParams tp;
  size_t smem = 0;
  return lmhead_tc_params(a.R, a.H, a.rows_per_cta, beside_smem, &tp, &smem);
}

// The CTA-pair form over ps.n passes (the tensor maps of the weight, its
// short tiles and each pass's rows; whole pairs of CTAs, a spare CTA
// reporting an empty range).
static cudaError_t launch_pair_passes(LmPasses ps, const TcParams& tp, size_t smem,
                                      cudaStream_t s, bool after_producer) {
  const LmArgs& a = ps.p[0];
  CUtensorMap wf, wt;
  XMaps x;
  memset(&x, 0, sizeof(x));
  const uint64_t w_inner = a.w_packed ? kKChunk : a.H;
  const uint64_t w_outer = a.w_packed ? (uint64_t)a.V * (a.H / kKChunk) : a.V;
  if (!make_map(&wf, a.w, w_inner, w_outer, kKChunk, kTileM, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
      !make_map(&wt, a.w, w_inner, w_outer, kKChunk, kTail, CU_TENSOR_MAP_L2_PROMOTION_L2_256B))
    return cudaErrorInvalidValue;
  for (int i = 0; i < ps.n; ++i) {
    if (!make_map(&x.m[i], ps.p[i].rows, a.H, ps.p[i].R, kKChunk, tp.npad / 2,
                  CU_TENSOR_MAP_L2_PROMOTION_L2_128B))
      return cudaErrorInvalidValue;
    ps.p[i].n_cta = (a.n_cta + 1) & ~1;
  }
  return launch_pair<8, 2>(wf, wt, x, ps, tp, smem, s, after_producer);
}

bool lmhead_tc_two_pass_ok(const LmArgs& a, const LmArgs& b) {
  TcParams tp;
  size_t smem = 0;
  return a.R > 128 && a.R <= 256 && b.R > 128 && b.R <= 256 && a.H == b.H && a.V == b.V &&
         a.w == b.w && a.n_cta == b.n_cta && a.rows_per_cta == b.rows_per_cta &&
         a.w_packed == b.w_packed && a.ctrl == b.ctrl && a.part != b.part &&
         a.n_cta <= kLmTeam * kLmMaxTeams && lmhead_tc2_params(256, a.H, &tp, &smem);
}

cudaError_t launch_lmhead_tc_two_pass(const LmArgs& a, const LmArgs& b, cudaStream_t s,
                                      bool after_producer) {
  TcParams tp;
  size_t smem = 0;
  if (!lmhead_tc_two_pass_ok(a, b) || !lmhead_tc2_params(256, a.H, &tp, &smem))
    return cudaErrorInvalidValue;
  LmPasses ps;
  memset(&ps, 0, sizeof(ps));
  ps.p[0] = a;
  ps.p[0].slot = 0;
  ps.p[1] = b;
  ps.p[1].slot = 1;
  ps.p[1].rows_ready = a.rows_ready;
  ps.n = 2;
  return launch_pair_passes(ps, tp, smem, s, after_producer);
}

cudaError_t launch_lmhead_tc(const LmArgs& a, cudaStream_t s, size_t beside_smem,
                             bool after_producer) {
  TcParams tp;
  size_t smem = 0;
  if (a.n_cta > kLmTeam * kLmMaxTeams) return cudaErrorInvalidValue;  // team tickets
  // From 129 rows on (full form): CTA pairs sharing each X chunk.  At 256
  // rows (7B vocabulary) 327 us a pass against 348 us for one CTA; at 128
  // rows the pair measured no faster (232 against 228 us) and the one-CTA
  // form stays.
  if (beside_smem == 0 && a.R > 128 && a.R <= 256 &&
      lmhead_tc2_params(256, a.H, &tp, &smem)) {
    LmPasses ps;
    memset(&ps, 0, sizeof(ps));
    ps.p[0] = a;
    ps.n = 1;
    return launch_pair_passes(ps, tp, smem, s, after_producer);
  }
  if (!lmhead_tc_params(a.R, a.H, a.rows_per_cta, beside_smem, &tp, &smem))
    return cudaErrorInvalidValue;
  CUtensorMap wf, wp, x;
  // Row-major: [V][H]; tiled: [V * H / 64][64], one 128-byte row per piece.
  const uint64_t w_inner = a.w_packed ? kKChunk : a.H;
  const uint64_t w_outer = a.w_packed ? (uint64_t)a.V * (a.H / kKChunk) : a.V;
  if (!make_map(&wf, a.w, w_inner, w_outer, kKChunk, kTileM, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
      !make_map(&wp, a.w, w_inner, w_outer, kKChunk, kBoxPart, CU_TENSOR_MAP_L2_PROMOTION_L2_256B) ||
      !make_map(&x, a.rows, a.H, a.R, kKChunk, tp.npad, CU_TENSOR_MAP_L2_PROMOTION_L2_128B))
    return cudaErrorInvalidValue;
#define FDL_LM_CASE(NCH)                                                   \
  case NCH:                                                                \
    if (tp.ksub == 4) return launch_nch<NCH, 4>(wf, wp, x, a, tp, smem, s, after_producer); \
    if (tp.ksub == 2) return launch_nch<NCH, 2>(wf, wp, x, a, tp, smem, s, after_producer); \
    return launch_nch<NCH, 1>(wf, wp, x, a, tp, smem, s, after_producer);
  switch (tp.npad / 32) {
    FDL_LM_CASE(1)
    FDL_LM_CASE(2)
    FDL_LM_CASE(4)
    FDL_LM_CASE(8)
  }
#undef FDL_LM_CASE
  return cudaErrorInvalidValue;
}

cudaError_t launch_pack_weight(const void* w, void* out, int V, int H, int rows_per_cta,
                               cudaStream_t s) {
  pack_weight_kernel<<<4 * kPlanSMs, 256, 0, s>>>(static_cast<const uint4*>(w),
                                                  static_cast<uint4*>(out), V, H / kKChunk,
                                                  rows_per_cta);
  return cudaGetLastError();
}

}  // namespace fdl
