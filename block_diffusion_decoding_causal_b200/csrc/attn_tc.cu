// Block-wise attention on the 5th-generation tensor cores (bf16, d = 128).
//
// The active unit's queries attend to [prefix cache | block rows | suffix
// cache] ("Fast-dLLM v2" section 3.4, Figure 7b and Level 3; technical review
// eq. (3) and section 3).  One (sequence, KV head, query-row tile) is an
// item: its rows are the unit's q_len positions x the group of query heads
// sharing the KV head (GQA packing: 8 x 7 = 56 rows at Qwen2.5-7B shapes),
// padded to the M = 128 tile.
//
// Stream-K split: every CTA reads the per-sequence lengths, cuts the
// concatenation of all items' 64-key chunks into equal contiguous ranges and
// takes its own, so the split follows the actual lengths and a CTA produces
// at most two partial results (its first and last item); items it covers
// whole are written out directly.  Per chunk:
//   warp 0   TMA: K and V [64 keys x 128] into one 32 KB stage (four 8 KB
//            boxes, 128-byte swizzle) of a STAGES-deep ring, a barrier pair
//            per half: S frees the K half, P V the V half; Q of each item by
//            a 3D box (d, head group, positions);
//   warp 1   tcgen05.mma: S = Q K^T (M 128, N 64, K 128) into one of two TMEM
//            S buffers, then, one chunk behind, O += P V (M 128, N 128, K 64)
//            with P read from TMEM and V MN-major from shared memory, into
//            the item's TMEM O buffer;
//   warps 2-5  softmax, one thread per row: S from TMEM, online max with a
//            lazy rescale (O in TMEM is rescaled only when the running max
//            grows by more than 2^8), P = exp2(S - m) as bf16 written back
//            over its S columns, and the item epilogue.
// Partial results (unnormalised O, m, l) go to the workspace.  Alone on the
// GPU (two CTAs per SM, three stages each where they fit, else two) a
// grid-stride merge kernel, launched as a programmatic dependent of this
// grid, combines them.  Beside the LM head (one CTA per SM, one stage,
// leaving the SM's other room to that kernel) the thread that writes a row's
// last partial merges the row itself.  No thread waits on another CTA.
#include <cudaTypedefs.h>

#include <mutex>

#include "fdl_common.cuh"
#include "fdl_plan.h"
#include "sm100.cuh"

namespace fdl {
namespace {

using namespace sm100;

constexpr int kCh = 64;                  // keys per chunk
// Rows of an item at most 64: the Q halves (d 0-63, 64-127) sit only the
// rows (rounded to 8) apart, 16 KB at most for both.  The MMA still reads 128
// rows per half; the rows past the item then fall on the other half or the
// K/V stage that follows, which only feeds S rows no softmax thread reads
// (rows of an M = 128 tile never mix).
// Bytes between the two d-halves of the Q buffer: the item's rows rounded up
// to the 8-row swizzle atom when they are at most 64, else 128 rows.
__host__ __device__ constexpr int q_region_for(int rows) {
  return rows <= 64 ? ((rows + 7) / 8) * 8 * 128 : 128 * 128;
}
constexpr int kKVRegion = kCh * 128;     // 64 keys x 64 bf16 (8 KB)
constexpr int kKVSlot = 4 * kKVRegion;   // K lo, K hi, V lo, V hi: one 32 KB stage
// K/V stages of the attention alone on the GPU (two CTAs per SM at 2) and
// beside the LM head (1).
constexpr int kMaxStages = 3;            // two CTAs per SM fit three stages when Q is small
constexpr int kQBufs = 1;                // Q is reloaded per item
constexpr int kSB = 2;                   // S buffers in TMEM; P overwrites its S
constexpr uint32_t kTmemCols = 256;      // S 2 x 64 columns, O 128 columns
constexpr uint32_t kOCol = kSB * 64;     // first column of O
constexpr int kThreads = 192;
constexpr float kRescale = 8.0f;         // log2-domain growth forcing a rescale
constexpr unsigned kDevTimeout = FDL_DEV_TIMEOUT;
constexpr int kMaxSeq = 256;

struct TcArgs {
  int B, Hq, Hkv, q_len, D, cap_p, cap_s, group, qpt, n_rt, n_cta, dual;
  float scale_log2;
  const int32_t* len_pre;
  const int32_t* len_suf;
  bf16* out;
  Control* ctrl;
  unsigned int* tickets;  // [items][128]: arrivals per (item, tile row)
  float* part_o;          // [2 * n_cta][128][128]
  float2* part_ml;        // [2 * n_cta][128]
  int inline_merge;       // the last CTA to finish a row of an item merges it
  int merge_wide;         // merge kernel: lanes over partials (many per item)
  int v_lag;              // V loads issued this many chunks behind K (0 or 1)
  int wait_inputs;        // programmatic launch: wait for the previous grid
                          // after the prologue, before any input is read
  int q_region;           // bytes between the two d-halves of the Q buffer
};

struct Maps {
  CUtensorMap q, kp, vp, kb, vb, ks, vs;
};

struct Smem {
  uint64_t k_full[kMaxStages], k_empty[kMaxStages];  // K half of a stage: free after S
  uint64_t v_full[kMaxStages], v_empty[kMaxStages];  // V half: free after P V
  uint64_t q_full[2], q_empty[2];
  uint64_t s_full[kSB], s_empty[kSB];   // S ready / S and its P free again
  uint64_t p_full[kSB];                 // P written into TMEM
  uint64_t o_full[2], o_empty[2];
  uint64_t drain;
  uint32_t tmem;
  // followed by the sequence table: cb [B + 1] (first global chunk of
  // sequence b), nc [B] (chunks per item), lp [B], ls [B] (lengths)
};

// Position in the chunk sequence of one CTA.
struct Cursor {
  int b, it, j;  // sequence, item within sequence, chunk within item
};

__device__ __forceinline__ Cursor locate(const int* cb, const int* nc, int B, long long g) {
  int lo = 0, hi = B - 1;
  while (lo < hi) {  // last b with cb[b] <= g
    const int mid = (lo + hi + 1) >> 1;
    if (cb[mid] <= g) lo = mid; else hi = mid - 1;
  }
  const int rem = (int)(g - cb[lo]);
  Cursor c;
  c.b = lo;
  c.it = rem / nc[lo];
  c.j = rem % nc[lo];
  return c;
}

__device__ __forceinline__ void advance(Cursor& c, const int* nc, int per_seq) {
  if (++c.j == nc[c.b]) {
    c.j = 0;
    if (++c.it == per_seq) {
      c.it = 0;
      ++c.b;
    }
  }
}

// CTA owning global chunk g: the largest i with floor(T i / n) <= g.
__device__ __forceinline__ int cta_of(long long g, long long T, int n) {
  return (int)(((g + 1) * n - 1) / T);
}

__device__ __forceinline__ long long cta_start(int i, long long T, int n) {
  return T * i / n;
}

// With fewer chunks than CTAs some ranges are empty; only non-empty ones
// between the first and last owner of an item touched it.
__device__ __forceinline__ bool cta_nonempty(int i, long long T, int n) {
  return cta_start(i, T, n) < cta_start(i + 1, T, n);
}

struct ChunkInfo {
  int seg;     // 0 prefix, 1 block, 2 suffix
  int key0;    // first key of the chunk within its segment
  int nvalid;  // valid keys in the chunk
};

// Chunks of one item: the prefix, the block rows (one chunk up to 64 rows;
// more when the recomputed rows of PrefixCache take the block's place) and
// the suffix, each cut into 64-key chunks.
__device__ __forceinline__ int item_chunks(int Lp, int Ls, int D) {
  return (Lp + kCh - 1) / kCh + (D + kCh - 1) / kCh + (Ls + kCh - 1) / kCh;
}

__device__ __forceinline__ ChunkInfo chunk_info(int j, int Lp, int Ls, int D) {
  const int ncp = (Lp + kCh - 1) / kCh;
  const int ncb = (D + kCh - 1) / kCh;
  ChunkInfo ci;
  if (j < ncp) {
    ci.seg = 0;
    ci.key0 = j * kCh;
    ci.nvalid = min(kCh, Lp - ci.key0);
  } else if (j < ncp + ncb) {
    ci.seg = 1;
    ci.key0 = (j - ncp) * kCh;
    ci.nvalid = min(kCh, D - ci.key0);
  } else {
    ci.seg = 2;
    ci.key0 = (j - ncp - ncb) * kCh;
    ci.nvalid = min(kCh, Ls - ci.key0);
  }
  return ci;
}



// 2^x with the PTX ex2.approx instruction (relative error near 2^-22,
// subnormal results flushed to zero): the softmax weights are rounded to
// bf16 right after, so the approximation is far below what is kept.
__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

// Partial slot of CTA j for the item whose chunks start at x_start: slot
// 2j holds a CTA's first item, 2j + 1 its last (when it is a different one).
__device__ __forceinline__ int partial_slot(int j, int cta_lo, long long x_start, long long T,
                                            int n) {
  return 2 * j + ((j == cta_lo && cta_start(j, T, n) != x_start) ? 1 : 0);
}

// Merge of one row of one item inside the attention kernel, by the thread
// of the CTA that wrote the row's last partial (used when the grid runs
// beside the LM head, where a separate merge launch would wait for that
// kernel).  The partials (O, m, l) of the CTAs cta_lo..cta_hi are combined
// with the usual max/sum rescaling, 32 columns at a time.
__device__ __noinline__ void merge_row_inline(const TcArgs& a, int r, int cta_lo, int cta_hi,
                                              long long x_start, long long T, int n,
                                              bf16* orow) {
  float M = kEmptyMax;
  for (int j = cta_lo; j <= cta_hi; ++j) {
    if (!cta_nonempty(j, T, n)) continue;
    M = fmaxf(M, __ldcg(&a.part_ml[(size_t)partial_slot(j, cta_lo, x_start, T, n) * 128 + r]).x);
  }
  float L = 0.f;
  for (int j = cta_lo; j <= cta_hi; ++j) {
    if (!cta_nonempty(j, T, n)) continue;
    const float2 ml = __ldcg(&a.part_ml[(size_t)partial_slot(j, cta_lo, x_start, T, n) * 128 + r]);
    L += ml.y * exp2f(ml.x - M);
  }
  const float inv = 1.f / L;
  for (int cc = 0; cc < 4; ++cc) {
    float acc[32];
#pragma unroll
    for (int t = 0; t < 32; ++t) acc[t] = 0.f;
    for (int j = cta_lo; j <= cta_hi; ++j) {
      if (!cta_nonempty(j, T, n)) continue;
      const int sl = partial_slot(j, cta_lo, x_start, T, n);
      const float w = exp2f(__ldcg(&a.part_ml[(size_t)sl * 128 + r]).x - M);
      const float4* src =
          reinterpret_cast<const float4*>(a.part_o + ((size_t)sl * 128 + r) * 128 + cc * 32);
      float4 v[8];
#pragma unroll
      for (int t = 0; t < 8; ++t) v[t] = __ldcg(src + t);
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        acc[4 * t] += v[t].x * w;
        acc[4 * t + 1] += v[t].y * w;
        acc[4 * t + 2] += v[t].z * w;
        acc[4 * t + 3] += v[t].w * w;
      }
    }
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      uint4 o;
      o.x = pack_bf16(acc[8 * t + 0] * inv, acc[8 * t + 1] * inv);
      o.y = pack_bf16(acc[8 * t + 2] * inv, acc[8 * t + 3] * inv);
      o.z = pack_bf16(acc[8 * t + 4] * inv, acc[8 * t + 5] * inv);
      o.w = pack_bf16(acc[8 * t + 6] * inv, acc[8 * t + 7] * inv);
      *reinterpret_cast<uint4*>(orow + cc * 32 + 8 * t) = o;
    }
  }
}

// Every split row of every item, one warp per (item, row), the tasks
// strided over `n_warps` warps of which this one is `first`.  The row's
// partials (CTAs cta_lo .. cta_hi of the attention grid of n CTAs over T
// chunks) are combined with the usual (max, sum) rescaling.  The lanes first
// work out which of 32 CTAs hold a partial of the item and where (one CTA
// each, in parallel: the split arithmetic is 64-bit), then the warp reads
// them sixteen at a time with every read in flight; lanes hold four of the
// 128 columns.
constexpr int kMergeBatch = 8;

__device__ __forceinline__ void merge_split_rows(const TcArgs& a, const int* cb, const int* nc,
                                                 long long T, int n, long long first,
                                                 long long n_warps) {
  const int lane = threadIdx.x & 31;
  const int per_seq = a.Hkv * a.n_rt;
  const int rows_full = a.qpt * a.group;
  const long long n_tasks = (long long)a.B * per_seq * rows_full;
  for (long long task = first; task < n_tasks; task += n_warps) {
    const int x = (int)(task / rows_full), r = (int)(task % rows_full);
    const int b = x / per_seq, it = x % per_seq;
    const long long x_start = cb[b] + (long long)it * nc[b];
    const long long x_end = x_start + nc[b];
    if (x_end <= x_start) continue;
    const int cta_lo = cta_of(x_start, T, n), cta_hi = cta_of(x_end - 1, T, n);
    if (cta_lo == cta_hi) continue;  // written directly by its only CTA
    const int kvh = it / a.n_rt, rt = it % a.n_rt;
    const int qpt_eff = min(a.qpt, a.q_len - rt * a.qpt);
    if (r >= qpt_eff * a.group) continue;
    float M = kEmptyMax, L = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    // CTA starts T i / n in 32-bit arithmetic when T n fits (always, at the
    // sizes the library takes; 64-bit otherwise).
    const bool narrow = T * n < (1ll << 32);
    const uint32_t T32 = (uint32_t)T, n32 = (uint32_t)n;
    for (int j0 = cta_lo; j0 <= cta_hi; j0 += 32) {
      const int j = j0 + lane;
      long long s0, s1;
      if (narrow) {
        s0 = (long long)(T32 * (uint32_t)j / n32);
        s1 = (long long)(T32 * (uint32_t)(j + 1) / n32);
      } else {
        s0 = cta_start(j, T, n);
        s1 = cta_start(j + 1, T, n);
      }
      const bool have = j <= cta_hi && s0 < s1;
      const int my_slot = 2 * j + ((j == cta_lo && s0 != x_start) ? 1 : 0);
      unsigned mask = __ballot_sync(0xffffffffu, have);
      while (mask != 0u) {
        const int cnt = min(kMergeBatch, __popc(mask));  // uniform across the warp
        float2 ml[kMergeBatch];
        float4 v[kMergeBatch];
#pragma unroll
        for (int u = 0; u < kMergeBatch; ++u) {
          if (u < cnt) {
            const int src = __ffs(mask) - 1;
            mask &= mask - 1u;
            const int sl = __shfl_sync(0xffffffffu, my_slot, src);
            ml[u] = __ldcg(&a.part_ml[(size_t)sl * 128 + r]);
            v[u] = __ldcg(reinterpret_cast<const float4*>(a.part_o + ((size_t)sl * 128 + r) * 128) +
                          lane);
          }
        }
#pragma unroll
        for (int u = 0; u < kMergeBatch; ++u) {
          if (u < cnt) {
            const float m_new = fmaxf(M, ml[u].x);
            const float f_old = ex2_fast(M - m_new), w = ex2_fast(ml[u].x - m_new);
            L = L * f_old + ml[u].y * w;
            acc.x = acc.x * f_old + v[u].x * w;
            acc.y = acc.y * f_old + v[u].y * w;
            acc.z = acc.z * f_old + v[u].z * w;
            acc.w = acc.w * f_old + v[u].w * w;
            M = m_new;
          }
        }
      }
    }
    const float inv = 1.f / L;
    const int pq = r / a.group, jq = r % a.group;
    bf16* dst = a.out + (((size_t)b * a.q_len + rt * a.qpt + pq) * a.Hq + kvh * a.group + jq) * 128;
    uint2 packed;
    packed.x = pack_bf16(acc.x * inv, acc.y * inv);
    packed.y = pack_bf16(acc.z * inv, acc.w * inv);
    reinterpret_cast<uint2*>(dst)[lane] = packed;
  }
}

template <int STAGES>
__global__ void __launch_bounds__(kThreads, 2)
attn_tc_kernel(const __grid_constant__ Maps maps, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = base;                               // kQBufs x 2 x q_region
  uint8_t* kv_smem = q_smem + kQBufs * 2 * a.q_region;  // STAGES x 32 KB
  Smem& S = *reinterpret_cast<Smem*>(kv_smem + STAGES * kKVSlot);
  int* const cb = reinterpret_cast<int*>(&S + 1);  // sequence table, sized by B
  int* const nc = cb + a.B + 1;
  int* const lp = nc + a.B;
  int* const ls = lp + a.B;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_seq = a.Hkv * a.n_rt;  // items per sequence
  const int rows_full = a.qpt * a.group;

  if (threadIdx.x == 0) {
    for (int i = 0; i < STAGES; ++i) {
      mbar_init(&S.k_full[i], 1);
      mbar_init(&S.k_empty[i], 1);
      mbar_init(&S.v_full[i], 1);
      mbar_init(&S.v_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&S.q_full[i], 1);
      mbar_init(&S.q_empty[i], 1);
      mbar_init(&S.o_full[i], 1);
      mbar_init(&S.o_empty[i], 128);
    }
    for (int i = 0; i < kSB; ++i) {
      mbar_init(&S.s_full[i], 1);
      mbar_init(&S.s_empty[i], 1);
      mbar_init(&S.p_full[i], 128);
    }
    mbar_init(&S.drain, 1);
    fence_barrier_init();
  }
  // Sequence table from the device-resident lengths: warp 0 reads 32
  // lengths at a time and prefix-sums the chunk counts with shuffles.
  auto build_table = [&]() {
    int run = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
      const int b = b0 + lane;
      int Lp = 0, Ls = 0, n_ch = 0;
      if (b < a.B) {
        Lp = a.len_pre[b];
        if (Lp < 0 || Lp > a.cap_p) {
          if (blockIdx.x == 0) atomicOr(&a.ctrl->status, FDL_DEV_BAD_PREFIX_LEN);
          Lp = 0;
        }
        if (a.dual) {
          Ls = a.len_suf[b];
          if (Ls < 0 || Ls > a.cap_s) {
            if (blockIdx.x == 0) atomicOr(&a.ctrl->status, FDL_DEV_BAD_SUFFIX_LEN);
            Ls = 0;
          }
        }
        n_ch = item_chunks(Lp, Ls, a.D);
      }
      int incl = n_ch * per_seq;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (b < a.B) {
        lp[b] = Lp;
        ls[b] = Ls;
        nc[b] = n_ch;
        cb[b] = run + incl - n_ch * per_seq;
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) cb[a.B] = run;
  };
  // Without a wait its length reads overlap the rest of the prologue.
  if (!a.wait_inputs && warp == 0) build_table();
  // Padding rows of the Q halves are never written by TMA: zero them once.
  const int q_rows = a.q_region / 128;
  for (int t = threadIdx.x; t < kQBufs * 2 * (q_rows - rows_full) * 8; t += kThreads) {
    const int per_region = (q_rows - rows_full) * 8;
    const int region = t / per_region, w = t % per_region;
    const int row = rows_full + w / 8, chunk = w % 8;
    *reinterpret_cast<uint4*>(q_smem + region * a.q_region + row * 128 + chunk * 16) =
        make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(&S.tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem;
  // Launched as a programmatic dependent of whatever ran before (a stand-
  // alone call): everything above overlapped that grid's tail; from here on
  // inputs are read and the workspace written, so wait for it to finish.
  if (a.wait_inputs) {
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (warp == 0) build_table();
    __syncthreads();
  }

  const long long T = cb[a.B];
  const int n = a.n_cta;
  const long long c_begin = cta_start(blockIdx.x, T, n);
  const long long c_end = cta_start(blockIdx.x + 1, T, n);
  bool failed = false;

  if (c_begin < c_end && warp == 0) {
    // -------------------------------------------------------------- TMA
    // A stage holds one chunk's K and V (16 KB each, two 8 KB boxes), with a
    // barrier per half: S = Q K^T releases the K half, P V the V half, so the
    // next K streams in while this chunk's softmax still runs.  Issue order
    // K(j), V(j - v_lag).  With 128-row tiles (compute-heavy) v_lag = 1: K's
    // slot frees (S(j - STAGES) done) before V's does, so K does not wait
    // behind V's slot (PrefixCache 42.7 -> 37.8 us); streaming decode keeps
    // each chunk's K and V together (v_lag = 0), V on time for its P V.
    if (lane == 0) {
      const int n_my = (int)(c_end - c_begin);
      const int lag = a.v_lag;
      int q_i = 0, prev_x = -1;
      Cursor ck = locate(cb, nc, a.B, c_begin), cv = ck;
      for (int j = 0; j < n_my + lag && !failed; ++j) {
        if (j < n_my) {
          const int x = ck.b * per_seq + ck.it;
          const int kvh = ck.it / a.n_rt, rt = ck.it % a.n_rt;
          const int slot = j % STAGES;
          if (!mbar_wait(&S.k_empty[slot], ((j / STAGES) & 1) ^ 1)) { failed = true; break; }
          // Streaming decode with a ring of several stages: K also waits for
          // the stage's V half, i.e. for the whole stage (measured faster:
          // batch 16, prefix 8192, 57.7 against 59.4 us with the early K).
          // The one-stage ring beside the LM head keeps the early K.
          if (lag == 0 && STAGES > 1 &&
              !mbar_wait(&S.v_empty[slot], ((j / STAGES) & 1) ^ 1)) { failed = true; break; }
          const ChunkInfo ci = chunk_info(ck.j, lp[ck.b], ls[ck.b], a.D);
          const int bk = ck.b * a.Hkv + kvh;
          const CUtensorMap* mk = ci.seg == 0 ? &maps.kp : (ci.seg == 1 ? &maps.kb : &maps.ks);
          const int row = ci.seg == 0 ? bk * a.cap_p + ci.key0
                                      : (ci.seg == 1 ? bk * a.D + ci.key0 : bk * a.cap_s + ci.key0);
          uint8_t* dst = kv_smem + slot * kKVSlot;
          mbar_arrive_expect_tx(&S.k_full[slot], 2 * kKVRegion);
          tma_load_2d(dst, mk, 0, row, &S.k_full[slot]);
          tma_load_2d(dst + kKVRegion, mk, 64, row, &S.k_full[slot]);
          // A new item's Q goes after its first K, so that load overlaps the
          // wait for the previous item's last S to release the Q buffer.
          if (x != prev_x) {
            const int qb = q_i % kQBufs;
            if (!mbar_wait(&S.q_empty[qb], ((q_i / kQBufs) & 1) ^ 1)) { failed = true; break; }
            mbar_arrive_expect_tx(&S.q_full[qb], 2u * 128u * (uint32_t)rows_full);
            const int z = ck.b * a.q_len + rt * a.qpt;
            tma_load_3d(q_smem + qb * 2 * a.q_region, &maps.q, 0, kvh * a.group, z,
                        &S.q_full[qb]);
            tma_load_3d(q_smem + qb * 2 * a.q_region + a.q_region, &maps.q, 64, kvh * a.group, z,
                        &S.q_full[qb]);
            ++q_i;
            prev_x = x;
          }
          advance(ck, nc, per_seq);
        }
        if (j >= lag) {
          const int i = j - lag;
          const int kvh = cv.it / a.n_rt;
          const int slot = i % STAGES;
          if (!mbar_wait(&S.v_empty[slot], ((i / STAGES) & 1) ^ 1)) { failed = true; break; }
          const ChunkInfo ci = chunk_info(cv.j, lp[cv.b], ls[cv.b], a.D);
          const int bk = cv.b * a.Hkv + kvh;
          const CUtensorMap* mv = ci.seg == 0 ? &maps.vp : (ci.seg == 1 ? &maps.vb : &maps.vs);
          const int row = ci.seg == 0 ? bk * a.cap_p + ci.key0
                                      : (ci.seg == 1 ? bk * a.D + ci.key0 : bk * a.cap_s + ci.key0);
          uint8_t* dst = kv_smem + slot * kKVSlot + 2 * kKVRegion;
          mbar_arrive_expect_tx(&S.v_full[slot], 2 * kKVRegion);
          tma_load_2d(dst, mv, 0, row, &S.v_full[slot]);
          tma_load_2d(dst + kKVRegion, mv, 64, row, &S.v_full[slot]);
          advance(cv, nc, per_seq);
        }
      }
      // Drain: every load issued has landed before this CTA can exit.
      for (int m = max(0, n_my - STAGES); m < n_my; ++m) {
        if (!mbar_wait(&S.k_full[m % STAGES], (m / STAGES) & 1)) failed = true;
        if (!mbar_wait(&S.v_full[m % STAGES], (m / STAGES) & 1)) failed = true;
      }
      for (int m = max(0, q_i - kQBufs); m < q_i; ++m)
        if (!mbar_wait(&S.q_full[m % kQBufs], (m / kQBufs) & 1)) failed = true;
    }
  } else if (c_begin < c_end && warp == 1) {
    // -------------------------------------------------------------- MMA
    // S for chunk i and P V for chunk j < i are issued as soon as each one's
    // inputs are ready (non-blocking probes), so the slot release that lets
    // the next loads start never waits on an unrelated load.
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, kCh);
      const uint32_t id_pv = idesc_bf16_f32(128, 128) | (1u << 16);  // V is MN-major
      const int n_my = (int)(c_end - c_begin);
      int is = 0, ip = 0, q_s = 0, o_i = 0, prev_xs = -1, prev_xp = -1;
      Cursor cs = locate(cb, nc, a.B, c_begin), cp = cs;
      long long t_last = clock64();
      while (ip < n_my) {
        bool progress = false;
        if (is < n_my) {
          const int x = cs.b * per_seq + cs.it;
          const bool first = x != prev_xs;
          const int slot = is % STAGES, sb = is % kSB;
          bool ready = first ? mbar_test(&S.q_full[q_s % kQBufs], (q_s / kQBufs) & 1) : true;
          ready = ready && mbar_test(&S.k_full[slot], (is / STAGES) & 1) &&
                  mbar_test(&S.s_empty[sb], ((is / kSB) & 1) ^ 1);
          if (ready) {
            if (first) {
              ++q_s;
              prev_xs = x;
            }
            const int qb = (q_s - 1) % kQBufs;
            const bool last = (is + 1 == n_my) || (cs.j + 1 == nc[cs.b]);
            tc_fence_after();
            const uint32_t q_base = smem_u32(q_smem + qb * 2 * a.q_region);
            const uint32_t k_base = smem_u32(kv_smem + slot * kKVSlot);
            const uint32_t d_s = tmem + (uint32_t)sb * kCh;
#pragma unroll
            for (int k = 0; k < 8; ++k)
              mma_bf16(d_s, desc_k_sw128(q_base + (k >> 2) * a.q_region + (k & 3) * 32),
                       desc_k_sw128(k_base + (k >> 2) * kKVRegion + (k & 3) * 32), id_s,
                       k ? 1u : 0u);
            mma_commit(&S.s_full[sb]);
            mma_commit(&S.k_empty[slot]);
            if (last) mma_commit(&S.q_empty[qb]);
            advance(cs, nc, per_seq);
            ++is;
            progress = true;
          }
        }
        if (ip < is) {
          const int x = cp.b * per_seq + cp.it;
          const bool first = x != prev_xp;
          const int pb = ip % kSB, vslot = ip % STAGES;
          bool ready = mbar_test(&S.p_full[pb], (ip / kSB) & 1) &&
                       mbar_test(&S.v_full[vslot], (ip / STAGES) & 1);
          if (first) ready = ready && mbar_test(&S.o_empty[0], (o_i & 1) ^ 1);
          if (ready) {
            if (first) prev_xp = x;
            const bool last = (ip + 1 == n_my) || (cp.j + 1 == nc[cp.b]);
            tc_fence_after();
            const uint32_t v_base = smem_u32(kv_smem + vslot * kKVSlot + 2 * kKVRegion);
            const uint32_t p_tmem = tmem + (uint32_t)pb * kCh;  // P over its S columns
            const uint32_t d_o = tmem + kOCol;
#pragma unroll
            for (int k = 0; k < kCh / 16; ++k)  // 16 keys = 8 packed columns of P
              mma_bf16_ts(d_o, p_tmem + k * 8, desc_mn_sw128(v_base + k * 2048, kKVRegion, 1024),
                          id_pv, (first && k == 0) ? 0u : 1u);
            mma_commit(&S.v_empty[vslot]);
            mma_commit(&S.s_empty[pb]);
            if (last) {
              mma_commit(&S.o_full[0]);
              ++o_i;
            }
            advance(cp, nc, per_seq);
            ++ip;
            progress = true;
          }
        }
        if (progress) {
          t_last = clock64();
        } else {
          if (clock64() - t_last > kWaitCycles) {
            failed = true;
            break;
          }
          // Nothing ready: yield the issue slots this sub-partition shares
          // with a softmax warp.
          __nanosleep(64);
        }
      }
      mma_commit(&S.drain);
      if (!mbar_wait(&S.drain, 0)) failed = true;
    }
  } else if (c_begin < c_end && warp >= 2) {
    // ------------------------------------------------- softmax + epilogue
    const int q4 = warp & 3;
    const int r = q4 * 32 + lane;  // TMEM lane = tile row
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    float m_used = kEmptyMax, l = 0.f;
    int s_i = 0, o_i = 0, prev_x = -1;
    const int first_x = [&] {
      const Cursor c0 = locate(cb, nc, a.B, c_begin);
      return c0.b * per_seq + c0.it;
    }();
    Cursor c = locate(cb, nc, a.B, c_begin);
    for (long long g = c_begin; g < c_end && !failed; ++g, advance(c, nc, per_seq)) {
      const int x = c.b * per_seq + c.it;
      const int first = x != prev_x;
      const int last = (g + 1 == c_end) || (c.j + 1 == nc[c.b]);
      const int kvh = c.it / a.n_rt, rt = c.it % a.n_rt;
      const int qpt_eff = min(a.qpt, a.q_len - rt * a.qpt);
      const int rows = qpt_eff * a.group;
      const bool warp_active = q4 * 32 < rows;
      if (first) {
        m_used = kEmptyMax;
        l = 0.f;
        prev_x = x;
      }
      const ChunkInfo ci = chunk_info(c.j, lp[c.b], ls[c.b], a.D);
      const int sb = s_i % kSB;
      if (!mbar_wait(&S.s_full[sb], (s_i / kSB) & 1)) { failed = true; break; }
      tc_fence_after();
      uint32_t sr[64];
      if (warp_active) {
        uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
        uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
        tmem_ld_32x32b_x32(tmem + lane_addr + (uint32_t)sb * kCh, lo);
        tmem_ld_32x32b_x32(tmem + lane_addr + (uint32_t)sb * kCh + 32, hi);
        tmem_ld_wait();
      }
      const int pb = sb;
      if (warp_active) {
        // Row maximum on the raw scores (the scale is positive); keys past
        // the chunk's valid count get the empty value, whose weight is 0.
        const float sc = a.scale_log2;
        if (ci.nvalid != kCh) {
#pragma unroll
          for (int jj = 0; jj < 64; ++jj)
            if (jj >= ci.nvalid) sr[jj] = __float_as_uint(kEmptyMax);
        }
        // Eight independent partial maxima, then a tree: short dependency
        // chains instead of one of 64.
        float pm[8];
#pragma unroll
        for (int t = 0; t < 8; ++t) pm[t] = __uint_as_float(sr[t]);
#pragma unroll
        for (int jj = 8; jj < 64; ++jj) pm[jj & 7] = fmaxf(pm[jj & 7], __uint_as_float(sr[jj]));
        const float rmax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                 fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
        const float cmax = rmax * sc;
        float alpha = 1.f;
        if (first) {
          m_used = cmax;
        } else if (cmax > m_used + kRescale) {
          alpha = ex2_fast(m_used - cmax);
          m_used = cmax;
        }
        // O rescale (warp-collective TMEM access) when any row needs it.
        if (__any_sync(0xffffffffu, alpha != 1.f)) {
          // P V of the previous chunk must be done before O is touched; its
          // S buffer's release says so (P V of chunk c - 1 - kSB is known
          // complete because S of chunk c was issued, so the parity cannot
          // be stale).
          const int pq = (s_i - 1) % kSB;
          if (!mbar_wait(&S.s_empty[pq], ((s_i - 1) / kSB) & 1)) { failed = true; }
          tc_fence_after();
          const uint32_t o_addr = tmem + lane_addr + kOCol;
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t ov[32];
            tmem_ld_32x32b_x32(o_addr + cc * 32, ov);
            tmem_ld_wait();
#pragma unroll
            for (int jj = 0; jj < 32; ++jj) ov[jj] = __float_as_uint(__uint_as_float(ov[jj]) * alpha);
            tmem_st_32x32b_x32(o_addr + cc * 32, ov);
          }
          tmem_st_wait();
        }
        l *= alpha;
        float ps[4] = {0.f, 0.f, 0.f, 0.f};  // independent partial sums
        uint32_t pk[32];
#pragma unroll
        for (int jj = 0; jj < 64; jj += 2) {
          const float p0 = ex2_fast(fmaf(__uint_as_float(sr[jj]), sc, -m_used));
          const float p1 = ex2_fast(fmaf(__uint_as_float(sr[jj + 1]), sc, -m_used));
          ps[(jj >> 1) & 3] += p0 + p1;
          pk[jj >> 1] = pack_bf16(p0, p1);
        }
        l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
        // P (bf16 pairs) over the first 32 columns of this chunk's S.
        tmem_st_32x32b_x32(tmem + lane_addr + (uint32_t)pb * kCh, pk);
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(&S.p_full[pb]);
      ++s_i;
      if (failed) break;
      if (!last) continue;

      // ----------------------------------------------------- item epilogue
      if (!mbar_wait(&S.o_full[0], o_i & 1)) { failed = true; break; }
      tc_fence_after();
      const long long x_start = cb[c.b] + (long long)c.it * nc[c.b];
      const long long x_end = x_start + nc[c.b];
      const int cta_lo = cta_of(x_start, T, n), cta_hi = cta_of(x_end - 1, T, n);
      const int p_pos = r / a.group, jh = r % a.group;
      const int qi = rt * a.qpt + p_pos;
      const bool row_ok = r < rows;
      bf16* orow = a.out + (((size_t)c.b * a.q_len + qi) * a.Hq + kvh * a.group + jh) * 128;
      const uint32_t o_addr = tmem + lane_addr + kOCol;
      if (cta_lo == cta_hi) {
        const float inv = 1.f / l;
        if (warp_active) {
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            uint32_t ov[32];
            tmem_ld_32x32b_x32(o_addr + cc * 32, ov);
            tmem_ld_wait();
            if (row_ok) {
#pragma unroll
              for (int t = 0; t < 4; ++t) {
                uint4 v;
                v.x = pack_bf16(__uint_as_float(ov[8 * t + 0]) * inv, __uint_as_float(ov[8 * t + 1]) * inv);
                v.y = pack_bf16(__uint_as_float(ov[8 * t + 2]) * inv, __uint_as_float(ov[8 * t + 3]) * inv);
                v.z = pack_bf16(__uint_as_float(ov[8 * t + 4]) * inv, __uint_as_float(ov[8 * t + 5]) * inv);
                v.w = pack_bf16(__uint_as_float(ov[8 * t + 6]) * inv, __uint_as_float(ov[8 * t + 7]) * inv);
                *reinterpret_cast<uint4*>(orow + cc * 32 + 8 * t) = v;
              }
            }
          }
        }
        tc_fence_before();
        mbar_arrive(&S.o_empty[0]);
        ++o_i;
        continue;
      }
      // Partial of this CTA: slot 2*cta for its first item, 2*cta+1 otherwise;
      // the merge kernel that follows combines the item's partials.
      const int slot = 2 * blockIdx.x + (x == first_x ? 0 : 1);
      float* po = a.part_o + ((size_t)slot * 128 + r) * 128;
      if (warp_active) {
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t ov[32];
          tmem_ld_32x32b_x32(o_addr + cc * 32, ov);
          tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int t = 0; t < 8; ++t)
              *reinterpret_cast<uint4*>(po + cc * 32 + 4 * t) =
                  make_uint4(ov[4 * t], ov[4 * t + 1], ov[4 * t + 2], ov[4 * t + 3]);
          }
        }
        if (row_ok) a.part_ml[(size_t)slot * 128 + r] = make_float2(m_used, l);
      }
      tc_fence_before();
      mbar_arrive(&S.o_empty[0]);
      ++o_i;
      if (a.inline_merge && row_ok) {
        // "Last to arrive" per (item, row): publish this partial, count it;
        // the thread that completes the count merges the row and rearms it.
        __threadfence();
        int parts = 0;
        for (int j = cta_lo; j <= cta_hi; ++j) parts += cta_nonempty(j, T, n) ? 1 : 0;
        unsigned int* tk = a.tickets + (size_t)x * 128 + r;
        if (atomicAdd(tk, 1u) == (unsigned int)(parts - 1)) {
          *tk = 0u;
          __threadfence();
          merge_row_inline(a, r, cta_lo, cta_hi, x_start, T, n, orow);
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (failed) atomicOr(&a.ctrl->status, kDevTimeout);
  // This CTA is done: the merge kernel may be scheduled once every CTA got
  // here (it still waits for the whole grid before reading a partial).
  // Triggered at entry instead, the merge's CTAs took the room of retiring
  // attention CTAs early and the pair ran slower (batch 1, prefix 8192: 34.5
  // against 18 us).
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // When launched beside the step's LM head, finish only after it did, so
  // that this grid's completion (which the merge waits for) covers both.
  // Alone (the wait after the prologue already returned) or without a
  // programmatic predecessor this returns at once.
  asm volatile("griddepcontrol.wait;" ::: "memory");
}

// The same merge for items spread over many CTAs (batch 1 or 4 at long
// prefixes: tens of partials per item): one warp per (item, row, quarter of
// the 128 columns), its lanes over the partials, 32 at a time.  Lane l reads
// partial l's (m, l) and its 32 columns of the quarter; the warp takes the
// maximum and the weighted sum of l with shuffles, then a reduce-scatter over
// the 32 x 32 weighted block leaves column c's sum in lane c.  One read round
// trip per 32 partials instead of one per eight.
__device__ __forceinline__ void merge_split_rows_wide(const TcArgs& a, const int* cb,
                                                      const int* nc, long long T, int n,
                                                      long long first, long long n_warps) {
  const int lane = threadIdx.x & 31;
  const int per_seq = a.Hkv * a.n_rt;
  const int rows_full = a.qpt * a.group;
  const long long n_tasks = (long long)a.B * per_seq * rows_full * 4;
  const bool narrow = T * n < (1ll << 32);
  const uint32_t T32 = (uint32_t)T, n32 = (uint32_t)n;
  for (long long task = first; task < n_tasks; task += n_warps) {
    const int cq = (int)(task & 3);
    const long long xr = task >> 2;
    const int x = (int)(xr / rows_full), r = (int)(xr % rows_full);
    const int b = x / per_seq, it = x % per_seq;
    const long long x_start = cb[b] + (long long)it * nc[b];
    const long long x_end = x_start + nc[b];
    if (x_end <= x_start) continue;
    const int cta_lo = cta_of(x_start, T, n), cta_hi = cta_of(x_end - 1, T, n);
    if (cta_lo == cta_hi) continue;
    const int kvh = it / a.n_rt, rt = it % a.n_rt;
    const int qpt_eff = min(a.qpt, a.q_len - rt * a.qpt);
    if (r >= qpt_eff * a.group) continue;
    float M = kEmptyMax, L = 0.f, acc = 0.f;  // acc: column cq * 32 + lane
    for (int j0 = cta_lo; j0 <= cta_hi; j0 += 32) {
      const int j = j0 + lane;
      long long s0, s1;
      if (narrow) {
        s0 = (long long)(T32 * (uint32_t)j / n32);
        s1 = (long long)(T32 * (uint32_t)(j + 1) / n32);
      } else {
        s0 = cta_start(j, T, n);
        s1 = cta_start(j + 1, T, n);
      }
      const bool have = j <= cta_hi && s0 < s1;
      float2 ml = make_float2(kEmptyMax, 0.f);
      float4 v[8];
      if (have) {
        const int sl = 2 * j + ((j == cta_lo && s0 != x_start) ? 1 : 0);
        ml = __ldcg(&a.part_ml[(size_t)sl * 128 + r]);
        const float4* src =
            reinterpret_cast<const float4*>(a.part_o + ((size_t)sl * 128 + r) * 128 + cq * 32);
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = __ldcg(src + t);
      } else {
#pragma unroll
        for (int t = 0; t < 8; ++t) v[t] = make_float4(0.f, 0.f, 0.f, 0.f);
      }
      float mc = ml.x;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) mc = fmaxf(mc, __shfl_xor_sync(0xffffffffu, mc, o));
      const float m_new = fmaxf(M, mc);
      const float w = have ? ex2_fast(ml.x - m_new) : 0.f;
      float lw = ml.y * w;
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) lw += __shfl_xor_sync(0xffffffffu, lw, o);
      const float f_old = ex2_fast(M - m_new);
      // Weighted 32 columns of this lane's partial, then a reduce-scatter:
      // after it lane c holds the sum over lanes of column c.
      float c32[32];
#pragma unroll
      for (int t = 0; t < 8; ++t) {
        c32[4 * t] = v[t].x * w;
        c32[4 * t + 1] = v[t].y * w;
        c32[4 * t + 2] = v[t].z * w;
        c32[4 * t + 3] = v[t].w * w;
      }
#pragma unroll
      for (int wdt = 16; wdt >= 1; wdt >>= 1) {
        const bool upper = (lane & wdt) != 0;
#pragma unroll
        for (int k = 0; k < wdt; ++k) {
          const float keep = upper ? c32[k + wdt] : c32[k];
          const float send = upper ? c32[k] : c32[k + wdt];
          c32[k] = keep + __shfl_xor_sync(0xffffffffu, send, wdt);
        }
      }
      acc = acc * f_old + c32[0];
      L = L * f_old + lw;
      M = m_new;
    }
    const int pq = r / a.group, jq = r % a.group;
    bf16* dst = a.out + (((size_t)b * a.q_len + rt * a.qpt + pq) * a.Hq + kvh * a.group + jq) * 128;
    dst[cq * 32 + lane] = __float2bfloat16_rn(acc / L);
  }
}

// Merge of the partials of every item the split spread over several CTAs,
// launched as a programmatic dependent of the attention grid: its CTAs are
// scheduled as the attention's retire, rebuild the sequence table from the
// lengths, and wait for the whole grid before reading a partial.  At most three CTAs per SM, eight warps each, every warp a
// (item, row) task at a time (few fat CTAs: the launch of one small CTA per
// (item, row block) cost more than the merge itself; three per SM keep about
// one task per warp in flight at batch 16).  Warp 0 first rebuilds
// the attention's sequence table from the device-resident lengths.
__global__ void __launch_bounds__(256, 3)
attn_merge_rows_kernel(const TcArgs a) {
  __shared__ int cb[kMaxSeq + 1];
  __shared__ int nc[kMaxSeq];
  // The step's LM head, launched behind this grid when its rows do not come
  // from the attention, may start on the SM room these CTAs leave; it
  // touches nothing this grid reads or writes.
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int per_seq = a.Hkv * a.n_rt;
  if (warp == 0) {
    int run = 0;
    for (int b0 = 0; b0 < a.B; b0 += 32) {
      const int b = b0 + lane;
      int n_ch = 0;
      if (b < a.B) {
        int Lp = a.len_pre[b];
        if (Lp < 0 || Lp > a.cap_p) Lp = 0;
        int Ls = 0;
        if (a.dual) {
          Ls = a.len_suf[b];
          if (Ls < 0 || Ls > a.cap_s) Ls = 0;
        }
        n_ch = item_chunks(Lp, Ls, a.D);
      }
      int incl = n_ch * per_seq;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      if (b < a.B) {
        nc[b] = n_ch;
        cb[b] = run + incl - n_ch * per_seq;
      }
      run += __shfl_sync(0xffffffffu, incl, 31);
    }
    if (lane == 0) cb[a.B] = run;
  }
  __syncthreads();
  // The lengths are inputs of the attention grid (complete before it began),
  // the partials its outputs: only these wait for the grid to finish.
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const long long warps = (long long)gridDim.x * (blockDim.x >> 5);
  const long long first = (long long)blockIdx.x * (blockDim.x >> 5) + warp;
  if (a.merge_wide)
    merge_split_rows_wide(a, cb, nc, cb[a.B], a.n_cta, first, warps);
  else
    merge_split_rows(a, cb, nc, cb[a.B], a.n_cta, first, warps);
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

// Rows of 128 bf16 (256 B), box [64 d x 64 rows], 128-byte swizzle.
bool map_rows(CUtensorMap* m, const void* base, uint64_t rows) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {128, rows};
  cuuint64_t strides[1] = {256};
  cuuint32_t box[2] = {64, kCh};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

// Q [B*q_len, Hq, 128] as a 3D map; box [64 d, group heads, qpt positions].
bool map_q(CUtensorMap* m, const void* base, int Hq, int BQ, int group, int qpt) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[3] = {128, (cuuint64_t)Hq, (cuuint64_t)BQ};
  cuuint64_t strides[2] = {256, (cuuint64_t)Hq * 256};
  cuuint32_t box[3] = {64, (cuuint32_t)group, (cuuint32_t)qpt};
  cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
         CUDA_SUCCESS;
}

}  // namespace

// Query positions per 128-row tile for a GQA group; 0 if unsupported.
int attn_tc_qpt(int q_len, int group) {
  if (group > 128) return 0;
  const int qpt = 128 / group;
  return qpt < q_len ? qpt : q_len;
}

size_t attn_tc_smem_bytes(int stages, int q_region, int B) {
  return 1024 + kQBufs * 2 * (size_t)q_region + stages * kKVSlot + sizeof(Smem) +
         sizeof(int) * (4 * (size_t)B + 1);
}

// Shared memory of one attention CTA (beside the LM head: one K/V stage).
// Stages of the attention alone on the GPU: three when two CTAs with three
// still fit on one SM (228 KB less a 1 KB reservation each), else two.
int attn_tc_alone_stages(int q_region, int B) {
  return 2 * (attn_tc_smem_bytes(3, q_region, B) + 1024) <= 228 * 1024 ? 3 : 2;
}

size_t attn_tc_smem_for(int q_len, int group, int B, bool beside) {
  const int qpt = attn_tc_qpt(q_len, group);
  const int q_region = q_region_for(qpt * group);
  return attn_tc_smem_bytes(beside ? 1 : attn_tc_alone_stages(q_region, B), q_region, B);
}


// Per-device host state of the attention launches: the dynamic shared memory
// each kernel variant was last opened up to (a driver call worth skipping on
// every launch).
constexpr int kMaxDev = 64;
static size_t g_smem_set[kMaxDev][kMaxStages + 1];
static std::mutex g_kern_mu;

static cudaError_t prepare_kernel(const void* kern, int stages, size_t smem) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(g_kern_mu);
  if (g_smem_set[dev][stages] < smem) {
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributePreferredSharedMemoryCarveout,
                             cudaSharedmemCarveoutMaxShared);
    if (e != cudaSuccess) return e;
    g_smem_set[dev][stages] = smem;
  }
  return cudaSuccess;
}

cudaError_t launch_attn_tc(const AttnArgs& a, float* part_o, float2* part_ml,
                           unsigned int* tickets, int n_cta, cudaStream_t s,
                           bool beside_prior) {
  const int qpt = attn_tc_qpt(a.q_len, a.group);
  if (a.d != 128 || qpt == 0 || a.B > kMaxSeq) return cudaErrorInvalidValue;
  Maps maps;
  const uint64_t bk = (uint64_t)a.B * a.Hkv;
  bool ok = map_q(&maps.q, a.q, a.Hq, a.B * a.q_len, a.group, qpt) &&
            map_rows(&maps.kb, a.k_blk, bk * a.D) && map_rows(&maps.vb, a.v_blk, bk * a.D);
  if (a.cap_p > 0) {
    ok = ok && map_rows(&maps.kp, a.k_pre, bk * a.cap_p) &&
         map_rows(&maps.vp, a.v_pre, bk * a.cap_p);
  } else {
    maps.kp = maps.kb;
    maps.vp = maps.vb;
  }
  if (a.k_suf != nullptr) {
    ok = ok && map_rows(&maps.ks, a.k_suf, bk * a.cap_s) &&
         map_rows(&maps.vs, a.v_suf, bk * a.cap_s);
  } else {
    maps.ks = maps.kb;
    maps.vs = maps.vb;
  }
  if (!ok) return cudaErrorInvalidValue;
  TcArgs t;
  t.B = a.B;
  t.Hq = a.Hq;
  t.Hkv = a.Hkv;
  t.q_len = a.q_len;
  t.D = a.D;
  t.cap_p = a.cap_p;
  t.cap_s = a.cap_s;
  t.group = a.group;
  t.qpt = qpt;
  t.n_rt = (a.q_len + qpt - 1) / qpt;
  // Items of more than 64 query rows (PrefixCache, long units), whose
  // partials are 64 KB fp32 tiles, and at least half as many items as
  // CTAs: one CTA per item, so that equal-length items are never split and
  // nothing is merged (at LLaDA-8B PrefixCache shapes the merge of the
  // stream-K split cost more than the imbalance does).  Everything else
  // keeps the full stream-K grid.
  const int n_items_all = a.B * a.Hkv * t.n_rt;
  if (!beside_prior && qpt * a.group > 64 && 2 * n_items_all >= n_cta &&
      n_items_all <= n_cta)
    n_cta = n_items_all;
  t.n_cta = n_cta;
  t.dual = a.k_suf != nullptr;
  t.scale_log2 = a.scale_log2;
  t.len_pre = a.len_pre;
  t.len_suf = a.len_suf;
  t.out = static_cast<bf16*>(a.out);
  t.ctrl = a.ctrl;
  t.tickets = tickets;
  t.part_o = part_o;
  t.part_ml = part_ml;
  t.inline_merge = beside_prior ? 1 : 0;
  t.merge_wide = 0;
  t.v_lag = qpt * a.group > 64 ? 1 : 0;
  // One sequence and one CTA per item (the PrefixCache shape): every item
  // has the same chunks, each CTA's range is exactly one item and there is
  // nothing to merge.
  const bool no_merge = !beside_prior && a.B == 1 && n_cta == n_items_all;
  // Programmatic launch.  Beside the LM head the attention reads nothing
  // that kernel writes and starts at once.  Alone it waits for its
  // predecessor after the prologue, so a call's launch and prologue overlap
  // the previous call's merge: 0.7-1.8 us a call at batch 1-16 (batch 4,
  // prefix 8192: 25.7 -> 24.0-24.3 us); the same time as before at the
  // PrefixCache shape, whose predecessor has no merge to hide behind.
  t.wait_inputs = beside_prior ? 0 : 1;
  t.q_region = q_region_for(qpt * a.group);
  // Beside the LM head: one K/V stage, so the SM's remaining shared memory
  // goes to that kernel's weight ring.
  const int stages = beside_prior ? 1 : attn_tc_alone_stages(t.q_region, a.B);
  const size_t smem = attn_tc_smem_bytes(stages, t.q_region, a.B);
  auto kern = stages == 1 ? attn_tc_kernel<1> : (stages == 2 ? attn_tc_kernel<2>
                                                             : attn_tc_kernel<3>);
  cudaError_t e = prepare_kernel(reinterpret_cast<const void*>(kern), stages, smem);
  if (e != cudaSuccess) return e;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  {
    cudaLaunchConfig_t mc = {};
    mc.gridDim = dim3(n_cta, 1, 1);
    mc.blockDim = dim3(kThreads, 1, 1);
    mc.dynamicSmemBytes = smem;
    mc.stream = s;
    mc.attrs = attr;
    mc.numAttrs = 1;
    e = cudaLaunchKernelEx(&mc, kern, maps, t);
    if (e != cudaSuccess) return e;
  }
  if (beside_prior) return cudaSuccess;  // merged inside the kernel
  if (no_merge) return cudaGetLastError();
  // The merge: up to three CTAs per SM, eight warps each, one (item, row)
  // task per warp at a time, or one (item, row, column quarter) with lanes
  // over the partials when an item has about 40 or more of them (batch 1 at
  // long prefixes: 17.9 against 23.4 us at prefix 8192; at batch 4, about 20
  // partials an item, the narrow form stays ahead: 24.7 against 27.5 us).
  t.merge_wide = n_cta / n_items_all + 1 >= 40 ? 1 : 0;
  const long long tasks = (long long)n_items_all * qpt * a.group * (t.merge_wide ? 4 : 1);
  const long long want = (tasks + 7) / 8;
  const long long cap = 3LL * kPlanCTAs;
  cudaLaunchConfig_t lc = {};
  lc.gridDim = dim3((unsigned)(want < cap ? (want < 1 ? 1 : want) : cap), 1, 1);
  lc.blockDim = dim3(256, 1, 1);
  lc.dynamicSmemBytes = 0;
  lc.stream = s;
  lc.attrs = attr;
  lc.numAttrs = 1;
  e = cudaLaunchKernelEx(&lc, attn_merge_rows_kernel, t);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace fdl
