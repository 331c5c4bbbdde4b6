// PrefixCache attention on the 5th-generation tensor cores (bf16, d = 128).
//
// Technical review, section 3 (and the PrefixCache branch of Algorithm 1):
// only the prompt and the finished answer are cached; the active block and
// the still-masked suffix after it (n rows) are recomputed every step, and
// their queries attend with full attention to the cached prefix rows
// [0, len_pre[b]) followed by their own n fresh K/V rows.  With n in the
// hundreds this is the compute-bound regime: S = Q K^T and O += P V at full
// 128-row tiles.
//
// An item is (sequence, KV head, 128-row query tile); its rows are query
// positions x the GQA group sharing the KV head.  One CTA per SM takes a PAIR
// of items of the same (sequence, KV head), which read the same keys, and
// streams each 64-key chunk of K and V once for both:
//   warp 0     TMA: Q of both tiles, then K and V of each chunk as one 32 KB
//              stage (four 8 KB boxes, 128-byte swizzle) through a 4-deep ring;
//   warp 1     tcgen05.mma for both tiles: S_t = Q_t K^T (M 128, N 64, K 128)
//              into one of two TMEM S buffers of tile t, then O_t += P_t V
//              (M 128, N 128, K 64) with P_t read from TMEM, each issued as
//              soon as its inputs are ready, so the tensor pipe works on one
//              tile while the other tile's softmax runs;
//   warps 2-5  softmax and epilogue of tile 0, warps 6-9 of tile 1: one
//              thread per row, online max with a lazy rescale of O in TMEM,
//              P = exp2(S - m) as bf16 written back over its S columns.
// TMEM: per tile two 64-column S buffers and a 128-column O (512 in all).
// A CTA loops over pairs; each item is written whole (no partial merge).
#include <cudaTypedefs.h>

#include <mutex>

#include "fdl_common.cuh"
#include "sm100.cuh"

namespace fdl {
namespace {

using namespace sm100;

constexpr int kCh = 64;                  // keys per chunk
constexpr int kKVRegion = kCh * 128;     // 64 keys x 64 bf16 (8 KB)
constexpr int kKVSlot = 4 * kKVRegion;   // K lo, K hi, V lo, V hi: one 32 KB stage
constexpr int kStages = 4;
constexpr int kQRegion = 128 * 128;      // one d-half of a 128-row tile (16 KB)
constexpr int kTiles = 2;
constexpr int kThreads = 320;            // TMA, MMA, 2 x 4 softmax warps
constexpr uint32_t kTmemCols = 512;      // per tile: S 2 x 64 + O 128
constexpr uint32_t kTileCols = 256;
constexpr uint32_t kOCol = 128;          // O's first column within a tile's 256
constexpr float kRescale = 8.0f;         // log2-domain growth forcing a rescale

struct PcArgs {
  int B, Hq, Hkv, q_len, D, cap_p, group, qpt, n_rt, n_pairs;
  float scale_log2;
  const int32_t* len_pre;
  bf16* out;
  Control* ctrl;
};

struct PcMaps {
  CUtensorMap q, kp, vp, kb, vb;
};

struct PcSmem {
  uint64_t kv_full[kStages], kv_empty[kStages];
  uint64_t q_full[kTiles], q_empty[kTiles];
  uint64_t s_full[kTiles][2], s_empty[kTiles][2];
  uint64_t p_full[kTiles][2];
  uint64_t o_full[kTiles], o_empty[kTiles];
  uint64_t drain;
  uint32_t tmem;
};

// Pair pr of the grid: (sequence, KV head, first row tile).
struct Pair {
  int b, kvh, rt0, n_t;  // n_t: tiles in the pair (2, or 1 for an odd last tile)
};

__device__ __forceinline__ Pair pair_of(const PcArgs& a, int pr) {
  const int per_head = (a.n_rt + 1) / 2;
  Pair p;
  p.b = pr / (a.Hkv * per_head);
  const int rem = pr % (a.Hkv * per_head);
  p.kvh = rem / per_head;
  p.rt0 = 2 * (rem % per_head);
  p.n_t = (p.rt0 + 1 < a.n_rt) ? 2 : 1;
  return p;
}

__device__ __forceinline__ int prefix_len(const PcArgs& a, int b) {
  const int Lp = a.len_pre[b];
  return (Lp < 0 || Lp > a.cap_p) ? 0 : Lp;
}

__device__ __forceinline__ int pair_chunks(int Lp, int D) {
  return (Lp + kCh - 1) / kCh + (D + kCh - 1) / kCh;
}

__device__ __forceinline__ uint32_t pack_bf16(float a, float b) {
  const __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<const uint32_t*>(&v);
}

__device__ __forceinline__ float ex2_fast(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__global__ void __launch_bounds__(kThreads, 1)
attn_pc_kernel(const __grid_constant__ PcMaps maps, const PcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* q_smem = base;                               // tiles x 2 halves x 16 KB
  uint8_t* kv_smem = q_smem + kTiles * 2 * kQRegion;    // stages x 32 KB
  PcSmem& S = *reinterpret_cast<PcSmem*>(kv_smem + kStages * kKVSlot);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows_full = a.qpt * a.group;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&S.kv_full[i], 1);
      mbar_init(&S.kv_empty[i], 1);
    }
    for (int t = 0; t < kTiles; ++t) {
      mbar_init(&S.q_full[t], 1);
      mbar_init(&S.q_empty[t], 1);
      mbar_init(&S.o_full[t], 1);
      mbar_init(&S.o_empty[t], 128);
      for (int i = 0; i < 2; ++i) {
        mbar_init(&S.s_full[t][i], 1);
        mbar_init(&S.s_empty[t][i], 1);
        mbar_init(&S.p_full[t][i], 128);
      }
    }
    mbar_init(&S.drain, 1);
    fence_barrier_init();
  }
  // Rows of a tile past the item's rows are never written by TMA: zero them
  // once (they only feed S rows no thread reads).
  for (int t = threadIdx.x; t < kTiles * 2 * (128 - rows_full) * 8; t += kThreads) {
    const int per_region = (128 - rows_full) * 8;
    const int region = t / per_region, w = t % per_region;
    const int row = rows_full + w / 8, chunk = w % 8;
    *reinterpret_cast<uint4*>(q_smem + region * kQRegion + row * 128 + chunk * 16) =
        make_uint4(0, 0, 0, 0);
  }
  fence_proxy_async_smem();
  if (warp == 1) tmem_alloc(&S.tmem, kTmemCols);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem;
  bool failed = false;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA
    if (lane == 0) {
      int kv_i = 0;
      int tp_cnt[kTiles] = {0, 0};  // pairs in which each tile took part
      for (int pr = blockIdx.x; pr < a.n_pairs && !failed; pr += gridDim.x) {
        const Pair p = pair_of(a, pr);
        const int Lp = prefix_len(a, p.b);
        const int n_ch = pair_chunks(Lp, a.D);
        const int ncp = (Lp + kCh - 1) / kCh;
        const int bk = p.b * a.Hkv + p.kvh;
        for (int j = 0; j < n_ch && !failed; ++j, ++kv_i) {
          const int slot = kv_i % kStages;
          if (!mbar_wait(&S.kv_empty[slot], ((kv_i / kStages) & 1) ^ 1)) { failed = true; break; }
          const bool pre = j < ncp;
          const CUtensorMap* mk = pre ? &maps.kp : &maps.kb;
          const CUtensorMap* mv = pre ? &maps.vp : &maps.vb;
          const int row = pre ? bk * a.cap_p + j * kCh : bk * a.D + (j - ncp) * kCh;
          uint8_t* dst = kv_smem + slot * kKVSlot;
          mbar_arrive_expect_tx(&S.kv_full[slot], kKVSlot);
          tma_load_2d(dst, mk, 0, row, &S.kv_full[slot]);
          tma_load_2d(dst + kKVRegion, mk, 64, row, &S.kv_full[slot]);
          tma_load_2d(dst + 2 * kKVRegion, mv, 0, row, &S.kv_full[slot]);
          tma_load_2d(dst + 3 * kKVRegion, mv, 64, row, &S.kv_full[slot]);
          if (j == 0) {
            // The pair's Q after its first K/V, so that load overlaps the wait
            // for the previous pair's last S to release the Q buffers.
            for (int t = 0; t < p.n_t; ++t) {
              if (!mbar_wait(&S.q_empty[t], (tp_cnt[t]++ & 1) ^ 1)) { failed = true; break; }
              mbar_arrive_expect_tx(&S.q_full[t], 2u * 128u * (uint32_t)rows_full);
              const int z = p.b * a.q_len + (p.rt0 + t) * a.qpt;
              uint8_t* qd = q_smem + t * 2 * kQRegion;
              tma_load_3d(qd, &maps.q, 0, p.kvh * a.group, z, &S.q_full[t]);
              tma_load_3d(qd + kQRegion, &maps.q, 64, p.kvh * a.group, z, &S.q_full[t]);
            }
          }
        }
      }
      // Drain: every load issued has landed before this CTA can exit.
      for (int m = max(0, kv_i - kStages); m < kv_i; ++m)
        if (!mbar_wait(&S.kv_full[m % kStages], (m / kStages) & 1)) failed = true;
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA
    if (lane == 0) {
      const uint32_t id_s = idesc_bf16_f32(128, kCh);
      const uint32_t id_pv = idesc_bf16_f32(128, 128) | (1u << 16);  // V is MN-major
      int kv_base = 0;          // global chunk index of the pair's first chunk
      int s_cnt[kTiles] = {0, 0}, p_cnt[kTiles] = {0, 0};  // per-tile S / PV issued
      int tp_cnt[kTiles] = {0, 0};  // pairs in which each tile took part
      long long t_last = clock64();
      for (int pr = blockIdx.x; pr < a.n_pairs && !failed; pr += gridDim.x) {
        const Pair p = pair_of(a, pr);
        const int n_ch = pair_chunks(prefix_len(a, p.b), a.D);
        int is[kTiles] = {0, 0}, ip[kTiles] = {0, 0};  // chunks issued in this pair
        bool q_ok[kTiles] = {false, false};
        bool o_ok[kTiles] = {false, false};
        while ((ip[0] < n_ch || (p.n_t > 1 && ip[1] < n_ch)) && !failed) {
          bool progress = false;
          for (int t = 0; t < p.n_t; ++t) {
            // S_t for chunk is[t]
            if (is[t] < n_ch) {
              const int g = kv_base + is[t], slot = g % kStages;
              const int sb = s_cnt[t] & 1;
              bool ready = q_ok[t] || mbar_test(&S.q_full[t], tp_cnt[t] & 1);
              if (ready) q_ok[t] = true;
              ready = ready && mbar_test(&S.kv_full[slot], (g / kStages) & 1) &&
                      mbar_test(&S.s_empty[t][sb], ((s_cnt[t] >> 1) & 1) ^ 1);
              if (ready) {
                tc_fence_after();
                const uint32_t q_base = smem_u32(q_smem + t * 2 * kQRegion);
                const uint32_t k_base = smem_u32(kv_smem + slot * kKVSlot);
                const uint32_t d_s = tmem + t * kTileCols + (uint32_t)sb * kCh;
#pragma unroll
                for (int k = 0; k < 8; ++k)
                  mma_bf16(d_s, desc_k_sw128(q_base + (k >> 2) * kQRegion + (k & 3) * 32),
                           desc_k_sw128(k_base + (k >> 2) * kKVRegion + (k & 3) * 32), id_s,
                           k ? 1u : 0u);
                mma_commit(&S.s_full[t][sb]);
                if (is[t] + 1 == n_ch) mma_commit(&S.q_empty[t]);
                ++is[t];
                ++s_cnt[t];
                progress = true;
              }
            }
            // O_t += P_t V for chunk ip[t]
            if (ip[t] < is[t]) {
              const int g = kv_base + ip[t], slot = g % kStages;
              const int pb = p_cnt[t] & 1;
              bool ready = mbar_test(&S.p_full[t][pb], (p_cnt[t] >> 1) & 1);
              if (ready && ip[t] == 0 && !o_ok[t]) {
                o_ok[t] = mbar_test(&S.o_empty[t], (tp_cnt[t] & 1) ^ 1);
                ready = o_ok[t];
              }
              if (ready) {
                tc_fence_after();
                const uint32_t v_base = smem_u32(kv_smem + slot * kKVSlot + 2 * kKVRegion);
                const uint32_t p_tmem = tmem + t * kTileCols + (uint32_t)pb * kCh;
                const uint32_t d_o = tmem + t * kTileCols + kOCol;
#pragma unroll
                for (int k = 0; k < kCh / 16; ++k)
                  mma_bf16_ts(d_o, p_tmem + k * 8,
                              desc_mn_sw128(v_base + k * 2048, kKVRegion, 1024), id_pv,
                              (ip[t] == 0 && k == 0) ? 0u : 1u);
                mma_commit(&S.s_empty[t][pb]);
                // The stage is free once every tile of the pair used it.
                const int other = 1 - t;
                if (p.n_t == 1 || ip[other] > ip[t]) mma_commit(&S.kv_empty[slot]);
                if (ip[t] + 1 == n_ch) mma_commit(&S.o_full[t]);
                ++ip[t];
                ++p_cnt[t];
                progress = true;
              }
            }
          }
          if (progress) {
            t_last = clock64();
          } else {
            if (clock64() - t_last > kWaitCycles) {
              failed = true;
              break;
            }
            __nanosleep(32);
          }
        }
        kv_base += n_ch;
        for (int t = 0; t < p.n_t; ++t) ++tp_cnt[t];
      }
      mma_commit(&S.drain);
      if (!mbar_wait(&S.drain, 0)) failed = true;
    }
  } else {
    // ---------------------------------------------- softmax + epilogue
    const int t = (warp - 2) >> 2;          // tile of this warpgroup
    const int q4 = warp & 3;                // TMEM lane quarter
    const int r = q4 * 32 + lane;           // tile row
    const uint32_t lane_addr = (uint32_t)(q4 * 32) << 16;
    const uint32_t t_base = tmem + lane_addr + t * kTileCols;
    int s_cnt = 0, tp_cnt = 0;              // chunks and pairs this tile took part in
    for (int pr = blockIdx.x; pr < a.n_pairs && !failed; pr += gridDim.x) {
      const Pair p = pair_of(a, pr);
      if (t >= p.n_t) continue;             // odd last tile: only tile 0 works
      const int Lp = prefix_len(a, p.b);
      const int n_ch = pair_chunks(Lp, a.D);
      const int ncp = (Lp + kCh - 1) / kCh;
      const int rt = p.rt0 + t;
      const int rows = min(a.qpt, a.q_len - rt * a.qpt) * a.group;
      const bool warp_active = q4 * 32 < rows;
      float m_used = kEmptyMax, l = 0.f;
      for (int j = 0; j < n_ch && !failed; ++j, ++s_cnt) {
        const int sb = s_cnt & 1;
        if (!mbar_wait(&S.s_full[t][sb], (s_cnt >> 1) & 1)) { failed = true; break; }
        tc_fence_after();
        const int nvalid = j < ncp ? min(kCh, Lp - j * kCh) : min(kCh, a.D - (j - ncp) * kCh);
        if (warp_active) {
          uint32_t sr[64];
          uint32_t (&lo)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[0]);
          uint32_t (&hi)[32] = *reinterpret_cast<uint32_t(*)[32]>(&sr[32]);
          tmem_ld_32x32b_x32(t_base + (uint32_t)sb * kCh, lo);
          tmem_ld_32x32b_x32(t_base + (uint32_t)sb * kCh + 32, hi);
          tmem_ld_wait();
          const float sc = a.scale_log2;
          if (nvalid != kCh) {
#pragma unroll
            for (int jj = 0; jj < 64; ++jj)
              if (jj >= nvalid) sr[jj] = __float_as_uint(kEmptyMax);
          }
          float pm[8];
#pragma unroll
          for (int u = 0; u < 8; ++u) pm[u] = __uint_as_float(sr[u]);
#pragma unroll
          for (int jj = 8; jj < 64; ++jj) pm[jj & 7] = fmaxf(pm[jj & 7], __uint_as_float(sr[jj]));
          const float rmax = fmaxf(fmaxf(fmaxf(pm[0], pm[1]), fmaxf(pm[2], pm[3])),
                                   fmaxf(fmaxf(pm[4], pm[5]), fmaxf(pm[6], pm[7])));
          const float cmax = rmax * sc;
          float alpha = 1.f;
          if (j == 0) {
            m_used = cmax;
          } else if (cmax > m_used + kRescale) {
            alpha = ex2_fast(m_used - cmax);
            m_used = cmax;
          }
          if (__any_sync(0xffffffffu, alpha != 1.f)) {
            // The previous chunk's P V must be done before O is touched; its
            // S buffer's release says so.
            const int pq = (s_cnt - 1) & 1;
            if (!mbar_wait(&S.s_empty[t][pq], ((s_cnt - 1) >> 1) & 1)) failed = true;
            tc_fence_after();
#pragma unroll
            for (int cc = 0; cc < 4; ++cc) {
              uint32_t ov[32];
              tmem_ld_32x32b_x32(t_base + kOCol + cc * 32, ov);
              tmem_ld_wait();
#pragma unroll
              for (int jj = 0; jj < 32; ++jj)
                ov[jj] = __float_as_uint(__uint_as_float(ov[jj]) * alpha);
              tmem_st_32x32b_x32(t_base + kOCol + cc * 32, ov);
            }
            tmem_st_wait();
          }
          l *= alpha;
          float ps[4] = {0.f, 0.f, 0.f, 0.f};
          uint32_t pk[32];
#pragma unroll
          for (int jj = 0; jj < 64; jj += 2) {
            const float p0 = ex2_fast(fmaf(__uint_as_float(sr[jj]), sc, -m_used));
            const float p1 = ex2_fast(fmaf(__uint_as_float(sr[jj + 1]), sc, -m_used));
            ps[(jj >> 1) & 3] += p0 + p1;
            pk[jj >> 1] = pack_bf16(p0, p1);
          }
          l += (ps[0] + ps[1]) + (ps[2] + ps[3]);
          tmem_st_32x32b_x32(t_base + (uint32_t)sb * kCh, pk);
          tmem_st_wait();
        }
        tc_fence_before();
        mbar_arrive(&S.p_full[t][sb]);
      }
      if (failed) break;
      // ------------------------------------------------------ item epilogue
      if (!mbar_wait(&S.o_full[t], tp_cnt++ & 1)) { failed = true; break; }
      tc_fence_after();
      if (warp_active) {
        const bool row_ok = r < rows;
        const int qi = rt * a.qpt + r / a.group, jh = r % a.group;
        bf16* orow =
            a.out + (((size_t)p.b * a.q_len + qi) * a.Hq + p.kvh * a.group + jh) * 128;
        const float inv = 1.f / l;
#pragma unroll
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t ov[32];
          tmem_ld_32x32b_x32(t_base + kOCol + cc * 32, ov);
          tmem_ld_wait();
          if (row_ok) {
#pragma unroll
            for (int u = 0; u < 4; ++u) {
              uint4 v;
              v.x = pack_bf16(__uint_as_float(ov[8 * u + 0]) * inv, __uint_as_float(ov[8 * u + 1]) * inv);
              v.y = pack_bf16(__uint_as_float(ov[8 * u + 2]) * inv, __uint_as_float(ov[8 * u + 3]) * inv);
              v.z = pack_bf16(__uint_as_float(ov[8 * u + 4]) * inv, __uint_as_float(ov[8 * u + 5]) * inv);
              v.w = pack_bf16(__uint_as_float(ov[8 * u + 6]) * inv, __uint_as_float(ov[8 * u + 7]) * inv);
              *reinterpret_cast<uint4*>(orow + cc * 32 + 8 * u) = v;
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&S.o_empty[t]);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
  if (failed) atomicOr(&a.ctrl->status, FDL_DEV_TIMEOUT);
}

PFN_cuTensorMapEncodeTiled_v12000 pc_encode_fn() {
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
bool pc_map_rows(CUtensorMap* m, const void* base, uint64_t rows) {
  auto fn = pc_encode_fn();
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
bool pc_map_q(CUtensorMap* m, const void* base, int Hq, int BQ, int group, int qpt) {
  auto fn = pc_encode_fn();
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

size_t attn_pc_smem_bytes() {
  return 1024 + (size_t)kTiles * 2 * kQRegion + (size_t)kStages * kKVSlot + sizeof(PcSmem);
}

// The paired-tile kernel serves items of more than 64 query rows (below
// that the decode-shaped kernel's split over keys is the better fit); the
// caller checks this.
cudaError_t launch_attn_pc(const AttnArgs& a, int n_sm, cudaStream_t s) {
  const int group = a.group;
  if (a.d != 128 || group > 128 || a.k_suf != nullptr) return cudaErrorInvalidValue;
  const int qpt = 128 / group < a.q_len ? 128 / group : a.q_len;
  PcMaps maps;
  const uint64_t bk = (uint64_t)a.B * a.Hkv;
  bool ok = pc_map_q(&maps.q, a.q, a.Hq, a.B * a.q_len, group, qpt) &&
            pc_map_rows(&maps.kb, a.k_blk, bk * a.D) && pc_map_rows(&maps.vb, a.v_blk, bk * a.D);
  if (a.cap_p > 0) {
    ok = ok && pc_map_rows(&maps.kp, a.k_pre, bk * a.cap_p) &&
         pc_map_rows(&maps.vp, a.v_pre, bk * a.cap_p);
  } else {
    maps.kp = maps.kb;
    maps.vp = maps.vb;
  }
  if (!ok) return cudaErrorInvalidValue;
  PcArgs t;
  t.B = a.B;
  t.Hq = a.Hq;
  t.Hkv = a.Hkv;
  t.q_len = a.q_len;
  t.D = a.D;
  t.cap_p = a.cap_p;
  t.group = group;
  t.qpt = qpt;
  t.n_rt = (a.q_len + qpt - 1) / qpt;
  t.n_pairs = a.B * a.Hkv * ((t.n_rt + 1) / 2);
  t.scale_log2 = a.scale_log2;
  t.len_pre = a.len_pre;
  t.out = static_cast<bf16*>(a.out);
  t.ctrl = a.ctrl;
  const size_t smem = attn_pc_smem_bytes();
  static std::mutex mu;
  static bool configured[64] = {};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!configured[dev]) {
      e = cudaFuncSetAttribute(attn_pc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)smem);
      if (e != cudaSuccess) return e;
      configured[dev] = true;
    }
  }
  const int grid = t.n_pairs < n_sm ? t.n_pairs : n_sm;
  attn_pc_kernel<<<grid, kThreads, smem, s>>>(maps, t);
  return cudaGetLastError();
}

}  // namespace fdl
