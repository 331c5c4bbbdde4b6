/*
 * fdl.h - C ABI of libfdl.so: one denoising step of the active block in
 * block-diffusion decoding (Fast-dLLM / Fast-dLLM v2), on one NVIDIA B200.
 *
 * The step (pages: "Fast-dLLM v2: Efficient Block-Diffusion LLM", section 3.4
 * "Inference Pipeline" and Figure 7b; "Fast-dLLM: Reusing Bidirectional State
 * and Spending Confidence on Parallel Tokens", sections 2-4):
 *   (a) attention of the active unit's queries over the block-level prefix
 *       KV cache, the block's own K/V (bidirectional within the block) and,
 *       for DualCache, the cached suffix of still-masked positions;
 *   (b) the LM-head contraction over the unit's hidden states fused with a
 *       full-vocabulary (max probability, argmax) reduction, then the
 *       confidence-threshold commit with its single-position fallback.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Pointers.  Every tensor pointer is a caller-owned DEVICE pointer (lengths
 *   included), 16-byte aligned, row-major and densely packed as documented.
 *   The library allocates no memory and keeps no state between calls: its
 *   only scratch is the caller's workspace `ws` (see fdl_workspace_size).
 * Streams.  `stream` is a cudaStream_t passed as void* (NULL = the legacy
 *   default stream).  All work is enqueued asynchronously on it; no entry
 *   point synchronises except fdl_get_status.
 * Types.  Floating tensors share cfg->dtype (FDL_F32 or FDL_BF16); conf is
 *   always float32, token ids int32, bitmaps uint8 (0/1).
 * Errors.  Arguments the host can check (NULL pointers, shapes, alignment,
 *   workspace size) are checked before any launch: the call returns a
 *   negative fdl_status with no side effects, and fdl_last_error() gives a
 *   message (thread-local).  Launch failures return FDL_ERR_CUDA.  Values the
 *   host cannot see (device-resident lengths outside [0, capacity]) are
 *   detected by the kernels: the sequence is processed as if the offending
 *   length were 0, a bit is set in the workspace status word, and
 *   fdl_get_status reports it.  No kernel traps.
 * Workspace.  `ws` must be at least fdl_workspace_size(cfg) bytes, 256-byte
 *   aligned, and zero-filled before its first use (cudaMemset or
 *   fdl_reset_workspace).  Every call leaves its counters at zero again, so
 *   a workspace can be reused for any number of calls on one stream.  Calls
 *   that overlap on the GPU must use different workspaces.
 */
#ifndef FDL_H_
#define FDL_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#define FDL_VERSION 1

typedef enum { FDL_F32 = 0, FDL_BF16 = 1 } fdl_dtype;

typedef enum {
  FDL_OK = 0,
  FDL_ERR_INVALID_ARG = -1,   /* bad pointer, shape, alignment or value      */
  FDL_ERR_UNSUPPORTED = -2,   /* valid but outside what the kernels handle   */
  FDL_ERR_WORKSPACE = -3,     /* workspace NULL, misaligned or too small     */
  FDL_ERR_CUDA = -4,          /* a CUDA call or launch failed                */
  FDL_ERR_DEVICE_STATUS = -5  /* fdl_get_status: a kernel flagged bad input  */
} fdl_status;

/* Device status bits (fdl_get_status). */
#define FDL_DEV_BAD_PREFIX_LEN 1u  /* len_pre[b] outside [0, cap_prefix] */
#define FDL_DEV_BAD_SUFFIX_LEN 2u  /* len_suf[b] outside [0, cap_suffix] */
#define FDL_DEV_TIMEOUT 4u         /* a kernel's bounded wait (about 1 s) ran out;
                                      its outputs are invalid and the workspace
                                      counters may be left non-zero: call
                                      fdl_reset_workspace before reusing it */

/*
 * Geometry and decoding parameters of one step.
 *
 * The pages state the problem as a prompt of length P, a generation length L
 * cut into blocks of block_size (D = 32 in all their experiments), sub-blocks
 * of q_len (8 by default) as the thresholding unit, a threshold tau and a
 * mask token.  One step works on block index k of the answer:
 *   prefix length Lp = P + k*D (prompt + finished blocks, exact cache);
 *   suffix length Ls = L - (k+1)*D (DualCache only: masked positions after
 *     the block, whose K/V are frozen);
 *   the active unit is block positions [q_off, q_off + q_len).
 * Lp and Ls are per sequence and live on the device (len_pre / len_suf);
 * cap_prefix / cap_suffix are the cache capacities (rows per (sequence, KV
 * head)).
 * Limits.  The fused step, the LM head and the commit entry points take
 * block_size <= 64, q_len <= 32 and batch * q_len <= 4096 (beyond 256 rows
 * the LM head makes one pass over the weight per group of whole sequences
 * that fits in 256 rows).  The attention entry points also take block_size
 * and q_len up to 4096 (PrefixCache: the recomputed rows), on the bf16,
 * head_dim 128 path with batch <= 256.
 */
typedef struct {
  int32_t batch;       /* B >= 1                                               */
  int32_t n_q_heads;   /* Hq; Hq % Hkv == 0                                    */
  int32_t n_kv_heads;  /* Hkv; query head h reads KV head h / (Hq / Hkv)       */
  int32_t head_dim;    /* d in {32, 64, 128}; softmax scale 1/sqrt(d)          */
  int32_t block_size;  /* D, 1..64 (attention entry points: up to 4096)      */
  int32_t q_off;       /* first block position of the active unit             */
  int32_t q_len;       /* unit length, 1..32, q_off + q_len <= D (attention
                          entry points: up to 4096)                           */
  int32_t cap_prefix;  /* prefix cache rows per (b, kv head), >= 0             */
  int32_t cap_suffix;  /* suffix cache rows per (b, kv head), >= 0 (DualCache) */
  int32_t hidden;      /* H: LM-head input width                               */
  int32_t vocab;       /* V >= 2                                               */
  int32_t mask_id;     /* the [MASK] token id, 0 <= mask_id < V                */
  int32_t shift;       /* 1: position p is predicted from the hidden state of
                          p - 1 (v2 token shift); 0: from p itself             */
  float tau;           /* commit iff confidence >= tau                         */
  int32_t dtype;       /* fdl_dtype of every floating tensor                   */
  int32_t w_layout;    /* FDL_W_ROW_MAJOR, or FDL_W_PACKED: w_lm as rewritten by
                          fdl_lmhead_pack_weight (bf16 only)                   */
} fdl_step_cfg;

/* Layouts of the LM-head weight (fdl_step_cfg.w_layout). */
#define FDL_W_ROW_MAJOR 0  /* w_lm [V, H] row-major                            */
#define FDL_W_PACKED 1     /* the tiled layout of fdl_lmhead_pack_weight         */

/* Library version (FDL_VERSION) and a thread-local description of the last
 * error returned on this thread ("" if none). */
int fdl_version(void);
const char* fdl_last_error(void);

/* Bytes of workspace any entry point needs for this configuration; 0 if the
 * configuration is invalid (fdl_last_error says why). */
size_t fdl_workspace_size(const fdl_step_cfg* cfg);

/* Zero a workspace (async memset on `stream`). */
int fdl_reset_workspace(void* ws, size_t ws_bytes, void* stream);

/*
 * Block-wise attention, v2 (stage a; "Fast-dLLM v2", section 3.4, Figure 7b
 * and Level 3; attention itself is eq. (3) of the technical review).
 *   For sequence b, query head h (KV head h / (Hq/Hkv)) and unit row r:
 *     out[b,r,h,:] = softmax(q[b,r,h,:] . K^T / sqrt(d)) V over the keys
 *     K = k_pre[b,kvh, 0:len_pre[b], :]  followed by  k_blk[b,kvh, 0:D, :]
 *   i.e. every cached earlier block (causal across blocks) and every row of
 *   the active block (bidirectional within it); later blocks do not exist.
 *   The block rows of the active unit are the fresh K/V the caller computed
 *   this step; the other block rows are its sub-block cache.
 * Layouts: q, out [B, q_len, Hq, d]; k_pre, v_pre [B, Hkv, cap_prefix, d];
 *   len_pre int32 [B]; k_blk, v_blk [B, Hkv, D, d].
 * fp32 accumulation; out is rounded to cfg->dtype.
 */
int fdl_block_attn(const fdl_step_cfg* cfg, const void* q, const void* k_pre,
                   const void* v_pre, const int32_t* len_pre, const void* k_blk,
                   const void* v_blk, void* out, void* ws, size_t ws_bytes,
                   void* stream);

/*
 * DualCache attention, v1 (stage a; technical review section 3 and its
 * Algorithm 1).  As fdl_block_attn with a third key segment,
 * the frozen suffix cache k_suf/v_suf [B, Hkv, cap_suffix, d], rows
 * 0:len_suf[b]; every key of prefix, block and suffix is visible (the
 * full-attention dLLMs DualCache accelerates).
 */
int fdl_dualcache_attn(const fdl_step_cfg* cfg, const void* q,
                       const void* k_pre, const void* v_pre,
                       const int32_t* len_pre, const void* k_blk,
                       const void* v_blk, const void* k_suf, const void* v_suf,
                       const int32_t* len_suf, void* out, void* ws,
                       size_t ws_bytes, void* stream);

/*
 * PrefixCache attention, v1 (technical review section 3 and the PrefixCache
 * branch of its Algorithm 1): only the prompt and the finished answer prefix
 * are cached; the active block and the masked suffix after it are
 * recomputed every step, and their queries attend, with full attention, to
 * the cached prefix and to their own fresh K/V.
 *   n = cfg->block_size = cfg->q_len recomputed rows (the active block and
 *   the suffix), cfg->q_off = 0 (else FDL_ERR_INVALID_ARG).  For sequence b,
 *   query head h (KV head kvh) and recomputed row r:
 *     out[b,r,h,:] = softmax(q[b,r,h,:] . K^T / sqrt(d)) V over
 *     K = k_pre[b,kvh, 0:len_pre[b], :] followed by k_fresh[b,kvh, 0:n, :].
 * Layouts: q, out [B, n, Hq, d]; k_pre, v_pre [B, Hkv, cap_prefix, d];
 *   len_pre int32 [B]; k_fresh, v_fresh [B, Hkv, n, d].  n up to 4096 on the
 *   bf16, head_dim 128 path (the 128-row query tiles are then full).
 * This is fdl_block_attn with the recomputed rows in the block's place.
 */
int fdl_prefixcache_attn(const fdl_step_cfg* cfg, const void* q, const void* k_pre,
                         const void* v_pre, const int32_t* len_pre, const void* k_fresh,
                         const void* v_fresh, void* out, void* ws, size_t ws_bytes,
                         void* stream);

/*
 * LM head + confidence (stage b, first half; "Fast-dLLM v2" Level 2 and
 * Algorithm 2 of the technical review, section 4).
 *   For each row i of rows [B*q_len, H] (already token-shifted: row
 *   (b, i) predicts block position q_off + i):
 *     l = w_lm . rows[i]  over the full vocabulary (w_lm [V, H] row-major,
 *     or, with cfg->w_layout = FDL_W_PACKED, the same weight as rewritten
 *     by fdl_lmhead_pack_weight; the results are identical),
 *     tok[i]  = argmax_v l_v (the lowest v on a tie),
 *     conf[i] = max softmax probability = 1 / sum_v exp(l_v - l_max).
 *   Logits never leave the chip.  Rows with row_active[i] == 0 report
 *   conf = -1 and tok = -1 (row_active may be NULL: all rows active).
 * Outputs: conf float32 [B, q_len], tok int32 [B, q_len].
 */
int fdl_lmhead_confidence(const fdl_step_cfg* cfg, const void* rows,
                          const void* w_lm, const uint8_t* row_active,
                          float* conf, int32_t* tok, void* ws, size_t ws_bytes,
                          void* stream);

/*
 * LM-head weight in its tiled form (no counterpart on the pages: a load-time
 * layout choice of this library, like a GEMM library's pre-transformed
 * weights).  Rewrites w_lm [V, H] row-major (bf16) into w_packed, the same
 * number of bytes (2 V H), so that every block the LM head streams — 128
 * vocabulary rows x 64 hidden columns of one CTA's range — is contiguous in
 * memory instead of 128 strided 128-byte pieces.  Call it once when the
 * weight is loaded; then pass w_packed as w_lm with cfg->w_layout =
 * FDL_W_PACKED to fdl_lmhead_confidence, fdl_lmhead_confidence_noalloc and
 * fdl_denoise_step.  The results are bit-identical to the row-major layout.
 * Only the vocabulary size and hidden width of cfg matter (the split of the
 * vocabulary over the CTAs is fixed by V); w_lm and w_packed must not
 * overlap.  bf16 and hidden % 64 == 0 only (else FDL_ERR_UNSUPPORTED).
 */
int fdl_lmhead_pack_weight(const fdl_step_cfg* cfg, const void* w_lm, void* w_packed,
                           void* stream);

/*
 * Threshold commit (stage b, second half; technical review Algorithm 2
 * section 4; "Fast-dLLM v2" Level 2 and the sub-block paragraph).
 *   Candidates C_b = unit positions p in [q_off, q_off+q_len) with
 *   block_tokens[b,p] == mask_id.  S_b = {p in C_b : conf[b,p-q_off] >= tau};
 *   if S_b is empty and C_b is not, S_b = {the p in C_b with the largest
 *   conf, the lowest p on a tie}.  Then block_tokens[b,p] = tok[b,p-q_off]
 *   for p in S_b (all at once).
 * In/out: block_tokens int32 [B, D].  Out: committed uint8 [B, D] (1 on S_b,
 *   0 elsewhere in the block), n_committed int32 [B] = |S_b|,
 *   n_masked_left int32 [B] = unit positions still equal to mask_id.
 */
int fdl_threshold_commit(const fdl_step_cfg* cfg, const float* conf,
                         const int32_t* tok, int32_t* block_tokens,
                         uint8_t* committed, int32_t* n_committed,
                         int32_t* n_masked_left, void* stream);

/* Selection rules of fdl_select_commit. */
#define FDL_SELECT_THRESHOLD 0 /* Algorithm 2: commit conf >= param (tau)    */
#define FDL_SELECT_FACTOR 1    /* Algorithm 3, eq. 13: factor f = param        */
#define FDL_SELECT_BUDGET 2    /* eq. 9: heterogeneous error budget (no param) */

/*
 * Commit with a chosen selection rule (technical review: section 4
 * Algorithm 2; section 6 eq. (13) and Algorithm 3; section 5.1 eq. (9)).
 * Candidates as in fdl_threshold_commit.  FDL_SELECT_THRESHOLD is
 * fdl_threshold_commit with tau = param.  FDL_SELECT_FACTOR sorts the
 * candidates by decreasing confidence (lower position first on ties) and
 * commits the first n for the largest n with (n + 1)(1 - c_(n)) < param.
 * FDL_SELECT_BUDGET commits the first n for the largest n with
 * sum_{j<=n} (1 - c_(j)) + (1 - c_(n)) < 1.  If no n qualifies, the most
 * confident candidate alone.  Outputs as fdl_threshold_commit.
 */
int fdl_select_commit(const fdl_step_cfg* cfg, int policy, float param,
                      const float* conf, const int32_t* tok,
                      int32_t* block_tokens, uint8_t* committed,
                      int32_t* n_committed, int32_t* n_masked_left, void* stream);

/*
 * One whole denoising step on one stream, no host synchronisation:
 *   attention (DualCache when k_suf != NULL, else block-causal) ->
 *   LM-head rows (hidden if given, else the attention output; then the token
 *   shift: with cfg->shift, row i is source row i-1 and row 0 is h_prev[b],
 *   the hidden state of the position before the unit) -> LM head +
 *   confidence on the rows whose target is still masked -> commit.
 * hidden: [B, q_len, H] or NULL (then H must equal Hq*d and the attention
 *   output, rounded to cfg->dtype, is used).  h_prev: [B, H], required iff
 *   cfg->shift.  attn_out: [B, q_len, Hq, d] or NULL (then it is kept in the
 *   workspace).  k_suf, v_suf, len_suf: all NULL or all set.  w_lm in the
 *   layout cfg->w_layout names, as for fdl_lmhead_confidence.
 * Outputs as fdl_lmhead_confidence and fdl_threshold_commit.
 */
int fdl_denoise_step(const fdl_step_cfg* cfg, const void* q, const void* k_pre,
                     const void* v_pre, const int32_t* len_pre,
                     const void* k_blk, const void* v_blk, const void* k_suf,
                     const void* v_suf, const int32_t* len_suf,
                     const void* hidden, const void* h_prev, const void* w_lm,
                     int32_t* block_tokens, void* attn_out, float* conf,
                     int32_t* tok, uint8_t* committed, int32_t* n_committed,
                     int32_t* n_masked_left, void* ws, size_t ws_bytes,
                     void* stream);

/*
 * LM head + confidence without a workspace (the pages have no counterpart;
 * this is a deployment convenience).  Same computation, arguments and
 * outputs as fdl_lmhead_confidence, minus `ws`.
 * For callers that cannot allocate device memory: a plugin inside another
 * engine that owns every allocation, a loop where allocation is forbidden
 * after start-up, or code that cannot reach the host framework's allocator.
 * The scratch is a fixed array inside libfdl (FDL_NOALLOC_SCRATCH_BYTES,
 * held by every GPU that loads the library until the process exits), so:
 *  - batch * q_len must be at most FDL_NOALLOC_MAX_ROWS (else
 *    FDL_ERR_UNSUPPORTED, before any launch);
 *  - the first call on a device (of this function or of the three
 *    fdl_lmhead_noalloc_* calls below) looks the array up, with that device
 *    current, and queues the zeroing of its control words on `stream`, ahead
 *    of its kernel: make that first call before any stream capture;
 *  - every call on a device shares the array and leaves its counters at zero;
 *    calls whose kernels overlap on the GPU (other streams, other threads)
 *    race on it and must be serialised by the caller;
 *  - device-detected failures (a bounded wait that ran out) set bits in the
 *    array's own status word, which fdl_get_status cannot see: read them with
 *    fdl_lmhead_noalloc_status.  While FDL_DEV_TIMEOUT is set every row
 *    reports conf = -1, tok = -1.
 * It calls no cudaMalloc, cudaFree or other allocating routine.
 */
#define FDL_NOALLOC_MAX_ROWS 128
#define FDL_NOALLOC_SCRATCH_BYTES 606464 /* 256 control bytes + 296 x 128 partials of 16 B */
int fdl_lmhead_confidence_noalloc(const fdl_step_cfg* cfg, const void* rows,
                                  const void* w_lm, const uint8_t* row_active,
                                  float* conf, int32_t* tok, void* stream);

/* The allocation-free LM head's status word: synchronise `stream`, read it
 * into *status (bits FDL_DEV_*) and clear it.  Returns FDL_ERR_DEVICE_STATUS
 * if any bit was set, FDL_OK otherwise.  Allocates nothing. */
int fdl_lmhead_noalloc_status(void* stream, uint32_t* status);

/* Zero all control words of the allocation-free LM head's array (status and
 * counters), on `stream`; for use after a device-detected failure.  Allocates
 * nothing. */
int fdl_lmhead_noalloc_reset(void* stream);

/* fdl_check_wait_timeout aimed at the allocation-free LM head's status word:
 * one CTA's bounded wait runs out after limit_cycles (1e3 .. 2e9) and sets
 * FDL_DEV_TIMEOUT there, which fdl_lmhead_noalloc_status then reports.
 * A diagnostic of this library (no counterpart on the pages). */
int fdl_lmhead_noalloc_check_wait_timeout(long long limit_cycles, void* stream);

/*
 * Loop control of the block decode (technical review Algorithm 1: repeat
 * steps for as long as masked positions remain in the block; "Fast-dLLM v2" Level 2).
 * Reads n_masked_left [B] (device) after a step and, each only if given:
 *   any_masked (device int32): 1 if any sequence still has a masked unit
 *     position, else 0;
 *   step_count (device int32): incremented by one;
 *   while_handle: a cudaGraphConditionalHandle (cast to integer, 0 = none)
 *     of the WHILE node that wraps the step in a CUDA graph; it is set to 1
 *     while a masked position is left AND the incremented step_count is
 *     below q_len, so the graph keeps stepping without the host and never
 *     loops more than q_len times (each step commits at least one position;
 *     only a committed token equal to mask_id can leave one masked).  A
 *     non-zero while_handle requires step_count (else FDL_ERR_INVALID_ARG),
 *     zeroed by the caller before each graph launch.
 * One tiny kernel; capturable.
 */
int fdl_unit_status(const fdl_step_cfg* cfg, const int32_t* n_masked_left,
                    int32_t* any_masked, int32_t* step_count,
                    unsigned long long while_handle, void* stream);

/*
 * Block-level KV cache append ("Fast-dLLM v2" Level 3): after the block is
 * fully decoded, copy its rows k_blk/v_blk [B, Hkv, D, d] into the prefix
 * cache k_pre/v_pre [B, Hkv, cap_prefix, d] at rows len_pre[b] .. +D, then
 * len_pre[b] += D, on the device.  A sequence whose cache would overflow is
 * left unchanged and flagged (FDL_DEV_BAD_PREFIX_LEN in the workspace).
 */
int fdl_append_block(const fdl_step_cfg* cfg, const void* k_blk,
                     const void* v_blk, void* k_pre, void* v_pre,
                     int32_t* len_pre, void* ws, size_t ws_bytes, void* stream);

/* Synchronise `stream`, read the workspace status word into *status (bits
 * FDL_DEV_*) and clear it.  Returns FDL_ERR_DEVICE_STATUS if any bit was
 * set, FDL_OK otherwise. */
int fdl_get_status(void* ws, void* stream, uint32_t* status);

/*
 * Failure-detection self-check (no counterpart on the pages; a diagnostic of
 * this library).  Launches one CTA that waits on an mbarrier nothing ever
 * arrives on, with the same bounded wait every kernel uses but a bound of
 * limit_cycles SM clocks (1e3 .. 2e9; 1e6 is about half a millisecond), so
 * the wait runs out: the kernel sets FDL_DEV_TIMEOUT in the workspace status
 * word and returns.  fdl_get_status then reports FDL_ERR_DEVICE_STATUS with
 * that bit, and the CUDA context stays usable.  ws: at least 256 bytes,
 * 256-byte aligned (only its control words are touched).
 */
int fdl_check_wait_timeout(void* ws, size_t ws_bytes, long long limit_cycles, void* stream);

#ifdef __cplusplus
}
#endif
#endif /* FDL_H_ */
