// CPU oracle for one denoising step of the active block: plain C++, fp64.
//
// TEST INFRASTRUCTURE.  Only the tests, the smoke check and the CPU-baseline
// and reference legs of the benchmark load this library.  It shares no source,
// header, table or helper with the CUDA library, and neither calls the other.
//
// Every routine writes out the plain definition the pages give, with naive
// loops: an explicit visibility mask over the whole key list, the masked
// softmax of every (sequence, head, query row) on its own, full-vocabulary
// logits kept in memory, and the selection rules as loops over positions.
// Nothing is blocked, fused or reordered beyond running independent
// (sequence, head) pairs, vocabulary ranges and rows on separate threads.
// Every dot product sums its terms in index order; -ffp-contract=off keeps
// the compiler from fusing a multiply with its add, so results do not depend
// on the host.
//
// Sources (page title, then the passage):
//  * "Fast-dLLM v2: Efficient Block-Diffusion LLM" (paper digest), section 3.4:
//    "Attention Mask Design" (the training mask M_full and the inference mask
//    of Figure 7b), "Step 5: Token shift for prediction", and "Inference
//    Pipeline" Levels 1-3 (block cache, confidence threshold, sub-blocks).
//  * "Fast-dLLM: Reusing Bidirectional State and Spending Confidence on
//    Parallel Tokens" (technical review): section 2 eq. (3) (attention),
//    section 3 (PrefixCache and DualCache), section 4 Algorithm 2 (threshold
//    selection with its fallback), section 5.1 eq. (9) (heterogeneous error
//    budget), section 6 eq. (13) with Algorithm 3 (factor selection).
//
// Readings where the pages are silent (each is listed in the design notes):
//  * GQA: query head h reads KV head h / (Hq / Hkv).
//  * argmax over the full vocabulary, lowest index on a tie; the confidence is
//    the largest softmax probability, 1 / sum_v exp(l_v - l_max).
//  * the commit keeps conf >= tau, with tau the float32 the library receives;
//    the fallback and the sort of the factor / budget rules put the lower
//    position first among equal confidences.
//  * token shift: the row predicting unit position q_off + i is the hidden
//    state at position q_off + i - 1; for i = 0 the caller's h_prev.
//  * the attention output is rounded once to the storage dtype (bf16: round to
//    nearest, ties to even) before it serves as an LM-head row.
// Parity unpinned: that rounding point, and the GPU's fp32 exponentials; the
// parity tolerances and decision margins cover both.

#include <cmath>
#include <cstdint>
#include <cstring>
#include <algorithm>
#include <limits>
#include <thread>
#include <vector>

namespace {

// ------------------------------------------------------------ storage types

// How an input array is stored: its elements are upcast to double exactly.
enum Stored { kF32 = 0, kBF16 = 1, kF64 = 2 };

double upcast(const void* base, int stored, size_t i) {
  if (stored == kF64) return static_cast<const double*>(base)[i];
  if (stored == kF32) return static_cast<double>(static_cast<const float*>(base)[i]);
  // bf16: the upper half of an IEEE binary32 bit pattern
  uint32_t bits = static_cast<uint32_t>(static_cast<const uint16_t*>(base)[i]) << 16;
  float f;
  std::memcpy(&f, &bits, sizeof f);
  return static_cast<double>(f);
}

// bfloat16 keeps 8 significant bits.  Write x = m * 2^e with 0.5 <= |m| < 1
// and keep nearbyint(m * 2^8) (the default rounding mode rounds half to even).
// Normal numbers only; the step never produces bf16 subnormals.
double round_bf16(double x) {
  if (x == 0.0 || !std::isfinite(x)) return x;
  int e = 0;
  double m = std::frexp(x, &e);
  return std::ldexp(std::nearbyint(m * 256.0), e - 8);
}

double round_to(double x, int stored) {
  if (stored == kBF16) return round_bf16(x);
  if (stored == kF32) return static_cast<double>(static_cast<float>(x));
  return x;
}

int thread_count(int requested) {
  if (requested > 0) return requested;
  unsigned n = std::thread::hardware_concurrency();
  return n ? static_cast<int>(n) : 1;
}

// Run body(i) for i in [0, n) over `threads` threads, contiguous ranges.
template <class F>
void parallel_for(int64_t n, int threads, F body) {
  threads = std::max<int64_t>(1, std::min<int64_t>(threads, n));
  if (threads == 1) {
    for (int64_t i = 0; i < n; ++i) body(i);
    return;
  }
  std::vector<std::thread> pool;
  for (int t = 0; t < threads; ++t) {
    int64_t lo = n * t / threads, hi = n * (t + 1) / threads;
    pool.emplace_back([=] { for (int64_t i = lo; i < hi; ++i) body(i); });
  }
  for (auto& th : pool) th.join();
}

// ------------------------------------------------------------------ masks

// Block index of an absolute position: the prompt is block 0, the generated
// answer is cut into blocks of D after it (v2 digest, Level 1).
int64_t block_id(int64_t pos, int64_t prompt_len, int64_t D) {
  return pos < prompt_len ? 0 : 1 + (pos - prompt_len) / D;
}

// Block-causal visibility (v2 digest, Figure 7b): a query sees every key of
// its own block (bidirectional inside the block) and of every earlier block
// (causal across blocks).  Full attention (technical review, section 3: the
// DualCache of a full-attention dLLM) sees every key.
bool visible(int64_t q_pos, int64_t k_pos, int64_t prompt_len, int64_t D, bool full) {
  if (full) return true;
  return block_id(k_pos, prompt_len, D) <= block_id(q_pos, prompt_len, D);
}

// ------------------------------------------------------------- attention

// One query row over an explicit key list (technical review eq. (3)):
// s_j = q.k_j / sqrt(d) for the visible keys, p = softmax(s), out = sum_j p_j v_j.
// Keys that are not visible take no part (their probability is exactly zero).
// Returns false if no key is visible (the output is then left at zero).
template <class KeyAt, class ValAt>
bool attend_row(int d, const double* q, int64_t n_keys, const uint8_t* vis,
                KeyAt key, ValAt val, double* out, std::vector<double>& s) {
  s.assign(n_keys, 0.0);
  const double scale = std::sqrt(static_cast<double>(d));
  double mx = -std::numeric_limits<double>::infinity();
  bool any = false;
  for (int64_t j = 0; j < n_keys; ++j) {
    if (!vis[j]) continue;
    double dot = 0.0;
    for (int c = 0; c < d; ++c) dot += q[c] * key(j, c);
    s[j] = dot / scale;
    if (!any || s[j] > mx) mx = s[j];
    any = true;
  }
  for (int c = 0; c < d; ++c) out[c] = 0.0;
  if (!any) return false;
  double sum = 0.0;
  for (int64_t j = 0; j < n_keys; ++j) {
    if (!vis[j]) continue;
    s[j] = std::exp(s[j] - mx);
    sum += s[j];
  }
  for (int64_t j = 0; j < n_keys; ++j) {
    if (!vis[j]) continue;
    const double p = s[j] / sum;
    for (int c = 0; c < d; ++c) out[c] += p * val(j, c);
  }
  return true;
}

struct AttnShape {
  int B, q_len, Hq, Hkv, d, D;
  int64_t cap_pre, cap_suf;
  int q_off;
};

// Attention of the active unit's queries (v2 digest, "Inference Pipeline"
// Level 3 and Figure 7b; technical review section 3 for DualCache).
// Keys of sequence b: prefix cache rows [0, len_pre[b]) at positions
// 0 .. Lp-1, the D block rows at Lp .. Lp+D-1 and, for DualCache, suffix cache
// rows [0, len_suf[b]) after them.  Query r of the unit sits at position
// Lp + q_off + r.  With a suffix the mask is full attention, otherwise
// block-causal.  `only` (may be null) limits the work to the flagged
// [b, r] query rows; the other rows of `out` are left as they are.
void attention_step(const AttnShape& a, int stored, const void* q, const void* k_pre,
                    const void* v_pre, const int64_t* len_pre, const int64_t* prompt_len,
                    const void* k_blk, const void* v_blk, const void* k_suf,
                    const void* v_suf, const int64_t* len_suf, const uint8_t* only,
                    double* out, int threads) {
  const bool dual = k_suf != nullptr;
  const int group = a.Hq / a.Hkv;
  parallel_for(static_cast<int64_t>(a.B) * a.Hq, thread_count(threads), [&](int64_t bh) {
    const int b = static_cast<int>(bh / a.Hq), h = static_cast<int>(bh % a.Hq);
    const int kvh = h / group;
    const int64_t Lp = len_pre[b];
    const int64_t Ls = dual ? len_suf[b] : 0;
    const int64_t n_keys = Lp + a.D + Ls;
    const size_t pre0 = (static_cast<size_t>(b) * a.Hkv + kvh) * a.cap_pre * a.d;
    const size_t blk0 = (static_cast<size_t>(b) * a.Hkv + kvh) * a.D * a.d;
    const size_t suf0 = (static_cast<size_t>(b) * a.Hkv + kvh) * a.cap_suf * a.d;
    auto elem = [&](const void* pre, const void* blk, const void* suf, int64_t j, int c) {
      if (j < Lp) return upcast(pre, stored, pre0 + j * a.d + c);
      if (j < Lp + a.D) return upcast(blk, stored, blk0 + (j - Lp) * a.d + c);
      return upcast(suf, stored, suf0 + (j - Lp - a.D) * a.d + c);
    };
    auto key = [&](int64_t j, int c) { return elem(k_pre, k_blk, k_suf, j, c); };
    auto val = [&](int64_t j, int c) { return elem(v_pre, v_blk, v_suf, j, c); };
    std::vector<uint8_t> vis(n_keys);
    std::vector<double> qrow(a.d), s;
    for (int r = 0; r < a.q_len; ++r) {
      if (only && !only[static_cast<size_t>(b) * a.q_len + r]) continue;
      const int64_t q_pos = Lp + a.q_off + r;
      for (int64_t j = 0; j < n_keys; ++j)
        vis[j] = visible(q_pos, j, prompt_len[b], a.D, dual);
      const size_t q0 = ((static_cast<size_t>(b) * a.q_len + r) * a.Hq + h) * a.d;
      for (int c = 0; c < a.d; ++c) qrow[c] = upcast(q, stored, q0 + c);
      attend_row(a.d, qrow.data(), n_keys, vis.data(), key, val, out + q0, s);
    }
  });
}

// PrefixCache attention (technical review, section 3, and the PrefixCache
// branch of Algorithm 1): only the prompt and the finished answer are cached;
// the n recomputed rows (the active block and the masked suffix after it)
// attend with full attention to the cached prefix rows [0, len_pre[b])
// followed by their own fresh K/V.
void prefixcache_attention(int B, int n, int Hq, int Hkv, int d, int64_t cap_pre,
                           int stored, const void* q, const void* k_pre,
                           const void* v_pre, const int64_t* len_pre,
                           const void* k_new, const void* v_new, double* out,
                           int threads) {
  const int group = Hq / Hkv;
  parallel_for(static_cast<int64_t>(B) * Hq, thread_count(threads), [&](int64_t bh) {
    const int b = static_cast<int>(bh / Hq), h = static_cast<int>(bh % Hq);
    const int kvh = h / group;
    const int64_t Lp = len_pre[b];
    const int64_t n_keys = Lp + n;
    const size_t pre0 = (static_cast<size_t>(b) * Hkv + kvh) * cap_pre * d;
    const size_t new0 = (static_cast<size_t>(b) * Hkv + kvh) * static_cast<size_t>(n) * d;
    auto key = [&](int64_t j, int c) {
      return j < Lp ? upcast(k_pre, stored, pre0 + j * d + c)
                    : upcast(k_new, stored, new0 + (j - Lp) * d + c);
    };
    auto val = [&](int64_t j, int c) {
      return j < Lp ? upcast(v_pre, stored, pre0 + j * d + c)
                    : upcast(v_new, stored, new0 + (j - Lp) * d + c);
    };
    std::vector<uint8_t> vis(n_keys, 1);
    std::vector<double> qrow(d), s;
    for (int r = 0; r < n; ++r) {
      const size_t q0 = ((static_cast<size_t>(b) * n + r) * Hq + h) * d;
      for (int c = 0; c < d; ++c) qrow[c] = upcast(q, stored, q0 + c);
      attend_row(d, qrow.data(), n_keys, vis.data(), key, val, out + q0, s);
    }
  });
}

// ------------------------------------------------------------- LM head

// Logits l = W h over the full vocabulary for the flagged rows, then per row:
// tok = argmax l (the lowest index on a tie), conf = the probability the
// softmax gives it = 1 / sum_v exp(l_v - l_max) (v2 digest, Level 2;
// technical review Algorithm 2), and the top-1 minus top-2 logit gap (a
// decision margin for the tests; 0 on a tie).  `rows` is [R, H] in fp64,
// `w` is [V, H] as stored.  The logits of all rows are held in memory.
void lmhead_confidence(int64_t R, int64_t V, int64_t H, const double* rows,
                       const void* w, int w_stored, const uint8_t* only,
                       int64_t* tok, double* conf, double* gap, int threads) {
  std::vector<int64_t> sel;
  for (int64_t r = 0; r < R; ++r)
    if (!only || only[r]) sel.push_back(r);
  const int64_t n = static_cast<int64_t>(sel.size());
  if (n == 0) return;
  // rows of the selected set, transposed to [H][n] so that one weight element
  // meets every selected row in turn
  std::vector<double> xt(static_cast<size_t>(H) * n);
  for (int64_t i = 0; i < n; ++i)
    for (int64_t k = 0; k < H; ++k) xt[k * n + i] = rows[sel[i] * H + k];
  std::vector<double> logits(static_cast<size_t>(n) * V);
  const int T = thread_count(threads);
  parallel_for(T, T, [&](int64_t t) {
    const int64_t v0 = V * t / T, v1 = V * (t + 1) / T;
    std::vector<double> wrow(H), acc(n);
    for (int64_t v = v0; v < v1; ++v) {
      for (int64_t k = 0; k < H; ++k) wrow[k] = upcast(w, w_stored, v * H + k);
      std::fill(acc.begin(), acc.end(), 0.0);
      // each logit l[i][v] = sum_k x[i][k] w[v][k], its terms added in k order
      for (int64_t k = 0; k < H; ++k) {
        const double wk = wrow[k];
        const double* x = &xt[k * n];
        for (int64_t i = 0; i < n; ++i) acc[i] += x[i] * wk;
      }
      for (int64_t i = 0; i < n; ++i) logits[i * V + v] = acc[i];
    }
  });
  parallel_for(n, T, [&](int64_t i) {
    const double* l = &logits[i * V];
    int64_t best = 0;
    double top1 = l[0], top2 = -std::numeric_limits<double>::infinity();
    for (int64_t v = 1; v < V; ++v) {
      if (l[v] > top1) {
        top2 = top1;
        top1 = l[v];
        best = v;
      } else if (l[v] > top2) {
        top2 = l[v];
      }
    }
    double sum = 0.0;
    for (int64_t v = 0; v < V; ++v) sum += std::exp(l[v] - top1);
    const int64_t r = sel[i];
    tok[r] = best;
    conf[r] = 1.0 / sum;
    gap[r] = V > 1 ? top1 - top2 : 0.0;
  });
}

// LM-head input rows with the token shift (v2 digest, section 3.4, Step 5):
// the row that predicts unit position q_off + i is the hidden state of the
// position before it, i.e. source row i - 1; row 0 takes the caller's h_prev
// (the last position before the unit).  Without the shift, row i is source
// row i.  src is [B, q_len, H], h_prev [B, H], rows [B, q_len, H].
void shifted_rows(int B, int q_len, int64_t H, int shift, const double* src,
                  const double* h_prev, double* rows) {
  for (int b = 0; b < B; ++b)
    for (int i = 0; i < q_len; ++i) {
      const double* from;
      if (!shift) from = src + (static_cast<size_t>(b) * q_len + i) * H;
      else if (i == 0) from = h_prev + static_cast<size_t>(b) * H;
      else from = src + (static_cast<size_t>(b) * q_len + i - 1) * H;
      double* to = rows + (static_cast<size_t>(b) * q_len + i) * H;
      for (int64_t k = 0; k < H; ++k) to[k] = from[k];
    }
}

// ------------------------------------------------------------ selection

enum Rule { kThreshold = 0, kFactor = 1, kBudget = 2 };

// Technical review Algorithm 2: S = {i in M : c_i >= tau}; if S is empty and
// M is not, S = {the position with the largest c_i} (the lowest position among
// equal confidences).
std::vector<int> threshold_select(const std::vector<int>& M, const double* c, double tau) {
  std::vector<int> S;
  for (int p : M)
    if (c[p] >= tau) S.push_back(p);
  if (S.empty() && !M.empty()) {
    int best = M[0];
    for (int p : M)
      if (c[p] > c[best]) best = p;
    S.push_back(best);
  }
  return S;
}

// M sorted by decreasing confidence, the lower position first on a tie
// (Algorithm 3 sorts by confidence; the tie order is a reading).
std::vector<int> by_confidence(std::vector<int> M, const double* c) {
  std::stable_sort(M.begin(), M.end(), [&](int a, int b) {
    if (c[a] != c[b]) return c[a] > c[b];
    return a < b;
  });
  return M;
}

// Technical review section 6, eq. (13) with Algorithm 3: with the positions in
// decreasing confidence c_(1) >= c_(2) >= ..., keep the largest n for which
// (n + 1) (1 - c_(n)) < f; if no n qualifies, the first position alone.
std::vector<int> factor_select(const std::vector<int>& M, const double* c, double f) {
  std::vector<int> order = by_confidence(M, c);
  size_t best = 0;
  for (size_t n = 1; n <= order.size(); ++n)
    if (static_cast<double>(n + 1) * (1.0 - c[order[n - 1]]) < f) best = n;
  if (best == 0) best = std::min<size_t>(1, order.size());
  order.resize(best);
  return order;
}

// Technical review section 5.1, eq. (9): errors eps_j = 1 - c_j; a group is
// certified when sum_j eps_j + max_j eps_j < 1.  With the positions in
// decreasing confidence, keep the largest certified prefix; if none, the first
// position alone.
bool budget_ok(const std::vector<double>& eps) {
  double sum = 0.0, mx = 0.0;
  for (double e : eps) {
    sum += e;
    mx = std::max(mx, e);
  }
  return sum + mx < 1.0;
}

std::vector<int> budget_select(const std::vector<int>& M, const double* c) {
  std::vector<int> order = by_confidence(M, c);
  size_t best = 0;
  std::vector<double> eps;
  for (size_t n = 1; n <= order.size(); ++n) {
    eps.push_back(1.0 - c[order[n - 1]]);
    if (budget_ok(eps)) best = n;
  }
  if (best == 0) best = std::min<size_t>(1, order.size());
  order.resize(best);
  return order;
}

std::vector<int> select(int rule, double param, const std::vector<int>& M, const double* c) {
  if (rule == kFactor) return factor_select(M, c, param);
  if (rule == kBudget) return budget_select(M, c);
  return threshold_select(M, c, param);
}

// The commit over the active unit [q_off, q_off + q_len) of every block
// (technical review Algorithm 2; the sub-block as the thresholding unit, v2
// digest "Sub-block size as a decoding granularity knob").  Candidates are
// the unit's positions still holding the mask token (v2 digest Level 1).
// conf / tok are [B, q_len], indexed by unit position.
void commit(int B, int D, int q_off, int q_len, int64_t mask_id, int rule, double param,
            const int64_t* block_tokens, const double* conf, const int64_t* tok,
            int64_t* new_tokens, uint8_t* committed, int64_t* n_committed,
            int64_t* n_masked_left) {
  std::vector<double> c(D);
  for (int b = 0; b < B; ++b) {
    const int64_t* bt = block_tokens + static_cast<size_t>(b) * D;
    int64_t* nt = new_tokens + static_cast<size_t>(b) * D;
    uint8_t* cm = committed + static_cast<size_t>(b) * D;
    std::vector<int> M;
    for (int p = 0; p < D; ++p) {
      nt[p] = bt[p];
      cm[p] = 0;
      c[p] = 0.0;
    }
    for (int p = q_off; p < q_off + q_len; ++p) {
      c[p] = conf[static_cast<size_t>(b) * q_len + (p - q_off)];
      if (bt[p] == mask_id) M.push_back(p);
    }
    std::vector<int> S = M.empty() ? std::vector<int>() : select(rule, param, M, c.data());
    for (int p : S) {
      nt[p] = tok[static_cast<size_t>(b) * q_len + (p - q_off)];
      cm[p] = 1;
    }
    n_committed[b] = static_cast<int64_t>(S.size());
    int64_t left = 0;
    for (int p = q_off; p < q_off + q_len; ++p) left += nt[p] == mask_id;
    n_masked_left[b] = left;
  }
}

}  // namespace

// =================================================================== C ABI
//
// Plain host pointers.  Arrays are row-major and contiguous; "stored" arrays
// are f32, bf16 (uint16 bit patterns) or f64 as the `stored` code says.
// Integer arrays are int64.  Nothing is allocated for the caller; nothing is
// kept between calls.  `threads` <= 0 means one per hardware thread.

extern "C" {

int orc_version(void) { return 2; }

void orc_round(int64_t n, const double* x, int stored, double* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = round_to(x[i], stored);
}

// M_full over the concatenation [x_t ; x_0] of length 2L (v2 digest,
// "Attention Mask Design"): [[M_BD, M_OBC], [0, M_BC]].  M_BD: noised i sees
// noised j iff they share a block.  M_OBC: noised i sees clean j iff j's block
// is strictly earlier.  M_BC: clean i sees clean j iff j's block is the same
// or earlier.  Clean never sees noised.  out is [2L, 2L].
void orc_training_mask(int64_t L, int64_t D, uint8_t* out) {
  const int64_t N = 2 * L;
  for (int64_t i = 0; i < N; ++i) {
    for (int64_t j = 0; j < N; ++j) {
      const bool qi_noised = i < L, kj_noised = j < L;
      const int64_t bi = (qi_noised ? i : i - L) / D;
      const int64_t bj = (kj_noised ? j : j - L) / D;
      bool v;
      if (qi_noised && kj_noised) v = bi == bj;          // M_BD
      else if (qi_noised) v = bj < bi;                    // M_OBC
      else if (kj_noised) v = false;                      // zero quadrant
      else v = bj <= bi;                                  // M_BC
      out[i * N + j] = v;
    }
  }
}

void orc_block_ids(int64_t n, const int64_t* pos, int64_t prompt_len, int64_t D,
                   int64_t* out) {
  for (int64_t i = 0; i < n; ++i) out[i] = block_id(pos[i], prompt_len, D);
}

void orc_inference_visibility(int64_t nq, const int64_t* q_pos, int64_t nk,
                              const int64_t* k_pos, int64_t prompt_len, int64_t D,
                              int full, uint8_t* out) {
  for (int64_t i = 0; i < nq; ++i)
    for (int64_t j = 0; j < nk; ++j)
      out[i * nk + j] = visible(q_pos[i], k_pos[j], prompt_len, D, full != 0);
}

// softmax(q k^T / sqrt(d)) v over an explicit [n, m] visibility mask
// (technical review eq. (3)); q [n, d], k and v [m, d], out [n, d], all fp64.
void orc_masked_attention(int64_t n, int64_t m, int d, const double* q, const double* k,
                          const double* v, const uint8_t* vis, double* out) {
  std::vector<double> s;
  auto key = [&](int64_t j, int c) { return k[j * d + c]; };
  auto val = [&](int64_t j, int c) { return v[j * d + c]; };
  for (int64_t i = 0; i < n; ++i)
    attend_row(d, q + i * d, m, vis + i * m, key, val, out + i * d, s);
}

void orc_attention_step(int B, int q_len, int Hq, int Hkv, int d, int D, int64_t cap_pre,
                        int64_t cap_suf, int q_off, int stored, const void* q,
                        const void* k_pre, const void* v_pre, const int64_t* len_pre,
                        const int64_t* prompt_len, const void* k_blk, const void* v_blk,
                        const void* k_suf, const void* v_suf, const int64_t* len_suf,
                        double* out, int threads) {
  AttnShape a{B, q_len, Hq, Hkv, d, D, cap_pre, cap_suf, q_off};
  attention_step(a, stored, q, k_pre, v_pre, len_pre, prompt_len, k_blk, v_blk, k_suf,
                 v_suf, len_suf, nullptr, out, threads);
}

void orc_prefixcache_attention(int B, int n, int Hq, int Hkv, int d, int64_t cap_pre,
                               int stored, const void* q, const void* k_pre,
                               const void* v_pre, const int64_t* len_pre,
                               const void* k_new, const void* v_new, double* out,
                               int threads) {
  prefixcache_attention(B, n, Hq, Hkv, d, cap_pre, stored, q, k_pre, v_pre, len_pre,
                        k_new, v_new, out, threads);
}

void orc_shifted_rows(int B, int q_len, int64_t H, int shift, const double* src,
                      const double* h_prev, double* rows) {
  shifted_rows(B, q_len, H, shift, src, h_prev, rows);
}

void orc_lmhead_confidence(int64_t R, int64_t V, int64_t H, const double* rows,
                           const void* w, int w_stored, int64_t* tok, double* conf,
                           double* gap, int threads) {
  lmhead_confidence(R, V, H, rows, w, w_stored, nullptr, tok, conf, gap, threads);
}

// Selection rules over one list of masked positions; conf is indexed by
// position.  Writes the selected positions in rule order and returns how many.
int orc_select(int rule, double param, int n_masked, const int* masked, const double* conf,
               int* out) {
  std::vector<int> M(masked, masked + n_masked);
  std::vector<int> S = M.empty() ? std::vector<int>() : select(rule, param, M, conf);
  for (size_t i = 0; i < S.size(); ++i) out[i] = S[i];
  return static_cast<int>(S.size());
}

int orc_budget_ok(int n, const double* eps) {
  return budget_ok(std::vector<double>(eps, eps + n)) ? 1 : 0;
}

void orc_commit(int B, int D, int q_off, int q_len, int64_t mask_id, int rule, double param,
                const int64_t* block_tokens, const double* conf, const int64_t* tok,
                int64_t* new_tokens, uint8_t* committed, int64_t* n_committed,
                int64_t* n_masked_left) {
  commit(B, D, q_off, q_len, mask_id, rule, param, block_tokens, conf, tok, new_tokens,
         committed, n_committed, n_masked_left);
}

// One denoising step of the active unit, from its definition:
//  1. attention of the unit's queries over the prefix (+ suffix) cache and the
//     block (v2 digest Figure 7b; technical review section 3);
//  2. that output rounded to the storage dtype;
//  3. the LM-head rows: `hidden` [B, q_len, H] if given, else the rounded
//     attention output (one layer chained), then the token shift (v2 digest,
//     Step 5): row i takes the source row i - 1, row 0 the caller's h_prev;
//  4. full-vocabulary argmax and confidence for the rows whose target position
//     still holds the mask token; the others report conf = -1 and tok = -1;
//  5. the threshold commit (tau as float32, compared in double).
// Also writes the decision margins the parity tests rely on: the logit gap of
// each active row and, where the fallback fires, the relative confidence gap
// between the two best candidates (+inf elsewhere).
//
// Incremental form: when `redo_q` / `redo_lm` are given ([B, q_len] flags),
// only the flagged attention query rows and LM-head rows are recomputed and
// every other value in `attn`, `conf`, `tok` and `logit_gap` is taken from
// what those buffers hold (the result of an earlier call on the same case);
// rounding, rows, commit and margins are always rebuilt.  Every row is
// independent of the others, so this gives exactly the result of a full call.
struct orc_step_cfg {
  int B, q_len, Hq, Hkv, d, D, q_off;
  int64_t cap_pre, cap_suf;
  int64_t H, V, mask_id;
  int shift, stored, w_stored, threads;
  float tau;
};

int orc_denoise_step(const orc_step_cfg* c, const void* q, const void* k_pre,
                     const void* v_pre, const int64_t* len_pre, const int64_t* prompt_len,
                     const void* k_blk, const void* v_blk, const void* k_suf,
                     const void* v_suf, const int64_t* len_suf, const void* hidden,
                     const void* h_prev, const void* w, const int64_t* block_tokens,
                     const uint8_t* redo_q, const uint8_t* redo_lm,
                     double* attn, double* attn_rounded, double* rows, uint8_t* active,
                     double* conf, int64_t* tok, double* logit_gap, int64_t* new_tokens,
                     uint8_t* committed, int64_t* n_committed, int64_t* n_masked_left,
                     double* cand_gap) {
  const int B = c->B, q_len = c->q_len;
  const int64_t H = c->H;
  if (c->Hkv <= 0 || c->Hq % c->Hkv != 0) return -1;
  if (hidden == nullptr && H != static_cast<int64_t>(c->Hq) * c->d) return -1;
  if (c->shift && h_prev == nullptr) return -1;
  const size_t n_attn = static_cast<size_t>(B) * q_len * c->Hq * c->d;
  const size_t n_rows = static_cast<size_t>(B) * q_len;

  // 1-2. attention and its rounding
  AttnShape a{B, q_len, c->Hq, c->Hkv, c->d, c->D, c->cap_pre, c->cap_suf, c->q_off};
  if (!redo_q) std::fill(attn, attn + n_attn, 0.0);
  attention_step(a, c->stored, q, k_pre, v_pre, len_pre, prompt_len, k_blk, v_blk, k_suf,
                 v_suf, len_suf, redo_q, attn, c->threads);
  for (size_t i = 0; i < n_attn; ++i) attn_rounded[i] = round_to(attn[i], c->stored);

  // 3. LM-head rows with the token shift
  std::vector<double> source(n_rows * H), prev;
  for (size_t i = 0; i < n_rows * static_cast<size_t>(H); ++i)
    source[i] = hidden ? upcast(hidden, c->stored, i) : attn_rounded[i];
  if (c->shift) {
    prev.resize(static_cast<size_t>(B) * H);
    for (size_t i = 0; i < prev.size(); ++i) prev[i] = upcast(h_prev, c->stored, i);
  }
  shifted_rows(B, q_len, H, c->shift, source.data(), prev.data(), rows);

  // 4. LM head over the rows whose target position is still masked
  std::vector<uint8_t> lm_rows(n_rows);
  for (int b = 0; b < B; ++b)
    for (int i = 0; i < q_len; ++i) {
      const size_t r = static_cast<size_t>(b) * q_len + i;
      active[r] = block_tokens[static_cast<size_t>(b) * c->D + c->q_off + i] == c->mask_id;
      lm_rows[r] = active[r] && (!redo_lm || redo_lm[r]);
    }
  lmhead_confidence(static_cast<int64_t>(n_rows), c->V, H, rows, w, c->w_stored,
                    lm_rows.data(), tok, conf, logit_gap, c->threads);
  for (size_t r = 0; r < n_rows; ++r)
    if (!active[r]) {
      conf[r] = -1.0;
      tok[r] = -1;
      logit_gap[r] = std::numeric_limits<double>::infinity();
    }

  // 5. threshold commit
  const double tau = static_cast<double>(c->tau);
  commit(B, c->D, c->q_off, q_len, c->mask_id, kThreshold, tau, block_tokens, conf, tok,
         new_tokens, committed, n_committed, n_masked_left);

  // margins of the fallback decision
  for (int b = 0; b < B; ++b) {
    std::vector<double> cs;
    for (int i = 0; i < q_len; ++i)
      if (active[static_cast<size_t>(b) * q_len + i])
        cs.push_back(conf[static_cast<size_t>(b) * q_len + i]);
    std::sort(cs.begin(), cs.end(), [](double x, double y) { return x > y; });
    cand_gap[b] = (cs.size() >= 2 && cs[0] < tau)
                      ? (cs[0] - cs[1]) / cs[0]
                      : std::numeric_limits<double>::infinity();
  }
  return 0;
}

}  // extern "C"
