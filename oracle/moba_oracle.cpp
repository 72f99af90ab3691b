// MoBA prefill forward: plain fp64 CPU oracle.
//
// TEST INFRASTRUCTURE ONLY. Only the tests, the smoke check and the bench's
// CPU-baseline leg may load this library. It shares no code, header or
// constant with the CUDA path and is never called by it.
//
// Sources (page title, section, equation):
//   [PT]  PaperTrace knowledge page "2.1.3 MoBA: 把历史块当成注意力专家"
//         (MoBA: history blocks as attention experts), sections 1-3.1, 5.2,
//         eq. (1)-(9), the worked example and Figure 1 of section 2.
//   [RD]  "MoBA：用于长上下文大语言模型的块注意力混合机制" (translated
//         official README): moba_naive = attention-mask view of the method.
//
// What is computed, per sequence b (cu_seqlens), query head h, kv head
// g = h / (Hq / Hkv), and query position p (0-indexed inside its sequence):
//   c      = floor(p / B)                       current block   [PT §2]
//   kbar_i = mean of the B raw keys of block i  (i < c)          [PT §1 eq.3]
//   s_i    = q_p . kbar_i                       (i < c only)     [PT §1 eq.3]
//   blocks later than c score -inf and are never chosen           [PT §2]
//   block c is always selected and uses one of the k slots        [PT §2, §2.1]
//   the other min(k-1, c) slots take the highest s_i, ties to the
//   lower block index (the pages leave ties open; lower index is the reading)
//   J      = all keys of the chosen history blocks + keys cB..p   [PT §2 eq.4-6]
//   o_p    = softmax(q K_J^T / sqrt(d)) V_J, ONE softmax over J   [PT §1 eq.4]
//   lse_p  = m + log(l)
// Every floating-point step is done in double; inputs are read exactly
// (bf16 bits widened, fp32 widened).
//
// Alternative routes to the same numbers, used by the tests as cross-checks:
//   oracle_forward_mask       builds the dense N x N boolean mask per head
//                             and runs masked dense softmax  ([RD] moba_naive,
//                             [PT §3.1] "naive implementation")
//   oracle_forward_two_branch keeps (m, l, u) for the current-block and the
//                             history branch and merges them with [PT §2]
//                             eq. (7)-(8).
//
// Routing variant ([PT §5.5], the paragraph on multi-head settings: a group
// of heads may share its candidate blocks, the routing score then has to
// aggregate the heads' needs): with shared routing every query head of a kv
// head's group gets the same blocks, chosen by the group's MEAN score
//   s_i = (1/grp) sum_{h in group} q_{p,h} . kbar_i
// under the same causal mask, forced own block and tie rule. (The pages do
// not fix the aggregate; the mean, which averages the heads' needs, is the
// reading taken.)
//
// Own-block variant ([PT §5.2], the paragraph on causal blocks: the own
// block's full mean would include keys after the query, so a correct gate
// either scores the own block by the mean of its keys up to the query -- the
// prefix mean -- or forces it in unscored; the forced branch is the default
// above). With the prefix mean, block c competes with the earlier blocks on
//   s_c = q_p . (1/(p - cB + 1)) sum_{j=cB..p} k_j
// and the k slots go to the best min(k, c+1) of blocks 0..c (ties to the lower
// index, so block c loses a tie). If block c is not chosen the query reads no
// key of its own block -- not even itself -- and its softmax runs over the
// chosen earlier blocks only (never empty: c = 0 leaves block 0 as the one
// candidate). With shared routing the group's mean of s_c is used.
//
// The *_routed entry points take routing as bit flags: bit 0 = shared by the
// group (0: per head, the default everywhere else), bit 1 = own block scored
// by its prefix mean (0: forced).
//
// Backward (oracle_backward_routed): gradients of L = sum(dO . O) with respect
// to q, k and v through the chosen blocks' keys. The block choice is a hard
// top-k and passes no gradient to the scores ([PT §5.3]: the top-k indices
// only build the mask; the loss flows back along the Q/K/V that were read).
// Per query row with candidate keys J, logits s_j = q.k_j / sqrt(d),
// P_j = softmax_J(s)_j, O = sum_j P_j v_j:
//   dP_j = dO . v_j,   D = sum_j P_j dP_j (= dO . O),   dS_j = P_j (dP_j - D)
//   dq  = sum_j dS_j k_j / sqrt(d),  dk_j += dS_j q / sqrt(d),  dv_j += P_j dO
// (the chain rule through the softmax; every query head adds into its kv
// head's dk, dv).

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <limits>
#include <vector>

#include <omp.h>

namespace {

constexpr int kBF16 = 0;
constexpr int kF32 = 1;

struct Problem {
  const void* q;
  const void* k;
  const void* v;
  int dtype;
  const int32_t* cu;  // [batch + 1]
  int batch, Hq, Hkv, d, B, topk;
  int shared;  // 1: the kv head's query heads share their blocks (mean score)
  int prefix;  // 1: the own block is scored by its prefix mean, not forced
};

bool routing_ok(int routing) { return routing >= 0 && routing <= 3; }

// Exact widening of a stored element to double.
inline double load(const void* p, int dtype, int64_t i) {
  if (dtype == kBF16) {
    uint32_t u = static_cast<uint32_t>(static_cast<const uint16_t*>(p)[i]) << 16;
    float f;
    std::memcpy(&f, &u, 4);
    return static_cast<double>(f);
  }
  return static_cast<double>(static_cast<const float*>(p)[i]);
}

inline int64_t q_off(const Problem& P, int64_t t, int h) {
  return (t * P.Hq + h) * static_cast<int64_t>(P.d);
}
inline int64_t kv_off(const Problem& P, int64_t t, int g) {
  return (t * P.Hkv + g) * static_cast<int64_t>(P.d);
}

int check(const Problem& P) {
  if (P.batch < 0 || P.Hq <= 0 || P.Hkv <= 0 || P.d <= 0 || P.B <= 0 ||
      P.topk <= 0 || P.Hq % P.Hkv != 0 || (P.dtype != kBF16 && P.dtype != kF32))
    return -1;
  for (int b = 0; b < P.batch; ++b)
    if (P.cu[b + 1] < P.cu[b]) return -1;
  return 0;
}

// Block means of one (sequence, kv head): [PT §1 eq.3]. Block i covers
// positions iB .. iB+B-1 of the sequence; a trailing partial block is
// averaged over the positions present (only full blocks are ever scored).
void block_means(const Problem& P, int b, int g, std::vector<double>& kbar) {
  const int64_t start = P.cu[b];
  const int64_t len = P.cu[b + 1] - start;
  const int64_t nb = (len + P.B - 1) / P.B;
  kbar.assign(static_cast<size_t>(nb * P.d), 0.0);
  for (int64_t i = 0; i < nb; ++i) {
    const int64_t j0 = i * P.B;
    const int64_t j1 = std::min<int64_t>(len, j0 + P.B);
    double* out = &kbar[static_cast<size_t>(i * P.d)];
    for (int64_t j = j0; j < j1; ++j)
      for (int x = 0; x < P.d; ++x) out[x] += load(P.k, P.dtype, kv_off(P, start + j, g) + x);
    const double inv_n = 1.0 / static_cast<double>(j1 - j0);
    for (int x = 0; x < P.d; ++x) out[x] *= inv_n;
  }
}

// Gate for one query: [PT §1 eq.3, §2, §2.1]. Writes the chosen blocks in
// ascending order (history first, then the current block c) padded with -1,
// and the relative score gap between the worst chosen and the best rejected
// candidate (infinity when nothing was left out). With P.prefix the own block
// is a scored candidate ([PT §5.2]) and may be left out; its keys are read at
// token kt (the query's token) of kv head g.
void select_blocks(const Problem& P, int64_t t, int h, int64_t p, const std::vector<double>& kbar,
                   int32_t* sel, double* gap, int64_t kt, int g) {
  const int64_t c = p / P.B;
  std::vector<std::pair<double, int64_t>> s;
  s.reserve(static_cast<size_t>(c + 1));
  const int grp = P.Hq / P.Hkv;
  const int h0 = P.shared ? (h / grp) * grp : h, nh_score = P.shared ? grp : 1;
  auto score = [&](const double* kb) {
    double sum = 0.0;
    for (int hh = h0; hh < h0 + nh_score; ++hh) {
      double acc = 0.0;
      for (int x = 0; x < P.d; ++x) acc += load(P.q, P.dtype, q_off(P, t, hh) + x) * kb[x];
      sum += acc;
    }
    return sum / nh_score;
  };
  for (int64_t i = 0; i < c; ++i) s.emplace_back(score(&kbar[static_cast<size_t>(i * P.d)]), i);
  if (P.prefix) {
    // prefix mean of the own block: keys cB .. p of the query's kv head
    const int64_t start = kt - p;
    std::vector<double> pm(static_cast<size_t>(P.d), 0.0);
    for (int64_t j = c * P.B; j <= p; ++j)
      for (int x = 0; x < P.d; ++x) pm[x] += load(P.k, P.dtype, kv_off(P, start + j, g) + x);
    for (int x = 0; x < P.d; ++x) pm[x] /= static_cast<double>(p - c * P.B + 1);
    s.emplace_back(score(pm.data()), c);
  }
  // Highest score first; equal scores: lower block index first.
  std::sort(s.begin(), s.end(), [](const std::pair<double, int64_t>& a,
                                   const std::pair<double, int64_t>& b2) {
    if (a.first != b2.first) return a.first > b2.first;
    return a.second < b2.second;
  });
  const int64_t n_cand = static_cast<int64_t>(s.size());
  const int64_t nh = std::min<int64_t>(P.prefix ? P.topk : P.topk - 1, n_cand);
  std::vector<int32_t> chosen;
  for (int64_t r = 0; r < nh; ++r) chosen.push_back(static_cast<int32_t>(s[r].second));
  if (!P.prefix) chosen.push_back(static_cast<int32_t>(c));
  std::sort(chosen.begin(), chosen.end());
  for (int r = 0; r < P.topk; ++r) sel[r] = r < static_cast<int>(chosen.size()) ? chosen[r] : -1;
  if (gap) {
    if (nh > 0 && nh < n_cand) {
      const double a = s[nh - 1].first, b2 = s[nh].first;
      const double den = std::max(std::max(std::fabs(a), std::fabs(b2)), 1e-30);
      *gap = std::fabs(a - b2) / den;
    } else {
      *gap = std::numeric_limits<double>::infinity();
    }
  }
}

// Whether the query reads its own block: always when it is forced, and with
// the prefix-mean gate only when the index row names it.
bool reads_own(const Problem& P, const int32_t* sel, int64_t c) {
  if (!P.prefix) return true;
  for (int r = 0; r < P.topk; ++r)
    if (sel[r] == c) return true;
  return false;
}

// Exact softmax attention of query (t, h) over the candidate keys of the
// chosen blocks: [PT §1 eq.4] with the current block causal [PT §2 eq.5].
// Entries of sel that are not in [0, c) are not history blocks; block c is
// attended up to position p (with P.prefix only if sel names it). Returns the
// number of keys attended.
// The query vector is read from Pq at (tq, hq): P itself, or a one-row view
// of the sampled q rows (oracle_forward_rows with q_rows).
int64_t attend_q(const Problem& P, const Problem& Pq, int b, int64_t t, int h, int64_t tq, int hq,
                 int64_t p, const int32_t* sel, double* o, double* lse) {
  const int64_t start = P.cu[b];
  const int g = h / (P.Hq / P.Hkv);
  const int64_t c = p / P.B;
  const double scale = 1.0 / std::sqrt(static_cast<double>(P.d));
  std::vector<int64_t> J;
  std::vector<int32_t> hist;
  for (int r = 0; r < P.topk; ++r)
    if (sel[r] >= 0 && sel[r] < c) hist.push_back(sel[r]);
  std::sort(hist.begin(), hist.end());
  hist.erase(std::unique(hist.begin(), hist.end()), hist.end());
  for (int32_t i : hist)
    for (int64_t j = static_cast<int64_t>(i) * P.B; j < static_cast<int64_t>(i + 1) * P.B; ++j)
      J.push_back(j);
  if (reads_own(P, sel, c))
    for (int64_t j = c * P.B; j <= p; ++j) J.push_back(j);

  std::vector<double> logit(J.size());
  double m = -std::numeric_limits<double>::infinity();
  for (size_t r = 0; r < J.size(); ++r) {
    double acc = 0.0;
    for (int x = 0; x < P.d; ++x)
      acc += load(Pq.q, P.dtype, q_off(Pq, tq, hq) + x) *
             load(P.k, P.dtype, kv_off(P, start + J[r], g) + x);
    logit[r] = acc * scale;
    m = std::max(m, logit[r]);
  }
  double l = 0.0;
  for (int x = 0; x < P.d; ++x) o[x] = 0.0;
  for (size_t r = 0; r < J.size(); ++r) {
    const double w = std::exp(logit[r] - m);
    l += w;
    for (int x = 0; x < P.d; ++x) o[x] += w * load(P.v, P.dtype, kv_off(P, start + J[r], g) + x);
  }
  for (int x = 0; x < P.d; ++x) o[x] /= l;
  if (lse) *lse = m + std::log(l);
  return static_cast<int64_t>(J.size());
}

// Backward contributions of one query row (t, h) at position p of sequence b:
// adds its dk, dv contributions to the kv head's rows of dk, dv and writes dq.
void backward_row(const Problem& P, const void* dout, int b, int64_t t, int h, int64_t p,
                  const int32_t* sel, double* dq, double* dk, double* dv) {
  const int64_t start = P.cu[b];
  const int g = h / (P.Hq / P.Hkv);
  const int64_t c = p / P.B;
  const double scale = 1.0 / std::sqrt(static_cast<double>(P.d));
  std::vector<int64_t> J;
  std::vector<int32_t> hist;
  for (int r = 0; r < P.topk; ++r)
    if (sel[r] >= 0 && sel[r] < c) hist.push_back(sel[r]);
  std::sort(hist.begin(), hist.end());
  hist.erase(std::unique(hist.begin(), hist.end()), hist.end());
  for (int32_t i : hist)
    for (int64_t j = static_cast<int64_t>(i) * P.B; j < static_cast<int64_t>(i + 1) * P.B; ++j)
      J.push_back(j);
  if (reads_own(P, sel, c))
    for (int64_t j = c * P.B; j <= p; ++j) J.push_back(j);
  const int d = P.d;
  std::vector<double> qv(d), dov(d);
  for (int x = 0; x < d; ++x) {
    qv[x] = load(P.q, P.dtype, q_off(P, t, h) + x);
    dov[x] = load(dout, P.dtype, q_off(P, t, h) + x);
  }
  std::vector<double> logit(J.size()), prob(J.size()), dp(J.size());
  double m = -std::numeric_limits<double>::infinity();
  for (size_t r = 0; r < J.size(); ++r) {
    double acc = 0.0;
    for (int x = 0; x < d; ++x) acc += qv[x] * load(P.k, P.dtype, kv_off(P, start + J[r], g) + x);
    logit[r] = acc * scale;
    m = std::max(m, logit[r]);
  }
  double l = 0.0;
  for (size_t r = 0; r < J.size(); ++r) l += (prob[r] = std::exp(logit[r] - m));
  double D = 0.0;
  for (size_t r = 0; r < J.size(); ++r) {
    prob[r] /= l;
    double acc = 0.0;
    for (int x = 0; x < d; ++x) acc += dov[x] * load(P.v, P.dtype, kv_off(P, start + J[r], g) + x);
    dp[r] = acc;
    D += prob[r] * acc;
  }
  double* dqr = dq + q_off(P, t, h);
  for (int x = 0; x < d; ++x) dqr[x] = 0.0;
  for (size_t r = 0; r < J.size(); ++r) {
    const double ds = prob[r] * (dp[r] - D);
    const int64_t kr = kv_off(P, start + J[r], g);
    for (int x = 0; x < d; ++x) {
      dqr[x] += ds * scale * load(P.k, P.dtype, kr + x);
      dk[kr + x] += ds * scale * qv[x];
      dv[kr + x] += prob[r] * dov[x];
    }
  }
}

int64_t attend(const Problem& P, int b, int64_t t, int h, int64_t p, const int32_t* sel, double* o,
               double* lse) {
  return attend_q(P, P, b, t, h, t, h, p, sel, o, lse);
}

// Sequence index of token t.
int seq_of(const Problem& P, int64_t t) {
  int b = 0;
  while (b + 1 <= P.batch && P.cu[b + 1] <= t) ++b;
  return b;
}

}  // namespace

extern "C" {

int oracle_num_threads() { return omp_get_max_threads(); }

// Block means, layout [batch][nb_max][Hkv][d]; slots past a sequence's last
// block are set to 0. [PT §1 eq.3]
int oracle_meanpool(const void* k, int dtype, const int32_t* cu, int batch, int Hkv, int d, int B,
                    int nb_max, double* kbar) {
  Problem P{nullptr, k, nullptr, dtype, cu, batch, Hkv, Hkv, d, B, 1};
  if (check(P)) return -1;
  std::memset(kbar, 0, sizeof(double) * static_cast<size_t>(batch) * nb_max * Hkv * d);
#pragma omp parallel for collapse(2) schedule(dynamic)
  for (int b = 0; b < batch; ++b)
    for (int g = 0; g < Hkv; ++g) {
      std::vector<double> kb;
      block_means(P, b, g, kb);
      const int64_t nb = static_cast<int64_t>(kb.size()) / d;
      for (int64_t i = 0; i < nb && i < nb_max; ++i)
        for (int x = 0; x < d; ++x)
          kbar[((static_cast<int64_t>(b) * nb_max + i) * Hkv + g) * d + x] = kb[i * d + x];
    }
  return 0;
}

// Gate + top-k for every (token, q head): idx [T][Hq][topk] int32, gap [T][Hq].
int oracle_gate_topk_routed(const void* q, const void* k, int dtype, const int32_t* cu, int batch,
                            int Hq, int Hkv, int d, int B, int topk, int routing, int32_t* idx,
                            double* gap) {
  Problem P{q, k, nullptr, dtype, cu, batch, Hq, Hkv, d, B, topk, routing & 1, routing >> 1};
  if (!routing_ok(routing)) return -1;
  if (check(P)) return -1;
  for (int b = 0; b < batch; ++b)
    for (int g = 0; g < Hkv; ++g) {
      std::vector<double> kb;
      block_means(P, b, g, kb);
      const int64_t len = cu[b + 1] - cu[b];
      const int grp = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic, 64)
      for (int64_t p = 0; p < len; ++p)
        for (int hh = 0; hh < grp; ++hh) {
          const int h = g * grp + hh;
          const int64_t t = cu[b] + p;
          select_blocks(P, t, h, p, kb, idx + (t * Hq + h) * topk, gap ? gap + t * Hq + h : nullptr,
                        t, g);
        }
    }
  return 0;
}

// Full forward by definition. If idx_in is non-null it supplies the chosen
// blocks per (token, head) instead of the gate (entries outside [0, c) are
// ignored; block c is always attended). idx_out, nkeys are optional.
int oracle_forward_routed(const void* q, const void* k, const void* v, int dtype,
                          const int32_t* cu, int batch, int Hq, int Hkv, int d, int B, int topk,
                          int routing, const int32_t* idx_in, double* out, double* lse,
                          int32_t* idx_out, int64_t* nkeys) {
  Problem P{q, k, v, dtype, cu, batch, Hq, Hkv, d, B, topk, routing & 1, routing >> 1};
  if (!routing_ok(routing)) return -1;
  if (check(P)) return -1;
  for (int b = 0; b < batch; ++b)
    for (int g = 0; g < Hkv; ++g) {
      std::vector<double> kb;
      if (!idx_in) block_means(P, b, g, kb);
      const int64_t len = cu[b + 1] - cu[b];
      const int grp = Hq / Hkv;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
      for (int64_t p = 0; p < len; ++p)
        for (int hh = 0; hh < grp; ++hh) {
          const int h = g * grp + hh;
          const int64_t t = cu[b] + p;
          std::vector<int32_t> sel(static_cast<size_t>(topk));
          if (idx_in)
            std::memcpy(sel.data(), idx_in + (t * Hq + h) * topk, sizeof(int32_t) * topk);
          else
            select_blocks(P, t, h, p, kb, sel.data(), nullptr, t, g);
          if (idx_out) std::memcpy(idx_out + (t * Hq + h) * topk, sel.data(), sizeof(int32_t) * topk);
          const int64_t n = attend(P, b, t, h, p, sel.data(), out + (t * Hq + h) * d,
                                   lse ? lse + t * Hq + h : nullptr);
          if (nkeys) nkeys[t * Hq + h] = n;
        }
    }
  return 0;
}

// Sampled forward: only the rows listed (row = t * Hq + h). Per row it
// writes out [nrows][d], lse [nrows], idx [nrows][topk], gap [nrows].
// If q_rows is non-null it holds the q vectors of the listed rows ([nrows][d],
// same dtype) and q is not read, so a caller need not hold all of q.
int oracle_forward_rows_routed(const void* q, const void* k, const void* v, int dtype,
                               const int32_t* cu, int batch, int Hq, int Hkv, int d, int B,
                               int topk, int routing, const int64_t* rows, int64_t nrows,
                               const int32_t* idx_in, double* out, double* lse, int32_t* idx_out,
                               double* gap, const void* q_rows) {
  Problem P{q, k, v, dtype, cu, batch, Hq, Hkv, d, B, topk, routing & 1, routing >> 1};
  // shared routing reads every head of the group: not with sampled q rows
  if (!routing_ok(routing) || ((routing & 1) && q_rows)) return -1;
  if (check(P)) return -1;
  const int64_t T = batch > 0 ? cu[batch] : 0;
  for (int64_t r = 0; r < nrows; ++r)
    if (rows[r] < 0 || rows[r] >= T * Hq) return -1;
  const int grp = Hq / Hkv;
  // Block means of every (sequence, kv head) that a sample touches.
  std::vector<int> need(static_cast<size_t>(batch) * Hkv, 0);
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t t = rows[r] / Hq;
    const int h = static_cast<int>(rows[r] % Hq);
    need[static_cast<size_t>(seq_of(P, t)) * Hkv + h / grp] = 1;
  }
  std::vector<std::vector<double>> means(static_cast<size_t>(batch) * Hkv);
  if (!idx_in) {
#pragma omp parallel for schedule(dynamic)
    for (int64_t bg = 0; bg < static_cast<int64_t>(batch) * Hkv; ++bg)
      if (need[bg]) block_means(P, static_cast<int>(bg / Hkv), static_cast<int>(bg % Hkv), means[bg]);
  }
#pragma omp parallel for schedule(dynamic, 4)
  for (int64_t r = 0; r < nrows; ++r) {
    const int64_t t = rows[r] / Hq;
    const int h = static_cast<int>(rows[r] % Hq);
    const int b = seq_of(P, t);
    const int64_t p = t - cu[b];
    // With q_rows, view row r as token 0 / head 0 of a one-row q array.
    Problem Pr = P;
    int64_t tq = t;
    int hq = h;
    if (q_rows) {
      Pr.q = static_cast<const char*>(q_rows) +
             r * static_cast<int64_t>(d) * (dtype == kBF16 ? 2 : 4);
      Pr.Hq = 1;
      tq = 0;
      hq = 0;
    }
    std::vector<int32_t> sel(static_cast<size_t>(topk));
    double gp = std::numeric_limits<double>::infinity();
    if (idx_in)
      std::memcpy(sel.data(), idx_in + r * topk, sizeof(int32_t) * topk);
    else
      select_blocks(Pr, tq, hq, p, means[static_cast<size_t>(b) * Hkv + h / grp], sel.data(),
                    &gp, t, h / grp);
    if (idx_out) std::memcpy(idx_out + r * topk, sel.data(), sizeof(int32_t) * topk);
    if (gap) gap[r] = gp;
    attend_q(P, Pr, b, t, h, tq, hq, p, sel.data(), out + r * d, lse ? lse + r : nullptr);
  }
  return 0;
}

// Per-head routing (the default) under the original names.
int oracle_gate_topk(const void* q, const void* k, int dtype, const int32_t* cu, int batch, int Hq,
                     int Hkv, int d, int B, int topk, int32_t* idx, double* gap) {
  return oracle_gate_topk_routed(q, k, dtype, cu, batch, Hq, Hkv, d, B, topk, 0, idx, gap);
}
int oracle_forward(const void* q, const void* k, const void* v, int dtype, const int32_t* cu,
                   int batch, int Hq, int Hkv, int d, int B, int topk, const int32_t* idx_in,
                   double* out, double* lse, int32_t* idx_out, int64_t* nkeys) {
  return oracle_forward_routed(q, k, v, dtype, cu, batch, Hq, Hkv, d, B, topk, 0, idx_in, out, lse,
                               idx_out, nkeys);
}
int oracle_forward_rows(const void* q, const void* k, const void* v, int dtype, const int32_t* cu,
                        int batch, int Hq, int Hkv, int d, int B, int topk, const int64_t* rows,
                        int64_t nrows, const int32_t* idx_in, double* out, double* lse,
                        int32_t* idx_out, double* gap, const void* q_rows) {
  return oracle_forward_rows_routed(q, k, v, dtype, cu, batch, Hq, Hkv, d, B, topk, 0, rows, nrows,
                                    idx_in, out, lse, idx_out, gap, q_rows);
}

// Backward by definition: dq [T][Hq][d], dk and dv [T][Hkv][d] (float64,
// overwritten). dout has q's shape and dtype. If idx_in is non-null it gives
// the chosen blocks per (token, q head), as in oracle_forward.
int oracle_backward_routed(const void* q, const void* k, const void* v, const void* dout, int dtype,
                           const int32_t* cu, int batch, int Hq, int Hkv, int d, int B, int topk,
                           int routing, const int32_t* idx_in, double* dq, double* dk,
                           double* dv) {
  Problem P{q, k, v, dtype, cu, batch, Hq, Hkv, d, B, topk, routing & 1, routing >> 1};
  if (check(P) || !routing_ok(routing) || !dout) return -1;
  const int64_t T = batch > 0 ? cu[batch] : 0;
  std::fill(dk, dk + T * Hkv * d, 0.0);
  std::fill(dv, dv + T * Hkv * d, 0.0);
  const int grp = Hq / Hkv;
  // one (sequence, kv head) per task: it alone writes that kv head's dk, dv
  // rows and its query heads' dq rows
#pragma omp parallel for schedule(dynamic)
  for (int64_t bg = 0; bg < static_cast<int64_t>(batch) * Hkv; ++bg) {
    const int b = static_cast<int>(bg / Hkv), g = static_cast<int>(bg % Hkv);
    std::vector<double> kb;
    if (!idx_in) block_means(P, b, g, kb);
    const int64_t len = cu[b + 1] - cu[b];
    std::vector<int32_t> sel(static_cast<size_t>(topk));
    for (int64_t p = 0; p < len; ++p)
      for (int hh = 0; hh < grp; ++hh) {
        const int h = g * grp + hh;
        const int64_t t = cu[b] + p;
        if (idx_in)
          std::memcpy(sel.data(), idx_in + (t * Hq + h) * topk, sizeof(int32_t) * topk);
        else
          select_blocks(P, t, h, p, kb, sel.data(), nullptr, t, g);
        backward_row(P, dout, b, t, h, p, sel.data(), dq, dk, dv);
      }
  }
  return 0;
}

// moba_naive view: per (sequence, head) build the dense boolean mask
// M[p][j] = (j <= p) and (block(j) is chosen for p), then run dense masked
// softmax row by row. Uses the gate's choice (or idx_in). [RD], [PT §3.1]
// With the prefix-mean gate (routing bit 1) the own block is on only when
// the row names it.
int oracle_forward_mask_routed(const void* q, const void* k, const void* v, int dtype,
                               const int32_t* cu, int batch, int Hq, int Hkv, int d, int B,
                               int topk, int routing, const int32_t* idx_in, double* out) {
  Problem P{q, k, v, dtype, cu, batch, Hq, Hkv, d, B, topk, routing & 1, routing >> 1};
  if (check(P) || !routing_ok(routing)) return -1;
  const int grp = Hq / Hkv;
  const double scale = 1.0 / std::sqrt(static_cast<double>(d));
  for (int b = 0; b < batch; ++b) {
    const int64_t start = cu[b];
    const int64_t len = cu[b + 1] - start;
#pragma omp parallel for schedule(dynamic)
    for (int h = 0; h < Hq; ++h) {
      const int g = h / grp;
      std::vector<double> kb;
      if (!idx_in) block_means(P, b, g, kb);
      std::vector<unsigned char> mask(static_cast<size_t>(len * len), 0);
      std::vector<int32_t> sel(static_cast<size_t>(topk));
      for (int64_t p = 0; p < len; ++p) {
        const int64_t t = start + p;
        if (idx_in)
          std::memcpy(sel.data(), idx_in + (t * Hq + h) * topk, sizeof(int32_t) * topk);
        else
          select_blocks(P, t, h, p, kb, sel.data(), nullptr, t, g);
        const int64_t c = p / B;
        for (int64_t j = 0; j <= p; ++j) {
          const int64_t bj = j / B;
          bool on = (bj == c) && !P.prefix;
          for (int r = 0; r < topk && !on; ++r) on = (sel[r] == bj);
          mask[static_cast<size_t>(p * len + j)] = on ? 1 : 0;
        }
      }
      std::vector<double> row(static_cast<size_t>(len));
      for (int64_t p = 0; p < len; ++p) {
        const int64_t t = start + p;
        double m = -std::numeric_limits<double>::infinity();
        for (int64_t j = 0; j < len; ++j) {
          if (!mask[static_cast<size_t>(p * len + j)]) continue;
          double acc = 0.0;
          for (int x = 0; x < d; ++x)
            acc += load(q, dtype, q_off(P, t, h) + x) * load(k, dtype, kv_off(P, start + j, g) + x);
          row[j] = acc * scale;
          m = std::max(m, row[j]);
        }
        double l = 0.0;
        double* o = out + (t * Hq + h) * d;
        for (int x = 0; x < d; ++x) o[x] = 0.0;
        for (int64_t j = 0; j < len; ++j) {
          if (!mask[static_cast<size_t>(p * len + j)]) continue;
          const double w = std::exp(row[j] - m);
          l += w;
          for (int x = 0; x < d; ++x) o[x] += w * load(v, dtype, kv_off(P, start + j, g) + x);
        }
        for (int x = 0; x < d; ++x) o[x] /= l;
      }
    }
  }
  return 0;
}

int oracle_forward_mask(const void* q, const void* k, const void* v, int dtype, const int32_t* cu,
                        int batch, int Hq, int Hkv, int d, int B, int topk, const int32_t* idx_in,
                        double* out) {
  return oracle_forward_mask_routed(q, k, v, dtype, cu, batch, Hq, Hkv, d, B, topk, 0, idx_in, out);
}

// Two-branch route: current block (causal, [PT §2 eq.5]) and history blocks
// (non-causal, eq.6) each keep (m, l, u); they are merged by eq.(7)-(8).
// With naive_sum != 0 it instead adds the two separately normalised outputs,
// the mistake [PT §2] warns against (kept so a test can show it differs).
int oracle_forward_two_branch(const void* q, const void* k, const void* v, int dtype,
                              const int32_t* cu, int batch, int Hq, int Hkv, int d, int B,
                              int topk, int naive_sum, double* out) {
  Problem P{q, k, v, dtype, cu, batch, Hq, Hkv, d, B, topk};
  if (check(P)) return -1;
  const int grp = Hq / Hkv;
  const double scale = 1.0 / std::sqrt(static_cast<double>(d));
  for (int b = 0; b < batch; ++b)
    for (int g = 0; g < Hkv; ++g) {
      std::vector<double> kb;
      block_means(P, b, g, kb);
      const int64_t start = cu[b];
      const int64_t len = cu[b + 1] - start;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
      for (int64_t p = 0; p < len; ++p)
        for (int hh = 0; hh < grp; ++hh) {
          const int h = g * grp + hh;
          const int64_t t = start + p;
          const int64_t c = p / B;
          std::vector<int32_t> sel(static_cast<size_t>(topk));
          select_blocks(P, t, h, p, kb, sel.data(), nullptr, t, g);
          // Branch statistics: m (max logit), l (sum of exp), u (unnormalised sum).
          auto branch = [&](const std::vector<int64_t>& J, double& m, double& l,
                            std::vector<double>& u) {
            m = -std::numeric_limits<double>::infinity();
            l = 0.0;
            u.assign(static_cast<size_t>(d), 0.0);
            std::vector<double> lg(J.size());
            for (size_t r = 0; r < J.size(); ++r) {
              double acc = 0.0;
              for (int x = 0; x < d; ++x)
                acc += load(q, dtype, q_off(P, t, h) + x) *
                       load(k, dtype, kv_off(P, start + J[r], g) + x);
              lg[r] = acc * scale;
              m = std::max(m, lg[r]);
            }
            for (size_t r = 0; r < J.size(); ++r) {
              const double w = std::exp(lg[r] - m);
              l += w;
              for (int x = 0; x < d; ++x) u[x] += w * load(v, dtype, kv_off(P, start + J[r], g) + x);
            }
          };
          std::vector<int64_t> Js, Jh;
          for (int64_t j = c * B; j <= p; ++j) Js.push_back(j);
          for (int r = 0; r < topk; ++r)
            if (sel[r] >= 0 && sel[r] < c)
              for (int64_t j = static_cast<int64_t>(sel[r]) * B; j < static_cast<int64_t>(sel[r] + 1) * B; ++j)
                Jh.push_back(j);
          double ms, ls, mh, lh;
          std::vector<double> us, uh;
          branch(Js, ms, ls, us);
          branch(Jh, mh, lh, uh);
          double* o = out + (t * Hq + h) * d;
          if (naive_sum) {
            for (int x = 0; x < d; ++x) o[x] = us[x] / ls + (lh > 0 ? uh[x] / lh : 0.0);
            continue;
          }
          // eq.(7)-(8); an empty history branch has l = 0 and contributes nothing.
          const double m = Jh.empty() ? ms : std::max(ms, mh);
          const double as = std::exp(ms - m);
          const double ah = Jh.empty() ? 0.0 : std::exp(mh - m);
          const double l = as * ls + ah * lh;
          for (int x = 0; x < d; ++x) o[x] = (as * us[x] + ah * uh[x]) / l;
        }
    }
  return 0;
}

// Dense causal softmax attention, [PT §1 eq.1] with the causal mask:
// every key j <= p of the query's own sequence.
int oracle_dense_causal(const void* q, const void* k, const void* v, int dtype, const int32_t* cu,
                        int batch, int Hq, int Hkv, int d, double* out, double* lse) {
  Problem P{q, k, v, dtype, cu, batch, Hq, Hkv, d, 1, 1};
  if (check(P)) return -1;
  const int grp = Hq / Hkv;
  const double scale = 1.0 / std::sqrt(static_cast<double>(d));
  for (int b = 0; b < batch; ++b) {
    const int64_t start = cu[b];
    const int64_t len = cu[b + 1] - start;
#pragma omp parallel for collapse(2) schedule(dynamic, 16)
    for (int64_t p = 0; p < len; ++p)
      for (int h = 0; h < Hq; ++h) {
        const int g = h / grp;
        const int64_t t = start + p;
        std::vector<double> lg(static_cast<size_t>(p + 1));
        double m = -std::numeric_limits<double>::infinity();
        for (int64_t j = 0; j <= p; ++j) {
          double acc = 0.0;
          for (int x = 0; x < d; ++x)
            acc += load(q, dtype, q_off(P, t, h) + x) * load(k, dtype, kv_off(P, start + j, g) + x);
          lg[j] = acc * scale;
          m = std::max(m, lg[j]);
        }
        double l = 0.0;
        double* o = out + (t * Hq + h) * d;
        for (int x = 0; x < d; ++x) o[x] = 0.0;
        for (int64_t j = 0; j <= p; ++j) {
          const double w = std::exp(lg[j] - m);
          l += w;
          for (int x = 0; x < d; ++x) o[x] += w * load(v, dtype, kv_off(P, start + j, g) + x);
        }
        for (int x = 0; x < d; ++x) o[x] /= l;
        if (lse) lse[t * Hq + h] = m + std::log(l);
      }
  }
  return 0;
}

}  // extern "C"
