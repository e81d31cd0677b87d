// Exact-attention oracle: plain, slow, fp64, CPU only.
//
// TEST INFRASTRUCTURE. Only the test suite, the package smoke check and the
// benchmark's CPU-baseline leg may load this code. It shares nothing with the
// CUDA library (no header, helper, table or constant): it is the definition of
// the operation written out, so a reader can check it against the sources by eye.
//
// Sources, cited by title and section:
//   [jsqmd]   "From GPU memory access to code: how FlashAttention makes large-model
//             training 3x faster" (jsqmd.com news 754333)
//   [intelli] "FlashAttention optimisation: breaking the performance bottleneck of
//             standard attention" (intelliparadigm.com)
//   [yunthe]  "Flash Attention-2: acceleration principle and GPU memory optimisation
//             in deployment" (yunthe.com)
//   [jos]     "A survey of key techniques of large language model pre-training
//             systems", Journal of Software 2026(1), p.218
//
// What it computes (per batch b and head h, with X[b,h] an N x d row-major matrix):
//   S = scale * Q K^T          [jos] attention definition (S = QK^T, P = Softmax(S),
//                              O = PV); the scaling by 1/sqrt(d) is [intelli] section 1
//                              step 2 and [yunthe] "standard attention" section; the
//                              scale is an argument here.
//   S[i][j] = -inf where key j is hidden from query i. Three masks, each optional,
//   combine by AND (a key is seen only if every mask given keeps it):
//     causal: keeps j <= i     [yunthe] "causal mask" troubleshooting item
//                              (is_causal=True); the query's own position is kept.
//     window (left, right): keeps i - left <= j <= i + right; a negative bound is
//                              no bound on that side. [yunthe] troubleshooting item 3
//                              (causal mask configuration), its sliding-window example
//                              (Longformer/Gemma style, a window-size pair such as
//                              (512, 512) given together with is_causal=True).
//     block mask M: keeps (i, j) iff M[i / 128][j / 128] != 0, M a row-major
//                              ceil(N/128) x ceil(N/128) byte matrix, the same for all
//                              heads. [intelli] section 7 item 2 (block-sparse
//                              FlashAttention: a sparse pattern over blocks) and [jos]
//                              p.218 (the algorithm extended to sparse attention); no
//                              page gives a block size for the mask, so it is the
//                              tile size 128 of [yunthe] "GPU memory optimisation
//                              strategy" (Block_Q = Block_K = 128).
//   A query row that sees no key at all has P = 0, O = 0 and L = -inf.
//   Dropout on P (optional): [jos] p.218 lists dropout among the operations fused into
//   the attention kernel. With drop probability p, Pd[i][j] = P[i][j] * Z[i][j] / (1 - p)
//   and O = Pd V; L stays the log-sum-exp of the logits (P is normalised before the
//   dropout). One Philox-4x32-10 block (Salmon, Moraes, Dror and Shaw, "Parallel
//   random numbers: as easy as 1, 2, 3", SC 2011) covers 4 queries x 4 keys: the block
//   at counter (j / 4, i / 4, bh, offset) under key (seed low 32 bits, seed high 32
//   bits), bh = b * H + h, gives query i its word i % 4 and key j byte j % 4 of that
//   word (byte 0 the least significant). Z[i][j] = 0 iff that byte is below
//   t = floor(256 p) (an integer decision), so the drop probability is t / 256: p
//   rounded down to a multiple of 1/256, and the factor 1/(1 - p) above is taken with
//   that rounded p, 256 / (256 - t).
//   m_i = max_j S[i][j]        [jsqmd] section 2.1, safe softmax
//   P[i][j] = exp(S[i][j] - m_i) / sum_j exp(S[i][j] - m_i)
//   O = P V
//   L_i = m_i + ln sum_j exp(S[i][j] - m_i)   natural-log log-sum-exp of the scaled
//                              logits: the normalisation statistics of [intelli]
//                              section 4.1, kept in log space as [intelli] 3.3 says.
//
// Backward, for the scalar loss l = <dO, O> (the sources only say "recompute",
// [intelli] section 4.2; the gradient is plain calculus of the definition above):
//   dV = P^T dO
//   dP = dO V^T
//   D_i = sum_j P[i][j] dP[i][j]   (equal to sum_k dO[i][k] O[i][k])
//   dS = P o (dP - D)              (softmax Jacobian, row by row)
//   With dropout: dV = Pd^T dO, dPd = dO V^T, dP = dPd o Z / (1 - p), and
//   D_i = sum_j P[i][j] dP[i][j] = sum_j Pd[i][j] dPd[i][j] (still rowsum(dO o O)).
//   dQ = scale * dS K
//   dK = scale * dS^T Q
//
// Every function materialises what the definition names (S, P, dP, dS) for one
// head, or one row, at a time; there is no blocking, no fusion and no online
// rescaling here. Parallelism is OpenMP over independent rows, which does not
// change the order of any sum within a row.
//
// Layout: all matrices contiguous, row-major [B, H, N, d]; L and D are [B, H, N].
// Every entry point returns 0 on success, nonzero on a bad argument or a failed
// allocation.

#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <limits>
#include <vector>

#ifdef _OPENMP
#include <omp.h>
#endif

namespace {

const double kNegInf = -std::numeric_limits<double>::infinity();

const int64_t kBlock = 128;  // block-mask granularity (rows and keys)

bool bad_shape(int64_t B, int64_t H, int64_t N, int64_t d) {
  return B < 0 || H < 0 || N < 0 || d <= 0;
}

// Which keys a query row sees: the AND of the three masks in the header.
struct Visibility {
  int causal;
  int64_t left, right;    // window bounds; negative = unbounded on that side
  const uint8_t* blocks;  // [nb x nb] row-major, nonzero = block kept; null = all kept
  int64_t nb;             // ceil(N / kBlock)

  bool sees(int64_t i, int64_t j) const {
    if (causal && j > i) return false;
    if (left >= 0 && j < i - left) return false;
    if (right >= 0 && j > i + right) return false;
    if (blocks && !blocks[(i / kBlock) * nb + j / kBlock]) return false;
    return true;
  }
};

Visibility make_vis(int64_t N, int causal, int64_t left, int64_t right,
                    const uint8_t* blocks) {
  return Visibility{causal, left, right, blocks, (N + kBlock - 1) / kBlock};
}

// Philox-4x32-10 as published: ten rounds; each multiplies words 0 and 2 by the two
// round multipliers (high and low halves of the 64-bit products), mixes in words 1
// and 3 and the round key, and permutes; the key grows by the two Weyl increments
// between rounds.
void philox4x32_10(const uint32_t ctr[4], uint32_t k0, uint32_t k1, uint32_t out[4]) {
  uint32_t x0 = ctr[0], x1 = ctr[1], x2 = ctr[2], x3 = ctr[3];
  for (int r = 0; r < 10; ++r) {
    if (r > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint64_t p0 = static_cast<uint64_t>(0xD2511F53u) * x0;
    const uint64_t p1 = static_cast<uint64_t>(0xCD9E8D57u) * x2;
    const uint32_t hi0 = static_cast<uint32_t>(p0 >> 32), lo0 = static_cast<uint32_t>(p0);
    const uint32_t hi1 = static_cast<uint32_t>(p1 >> 32), lo1 = static_cast<uint32_t>(p1);
    x0 = hi1 ^ x1 ^ k0;
    x1 = lo1;
    x2 = hi0 ^ x3 ^ k1;
    x3 = lo0;
  }
  out[0] = x0;
  out[1] = x1;
  out[2] = x2;
  out[3] = x3;
}

// Dropout on P (see the header). p = 0 is no dropout.
struct Dropout {
  double p;
  uint64_t seed;
  uint32_t offset;
  uint32_t threshold;  // a key is dropped iff its Philox byte is below this (0..255)

  bool on() const { return p > 0.0; }
  // Z[i][j] of head bh, as 0 or 1
  bool keep(int64_t bh, int64_t i, int64_t j) const {
    if (!on()) return true;
    const uint32_t ctr[4] = {static_cast<uint32_t>(j / 4), static_cast<uint32_t>(i / 4),
                             static_cast<uint32_t>(bh), offset};
    uint32_t w[4];
    philox4x32_10(ctr, static_cast<uint32_t>(seed), static_cast<uint32_t>(seed >> 32), w);
    const uint32_t byte = (w[i % 4] >> (8 * (j % 4))) & 0xffu;
    return byte >= threshold;
  }
  // Pd / P for (i, j): Z / (1 - t/256)
  double factor(int64_t bh, int64_t i, int64_t j) const {
    if (!on()) return 1.0;
    return keep(bh, i, j) ? 256.0 / (256.0 - threshold) : 0.0;
  }
};

Dropout make_dropout(double p, uint64_t seed, uint32_t offset) {
  double t = std::floor(p * 256.0);
  if (t > 255.0) t = 255.0;
  if (!(t > 0.0)) t = 0.0;
  return Dropout{p, seed, offset, static_cast<uint32_t>(t)};
}

bool bad_dropout(double p) { return !(p >= 0.0 && p < 1.0); }

// One row of scaled, masked logits: s[j] = scale * <q_i, k_j>, -inf where the
// key is hidden.
void logits_row(const double* q, const double* K, int64_t N, int64_t d, double scale,
                const Visibility& vis, int64_t i, double* s) {
  for (int64_t j = 0; j < N; ++j) {
    if (!vis.sees(i, j)) {
      s[j] = kNegInf;
      continue;
    }
    const double* k = K + j * d;
    double acc = 0.0;
    for (int64_t c = 0; c < d; ++c) acc += q[c] * k[c];
    s[j] = scale * acc;
  }
}

// Safe softmax of one row ([jsqmd] section 2.1): subtract the row max,
// exponentiate, divide by the sum. Writes p and returns the natural-log
// log-sum-exp m + ln(sum). A row with every entry masked gets p = 0 and -inf.
double safe_softmax_row(const double* s, int64_t N, double* p) {
  double m = kNegInf;
  for (int64_t j = 0; j < N; ++j) m = s[j] > m ? s[j] : m;
  if (m == kNegInf) {
    for (int64_t j = 0; j < N; ++j) p[j] = 0.0;
    return kNegInf;
  }
  double sum = 0.0;
  for (int64_t j = 0; j < N; ++j) {
    p[j] = std::exp(s[j] - m);
    sum += p[j];
  }
  for (int64_t j = 0; j < N; ++j) p[j] /= sum;
  return m + std::log(sum);
}

}  // namespace

extern "C" {

// Number of OpenMP threads the oracle will use (1 without OpenMP).
int oracle_num_threads(void) {
#ifdef _OPENMP
  return omp_get_max_threads();
#else
  return 1;
#endif
}

void oracle_set_num_threads(int n) {
#ifdef _OPENMP
  if (n > 0) omp_set_num_threads(n);
#else
  (void)n;
#endif
}

// Philox-4x32-10 of one counter under one key (for the generator's own pins).
void oracle_philox4x32_10(const uint32_t* ctr, uint32_t k0, uint32_t k1, uint32_t* out) {
  philox4x32_10(ctr, k0, k1, out);
}

// The row-stochastic matrix P = softmax(S) of one head, N x N, into P.
int oracle_attention_probs(const double* Q, const double* K, int64_t N, int64_t d,
                           double scale, int causal, int64_t left, int64_t right,
                           const uint8_t* blocks, double* P) {
  if (bad_shape(1, 1, N, d) || !Q || !K || !P) return 1;
  const Visibility vis = make_vis(N, causal, left, right, blocks);
#pragma omp parallel
  {
    std::vector<double> s(N);
#pragma omp for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
      logits_row(Q + i * d, K, N, d, scale, vis, i, s.data());
      safe_softmax_row(s.data(), N, P + i * N);
    }
  }
  return 0;
}

// Full forward: O [B,H,N,d] and L [B,H,N]. Materialises S and P (N x N) of one
// head at a time.
int oracle_attention_forward(const double* Q, const double* K, const double* V, int64_t B,
                             int64_t H, int64_t N, int64_t d, double scale, int causal,
                             int64_t left, int64_t right, const uint8_t* blocks, double p_drop,
                             uint64_t seed, uint32_t offset, double* O, double* L) {
  if (bad_shape(B, H, N, d) || !Q || !K || !V || !O || !L || bad_dropout(p_drop)) return 1;
  const Visibility vis = make_vis(N, causal, left, right, blocks);
  const Dropout drop = make_dropout(p_drop, seed, offset);
  if (N == 0) return 0;
  std::vector<double> P;
  try {
    P.resize(static_cast<size_t>(N) * N);
  } catch (...) {
    return 2;
  }
  for (int64_t bh = 0; bh < B * H; ++bh) {
    const double* q = Q + bh * N * d;
    const double* k = K + bh * N * d;
    const double* v = V + bh * N * d;
    double* o = O + bh * N * d;
    double* l = L + bh * N;
    // S then P, row by row (P overwrites S in place).
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
      double* row = P.data() + i * N;
      logits_row(q + i * d, k, N, d, scale, vis, i, row);
      std::vector<double> s(row, row + N);
      l[i] = safe_softmax_row(s.data(), N, row);
    }
    // O = Pd V (Pd = P without dropout)
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
      const double* p = P.data() + i * N;
      double* oi = o + i * d;
      for (int64_t c = 0; c < d; ++c) oi[c] = 0.0;
      for (int64_t j = 0; j < N; ++j) {
        const double pij = p[j] * drop.factor(bh, i, j);
        const double* vj = v + j * d;
        for (int64_t c = 0; c < d; ++c) oi[c] += pij * vj[c];
      }
    }
  }
  return 0;
}

// Full backward by calculus: dQ, dK, dV [B,H,N,d] and D [B,H,N] (D = rowsum(P o dP)).
// Materialises P, dP and dS (N x N) of one head at a time. If Dcheck is non-null it
// receives, per row, sum_k dO[i][k] * O[i][k] computed from O = P V, the second
// way of forming D; the two must agree.
int oracle_attention_backward(const double* Q, const double* K, const double* V,
                              const double* dO, int64_t B, int64_t H, int64_t N, int64_t d,
                              double scale, int causal, int64_t left, int64_t right,
                              const uint8_t* blocks, double p_drop, uint64_t seed,
                              uint32_t offset, double* dQ, double* dK, double* dV, double* D,
                              double* Dcheck) {
  if (bad_shape(B, H, N, d) || !Q || !K || !V || !dO || !dQ || !dK || !dV || !D ||
      bad_dropout(p_drop))
    return 1;
  const Visibility vis = make_vis(N, causal, left, right, blocks);
  const Dropout drop = make_dropout(p_drop, seed, offset);
  if (N == 0) return 0;
  std::vector<double> P, dS;
  try {
    P.resize(static_cast<size_t>(N) * N);
    dS.resize(static_cast<size_t>(N) * N);
  } catch (...) {
    return 2;
  }
  for (int64_t bh = 0; bh < B * H; ++bh) {
    const double* q = Q + bh * N * d;
    const double* k = K + bh * N * d;
    const double* v = V + bh * N * d;
    const double* go = dO + bh * N * d;
    double* gq = dQ + bh * N * d;
    double* gk = dK + bh * N * d;
    double* gv = dV + bh * N * d;
    double* Dh = D + bh * N;
    // P = softmax(S)
#pragma omp parallel
    {
      std::vector<double> s(N);
#pragma omp for schedule(static)
      for (int64_t i = 0; i < N; ++i) {
        logits_row(q + i * d, k, N, d, scale, vis, i, s.data());
        safe_softmax_row(s.data(), N, P.data() + i * N);
      }
    }
    // dP = (dO V^T) o Z / (1 - p), D_i = sum_j P_ij dP_ij, dS = P o (dP - D); dS holds
    // dP first.
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
      const double* goi = go + i * d;
      double* dsi = dS.data() + i * N;
      const double* pi = P.data() + i * N;
      double Di = 0.0;
      for (int64_t j = 0; j < N; ++j) {
        const double* vj = v + j * d;
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c) acc += goi[c] * vj[c];
        dsi[j] = acc * drop.factor(bh, i, j);
        Di += pi[j] * dsi[j];
      }
      Dh[i] = Di;
      for (int64_t j = 0; j < N; ++j) dsi[j] = pi[j] * (dsi[j] - Di);
      if (Dcheck) {
        // O_i = sum_j Pd_ij V_j, then sum_k dO_ik O_ik
        double Dc = 0.0;
        for (int64_t c = 0; c < d; ++c) {
          double oic = 0.0;
          for (int64_t j = 0; j < N; ++j) oic += pi[j] * drop.factor(bh, i, j) * v[j * d + c];
          Dc += goi[c] * oic;
        }
        Dcheck[bh * N + i] = Dc;
      }
    }
    // dQ = scale * dS K
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < N; ++i) {
      const double* dsi = dS.data() + i * N;
      double* gqi = gq + i * d;
      for (int64_t c = 0; c < d; ++c) gqi[c] = 0.0;
      for (int64_t j = 0; j < N; ++j) {
        const double* kj = k + j * d;
        for (int64_t c = 0; c < d; ++c) gqi[c] += dsi[j] * kj[c];
      }
      for (int64_t c = 0; c < d; ++c) gqi[c] *= scale;
    }
    // dK = scale * dS^T Q, dV = P^T dO
#pragma omp parallel for schedule(static)
    for (int64_t j = 0; j < N; ++j) {
      double* gkj = gk + j * d;
      double* gvj = gv + j * d;
      for (int64_t c = 0; c < d; ++c) {
        gkj[c] = 0.0;
        gvj[c] = 0.0;
      }
      for (int64_t i = 0; i < N; ++i) {
        const double ds = dS[i * N + j];
        const double p = P[i * N + j] * drop.factor(bh, i, j);
        const double* qi = q + i * d;
        const double* goi = go + i * d;
        for (int64_t c = 0; c < d; ++c) {
          gkj[c] += ds * qi[c];
          gvj[c] += p * goi[c];
        }
      }
      for (int64_t c = 0; c < d; ++c) gkj[c] *= scale;
    }
  }
  return 0;
}

// Forward restricted to selected query rows: for r in [0, R), row rows[r] of head
// heads[r] (head index bh = b * H + h). Writes O_r [R, d] and L_r [R]. The same
// definition as oracle_attention_forward, one materialised row of S and P each.
int oracle_attention_forward_rows(const double* Q, const double* K, const double* V,
                                  int64_t B, int64_t H, int64_t N, int64_t d, double scale,
                                  int causal, int64_t left, int64_t right,
                                  const uint8_t* blocks, double p_drop, uint64_t seed,
                                  uint32_t offset, int64_t R, const int64_t* heads,
                                  const int64_t* rows, double* O_r, double* L_r) {
  if (bad_shape(B, H, N, d) || R < 0 || (R > 0 && (!heads || !rows || !O_r || !L_r)) ||
      bad_dropout(p_drop))
    return 1;
  const Visibility vis = make_vis(N, causal, left, right, blocks);
  const Dropout drop = make_dropout(p_drop, seed, offset);
  for (int64_t r = 0; r < R; ++r)
    if (heads[r] < 0 || heads[r] >= B * H || rows[r] < 0 || rows[r] >= N) return 1;
#pragma omp parallel
  {
    std::vector<double> s(N), p(N);
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < R; ++r) {
      const int64_t bh = heads[r], i = rows[r];
      const double* k = K + bh * N * d;
      const double* v = V + bh * N * d;
      logits_row(Q + (bh * N + i) * d, k, N, d, scale, vis, i, s.data());
      L_r[r] = safe_softmax_row(s.data(), N, p.data());
      double* o = O_r + r * d;
      for (int64_t c = 0; c < d; ++c) o[c] = 0.0;
      for (int64_t j = 0; j < N; ++j) {
        const double pd = p[j] * drop.factor(bh, i, j);
        for (int64_t c = 0; c < d; ++c) o[c] += pd * v[j * d + c];
      }
    }
  }
  return 0;
}

// dQ restricted to selected query rows (same selection convention as
// oracle_attention_forward_rows). Row i needs only its own P row and dP row:
// D_i = sum_j P_ij dP_ij, dQ_i = scale * sum_j P_ij (dP_ij - D_i) K_j.
int oracle_attention_backward_dq_rows(const double* Q, const double* K, const double* V,
                                      const double* dO, int64_t B, int64_t H, int64_t N,
                                      int64_t d, double scale, int causal, int64_t left,
                                      int64_t right, const uint8_t* blocks, double p_drop,
                                      uint64_t seed, uint32_t offset, int64_t R,
                                      const int64_t* heads, const int64_t* rows,
                                      double* dQ_r, double* D_r) {
  if (bad_shape(B, H, N, d) || R < 0 || (R > 0 && (!heads || !rows || !dQ_r || !D_r)) ||
      bad_dropout(p_drop))
    return 1;
  const Visibility vis = make_vis(N, causal, left, right, blocks);
  const Dropout drop = make_dropout(p_drop, seed, offset);
  for (int64_t r = 0; r < R; ++r)
    if (heads[r] < 0 || heads[r] >= B * H || rows[r] < 0 || rows[r] >= N) return 1;
#pragma omp parallel
  {
    std::vector<double> s(N), p(N), dp(N);
#pragma omp for schedule(dynamic, 4)
    for (int64_t r = 0; r < R; ++r) {
      const int64_t bh = heads[r], i = rows[r];
      const double* k = K + bh * N * d;
      const double* v = V + bh * N * d;
      const double* goi = dO + (bh * N + i) * d;
      logits_row(Q + (bh * N + i) * d, k, N, d, scale, vis, i, s.data());
      safe_softmax_row(s.data(), N, p.data());
      double Di = 0.0;
      for (int64_t j = 0; j < N; ++j) {
        double acc = 0.0;
        for (int64_t c = 0; c < d; ++c) acc += goi[c] * v[j * d + c];
        dp[j] = acc * drop.factor(bh, i, j);
        Di += p[j] * dp[j];
      }
      D_r[r] = Di;
      double* g = dQ_r + r * d;
      for (int64_t c = 0; c < d; ++c) g[c] = 0.0;
      for (int64_t j = 0; j < N; ++j) {
        const double ds = p[j] * (dp[j] - Di);
        for (int64_t c = 0; c < d; ++c) g[c] += ds * k[j * d + c];
      }
      for (int64_t c = 0; c < d; ++c) g[c] *= scale;
    }
  }
  return 0;
}

// dK and dV restricted to selected key rows j of one head bh. Column j of P needs
// every row's normaliser and every row's D, so the caller passes L [N] and D [N]
// of that head as this oracle computed them (oracle_attention_forward_rows over all
// rows for L; oracle_attention_backward_dq_rows for D):
//   P_ij = exp(S_ij - L_i), dS_ij = P_ij (dO_i . V_j - D_i),
//   dV_j = sum_i P_ij dO_i,  dK_j = scale * sum_i dS_ij Q_i.
int oracle_attention_backward_dkdv_rows(const double* Q, const double* K, const double* V,
                                        const double* dO, int64_t B, int64_t H, int64_t N,
                                        int64_t d, double scale, int causal, int64_t left,
                                        int64_t right, const uint8_t* blocks, double p_drop,
                                        uint64_t seed, uint32_t offset, int64_t bh,
                                        const double* L, const double* D, int64_t R,
                                        const int64_t* keys, double* dK_r, double* dV_r) {
  if (bad_shape(B, H, N, d) || bh < 0 || bh >= B * H || R < 0 || !L || !D ||
      (R > 0 && (!keys || !dK_r || !dV_r)) || bad_dropout(p_drop))
    return 1;
  const Visibility vis = make_vis(N, causal, left, right, blocks);
  const Dropout drop = make_dropout(p_drop, seed, offset);
  for (int64_t r = 0; r < R; ++r)
    if (keys[r] < 0 || keys[r] >= N) return 1;
  const double* q = Q + bh * N * d;
  const double* k = K + bh * N * d;
  const double* v = V + bh * N * d;
  const double* go = dO + bh * N * d;
#pragma omp parallel for schedule(dynamic, 1)
  for (int64_t r = 0; r < R; ++r) {
    const int64_t j = keys[r];
    const double* kj = k + j * d;
    const double* vj = v + j * d;
    double* gk = dK_r + r * d;
    double* gv = dV_r + r * d;
    for (int64_t c = 0; c < d; ++c) {
      gk[c] = 0.0;
      gv[c] = 0.0;
    }
    for (int64_t i = 0; i < N; ++i) {
      if (!vis.sees(i, j)) continue;
      const double* qi = q + i * d;
      const double* goi = go + i * d;
      double sij = 0.0, dpij = 0.0;
      for (int64_t c = 0; c < d; ++c) {
        sij += qi[c] * kj[c];
        dpij += goi[c] * vj[c];
      }
      const double pij = std::exp(scale * sij - L[i]);
      const double f = drop.factor(bh, i, j);
      const double dsij = pij * (dpij * f - D[i]);
      for (int64_t c = 0; c < d; ++c) {
        gv[c] += pij * f * goi[c];
        gk[c] += dsij * qi[c];
      }
    }
    for (int64_t c = 0; c < d; ++c) gk[c] *= scale;
  }
  return 0;
}

}  // extern "C"
