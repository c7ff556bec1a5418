// Test infrastructure only: the fp64 CPU oracle for causal linear attention.
//
// Only the tests, the package's smoke entry and the benchmark's CPU-baseline /
// reference arm may load this library.  The product path (the CUDA library) never
// calls it and shares no code with it.
//
// What it computes is the plain definition of causal linear attention, one token at a
// time, in double precision:
//
//   phi(x)  = x + 1 for x > 0, exp(x) otherwise (ELU with alpha = 1, plus one), or the
//             identity.  Source: "Linear Attention and Retentive Networks: How Recurrent
//             Duals and Chunkwise Tiling Eliminate the Quadratic Bottleneck", section
//             "The Associative Property and Linear Kernel Formulation" (the kernel
//             feature map that makes the similarity separable).
//   S_t     = gamma * S_{t-1} + phi(k_t) v_t^T      (dk x dv)
//   Z_t     = gamma * Z_{t-1} + phi(k_t)            (dk)
//   o_t     = phi(q_t) S_t / (phi(q_t) . Z_t + eps)  (normalised) or phi(q_t) S_t.
//             Sources: the same page, "The Recurrent Dual" (undecayed state, normaliser
//             and ratio readout) and "2. The Three Computation Paradigms / B. Recurrent
//             Representation" (the per-head scalar decay gamma, unnormalised readout);
//             "Log-Depth Chunked Linear-Attention Scan", "Mathematical statement" (S_t and
//             Z_t as sums over i <= t, so token t is included in its own state) and
//             "Implementation notes" (the ratio with "+ eps" in the denominator).
//
// gamma == NULL means no decay (gamma = 1).  Token t is counted in its own state
// (inclusive sums).  The decay multiplies the previous state only; the current token
// enters with weight gamma^0 = 1.  When both decay and normalisation are requested the
// normaliser decays the same way as the state.
//
// Inputs are float32 arrays: the GPU path's bf16 inputs are widened to float32 exactly
// before they are passed here, so both sides see identical values.  All arithmetic is
// double precision, built without fast-math.  Work is split over (b, h) pairs only,
// with std::thread; each pair is an independent token loop.
//
// Layouts (all contiguous, row-major):
//   q, k   [B, H, T, dk]      v [B, H, T, dv]      out [B, H, T, dv]  (may be NULL)
//   S_init, S_final [B, H, dk, dv]   (S[i][j], i = key feature, j = value feature)
//   Z_init, Z_final [B, H, dk]
//   gamma [H] (double) or NULL.
// S_init / Z_init may be NULL (zero initial state); the outputs may be NULL (skipped).
//
// la_oracle_backward differentiates both forms by hand, token by token (the chain rule
// through the recurrence; see backward_pair), for the backward pass.  la_oracle_gla_forward
// runs the gated (data-dependent decay) recurrence (see gla_pair), la_oracle_gla_backward its
// gradients (see gla_backward_pair).

#include <algorithm>
#include <cmath>
#include <cstddef>
#include <cstdint>
#include <thread>
#include <vector>

namespace {

inline double feature_map(double x, int fm) {
  if (fm == 0) return x;                    // identity
  return x > 0.0 ? x + 1.0 : std::exp(x);   // ELU(alpha = 1) + 1
}

struct Problem {
  const float* q;
  const float* k;
  const float* v;
  int B, H;
  long long T;
  int dk, dv, fm;
  const double* gamma;
  int normalize;
  double eps;
  const double* S_init;
  const double* Z_init;
  double* out;
  double* S_final;
  double* Z_final;
};

// The token loop for one (b, h) pair.
void run_pair(const Problem& p, long long bh) {
  const int dk = p.dk, dv = p.dv;
  const long long T = p.T;
  const int h = static_cast<int>(bh % p.H);
  const double g = p.gamma ? p.gamma[h] : 1.0;

  std::vector<double> S(static_cast<size_t>(dk) * dv, 0.0), Z(dk, 0.0);
  if (p.S_init)
    for (size_t e = 0; e < S.size(); ++e) S[e] = p.S_init[bh * dk * dv + e];
  if (p.Z_init)
    for (int i = 0; i < dk; ++i) Z[i] = p.Z_init[bh * dk + i];

  std::vector<double> fq(dk), fk(dk), num(dv);
  const float* q = p.q + bh * T * dk;
  const float* k = p.k + bh * T * dk;
  const float* v = p.v + bh * T * dv;
  double* out = p.out ? p.out + bh * T * dv : nullptr;

  for (long long t = 0; t < T; ++t) {
    for (int i = 0; i < dk; ++i) {
      fq[i] = feature_map(static_cast<double>(q[t * dk + i]), p.fm);
      fk[i] = feature_map(static_cast<double>(k[t * dk + i]), p.fm);
    }
    const float* vt = v + t * dv;
    // State update: decay the past, then add the current token's outer product.
    for (int i = 0; i < dk; ++i) {
      double* Si = &S[static_cast<size_t>(i) * dv];
      for (int j = 0; j < dv; ++j) Si[j] = g * Si[j] + fk[i] * static_cast<double>(vt[j]);
      Z[i] = g * Z[i] + fk[i];
    }
    if (!out) continue;
    // Readout with the inclusive state.
    for (int j = 0; j < dv; ++j) num[j] = 0.0;
    double den = 0.0;
    for (int i = 0; i < dk; ++i) {
      const double* Si = &S[static_cast<size_t>(i) * dv];
      for (int j = 0; j < dv; ++j) num[j] += fq[i] * Si[j];
      den += fq[i] * Z[i];
    }
    double* ot = out + t * dv;
    if (p.normalize) {
      for (int j = 0; j < dv; ++j) ot[j] = num[j] / (den + p.eps);
    } else {
      for (int j = 0; j < dv; ++j) ot[j] = num[j];
    }
  }

  if (p.S_final)
    for (size_t e = 0; e < S.size(); ++e) p.S_final[bh * dk * dv + e] = S[e];
  if (p.Z_final)
    for (int i = 0; i < dk; ++i) p.Z_final[bh * dk + i] = Z[i];
}

// Backward for one (b, h) pair.  With do_t = dL/do_t, dS_final = dL/dS_final and
// dZ_final = dL/dZ_final (or zero), differentiating the recurrence above one token at a
// time.  The output is o_t = n_t / d_t with n_t = phi(q_t) S_t and d_t = phi(q_t) . Z_t
// + eps (normalised form), or o_t = n_t (unnormalised: d_t = 1 and no Z terms).  So
//   dn_t = do_t / d_t,   dd_t = -(do_t . n_t) / d_t^2            (dd_t = 0 unnormalised)
//   dphi(q_t) = S_t dn_t + Z_t dd_t                              (forward sweep)
//   G_t = phi(q_t) dn_t^T + gamma G_{t+1},  G_{T-1} = phi(q_{T-1}) dn_{T-1}^T + dS_final
//   g_t = phi(q_t) dd_t   + gamma g_{t+1},  g_{T-1} = phi(q_{T-1}) dd_{T-1}   + dZ_final
//   dphi(k_t) = G_t v_t + g_t,   dv_t = G_t^T phi(k_t)           (reverse sweep)
//   dS_init = gamma G_0,   dZ_init = gamma g_0
// and dq = dphi(q) * phi'(q), dk = dphi(k) * phi'(k) with phi' = 1 (identity) or
// 1 for x > 0, exp(x) otherwise (ELU + 1).
struct BackwardProblem {
  const float* q;
  const float* k;
  const float* v;
  const double* dout;
  int H;
  long long T;
  int dk, dv, fm;
  const double* gamma;
  int normalize;
  double eps;
  const double* S_init;
  const double* Z_init;
  const double* dS_final;
  const double* dZ_final;
  double* dq;
  double* dk_out;
  double* dv_out;
  double* dS_init;
  double* dZ_init;
};

inline double feature_map_derivative(double x, int fm) {
  if (fm == 0) return 1.0;
  return x > 0.0 ? 1.0 : std::exp(x);
}

void backward_pair(const BackwardProblem& p, long long bh) {
  const int dk = p.dk, dv = p.dv;
  const long long T = p.T;
  const int h = static_cast<int>(bh % p.H);
  const double g = p.gamma ? p.gamma[h] : 1.0;
  const float* q = p.q + bh * T * dk;
  const float* k = p.k + bh * T * dk;
  const float* v = p.v + bh * T * dv;
  const double* dout = p.dout + bh * T * dv;

  // Forward sweep: S_t and Z_t, the output's numerator and denominator, the gradients
  // that reach them (kept for the reverse sweep), and dphi(q_t).
  std::vector<double> S(static_cast<size_t>(dk) * dv, 0.0), Z(dk, 0.0), fq(dk), n(dv);
  std::vector<double> dn(static_cast<size_t>(T) * dv), dd(static_cast<size_t>(T), 0.0);
  if (p.S_init)
    for (size_t e = 0; e < S.size(); ++e) S[e] = p.S_init[bh * dk * dv + e];
  if (p.normalize && p.Z_init)
    for (int i = 0; i < dk; ++i) Z[i] = p.Z_init[bh * dk + i];
  for (long long t = 0; t < T; ++t) {
    for (int i = 0; i < dk; ++i) {
      const double fk = feature_map(static_cast<double>(k[t * dk + i]), p.fm);
      double* Si = &S[static_cast<size_t>(i) * dv];
      for (int j = 0; j < dv; ++j) Si[j] = g * Si[j] + fk * static_cast<double>(v[t * dv + j]);
      Z[i] = g * Z[i] + fk;
      const double xq = q[t * dk + i];
      fq[i] = feature_map(xq, p.fm);
    }
    double den = 1.0, don = 0.0;
    if (p.normalize) {
      den = p.eps;
      for (int i = 0; i < dk; ++i) den += Z[i] * fq[i];
    }
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int i = 0; i < dk; ++i) acc += fq[i] * S[static_cast<size_t>(i) * dv + j];
      n[j] = acc;
      don += dout[t * dv + j] * acc;
      dn[static_cast<size_t>(t) * dv + j] = dout[t * dv + j] / den;
    }
    if (p.normalize) dd[static_cast<size_t>(t)] = -don / (den * den);
    for (int i = 0; i < dk; ++i) {
      const double* Si = &S[static_cast<size_t>(i) * dv];
      double acc = 0.0;
      for (int j = 0; j < dv; ++j) acc += Si[j] * dn[static_cast<size_t>(t) * dv + j];
      acc += Z[i] * dd[static_cast<size_t>(t)];
      const double x = static_cast<double>(q[t * dk + i]);
      p.dq[(bh * T + t) * dk + i] = acc * feature_map_derivative(x, p.fm);
    }
  }

  // Reverse sweep: G accumulates phi(q_t) dn_t^T, g accumulates phi(q_t) dd_t, and both
  // decay by gamma between tokens.
  std::vector<double> G(static_cast<size_t>(dk) * dv, 0.0), gz(dk, 0.0), fk(dk);
  if (p.dS_final)
    for (size_t e = 0; e < G.size(); ++e) G[e] = p.dS_final[bh * dk * dv + e];
  if (p.normalize && p.dZ_final)
    for (int i = 0; i < dk; ++i) gz[i] = p.dZ_final[bh * dk + i];
  for (long long t = T - 1; t >= 0; --t) {
    const double* dnt = &dn[static_cast<size_t>(t) * dv];
    for (int i = 0; i < dk; ++i) {
      const double fqi = feature_map(static_cast<double>(q[t * dk + i]), p.fm);
      double* Gi = &G[static_cast<size_t>(i) * dv];
      for (int j = 0; j < dv; ++j) Gi[j] += fqi * dnt[j];
      gz[i] += fqi * dd[static_cast<size_t>(t)];
      fk[i] = feature_map(static_cast<double>(k[t * dk + i]), p.fm);
    }
    for (int i = 0; i < dk; ++i) {
      const double* Gi = &G[static_cast<size_t>(i) * dv];
      double acc = gz[i];
      for (int j = 0; j < dv; ++j) acc += Gi[j] * static_cast<double>(v[t * dv + j]);
      const double x = static_cast<double>(k[t * dk + i]);
      p.dk_out[(bh * T + t) * dk + i] = acc * feature_map_derivative(x, p.fm);
    }
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int i = 0; i < dk; ++i) acc += G[static_cast<size_t>(i) * dv + j] * fk[i];
      p.dv_out[(bh * T + t) * dv + j] = acc;
    }
    for (double& x : G) x *= g;  // G_{t-1} receives gamma G_t
    for (double& x : gz) x *= g;
  }
  if (p.dS_init)
    for (size_t e = 0; e < G.size(); ++e) p.dS_init[bh * dk * dv + e] = G[e];
  if (p.dZ_init)
    for (int i = 0; i < dk; ++i) p.dZ_init[bh * dk + i] = p.normalize ? gz[i] : 0.0;
}

// Gated linear attention ("Linear Attention and Retentive Networks ...", Gated Linear
// Attention (GLA) and Hardware-Software Co-Design: the update S_t = G_t (.) S_{t-1} +
// k_t^T v_t with the gate G_t = alpha_t 1^T), one (b, h) pair, token by token:
//   S_t[i][j] = alpha_t[i] S_{t-1}[i][j] + k_t[i] v_t[j],   o_t[j] = sum_i q_t[i] S_t[i][j]
// with S_{-1} = S_init (or zero).  No feature map and no normalisation, as on that page.
struct GlaProblem {
  const float* q;
  const float* k;
  const float* v;
  const float* alpha;
  long long T;
  int dk, dv;
  const double* S_init;
  double* out;
  double* S_final;
};

void gla_pair(const GlaProblem& p, long long bh) {
  const int dk = p.dk, dv = p.dv;
  const long long T = p.T;
  const float* q = p.q + bh * T * dk;
  const float* k = p.k + bh * T * dk;
  const float* v = p.v + bh * T * dv;
  const float* al = p.alpha + bh * T * dk;
  std::vector<double> S(static_cast<size_t>(dk) * dv, 0.0);
  if (p.S_init)
    for (size_t e = 0; e < S.size(); ++e) S[e] = p.S_init[bh * dk * dv + e];
  for (long long t = 0; t < T; ++t) {
    for (int i = 0; i < dk; ++i) {
      const double gate = static_cast<double>(al[t * dk + i]);
      const double ki = static_cast<double>(k[t * dk + i]);
      double* Si = &S[static_cast<size_t>(i) * dv];
      for (int j = 0; j < dv; ++j) Si[j] = gate * Si[j] + ki * static_cast<double>(v[t * dv + j]);
    }
    if (p.out) {
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i)
          acc += static_cast<double>(q[t * dk + i]) * S[static_cast<size_t>(i) * dv + j];
        p.out[(bh * T + t) * dv + j] = acc;
      }
    }
  }
  if (p.S_final)
    for (size_t e = 0; e < S.size(); ++e) p.S_final[bh * dk * dv + e] = S[e];
}

// Gradients of the gated loop (see gla_pair) for L = <dout, out> + <dS_final, S_final>, by
// the chain rule one token at a time: with G_t = dL/dS_t,
//   dq_t[i] = sum_j S_t[i][j] do_t[j]                        (forward sweep)
//   G_t = q_t do_t^T + diag(alpha_{t+1}) G_{t+1},  G_{T-1} = q_{T-1} do_{T-1}^T + dS_final
//   dk_t[i] = sum_j G_t[i][j] v_t[j],  dv_t[j] = sum_i G_t[i][j] k_t[i]
//   dalpha_t[i] = sum_j G_t[i][j] S_{t-1}[i][j],  dS_init = diag(alpha_0) G_0
// The reverse sweep needs S_{t-1}: the forward sweep keeps S every kGlaCheck tokens and each
// block is recomputed from its checkpoint.  kGlaCheck is about sqrt(T) (at least 64), so the
// checkpoints and one block's states take O(sqrt(T) dk dv) memory per thread; the values are
// the same for any interval (the recomputation repeats the forward sweep's operations).
constexpr long long kGlaCheckMin = 64;

struct GlaBackwardProblem {
  const float* q;
  const float* k;
  const float* v;
  const float* alpha;
  const double* dout;
  long long T;
  int dk, dv;
  const double* S_init;
  const double* dS_final;
  double* dq;
  double* dk_out;
  double* dv_out;
  double* dalpha;
  double* dS_init;
};

void gla_backward_pair(const GlaBackwardProblem& p, long long bh) {
  const int dk = p.dk, dv = p.dv;
  const long long T = p.T;
  const size_t sd = static_cast<size_t>(dk) * dv;
  const float* q = p.q + bh * T * dk;
  const float* k = p.k + bh * T * dk;
  const float* v = p.v + bh * T * dv;
  const float* al = p.alpha + bh * T * dk;
  const double* dout = p.dout + bh * T * dv;
  const long long kGlaCheck = std::max<long long>(
      kGlaCheckMin, static_cast<long long>(std::ceil(std::sqrt(static_cast<double>(T)))));
  auto step = [&](std::vector<double>& S, long long t) {  // S_{t-1} -> S_t
    for (int i = 0; i < dk; ++i) {
      const double gate = static_cast<double>(al[t * dk + i]), ki = static_cast<double>(k[t * dk + i]);
      for (int j = 0; j < dv; ++j)
        S[static_cast<size_t>(i) * dv + j] = gate * S[static_cast<size_t>(i) * dv + j] +
                                             ki * static_cast<double>(v[t * dv + j]);
    }
  };
  // Forward sweep: dq, and S before every block of kGlaCheck tokens.
  const long long nblk = (T + kGlaCheck - 1) / kGlaCheck;
  std::vector<double> S(sd, 0.0), checks(static_cast<size_t>(nblk) * sd);
  if (p.S_init)
    for (size_t e = 0; e < sd; ++e) S[e] = p.S_init[bh * sd + e];
  for (long long t = 0; t < T; ++t) {
    if (t % kGlaCheck == 0) std::copy(S.begin(), S.end(), checks.begin() + (t / kGlaCheck) * sd);
    step(S, t);
    for (int i = 0; i < dk; ++i) {
      double acc = 0.0;
      for (int j = 0; j < dv; ++j) acc += S[static_cast<size_t>(i) * dv + j] * dout[t * dv + j];
      p.dq[(bh * T + t) * dk + i] = acc;
    }
  }
  // Reverse sweep, block by block from the last.
  std::vector<double> G(sd, 0.0), prev(static_cast<size_t>(kGlaCheck) * sd);
  if (p.dS_final)
    for (size_t e = 0; e < sd; ++e) G[e] = p.dS_final[bh * sd + e];
  for (long long b = nblk - 1; b >= 0; --b) {
    const long long t0 = b * kGlaCheck, t1 = std::min(T, t0 + kGlaCheck);
    std::vector<double> Sb(checks.begin() + b * sd, checks.begin() + (b + 1) * sd);
    for (long long t = t0; t < t1; ++t) {  // prev[t - t0] = S_{t-1}
      std::copy(Sb.begin(), Sb.end(), prev.begin() + (t - t0) * sd);
      step(Sb, t);
    }
    for (long long t = t1 - 1; t >= t0; --t) {
      const double* Sp = &prev[(t - t0) * sd];
      for (int i = 0; i < dk; ++i) {
        const double qi = static_cast<double>(q[t * dk + i]);
        for (int j = 0; j < dv; ++j) G[static_cast<size_t>(i) * dv + j] += qi * dout[t * dv + j];
      }
      for (int i = 0; i < dk; ++i) {
        double gk = 0.0, ga = 0.0;
        for (int j = 0; j < dv; ++j) {
          gk += G[static_cast<size_t>(i) * dv + j] * static_cast<double>(v[t * dv + j]);
          ga += G[static_cast<size_t>(i) * dv + j] * Sp[static_cast<size_t>(i) * dv + j];
        }
        p.dk_out[(bh * T + t) * dk + i] = gk;
        p.dalpha[(bh * T + t) * dk + i] = ga;
      }
      for (int j = 0; j < dv; ++j) {
        double acc = 0.0;
        for (int i = 0; i < dk; ++i)
          acc += G[static_cast<size_t>(i) * dv + j] * static_cast<double>(k[t * dk + i]);
        p.dv_out[(bh * T + t) * dv + j] = acc;
      }
      for (int i = 0; i < dk; ++i) {  // G_{t-1} receives diag(alpha_t) G_t
        const double at = al[t * dk + i];
        for (int j = 0; j < dv; ++j) G[static_cast<size_t>(i) * dv + j] *= at;
      }
    }
  }
  if (p.dS_init)
    for (size_t e = 0; e < sd; ++e) p.dS_init[bh * sd + e] = G[e];
}

}  // namespace

extern "C" {

// Gradients of the gated loop (see gla_backward_pair).  dout [B, H, T, dv] double,
// dS_final [B, H, dk, dv] double or NULL; writes dq, dk, dalpha [B, H, T, dk], dv
// [B, H, T, dv] and dS_init [B, H, dk, dv] (may be NULL), all double.
int la_oracle_gla_backward(const float* q, const float* k, const float* v, const float* alpha,
                           const double* dout, int B, int H, long long T, int dk, int dv,
                           const double* S_init, const double* dS_final, double* dq,
                           double* dk_out, double* dv_out, double* dalpha, double* dS_init,
                           int nthreads) {
  if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return 1;
  if (T > 0 && (!q || !k || !v || !alpha || !dout || !dq || !dk_out || !dv_out || !dalpha))
    return 1;
  const long long BH = static_cast<long long>(B) * H;
  if (BH == 0) return 0;
  GlaBackwardProblem p{q, k, v, alpha, dout, T, dk, dv, S_init, dS_final, dq, dk_out, dv_out,
                       dalpha, dS_init};
  long long workers = nthreads > 0 ? nthreads
                                   : static_cast<long long>(std::thread::hardware_concurrency());
  if (workers < 1) workers = 1;
  if (workers > BH) workers = BH;
  std::vector<std::thread> pool;
  for (long long w = 0; w < workers; ++w)
    pool.emplace_back([&p, w, workers, BH]() {
      for (long long bh = w; bh < BH; bh += workers) gla_backward_pair(p, bh);
    });
  for (auto& th : pool) th.join();
  return 0;
}


// Gated linear attention forward (see gla_pair).  alpha [B, H, T, dk] float32 gates;
// S_init [B, H, dk, dv] double or NULL; out [B, H, T, dv] and S_final double (each may be
// NULL).  Returns 0, or 1 on an invalid argument.
int la_oracle_gla_forward(const float* q, const float* k, const float* v, const float* alpha,
                          int B, int H, long long T, int dk, int dv, const double* S_init,
                          double* out, double* S_final, int nthreads) {
  if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return 1;
  if (T > 0 && (!q || !k || !v || !alpha)) return 1;
  const long long BH = static_cast<long long>(B) * H;
  if (BH == 0) return 0;
  GlaProblem p{q, k, v, alpha, T, dk, dv, S_init, out, S_final};
  long long workers = nthreads > 0 ? nthreads
                                   : static_cast<long long>(std::thread::hardware_concurrency());
  if (workers < 1) workers = 1;
  if (workers > BH) workers = BH;
  std::vector<std::thread> pool;
  for (long long w = 0; w < workers; ++w)
    pool.emplace_back([&p, w, workers, BH]() {
      for (long long bh = w; bh < BH; bh += workers) gla_pair(p, bh);
    });
  for (auto& th : pool) th.join();
  return 0;
}


// Returns 0 on success, 1 on an invalid argument.  nthreads <= 0 means one thread per
// hardware thread (capped at B*H).
int la_oracle_forward(const float* q, const float* k, const float* v, int B, int H,
                      long long T, int dk, int dv, int feature_map_id,
                      const double* gamma, int normalize, double eps,
                      const double* S_init, const double* Z_init, double* out,
                      double* S_final, double* Z_final, int nthreads) {
  if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return 1;
  if (feature_map_id != 0 && feature_map_id != 1) return 1;
  if (T > 0 && (!q || !k || !v)) return 1;
  const long long BH = static_cast<long long>(B) * H;
  if (BH == 0) return 0;

  Problem p{q, k, v, B, H, T, dk, dv, feature_map_id, gamma, normalize, eps,
            S_init, Z_init, out, S_final, Z_final};

  long long workers = nthreads > 0 ? nthreads
                                   : static_cast<long long>(std::thread::hardware_concurrency());
  if (workers < 1) workers = 1;
  if (workers > BH) workers = BH;

  if (workers == 1) {
    for (long long bh = 0; bh < BH; ++bh) run_pair(p, bh);
    return 0;
  }
  std::vector<std::thread> pool;
  pool.reserve(static_cast<size_t>(workers));
  for (long long w = 0; w < workers; ++w) {
    pool.emplace_back([&p, w, workers, BH]() {
      for (long long bh = w; bh < BH; bh += workers) run_pair(p, bh);
    });
  }
  for (auto& th : pool) th.join();
  return 0;
}

// Backward (see backward_pair).  dout [B, H, T, dv] (double), dS_final [B, H, dk, dv] and
// dZ_final [B, H, dk] or NULL, S_init / Z_init as in la_oracle_forward.  Writes dq, dk
// [B, H, T, dk], dv [B, H, T, dv], dS_init [B, H, dk, dv] and dZ_init [B, H, dk] (each
// may be NULL; dZ_init is zero for the unnormalised form), all double.
int la_oracle_backward(const float* q, const float* k, const float* v, const double* dout,
                       int B, int H, long long T, int dk, int dv, int feature_map_id,
                       const double* gamma, int normalize, double eps, const double* S_init,
                       const double* Z_init, const double* dS_final, const double* dZ_final,
                       double* dq, double* dk_out, double* dv_out, double* dS_init,
                       double* dZ_init, int nthreads) {
  if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return 1;
  if (feature_map_id != 0 && feature_map_id != 1) return 1;
  if (T > 0 && (!q || !k || !v || !dout || !dq || !dk_out || !dv_out)) return 1;
  const long long BH = static_cast<long long>(B) * H;
  if (BH == 0) return 0;
  BackwardProblem p{q, k, v, dout, H, T, dk, dv, feature_map_id, gamma, normalize, eps,
                    S_init, Z_init, dS_final, dZ_final, dq, dk_out, dv_out, dS_init, dZ_init};
  long long workers = nthreads > 0 ? nthreads
                                   : static_cast<long long>(std::thread::hardware_concurrency());
  if (workers < 1) workers = 1;
  if (workers > BH) workers = BH;
  std::vector<std::thread> pool;
  for (long long w = 0; w < workers; ++w)
    pool.emplace_back([&p, w, workers, BH]() {
      for (long long bh = w; bh < BH; bh += workers) backward_pair(p, bh);
    });
  for (auto& th : pool) th.join();
  return 0;
}

// The feature map alone, element-wise, for direct checks against closed forms.
int la_oracle_feature_map(const double* x, double* y, long long n, int feature_map_id) {
  if (feature_map_id != 0 && feature_map_id != 1) return 1;
  for (long long e = 0; e < n; ++e) y[e] = feature_map(x[e], feature_map_id);
  return 0;
}

}  // extern "C"
