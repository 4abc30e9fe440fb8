// Lizard hybrid attention: plain fp64 CPU oracle.
//
// TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously-correct
// definition that the CUDA library is checked against.  Only the tests, the
// smoke check and the CPU-baseline leg of the benchmark may load it; the
// product path never does.  It shares no code, header or table with the CUDA
// sources.
//
// Source of the definitions: "Lizard: An Efficient Linearization Framework
// for Large Language Models" (gist.science technical summary, section 2a
// "hybrid attention architecture"):
//   * gated linear attention: constant-size state S_i = Gamma_i S_{i-1} +
//     phi(k_i) v_i^T with a learnable per-dimension gate Gamma_i;
//   * anchor (sliding-window) softmax attention with learnable meta-memory
//     tokens that act as attention sinks in the softmax denominator;
//   * output = Y_gate + alpha * Y_anchor (weighted sum).
// Section 2c of the same summary (hardware-aware algorithm) motivates the
// chunked form, which is an exact rearrangement of the recurrence; it is
// implemented here only so that the identity can be tested.
//
// Readings taken where the page is silent:
//   * Gamma_t = diag(exp(g_t)) with g_t <= 0 the log-gate (a per-key-dim
//     vector); the state is decayed first, then the current token is added,
//     and the output reads the updated state: o_t = q_t^T S_t.
//   * phi is applied upstream: q and k arrive already featurized.
//   * the window holds keys j in [t-w+1, t] (w keys including the current
//     token); meta tokens are [H, M, d], shared across the batch, always
//     visible; their logits use the same scale as the window logits.
//   * meta values: meta_v == NULL is the sink-only reading (the meta tokens
//     add to the denominator only); a non-NULL meta_v adds p_m * mv_m to the
//     numerator.
//   * alpha is a plain scalar.
//
// Layouts (all row-major, contiguous):
//   q, k, g : [B, H, T, dk]     v, o : [B, H, T, dv]
//   h0, hT  : [B, H, dk, dv]    lse  : [B, H, T]
//   meta_k  : [H, M, dk]        meta_v : [H, M, dv]
// Every function returns 0 on success and a negative number on a bad
// argument.  Work is split over (batch, head) pairs with std::thread.

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdint>
#include <cstring>
#include <functional>
#include <thread>
#include <vector>

namespace {

void parallel_for(int n, int nthreads, const std::function<void(int)>& fn) {
  if (nthreads <= 0) nthreads = (int)std::thread::hardware_concurrency();
  if (nthreads <= 0) nthreads = 1;
  nthreads = std::min(nthreads, std::max(n, 1));
  std::atomic<int> next(0);
  auto worker = [&]() {
    for (;;) {
      int i = next.fetch_add(1);
      if (i >= n) break;
      fn(i);
    }
  };
  if (nthreads == 1) {
    worker();
    return;
  }
  std::vector<std::thread> pool;
  for (int t = 0; t < nthreads; ++t) pool.emplace_back(worker);
  for (auto& th : pool) th.join();
}

// ---------------------------------------------------------------------------
// Gated linear attention, token by token (section 2a, state update equation).
// ---------------------------------------------------------------------------
void gla_fwd_one(int T, int dk, int dv, const double* q, const double* k,
                 const double* v, const double* g, const double* h0,
                 double* o, double* hT) {
  std::vector<double> S((size_t)dk * dv, 0.0);
  if (h0) std::memcpy(S.data(), h0, sizeof(double) * dk * dv);
  for (int t = 0; t < T; ++t) {
    const double* qt = q + (size_t)t * dk;
    const double* kt = k + (size_t)t * dk;
    const double* vt = v + (size_t)t * dv;
    const double* gt = g + (size_t)t * dk;
    // S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T
    for (int i = 0; i < dk; ++i) {
      double decay = std::exp(gt[i]);
      for (int j = 0; j < dv; ++j)
        S[(size_t)i * dv + j] = decay * S[(size_t)i * dv + j] + kt[i] * vt[j];
    }
    // o_t = q_t^T S_t
    double* ot = o + (size_t)t * dv;
    for (int j = 0; j < dv; ++j) {
      double acc = 0.0;
      for (int i = 0; i < dk; ++i) acc += qt[i] * S[(size_t)i * dv + j];
      ot[j] = acc;
    }
  }
  if (hT) std::memcpy(hT, S.data(), sizeof(double) * dk * dv);
}

// ---------------------------------------------------------------------------
// Chunked form of the same recurrence (the rearrangement that section 2c
// builds on): inside a chunk the cumulative log-gate b_t = sum of g over the
// chunk up to t (inclusive) gives
//   o_t = (q_t * exp(b_t))^T S_prev + sum_{s<=t} [sum_i q_t,i k_s,i exp(b_t,i - b_s,i)] v_s
//   S   = diag(exp(b_last)) S_prev + sum_s diag(exp(b_last - b_s)) k_s v_s^T
// Exponentials are taken elementwise in fp64; this exists only for the
// chunked-equals-recurrent identity test.
// ---------------------------------------------------------------------------
void gla_chunked_one(int T, int dk, int dv, int C, const double* q,
                     const double* k, const double* v, const double* g,
                     const double* h0, double* o, double* hT) {
  std::vector<double> S((size_t)dk * dv, 0.0);
  if (h0) std::memcpy(S.data(), h0, sizeof(double) * dk * dv);
  std::vector<double> b((size_t)C * dk);
  std::vector<double> Snew((size_t)dk * dv);
  for (int c0 = 0; c0 < T; c0 += C) {
    int n = std::min(C, T - c0);
    for (int i = 0; i < dk; ++i) {
      double run = 0.0;
      for (int r = 0; r < n; ++r) {
        run += g[(size_t)(c0 + r) * dk + i];
        b[(size_t)r * dk + i] = run;
      }
    }
    for (int r = 0; r < n; ++r) {
      const double* qt = q + (size_t)(c0 + r) * dk;
      double* ot = o + (size_t)(c0 + r) * dv;
      for (int j = 0; j < dv; ++j) ot[j] = 0.0;
      // inter-chunk part
      for (int i = 0; i < dk; ++i) {
        double qi = qt[i] * std::exp(b[(size_t)r * dk + i]);
        for (int j = 0; j < dv; ++j) ot[j] += qi * S[(size_t)i * dv + j];
      }
      // intra-chunk part
      for (int s = 0; s <= r; ++s) {
        const double* ks = k + (size_t)(c0 + s) * dk;
        const double* vs = v + (size_t)(c0 + s) * dv;
        double a = 0.0;
        for (int i = 0; i < dk; ++i)
          a += qt[i] * ks[i] *
               std::exp(b[(size_t)r * dk + i] - b[(size_t)s * dk + i]);
        for (int j = 0; j < dv; ++j) ot[j] += a * vs[j];
      }
    }
    const double* blast = b.data() + (size_t)(n - 1) * dk;
    for (int i = 0; i < dk; ++i) {
      double decay = std::exp(blast[i]);
      for (int j = 0; j < dv; ++j) Snew[(size_t)i * dv + j] = decay * S[(size_t)i * dv + j];
    }
    for (int s = 0; s < n; ++s) {
      const double* ks = k + (size_t)(c0 + s) * dk;
      const double* vs = v + (size_t)(c0 + s) * dv;
      for (int i = 0; i < dk; ++i) {
        double f = ks[i] * std::exp(blast[i] - b[(size_t)s * dk + i]);
        for (int j = 0; j < dv; ++j) Snew[(size_t)i * dv + j] += f * vs[j];
      }
    }
    S.swap(Snew);
  }
  if (hT) std::memcpy(hT, S.data(), sizeof(double) * dk * dv);
}

// ---------------------------------------------------------------------------
// Sliding-window softmax attention with meta-memory sinks (section 2a,
// "anchor window attention"), brute force per query.
// ---------------------------------------------------------------------------
void swa_fwd_one(int T, int dk, int dv, int w, int M, double scale,
                 const double* q, const double* k, const double* v,
                 const double* mk, const double* mv, double* o, double* lse) {
  std::vector<double> logit((size_t)w + M);
  for (int t = 0; t < T; ++t) {
    const double* qt = q + (size_t)t * dk;
    int lo = std::max(0, t - w + 1);
    int nwin = t - lo + 1;
    double mu = -INFINITY;
    for (int j = lo; j <= t; ++j) {
      double a = 0.0;
      for (int i = 0; i < dk; ++i) a += qt[i] * k[(size_t)j * dk + i];
      a *= scale;
      logit[j - lo] = a;
      mu = std::max(mu, a);
    }
    for (int m = 0; m < M; ++m) {
      double a = 0.0;
      for (int i = 0; i < dk; ++i) a += qt[i] * mk[(size_t)m * dk + i];
      a *= scale;
      logit[nwin + m] = a;
      mu = std::max(mu, a);
    }
    double l = 0.0;
    double* ot = o + (size_t)t * dv;
    for (int j = 0; j < dv; ++j) ot[j] = 0.0;
    for (int j = lo; j <= t; ++j) {
      double p = std::exp(logit[j - lo] - mu);
      l += p;
      for (int c = 0; c < dv; ++c) ot[c] += p * v[(size_t)j * dv + c];
    }
    for (int m = 0; m < M; ++m) {
      double p = std::exp(logit[nwin + m] - mu);
      l += p;  // a sink always enters the denominator
      if (mv)
        for (int c = 0; c < dv; ++c) ot[c] += p * mv[(size_t)m * dv + c];
    }
    for (int c = 0; c < dv; ++c) ot[c] /= l;
    if (lse) lse[t] = mu + std::log(l);
  }
}

// ---------------------------------------------------------------------------
// Gradient of the gated recurrence, written out by hand (needed because the
// first training stage regresses attention outputs, section 2b).  With
// dS = total dL/dS_t accumulated in reverse:
//   dS_t  = q_t dO_t^T + diag(exp(g_{t+1})) dS_{t+1}   (dS_{T-1} also gets dhT)
//   dq_t  = S_t dO_t,  dk_t = dS_t v_t,  dv_t = dS_t^T k_t
//   dg_t,i = exp(g_t,i) * sum_j dS_t,ij S_{t-1},ij
//   dh0   = diag(exp(g_0)) dS_0
// States are checkpointed every CK tokens and recomputed per segment.
// ---------------------------------------------------------------------------
void gla_bwd_one(int T, int dk, int dv, const double* q, const double* k,
                 const double* v, const double* g, const double* h0,
                 const double* dO, const double* dhT, double* dq, double* dkk,
                 double* dvv, double* dg, double* dh0) {
  const int CK = 64;
  const size_t SS = (size_t)dk * dv;
  int nseg = (T + CK - 1) / CK;
  // ckpt[c] = state before the first token of segment c
  std::vector<double> ckpt((size_t)std::max(nseg, 1) * SS, 0.0);
  std::vector<double> S(SS, 0.0);
  if (h0) std::memcpy(S.data(), h0, sizeof(double) * SS);
  for (int c = 0; c < nseg; ++c) {
    std::memcpy(ckpt.data() + (size_t)c * SS, S.data(), sizeof(double) * SS);
    int t1 = std::min(T, (c + 1) * CK);
    for (int t = c * CK; t < t1; ++t)
      for (int i = 0; i < dk; ++i) {
        double decay = std::exp(g[(size_t)t * dk + i]);
        for (int j = 0; j < dv; ++j)
          S[(size_t)i * dv + j] =
              decay * S[(size_t)i * dv + j] + k[(size_t)t * dk + i] * v[(size_t)t * dv + j];
      }
  }
  std::vector<double> dS(SS, 0.0);
  if (dhT) std::memcpy(dS.data(), dhT, sizeof(double) * SS);
  // states[r] = S_{t0-1+r}, r = 0..n
  std::vector<double> states((size_t)(CK + 1) * SS);
  for (int c = nseg - 1; c >= 0; --c) {
    int t0 = c * CK, t1 = std::min(T, (c + 1) * CK);
    std::memcpy(states.data(), ckpt.data() + (size_t)c * SS, sizeof(double) * SS);
    for (int t = t0; t < t1; ++t) {
      const double* prev = states.data() + (size_t)(t - t0) * SS;
      double* cur = states.data() + (size_t)(t - t0 + 1) * SS;
      for (int i = 0; i < dk; ++i) {
        double decay = std::exp(g[(size_t)t * dk + i]);
        for (int j = 0; j < dv; ++j)
          cur[(size_t)i * dv + j] =
              decay * prev[(size_t)i * dv + j] + k[(size_t)t * dk + i] * v[(size_t)t * dv + j];
      }
    }
    for (int t = t1 - 1; t >= t0; --t) {
      const double* St = states.data() + (size_t)(t - t0 + 1) * SS;
      const double* Sp = states.data() + (size_t)(t - t0) * SS;
      const double* qt = q + (size_t)t * dk;
      const double* kt = k + (size_t)t * dk;
      const double* vt = v + (size_t)t * dv;
      const double* gt = g + (size_t)t * dk;
      const double* dot = dO + (size_t)t * dv;
      for (int i = 0; i < dk; ++i)
        for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] += qt[i] * dot[j];
      for (int i = 0; i < dk; ++i) {
        double a = 0.0, bsum = 0.0, gsum = 0.0;
        for (int j = 0; j < dv; ++j) {
          a += St[(size_t)i * dv + j] * dot[j];
          bsum += dS[(size_t)i * dv + j] * vt[j];
          gsum += dS[(size_t)i * dv + j] * Sp[(size_t)i * dv + j];
        }
        dq[(size_t)t * dk + i] = a;
        dkk[(size_t)t * dk + i] = bsum;
        dg[(size_t)t * dk + i] = std::exp(gt[i]) * gsum;
      }
      for (int j = 0; j < dv; ++j) {
        double a = 0.0;
        for (int i = 0; i < dk; ++i) a += dS[(size_t)i * dv + j] * kt[i];
        dvv[(size_t)t * dv + j] = a;
      }
      for (int i = 0; i < dk; ++i) {
        double decay = std::exp(gt[i]);
        for (int j = 0; j < dv; ++j) dS[(size_t)i * dv + j] *= decay;
      }
    }
  }
  if (dh0) std::memcpy(dh0, dS.data(), sizeof(double) * SS);
}

// ---------------------------------------------------------------------------
// Gradient of the window + meta softmax (textbook softmax Jacobian, per
// query).  dO here is dL/d(o_swa).  Key gradients accumulate over the
// queries that see the key; meta gradients are written per (batch, head)
// into dmk_part / dmv_part and summed over the batch by the caller.
// ---------------------------------------------------------------------------
void swa_bwd_one(int T, int dk, int dv, int w, int M, double scale,
                 const double* q, const double* k, const double* v,
                 const double* mk, const double* mv, const double* dO,
                 double* dq, double* dkk, double* dvv, double* dmk_part,
                 double* dmv_part) {
  std::vector<double> logit((size_t)w + M), p((size_t)w + M), dp((size_t)w + M);
  std::vector<double> ot(dv);
  for (size_t x = 0; x < (size_t)T * dk; ++x) dkk[x] = 0.0;
  for (size_t x = 0; x < (size_t)T * dv; ++x) dvv[x] = 0.0;
  for (int t = 0; t < T; ++t) {
    const double* qt = q + (size_t)t * dk;
    const double* dot = dO + (size_t)t * dv;
    int lo = std::max(0, t - w + 1);
    int nwin = t - lo + 1;
    int nall = nwin + M;
    double mu = -INFINITY;
    for (int x = 0; x < nall; ++x) {
      const double* key = x < nwin ? k + (size_t)(lo + x) * dk : mk + (size_t)(x - nwin) * dk;
      double a = 0.0;
      for (int i = 0; i < dk; ++i) a += qt[i] * key[i];
      logit[x] = a * scale;
      mu = std::max(mu, logit[x]);
    }
    double l = 0.0;
    for (int x = 0; x < nall; ++x) {
      p[x] = std::exp(logit[x] - mu);
      l += p[x];
    }
    for (int x = 0; x < nall; ++x) p[x] /= l;
    for (int c = 0; c < dv; ++c) ot[c] = 0.0;
    for (int x = 0; x < nall; ++x) {
      const double* val = x < nwin ? v + (size_t)(lo + x) * dv
                                   : (mv ? mv + (size_t)(x - nwin) * dv : nullptr);
      double d = 0.0;
      if (val) {
        for (int c = 0; c < dv; ++c) {
          d += dot[c] * val[c];
          ot[c] += p[x] * val[c];
        }
      }
      dp[x] = d;
    }
    double D = 0.0;  // = dO_t . o_t = sum_x p_x dp_x
    for (int c = 0; c < dv; ++c) D += dot[c] * ot[c];
    double* dqt = dq + (size_t)t * dk;
    for (int i = 0; i < dk; ++i) dqt[i] = 0.0;
    for (int x = 0; x < nall; ++x) {
      double ds = p[x] * (dp[x] - D);  // dL/dlogit_x
      const double* key;
      double* dkey;
      double* dval;
      if (x < nwin) {
        key = k + (size_t)(lo + x) * dk;
        dkey = dkk + (size_t)(lo + x) * dk;
        dval = dvv + (size_t)(lo + x) * dv;
      } else {
        key = mk + (size_t)(x - nwin) * dk;
        dkey = dmk_part + (size_t)(x - nwin) * dk;
        dval = mv ? dmv_part + (size_t)(x - nwin) * dv : nullptr;
      }
      for (int i = 0; i < dk; ++i) {
        dqt[i] += scale * ds * key[i];
        dkey[i] += scale * ds * qt[i];
      }
      if (dval)
        for (int c = 0; c < dv; ++c) dval[c] += p[x] * dot[c];
    }
  }
}

}  // namespace

extern "C" {

int oracle_gla_fwd(int B, int H, int T, int dk, int dv, const double* q,
                   const double* k, const double* v, const double* g,
                   const double* h0, double* o, double* hT, int nthreads) {
  if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return -1;
  parallel_for(B * H, nthreads, [&](int bh) {
    size_t tk = (size_t)bh * T * dk, tv = (size_t)bh * T * dv, ss = (size_t)bh * dk * dv;
    gla_fwd_one(T, dk, dv, q + tk, k + tk, v + tv, g + tk, h0 ? h0 + ss : nullptr,
                o + tv, hT ? hT + ss : nullptr);
  });
  return 0;
}

int oracle_gla_chunked_fwd(int B, int H, int T, int dk, int dv, int C,
                           const double* q, const double* k, const double* v,
                           const double* g, const double* h0, double* o,
                           double* hT, int nthreads) {
  if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0 || C <= 0) return -1;
  parallel_for(B * H, nthreads, [&](int bh) {
    size_t tk = (size_t)bh * T * dk, tv = (size_t)bh * T * dv, ss = (size_t)bh * dk * dv;
    gla_chunked_one(T, dk, dv, C, q + tk, k + tk, v + tv, g + tk,
                    h0 ? h0 + ss : nullptr, o + tv, hT ? hT + ss : nullptr);
  });
  return 0;
}

int oracle_swa_meta_fwd(int B, int H, int T, int dk, int dv, int w, int M,
                        double scale, const double* q, const double* k,
                        const double* v, const double* mk, const double* mv,
                        double* o, double* lse, int nthreads) {
  if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0 || w < 1 || M < 0) return -1;
  if (M > 0 && !mk) return -1;
  parallel_for(B * H, nthreads, [&](int bh) {
    int h = bh % H;
    size_t tk = (size_t)bh * T * dk, tv = (size_t)bh * T * dv;
    swa_fwd_one(T, dk, dv, w, M, scale, q + tk, k + tk, v + tv,
                M ? mk + (size_t)h * M * dk : nullptr,
                (M && mv) ? mv + (size_t)h * M * dv : nullptr, o + tv,
                lse ? lse + (size_t)bh * T : nullptr);
  });
  return 0;
}

// o = o_gla + alpha * o_swa  (section 2a, final output).  o_swa, lse, hT are
// optional extra outputs.
int oracle_hybrid_fwd(int B, int H, int T, int dk, int dv, int w, int M,
                      double scale, double alpha, const double* q,
                      const double* k, const double* v, const double* g,
                      const double* mk, const double* mv, const double* h0,
                      double* o, double* hT, double* lse, double* o_swa,
                      int nthreads) {
  if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0 || w < 1 || M < 0) return -1;
  if (M > 0 && !mk) return -1;
  parallel_for(B * H, nthreads, [&](int bh) {
    int h = bh % H;
    size_t tk = (size_t)bh * T * dk, tv = (size_t)bh * T * dv, ss = (size_t)bh * dk * dv;
    std::vector<double> og((size_t)T * dv), os((size_t)T * dv);
    gla_fwd_one(T, dk, dv, q + tk, k + tk, v + tv, g + tk, h0 ? h0 + ss : nullptr,
                og.data(), hT ? hT + ss : nullptr);
    swa_fwd_one(T, dk, dv, w, M, scale, q + tk, k + tk, v + tv,
                M ? mk + (size_t)h * M * dk : nullptr,
                (M && mv) ? mv + (size_t)h * M * dv : nullptr, os.data(),
                lse ? lse + (size_t)bh * T : nullptr);
    for (size_t x = 0; x < (size_t)T * dv; ++x) {
      o[tv + x] = og[x] + alpha * os[x];
      if (o_swa) o_swa[tv + x] = os[x];
    }
  });
  return 0;
}

int oracle_gla_bwd(int B, int H, int T, int dk, int dv, const double* q,
                   const double* k, const double* v, const double* g,
                   const double* h0, const double* dO, const double* dhT,
                   double* dq, double* dkk, double* dvv, double* dg,
                   double* dh0, int nthreads) {
  if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0) return -1;
  parallel_for(B * H, nthreads, [&](int bh) {
    size_t tk = (size_t)bh * T * dk, tv = (size_t)bh * T * dv, ss = (size_t)bh * dk * dv;
    gla_bwd_one(T, dk, dv, q + tk, k + tk, v + tv, g + tk, h0 ? h0 + ss : nullptr,
                dO + tv, dhT ? dhT + ss : nullptr, dq + tk, dkk + tk, dvv + tv,
                dg + tk, dh0 ? dh0 + ss : nullptr);
  });
  return 0;
}

// dO is dL/d(o_swa).  dmk [H,M,dk] and dmv [H,M,dv] are summed over the batch
// and the sequence; dmv is skipped in sink-only mode (mv == NULL).
int oracle_swa_meta_bwd(int B, int H, int T, int dk, int dv, int w, int M,
                        double scale, const double* q, const double* k,
                        const double* v, const double* mk, const double* mv,
                        const double* dO, double* dq, double* dkk, double* dvv,
                        double* dmk, double* dmv, int nthreads) {
  if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0 || w < 1 || M < 0) return -1;
  if (M > 0 && !mk) return -1;
  std::vector<double> pk((size_t)B * H * std::max(M, 1) * dk, 0.0);
  std::vector<double> pv((size_t)B * H * std::max(M, 1) * dv, 0.0);
  parallel_for(B * H, nthreads, [&](int bh) {
    int h = bh % H;
    size_t tk = (size_t)bh * T * dk, tv = (size_t)bh * T * dv;
    swa_bwd_one(T, dk, dv, w, M, scale, q + tk, k + tk, v + tv,
                M ? mk + (size_t)h * M * dk : nullptr,
                (M && mv) ? mv + (size_t)h * M * dv : nullptr, dO + tv, dq + tk,
                dkk + tk, dvv + tv, pk.data() + (size_t)bh * M * dk,
                pv.data() + (size_t)bh * M * dv);
  });
  if (M > 0) {
    if (dmk) {
      for (size_t x = 0; x < (size_t)H * M * dk; ++x) dmk[x] = 0.0;
      for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
          for (size_t x = 0; x < (size_t)M * dk; ++x)
            dmk[(size_t)h * M * dk + x] += pk[((size_t)b * H + h) * M * dk + x];
    }
    if (dmv && mv) {
      for (size_t x = 0; x < (size_t)H * M * dv; ++x) dmv[x] = 0.0;
      for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
          for (size_t x = 0; x < (size_t)M * dv; ++x)
            dmv[(size_t)h * M * dv + x] += pv[((size_t)b * H + h) * M * dv + x];
    }
  }
  return 0;
}

// Gradient of o = o_gla + alpha * o_swa: the gated branch sees dO, the window
// branch sees alpha * dO, and dalpha = sum over all (b,h,t) of dO_t . o_swa_t.
int oracle_hybrid_bwd(int B, int H, int T, int dk, int dv, int w, int M,
                      double scale, double alpha, const double* q,
                      const double* k, const double* v, const double* g,
                      const double* mk, const double* mv, const double* h0,
                      const double* dO, const double* dhT, double* dq,
                      double* dkk, double* dvv, double* dg, double* dh0,
                      double* dmk, double* dmv, double* dalpha, int nthreads) {
  if (B < 0 || H < 0 || T < 0 || dk <= 0 || dv <= 0 || w < 1 || M < 0) return -1;
  if (M > 0 && !mk) return -1;
  int n = B * H;
  std::vector<double> pk((size_t)n * std::max(M, 1) * dk, 0.0);
  std::vector<double> pv((size_t)n * std::max(M, 1) * dv, 0.0);
  std::vector<double> pa((size_t)std::max(n, 1), 0.0);
  parallel_for(n, nthreads, [&](int bh) {
    int h = bh % H;
    size_t tk = (size_t)bh * T * dk, tv = (size_t)bh * T * dv, ss = (size_t)bh * dk * dv;
    gla_bwd_one(T, dk, dv, q + tk, k + tk, v + tv, g + tk, h0 ? h0 + ss : nullptr,
                dO + tv, dhT ? dhT + ss : nullptr, dq + tk, dkk + tk, dvv + tv,
                dg + tk, dh0 ? dh0 + ss : nullptr);
    std::vector<double> adO((size_t)T * dv);
    for (size_t x = 0; x < (size_t)T * dv; ++x) adO[x] = alpha * dO[tv + x];
    std::vector<double> sq((size_t)T * dk), sk((size_t)T * dk), sv((size_t)T * dv);
    swa_bwd_one(T, dk, dv, w, M, scale, q + tk, k + tk, v + tv,
                M ? mk + (size_t)h * M * dk : nullptr,
                (M && mv) ? mv + (size_t)h * M * dv : nullptr, adO.data(),
                sq.data(), sk.data(), sv.data(), pk.data() + (size_t)bh * M * dk,
                pv.data() + (size_t)bh * M * dv);
    // dalpha part: sum_t dO_t . o_swa_t with o_swa recomputed
    std::vector<double> os((size_t)T * dv);
    swa_fwd_one(T, dk, dv, w, M, scale, q + tk, k + tk, v + tv,
                M ? mk + (size_t)h * M * dk : nullptr,
                (M && mv) ? mv + (size_t)h * M * dv : nullptr, os.data(), nullptr);
    double s = 0.0;
    for (size_t x = 0; x < (size_t)T * dv; ++x) s += dO[tv + x] * os[x];
    pa[bh] = s;
    for (size_t x = 0; x < (size_t)T * dk; ++x) {
      dq[tk + x] += sq[x];
      dkk[tk + x] += sk[x];
    }
    for (size_t x = 0; x < (size_t)T * dv; ++x) dvv[tv + x] += sv[x];
  });
  if (M > 0) {
    if (dmk) {
      for (size_t x = 0; x < (size_t)H * M * dk; ++x) dmk[x] = 0.0;
      for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
          for (size_t x = 0; x < (size_t)M * dk; ++x)
            dmk[(size_t)h * M * dk + x] += pk[((size_t)b * H + h) * M * dk + x];
    }
    if (dmv && mv) {
      for (size_t x = 0; x < (size_t)H * M * dv; ++x) dmv[x] = 0.0;
      for (int b = 0; b < B; ++b)
        for (int h = 0; h < H; ++h)
          for (size_t x = 0; x < (size_t)M * dv; ++x)
            dmv[(size_t)h * M * dv + x] += pv[((size_t)b * H + h) * M * dv + x];
    }
  }
  if (dalpha) {
    double s = 0.0;
    for (int x = 0; x < n; ++x) s += pa[x];
    *dalpha = s;
  }
  return 0;
}

// One constant-memory generation step for Bd sequences (section 2a: the
// fixed-size state replaces the growing KV cache).  In place:
//   state [Bd,H,dk,dv], kring [Bd,H,w,dk], vring [Bd,H,w,dv], pos [Bd].
// Per sequence b with p = pos[b]: the new key/value go to ring slot p mod w;
// S = diag(exp(g)) S + k v^T; o_gla = q^T S; the window is the last
// min(p+1, w) tokens (the new one included) plus the M meta tokens;
// o = o_gla + alpha * o_swa; pos[b] = p + 1.
int oracle_decode_step(int Bd, int H, int dk, int dv, int w, int M,
                       double scale, double alpha, double* state,
                       double* kring, double* vring, int64_t* pos,
                       const double* q, const double* k, const double* v,
                       const double* g, const double* mk, const double* mv,
                       double* o, int nthreads) {
  if (Bd < 0 || H < 0 || dk <= 0 || dv <= 0 || w < 1 || M < 0) return -1;
  if (M > 0 && !mk) return -1;
  for (int b = 0; b < Bd; ++b)
    if (pos[b] < 0) return -1;
  parallel_for(Bd * H, nthreads, [&](int bh) {
    int b = bh / H, h = bh % H;
    int64_t p = pos[b];
    int slot = (int)(p % w);
    const double* qt = q + (size_t)bh * dk;
    const double* kt = k + (size_t)bh * dk;
    const double* vt = v + (size_t)bh * dv;
    const double* gt = g + (size_t)bh * dk;
    double* S = state + (size_t)bh * dk * dv;
    double* kr = kring + (size_t)bh * w * dk;
    double* vr = vring + (size_t)bh * w * dv;
    for (int i = 0; i < dk; ++i) kr[(size_t)slot * dk + i] = kt[i];
    for (int j = 0; j < dv; ++j) vr[(size_t)slot * dv + j] = vt[j];
    std::vector<double> og(dv, 0.0), os(dv, 0.0);
    for (int i = 0; i < dk; ++i) {
      double decay = std::exp(gt[i]);
      for (int j = 0; j < dv; ++j)
        S[(size_t)i * dv + j] = decay * S[(size_t)i * dv + j] + kt[i] * vt[j];
    }
    for (int j = 0; j < dv; ++j)
      for (int i = 0; i < dk; ++i) og[j] += qt[i] * S[(size_t)i * dv + j];
    int nwin = (int)std::min<int64_t>(p + 1, w);
    std::vector<double> logit((size_t)nwin + M);
    std::vector<int> slots(nwin);
    double mu = -INFINITY;
    for (int x = 0; x < nwin; ++x) {
      int64_t tok = p - x;  // tokens p, p-1, ..., p-nwin+1
      slots[x] = (int)(tok % w);
      double a = 0.0;
      for (int i = 0; i < dk; ++i) a += qt[i] * kr[(size_t)slots[x] * dk + i];
      logit[x] = a * scale;
      mu = std::max(mu, logit[x]);
    }
    for (int m = 0; m < M; ++m) {
      const double* key = mk + ((size_t)h * M + m) * dk;
      double a = 0.0;
      for (int i = 0; i < dk; ++i) a += qt[i] * key[i];
      logit[nwin + m] = a * scale;
      mu = std::max(mu, logit[nwin + m]);
    }
    double l = 0.0;
    for (int x = 0; x < nwin; ++x) {
      double pr = std::exp(logit[x] - mu);
      l += pr;
      for (int j = 0; j < dv; ++j) os[j] += pr * vr[(size_t)slots[x] * dv + j];
    }
    for (int m = 0; m < M; ++m) {
      double pr = std::exp(logit[nwin + m] - mu);
      l += pr;
      if (mv)
        for (int j = 0; j < dv; ++j) os[j] += pr * mv[((size_t)h * M + m) * dv + j];
    }
    for (int j = 0; j < dv; ++j) o[(size_t)bh * dv + j] = og[j] + alpha * os[j] / l;
  });
  for (int b = 0; b < Bd; ++b) pos[b] += 1;
  return 0;
}

// Gate from its logit (section 2a: the learnable gate is Gamma_i =
// sigma(W_gamma x_i), so the logit z = W_gamma x_i arrives from the
// projection upstream).  The log-gate the recurrence uses is
//   g = scale * log sigma(z)  (<= 0; scale > 0 a temperature, 1 on the page)
// with log sigma(z) = -log(1 + e^{-z}) taken in the form that does not
// overflow for either sign of z.  n elements; g_out may alias nothing.
int oracle_gate_from_logits(int64_t n, const double* z, double scale, double* g_out) {
  if (n < 0 || !(scale > 0.0)) return -1;
  if (n > 0 && (!z || !g_out)) return -1;
  for (int64_t x = 0; x < n; ++x) {
    const double v = z[x];
    const double ls = v >= 0.0 ? -std::log1p(std::exp(-v)) : v - std::log1p(std::exp(v));
    g_out[x] = scale * ls;
  }
  return 0;
}

// Chain rule through that map: dL/dz = dL/dg * scale * sigma(-z), with
// sigma(-z) = 1 / (1 + e^{z}) taken without overflow.
int oracle_dlogits(int64_t n, const double* z, double scale, const double* dg, double* dz) {
  if (n < 0 || !(scale > 0.0)) return -1;
  if (n > 0 && (!z || !dg || !dz)) return -1;
  for (int64_t x = 0; x < n; ++x) {
    const double v = z[x];
    const double sneg = v >= 0.0 ? std::exp(-v) / (1.0 + std::exp(-v)) : 1.0 / (1.0 + std::exp(v));
    dz[x] = dg[x] * scale * sneg;
  }
  return 0;
}

// The projections in front of the operator (section 2a: the gate is
// Gamma_i = sigma(W_gamma x_i); the state update takes phi(k_i) and the output
// reads q_i).  For hidden states x [B][T][Dm] and weights W [H*dk][Dm] (one
// row per output feature): q = x Wq^T and k = x Wk^T with phi the identity
// (the pages do not define phi; reading: the operator receives the featurised
// keys), g = scale * log sigma(x Wg^T) through oracle_gate_from_logits.
// Outputs in the operator's layout [B][H][T][dk]; a NULL weight skips its
// output.
int oracle_qkg_projection(int B, int T, int Dm, int H, int dk, const double* x, const double* Wq,
                          const double* Wk, const double* Wg, double scale, double* q, double* k,
                          double* g) {
  if (B < 0 || T < 0 || Dm < 1 || H < 1 || dk < 1 || !(scale > 0.0)) return -1;
  const double* W[3] = {Wq, Wk, Wg};
  double* out[3] = {q, k, g};
  std::vector<double> z((size_t)dk);
  for (int which = 0; which < 3; ++which) {
    if (!W[which]) continue;
    if (!out[which] || (B * T > 0 && !x)) return -1;
    for (int b = 0; b < B; ++b)
      for (int t = 0; t < T; ++t) {
        const double* xr = x + ((size_t)b * T + t) * Dm;
        for (int h = 0; h < H; ++h) {
          for (int i = 0; i < dk; ++i) {
            const double* wr = W[which] + ((size_t)h * dk + i) * Dm;
            double acc = 0.0;
            for (int c = 0; c < Dm; ++c) acc += xr[c] * wr[c];
            z[i] = acc;
          }
          double* dst = out[which] + (((size_t)b * H + h) * T + t) * dk;
          if (which == 2) {
            if (oracle_gate_from_logits(dk, z.data(), scale, dst) != 0) return -1;
          } else {
            for (int i = 0; i < dk; ++i) dst[i] = z[i];
          }
        }
      }
  }
  return 0;
}

// Stage-1 distillation loss (section 2b, "training strategy": the first
// stage trains the hybrid attention to reproduce the teacher's attention
// output under a mean-squared-error loss).  Reading: the mean runs over every
// element of the output tensor (n = B*H*T*dv elements):
//   loss = (1/n) sum_x (o_x - target_x)^2,   dO_x = dloss/do_x = 2 (o_x - target_x) / n.
// dO may be NULL.  n == 0 gives loss 0.
int oracle_mse_loss(int64_t n, const double* o, const double* target, double* loss,
                    double* dO) {
  if (n < 0 || !loss) return -1;
  if (n > 0 && (!o || !target)) return -1;
  double s = 0.0;
  for (int64_t x = 0; x < n; ++x) {
    const double diff = o[x] - target[x];
    s += diff * diff;
    if (dO) dO[x] = 2.0 * diff / (double)n;
  }
  *loss = n > 0 ? s / (double)n : 0.0;
  return 0;
}

}  // extern "C"
