// Gated linear attention, chunked, fp32 SIMT arithmetic (fp32 or bf16 I/O).
//
// Recurrence (Lizard technical summary, section 2a, state update equation):
//   S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T,   o_t = q_t^T S_t.
// Chunked form over 16-token chunks with b_t the inclusive running sum of g
// inside the chunk and b_l its value at the chunk's last row:
//   o_t  = (q_t * e^{b_t})^T S_prev + sum_{s<=t} A[t][s] v_s
//   A[t][s] = sum_i q_t,i k_s,i e^{b_t,i - b_s,i}
//           = sum_i (q_t,i e^{b_t,i - b_l,i}) (k_s,i e^{b_l,i - b_s,i})
//   S    = diag(e^{b_l}) S_prev + sum_s (k_s * e^{b_l - b_s}) v_s^T
// Every factor above is <= 1 except q*e^{b_t-b_l} (<= e^{span}); when the
// chunk's gate span exceeds kSpanLimit the scores take exp(b_t-b_s) per
// element instead.  This is the fp32 I/O path and the reference structure
// for the tensor-core kernels.
#include "common.cuh"
#include "kernels.h"

namespace lz {
namespace {

constexpr int SC = kSimtChunk;  // 16 rows per chunk
constexpr int DVT = 32;         // value columns per CTA
constexpr int NT = 256;         // threads (== SC * SC)
static_assert(NT == SC * SC, "score tile mapping needs one thread per pair");

template <int DK>
constexpr size_t fwd_smem_floats() {
  return (size_t)SC * DK + 3 * SC * (DK + 1) + SC * DVT + DK * DVT + SC * (SC + 1) + DK;
}

template <typename IO, int DK>
__global__ void __launch_bounds__(NT) gla_fwd_simt_kernel(GlaFwdParams p) {
  extern __shared__ float smem[];
  constexpr int DKP = DK + 1;
  float* bs = smem;               // [SC][DK]   running log-gate
  float* qi = bs + SC * DK;       // [SC][DKP]  q e^{b}
  float* qt = qi + SC * DKP;      // [SC][DKP]  q e^{b - b_l}
  float* kt = qt + SC * DKP;      // [SC][DKP]  k e^{b_l - b}
  float* vs = kt + SC * DKP;      // [SC][DVT]
  float* S = vs + SC * DVT;       // [DK][DVT]
  float* A = S + DK * DVT;        // [SC][SC+1]
  float* el = A + SC * (SC + 1);  // [DK] e^{b_l}
  __shared__ int slow;

  const int tid = threadIdx.x;
  const int j0 = blockIdx.x * DVT;
  const int bh = blockIdx.y;
  const int T = p.T, DV = p.dv;
  const IO* q = (const IO*)p.q + (size_t)bh * T * DK;
  const IO* k = (const IO*)p.k + (size_t)bh * T * DK;
  const IO* v = (const IO*)p.v + (size_t)bh * T * DV;
  const float* g = p.g + (size_t)bh * T * DK;
  const bool want_o = p.o != nullptr;

  for (int x = tid; x < DK * DVT; x += NT) {
    int i = x / DVT, j = x % DVT;
    S[x] = p.h0 ? p.h0[((size_t)bh * DK + i) * DV + j0 + j] : 0.f;
  }
  const int nchunks = (T + SC - 1) / SC;
  for (int c = 0; c < nchunks; ++c) {
    const int c0 = c * SC;
    const int n = min(SC, T - c0);
    __syncthreads();
    if (p.states) {
      float* dst = p.states + ((size_t)bh * nchunks + c) * DK * DV + j0;
      for (int x = tid; x < DK * DVT; x += NT) {
        int i = x / DVT, j = x % DVT;
        dst[(size_t)i * DV + j] = S[x];
      }
    }
    for (int x = tid; x < SC * DK; x += NT) {
      int r = x / DK, i = x % DK;
      bs[x] = (r < n) ? g[(size_t)(c0 + r) * DK + i] : 0.f;
    }
    for (int x = tid; x < SC * DVT; x += NT) {
      int r = x / DVT, j = x % DVT;
      vs[x] = (r < n) ? ldf(v + (size_t)(c0 + r) * DV + j0 + j) : 0.f;
    }
    if (tid == 0) slow = 0;
    __syncthreads();
    for (int i = tid; i < DK; i += NT) {
      float run = 0.f;
#pragma unroll
      for (int r = 0; r < SC; ++r) {
        run += bs[r * DK + i];
        bs[r * DK + i] = run;
      }
      el[i] = expf(run);
      if (-run > kSpanLimit) slow = 1;
    }
    __syncthreads();
    for (int x = tid; x < SC * DK; x += NT) {
      int r = x / DK, i = x % DK;
      float b = bs[x], bl = bs[(SC - 1) * DK + i];
      float qv = (r < n) ? ldf(q + (size_t)(c0 + r) * DK + i) : 0.f;
      float kv = (r < n) ? ldf(k + (size_t)(c0 + r) * DK + i) : 0.f;
      qi[r * DKP + i] = qv * expf(b);
      qt[r * DKP + i] = qv * expf(b - bl);
      kt[r * DKP + i] = kv * expf(bl - b);
    }
    __syncthreads();
    if (want_o) {
      const int t = tid / SC, s = tid % SC;
      float a = 0.f;
      if (s <= t && t < n) {
        if (!slow) {
#pragma unroll 8
          for (int i = 0; i < DK; ++i) a += qt[t * DKP + i] * kt[s * DKP + i];
        } else {
          const IO* qr = q + (size_t)(c0 + t) * DK;
          const IO* kr = k + (size_t)(c0 + s) * DK;
          for (int i = 0; i < DK; ++i)
            a += ldf(qr + i) * ldf(kr + i) * expf(bs[t * DK + i] - bs[s * DK + i]);
        }
      }
      A[t * (SC + 1) + s] = a;
      __syncthreads();
      for (int x = tid; x < SC * DVT; x += NT) {
        int t2 = x / DVT, j = x % DVT;
        if (t2 >= n) continue;
        float acc = 0.f;
#pragma unroll 8
        for (int i = 0; i < DK; ++i) acc += qi[t2 * DKP + i] * S[i * DVT + j];
        for (int s2 = 0; s2 <= t2; ++s2) acc += A[t2 * (SC + 1) + s2] * vs[s2 * DVT + j];
        size_t off = ((size_t)bh * T + c0 + t2) * DV + j0 + j;
        if (p.add) acc += p.alpha * p.add[off];
        ((IO*)p.o)[off] = from_f<IO>(acc);
      }
      __syncthreads();
    }
    for (int x = tid; x < DK * DVT; x += NT) {
      int i = x / DVT, j = x % DVT;
      float acc = el[i] * S[x];
#pragma unroll
      for (int s2 = 0; s2 < SC; ++s2) acc += kt[s2 * DKP + i] * vs[s2 * DVT + j];
      S[x] = acc;
    }
  }
  __syncthreads();
  if (p.hT) {
    for (int x = tid; x < DK * DVT; x += NT) {
      int i = x / DVT, j = x % DVT;
      p.hT[((size_t)bh * DK + i) * DV + j0 + j] = S[x];
    }
  }
}

// Backward, one CTA per (batch, head), reverse walk over 16-token chunks.
// G is the gradient carried into the chunk from the future,
//   G = diag(e^{g_{next}}) dL/dS_{next}  (dhT at the end),
// and for t in the chunk (B[t][s] = dO_t . v_s, A as in the forward):
//   dq_t = e^{b_t} * (S_prev dO_t) + sum_{s<=t} B[t][s] k_s e^{b_t - b_s}
//   dk_t = e^{b_l - b_t} * (G v_t) + sum_{u>=t} B[u][t] q_u e^{b_u - b_t}
//   dv_t = (k_t e^{b_l - b_t})^T G + sum_{u>=t} A[u][t] dO_u
//   G   <- diag(e^{b_l}) G + sum_u (q_u e^{b_u})^T dO_u
// and dg is the reverse running sum of q*dq - k*dk, seeded with
// sum_j dhT_ij hT_ij at the last token (o and hT see the running log-gate
// only through q e^{G_t}, k e^{-G_s} and hT's factor e^{G_{T-1}}).
template <int DK, int DV>
constexpr size_t bwd_smem_floats() {
  return (size_t)DK * (DV + 1) + (DK / 2) * (DV + 1) + SC * DK + 7 * SC * (DK + 1) +
         2 * SC * (DV + 1) + 2 * SC * (SC + 1) + DK;
}

template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(NT) gla_bwd_simt_kernel(GlaBwdParams p) {
  extern __shared__ float smem[];
  constexpr int DKP = DK + 1, DVP = DV + 1, HK = DK / 2;
  float* G = smem;               // [DK][DVP]
  float* Sp = G + DK * DVP;      // [HK][DVP] half of S_prev
  float* bs = Sp + HK * DVP;     // [SC][DK]
  float* qs = bs + SC * DK;      // [SC][DKP]
  float* ks = qs + SC * DKP;
  float* qt = ks + SC * DKP;     // q e^{b - b_l}
  float* kt = qt + SC * DKP;     // k e^{b_l - b}
  float* qi = kt + SC * DKP;     // q e^{b}
  float* dqs = qi + SC * DKP;
  float* dks = dqs + SC * DKP;
  float* vs = dks + SC * DKP;    // [SC][DVP]
  float* dos = vs + SC * DVP;    // [SC][DVP]
  float* A = dos + SC * DVP;     // [SC][SC+1]
  float* Bm = A + SC * (SC + 1);
  float* el = Bm + SC * (SC + 1);  // [DK]
  __shared__ int slow;

  const int tid = threadIdx.x;
  const int bh = blockIdx.x;
  const int T = p.T;
  const size_t tk = (size_t)bh * T * DK, tv = (size_t)bh * T * DV;
  const IO* q = (const IO*)p.q + tk;
  const IO* k = (const IO*)p.k + tk;
  const IO* v = (const IO*)p.v + tv;
  const IO* dO = (const IO*)p.dO + tv;
  const float* g = p.g + tk;
  const int nchunks = (T + SC - 1) / SC;

  for (int x = tid; x < DK * DV; x += NT) {
    int i = x / DV, j = x % DV;
    G[i * DVP + j] = p.dhT ? p.dhT[(size_t)bh * DK * DV + x] : 0.f;
  }
  float run = 0.f;  // reverse running sum for dg (thread tid < DK owns dim tid)
  if (p.dhT && tid < DK) {
    const float* hTr = p.hT + ((size_t)bh * DK + tid) * DV;
    const float* dhr = p.dhT + ((size_t)bh * DK + tid) * DV;
    for (int j = 0; j < DV; ++j) run += dhr[j] * hTr[j];
  }

  for (int c = nchunks - 1; c >= 0; --c) {
    const int c0 = c * SC;
    const int n = min(SC, T - c0);
    __syncthreads();
    for (int x = tid; x < SC * DK; x += NT) {
      int r = x / DK, i = x % DK;
      bool ok = r < n;
      size_t off = (size_t)(c0 + r) * DK + i;
      bs[x] = ok ? g[off] : 0.f;
      qs[r * DKP + i] = ok ? ldf(q + off) : 0.f;
      ks[r * DKP + i] = ok ? ldf(k + off) : 0.f;
    }
    for (int x = tid; x < SC * DV; x += NT) {
      int r = x / DV, j = x % DV;
      bool ok = r < n;
      size_t off = (size_t)(c0 + r) * DV + j;
      vs[r * DVP + j] = ok ? ldf(v + off) : 0.f;
      dos[r * DVP + j] = ok ? ldf(dO + off) : 0.f;
    }
    if (tid == 0) slow = 0;
    __syncthreads();
    for (int i = tid; i < DK; i += NT) {
      float rs = 0.f;
#pragma unroll
      for (int r = 0; r < SC; ++r) {
        rs += bs[r * DK + i];
        bs[r * DK + i] = rs;
      }
      el[i] = expf(rs);
      if (-rs > kSpanLimit) slow = 1;
    }
    __syncthreads();
    for (int x = tid; x < SC * DK; x += NT) {
      int r = x / DK, i = x % DK;
      float b = bs[x], bl = bs[(SC - 1) * DK + i];
      float qv = qs[r * DKP + i], kv = ks[r * DKP + i];
      qi[r * DKP + i] = qv * expf(b);
      qt[r * DKP + i] = qv * expf(b - bl);
      kt[r * DKP + i] = kv * expf(bl - b);
    }
    __syncthreads();
    {
      const int t = tid / SC, s = tid % SC;
      float a = 0.f, bm = 0.f;
      if (s <= t) {
        if (!slow) {
#pragma unroll 8
          for (int i = 0; i < DK; ++i) a += qt[t * DKP + i] * kt[s * DKP + i];
        } else {
          for (int i = 0; i < DK; ++i)
            a += qs[t * DKP + i] * ks[s * DKP + i] * expf(bs[t * DK + i] - bs[s * DK + i]);
        }
#pragma unroll 8
        for (int j = 0; j < DV; ++j) bm += dos[t * DVP + j] * vs[s * DVP + j];
      }
      A[t * (SC + 1) + s] = a;
      Bm[t * (SC + 1) + s] = bm;
    }
    // dq, in two halves of the key dim so that only half of S_prev is staged
    const float* Sg = p.states + ((size_t)bh * nchunks + c) * DK * DV;
    for (int half = 0; half < 2; ++half) {
      __syncthreads();
      for (int x = tid; x < HK * DV; x += NT) {
        int il = x / DV, j = x % DV;
        Sp[il * DVP + j] = Sg[(size_t)(half * HK + il) * DV + j];
      }
      __syncthreads();
      for (int x = tid; x < SC * HK; x += NT) {
        int t = x / HK, il = x % HK, i = half * HK + il;
        float inter = 0.f;
#pragma unroll 8
        for (int j = 0; j < DV; ++j) inter += dos[t * DVP + j] * Sp[il * DVP + j];
        float b = bs[t * DK + i], bl = bs[(SC - 1) * DK + i];
        float intra = 0.f;
        if (!slow) {
          for (int s = 0; s <= t; ++s) intra += Bm[t * (SC + 1) + s] * kt[s * DKP + i];
          intra *= expf(b - bl);
        } else {
          for (int s = 0; s <= t; ++s)
            intra += Bm[t * (SC + 1) + s] * ks[s * DKP + i] * expf(b - bs[s * DK + i]);
        }
        float dqv = expf(b) * inter + intra;
        dqs[t * DKP + i] = dqv;
        if (t < n) {
          size_t off = tk + (size_t)(c0 + t) * DK + i;
          float outv = dqv + (p.add_dq ? p.add_dq[off] : 0.f);
          ((IO*)p.dq)[off] = from_f<IO>(outv);
        }
      }
    }
    // dk
    for (int x = tid; x < SC * DK; x += NT) {
      int t = x / DK, i = x % DK;
      float b = bs[t * DK + i], bl = bs[(SC - 1) * DK + i];
      float inter = 0.f;
#pragma unroll 8
      for (int j = 0; j < DV; ++j) inter += G[i * DVP + j] * vs[t * DVP + j];
      float dkv;
      if (!slow) {
        float intra = 0.f;  // sum_u B[u][t] q_u e^{b_u - b_l}
        for (int u = t; u < SC; ++u) intra += Bm[u * (SC + 1) + t] * qt[u * DKP + i];
        dkv = expf(bl - b) * (inter + intra);
      } else {
        float intra = 0.f;  // sum_u B[u][t] q_u e^{b_u - b_t}, elementwise
        for (int u = t; u < SC; ++u)
          intra += Bm[u * (SC + 1) + t] * qs[u * DKP + i] * expf(bs[u * DK + i] - b);
        dkv = expf(bl - b) * inter + intra;
      }
      dks[t * DKP + i] = dkv;
      if (t < n) {
        size_t off = tk + (size_t)(c0 + t) * DK + i;
        float outv = dkv + (p.add_dk ? p.add_dk[off] : 0.f);
        ((IO*)p.dk)[off] = from_f<IO>(outv);
      }
    }
    // dv
    for (int x = tid; x < SC * DV; x += NT) {
      int t = x / DV, j = x % DV;
      if (t >= n) continue;
      float acc = 0.f;
      for (int u = t; u < SC; ++u) acc += A[u * (SC + 1) + t] * dos[u * DVP + j];
#pragma unroll 8
      for (int i = 0; i < DK; ++i) acc += kt[t * DKP + i] * G[i * DVP + j];
      size_t off = tv + (size_t)(c0 + t) * DV + j;
      float outv = acc + (p.add_dv ? p.add_dv[off] : 0.f);
      ((IO*)p.dv)[off] = from_f<IO>(outv);
    }
    __syncthreads();
    if (tid < DK) {
      const int i = tid;
      for (int t = n - 1; t >= 0; --t) {
        run += qs[t * DKP + i] * dqs[t * DKP + i] - ks[t * DKP + i] * dks[t * DKP + i];
        p.dg[tk + (size_t)(c0 + t) * DK + i] = run;
      }
    }
    for (int x = tid; x < DK * DV; x += NT) {
      int i = x / DV, j = x % DV;
      float acc = el[i] * G[i * DVP + j];
#pragma unroll
      for (int u = 0; u < SC; ++u) acc += qi[u * DKP + i] * dos[u * DVP + j];
      G[i * DVP + j] = acc;
    }
  }
  __syncthreads();
  if (p.dh0) {
    for (int x = tid; x < DK * DV; x += NT) {
      int i = x / DV, j = x % DV;
      p.dh0[(size_t)bh * DK * DV + x] = G[i * DVP + j];
    }
  }
}

template <typename IO, int DK>
cudaError_t fwd_launch(const GlaFwdParams& p, cudaStream_t s) {
  size_t bytes = fwd_smem_floats<DK>() * sizeof(float);
  auto kern = gla_fwd_simt_kernel<IO, DK>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.dv / DVT, p.B * p.H);
  {
    ScopedTiming tm(p.o ? "gla_fwd_simt" : "gla_state_pass_simt", s);
    kern<<<grid, NT, bytes, s>>>(p);
  }
  return cudaGetLastError();
}

template <typename IO, int DK, int DV>
cudaError_t bwd_launch(const GlaBwdParams& p, cudaStream_t s) {
  size_t bytes = bwd_smem_floats<DK, DV>() * sizeof(float);
  auto kern = gla_bwd_simt_kernel<IO, DK, DV>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  {
    ScopedTiming tm("gla_bwd_simt", s);
    kern<<<p.B * p.H, NT, bytes, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_gla_fwd_simt(const GlaFwdParams& p, bool bf16, cudaStream_t s) {
  if (p.B * p.H == 0) return cudaSuccess;  // T == 0 still copies h0 to hT
  if (p.dk == 64) return bf16 ? fwd_launch<lz::bf16, 64>(p, s) : fwd_launch<float, 64>(p, s);
  return bf16 ? fwd_launch<lz::bf16, 128>(p, s) : fwd_launch<float, 128>(p, s);
}

cudaError_t launch_gla_bwd_simt(const GlaBwdParams& p, bool bf16, cudaStream_t s) {
  if (p.B * p.H == 0) return cudaSuccess;  // T == 0 still writes dh0 = dhT
#define LZ_BWD(DK_, DV_)                                                          \
  if (p.dkd == DK_ && p.dvd == DV_)                                               \
    return bf16 ? bwd_launch<lz::bf16, DK_, DV_>(p, s) : bwd_launch<float, DK_, DV_>(p, s);
  LZ_BWD(64, 64)
  LZ_BWD(64, 128)
  LZ_BWD(128, 64)
  LZ_BWD(128, 128)
#undef LZ_BWD
  return cudaErrorInvalidValue;
}

}  // namespace lz
