// Chunked gated linear attention backward on the tensor cores (bf16 I/O,
// fp32 accumulation, dk = dv = 128).
//
// Gradient of S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T, o_t = q_t^T S_t (the
// attention-output regression of the first training stage, Lizard technical
// summary section 2b, needs it).  Reverse walk over 64-token chunks with
// b_t the running log-gate inside the chunk, b_l its last value, G the
// gradient carried in from later chunks (dL/dhT at the end), S_prev the state
// before the chunk, B[t][s] = dO_t . v_s and A[t][s] = sum_i q_t k_s e^{b_t-b_s}
// (both for s <= t):
//   dq_t = e^{b_t} (S_prev dO_t) + sum_{s<=t} B[t][s] k_s e^{b_t - b_s}
//   dk_t = e^{b_l - b_t} (G v_t) + sum_{u>=t} B[u][t] q_u e^{b_u - b_t}
//   dv_t = (k_t e^{b_l - b_t})^T G + sum_{u>=t} A[u][t] dO_u
//   G   <- diag(e^{b_l}) G + sum_u (q_u e^{b_u})^T dO_u
//   dg   : from the gate's direct gradient e^{g_t} <dS_t, S_{t-1}> per key dim,
//          which at the chunk's first row is
//            seed = e^{b_l} <G, S_prev> + sum_u q_u * dq_inter_u
//          (dq_inter_u = e^{b_u} S_prev dO_u), and inside the chunk
//            dg_t = seed - sum_{u<t} (q_u dq_u - k_u dk_u)
//          so rounding errors add up over one chunk, not the whole sequence.
//
// Work split: a cluster of two CTAs per (batch, head); CTA r owns key dims
// [64r, 64r+64).  dq, dk, dg and its half of G are complete inside the CTA;
// dv is a sum over key dims, so each CTA sends the partial dv of the peer's
// 64 value columns through distributed shared memory every chunk and adds
// the peer's share to its own before storing.
//
// Gate factors follow the forward kernel: per key dim, one reference row
// (the end of the chunk's first half) when each 32-row half decays by at
// most e^-60 ("tame"), otherwise 16-row sub-block references with per-pair
// factors F_IJ; diagonal blocks whose decay is below e^-60 use elementwise
// exponents.  With Eq (q side) and Ek (k side) the factors that make
// Qf = q Eq, Kf = k Ek:
//   dq = Eq * [ ci * (dO S_prev^T) + sum_J B_IJ (Kf_J * F_IJ) ]
//   dk = Ek * [ ck * (v G^T)       + sum_J B_JI^T (Qf_J * F_JI) ]
// with ci = e^{b_t}/Eq and ck = e^{b_l - b_t}/Ek constant per (sub-block,
// key dim).
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"

namespace cg = cooperative_groups;

namespace lz {
namespace {

constexpr int C = 64;
constexpr int SB = 16;
constexpr int NSB = C / SB;
constexpr int DK = 128;
constexpr int DV = 128;
constexpr int DKH = 64;        // key dims per CTA
constexpr int NT = 256;
constexpr int KP = DKH + 8;    // padded row of the [rows][64 dims] operands
constexpr int VP = DV + 8;     // padded row of the v / dO tiles
constexpr int RP = DKH + 2;    // dg staging row (even: float2 access)
constexpr int NPAIR = NSB * (NSB + 1) / 2;
__device__ constexpr float kMinBlockDecay = 8.75651076e-27f;  // e^-60

// [rows][128] bf16 tile with its 16-byte chunks XOR-swizzled by row
__device__ __forceinline__ int swz(int row, int col) {
  return row * 128 + ((((col >> 3) ^ row) & 15) << 3) + (col & 7);
}

struct BwdSmem {
  bf16 q[2][C * DKH];
  bf16 k[2][C * DKH];
  bf16 v[2][C * VP];
  bf16 dO[2][C * VP];
  float g[C * DKH];
  bf16 sp[DKH * DV];   // state before the chunk, rows = this CTA's key dims (swizzled)
  bf16 qf[C * KP];
  bf16 kf[C * KP];
  bf16 qi[C * KP];     // q e^{b}
  bf16 ks[C * KP];     // k e^{b_l - b}
  bf16 eqf[C * KP];    // Eq
  bf16 ekf[C * KP];    // Ek
  bf16 g16[DKH * DV];  // carried gradient G, bf16 (swizzled)
  float red[C * RP];   // q*dq - k*dk for the dg scan; then the peer's dv share
  float dec[NSB][DKH];
  float fac[NPAIR][DKH];
  float ci[NSB][DKH];
  float ck[NSB][DKH];
  float ec[DKH];
  float qdqi[NSB][DKH];  // per sub-block column sums of q * dq_inter
  float gsp[2][DKH];     // <G, S_prev> per key dim, two value halves
  float tot[NSB][DKH];
};

static_assert(sizeof(BwdSmem) <= 232448, "shared memory per block exceeds 227 KB");

__device__ __forceinline__ int pair_index(int I, int J) { return I * (I + 1) / 2 + J; }

// Transposed diagonal scores A^T[t][u] = sum_i q_u,i k_t,i exp(sum_{x=t+1..u} g_x,i)
// for u >= t inside sub-block I (this CTA's key dims only), at the lane's
// fragment positions.  q, k: stage tiles [C][DKH]; g: global, first row of
// the chunk, row stride DK, already offset to this CTA's dims.
__device__ __noinline__ void diag_at_elementwise(const bf16* q, const bf16* k, const float* g,
                                                 int rows, int I, int lane, float (*acc)[4]) {
  const int gr = lane >> 2, gc = (lane & 3) * 2;
  for (int nt = 0; nt < 2; ++nt)
    for (int e = 0; e < 4; ++e) {
      const int t = gr + (e >> 1) * 8, u = nt * 8 + gc + (e & 1);
      const int rt = SB * I + t, ru = SB * I + u;
      float a = 0.f;
      if (u >= t && ru < rows) {
        for (int i = 0; i < DKH; ++i) {
          float lg = 0.f;
          for (int x = rt + 1; x <= ru; ++x) lg += g[(size_t)x * DK + i];
          a += __bfloat162float(q[ru * DKH + i]) * __bfloat162float(k[rt * DKH + i]) * __expf(lg);
        }
      }
      acc[nt][e] = a;
    }
}

// Same for B-side products: E[t][s] = exp(sum_{x=s+1..t} g_x) is needed
// elementwise only through A; B carries no gate, so dq/dk intra terms of a
// slow diagonal block are rebuilt from these per-dim factors.
__device__ __noinline__ void diag_gate_elementwise(const float* g, int rows, int I, int t, int s,
                                                   int i, float* out) {
  // exp(sum_{x=s+1..t} g_x,i) for one (t, s, i); t, s relative to sub-block I
  float lg = 0.f;
  for (int x = SB * I + s + 1; x <= SB * I + t && x < rows; ++x) lg += g[(size_t)x * DK + i];
  *out = __expf(lg);
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NT, 1)
    gla_bwd_mma_kernel(GlaBwdParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  BwdSmem& sm = *reinterpret_cast<BwdSmem*>(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, gc = (lane & 3) * 2;
  const int half = blockIdx.x;  // == rank in the cluster
  const int i0 = half * DKH;    // first key dim of this CTA
  const int bh = blockIdx.y;
  const int T = p.T;
  const size_t tk = (size_t)bh * T * DK, tv = (size_t)bh * T * DV;
  const bf16* q = (const bf16*)p.q + tk;
  const bf16* k = (const bf16*)p.k + tk;
  const bf16* v = (const bf16*)p.v + tv;
  const bf16* dO = (const bf16*)p.dO + tv;
  const float* g = p.g + tk;
  const bf16* st16 = (const bf16*)p.states16;
  const int nchunks = (T + C - 1) / C;
  float* peer_red = cluster.map_shared_rank(sm.red, half ^ 1);

  auto issue_tiles = [&](int c, int st) {
    const int c0 = c * C;
    for (int x = tid; x < C * DKH / 8; x += NT) {
      const int r = x / (DKH / 8), cc = x % (DKH / 8);
      const bool ok = c0 + r < T;
      const size_t off = (size_t)(ok ? c0 + r : 0) * DK + i0 + cc * 8;
      cp_async16(&sm.q[st][r * DKH + cc * 8], q + off, ok ? 16 : 0);
      cp_async16(&sm.k[st][r * DKH + cc * 8], k + off, ok ? 16 : 0);
    }
    for (int x = tid; x < C * DV / 8; x += NT) {
      const int r = x / (DV / 8), cc = x % (DV / 8);
      const bool ok = c0 + r < T;
      const size_t off = (size_t)(ok ? c0 + r : 0) * DV + cc * 8;
      cp_async16(&sm.v[st][r * VP + cc * 8], v + off, ok ? 16 : 0);
      cp_async16(&sm.dO[st][r * VP + cc * 8], dO + off, ok ? 16 : 0);
    }
    cp_async_commit();
  };
  auto issue_g = [&](int c) {
    const int c0 = c * C;
    for (int x = tid; x < C * DKH / 4; x += NT) {
      const int r = x / (DKH / 4), cc = x % (DKH / 4);
      const bool ok = c0 + r < T;
      const size_t off = (size_t)(ok ? c0 + r : 0) * DK + i0 + cc * 4;
      cp_async16(&sm.g[r * DKH + cc * 4], g + off, ok ? 16 : 0);
    }
    cp_async_commit();
  };
  auto issue_sp = [&](int c) {
    const bf16* src = st16 + ((size_t)bh * nchunks + c) * DK * DV + (size_t)i0 * DV;
    for (int x = tid; x < DKH * DV / 8; x += NT) {
      const int r = x / (DV / 8), cc = x % (DV / 8);
      cp_async16(&sm.sp[swz(r, cc * 8)], src + (size_t)r * DV + cc * 8, 16);
    }
    cp_async_commit();
  };

  // ---- carried gradient G: warp -> (key-dim tile mt, value half nh) --------
  const int mt = warp & 3, gnh = warp >> 2;
  float G[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = i0 + 16 * mt + gr + 8 * hh, j = 64 * gnh + nt * 8 + gc;
      float a = 0.f, b = 0.f;
      if (p.dhT) {
        const float* src = p.dhT + ((size_t)bh * DK + i) * DV + j;
        a = src[0];
        b = src[1];
      }
      G[nt][2 * hh] = a;
      G[nt][2 * hh + 1] = b;
    }
  auto write_g16 = [&]() {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int r = 16 * mt + gr + 8 * hh, j = 64 * gnh + nt * 8 + gc;
        *reinterpret_cast<uint32_t*>(&sm.g16[swz(r, j)]) = pack_bf16(G[nt][2 * hh], G[nt][2 * hh + 1]);
      }
  };
  write_g16();
  if (nchunks > 0) {
    issue_tiles(nchunks - 1, 0);
    issue_g(nchunks - 1);
    issue_sp(nchunks - 1);
  }
  for (int it = 0; it < nchunks; ++it) {
    const int c = nchunks - 1 - it;
    const int st = it & 1;
    const int c0 = c * C;
    const int rows = T - c0;  // valid rows in this chunk (may exceed C)
    cp_async_wait<0>();
    __syncthreads();
    if (c > 0) issue_tiles(c - 1, st ^ 1);

    // ---- prep 1: per key dim cumulative gate products -----------------------
    const int K = tid >> 6, i = tid & 63, r0 = K * SB;
    float qfac[SB], kfac[SB];
    {
      float e[SB];
#pragma unroll
      for (int r = 0; r < SB; ++r) e[r] = __expf(sm.g[(r0 + r) * DKH + i]);
      float run = 1.f;
#pragma unroll
      for (int r = SB - 1; r >= 0; --r) {
        kfac[r] = run;
        run *= e[r];
      }
      run = 1.f;
#pragma unroll
      for (int r = 0; r < SB; ++r) {
        run *= e[r];
        qfac[r] = run;
      }
      sm.dec[K][i] = run;
    }
    __syncthreads();
    if (c > 0) issue_g(c - 1);
    // ---- prep 2: operands and factor tables -------------------------------
    int flags;
    {
      const float d0 = sm.dec[0][i], d1 = sm.dec[1][i], d2 = sm.dec[2][i], d3 = sm.dec[3][i];
      const float dk4[NSB] = {d0, d1, d2, d3};
      const bool tame = (d0 * d1 >= kMinBlockDecay) && (d2 * d3 >= kMinBlockDecay);
      const bool bad = !tame && !(d0 >= kMinBlockDecay && d1 >= kMinBlockDecay &&
                                  d2 >= kMinBlockDecay && d3 >= kMinBlockDecay);
      float rq = 1.f, rk = 1.f;
      if (tame) {
        rq = K == 0 ? 1.f / (d0 * d1) : K == 1 ? 1.f / d1 : K == 2 ? 1.f : d2;
        rk = K == 0 ? d1 : K == 1 ? 1.f : K == 2 ? 1.f / d2 : 1.f / (d2 * d3);
      }
      float eqk = 1.f, ksk = 1.f;
#pragma unroll
      for (int J = 0; J < NSB; ++J) {
        if (J < K) eqk *= dk4[J];
        if (J > K) ksk *= dk4[J];
      }
      // inter factors for sub-block K: e^{b_t}/Eq and e^{b_l - b_t}/Ek
      sm.ci[K][i] = tame ? d0 * d1 : eqk;
      sm.ck[K][i] = tame ? d2 * d3 : ksk;
#pragma unroll
      for (int I = 0; I < NSB; ++I)
#pragma unroll
        for (int J = 0; J <= I; ++J) {
          if (pair_index(I, J) % NSB != K) continue;
          float f = 1.f;
          if (!tame) {
            if (J == I) {
              f = 1.f / fmaxf(dk4[I], 1e-30f);
            } else {
#pragma unroll
              for (int Kp = 0; Kp < NSB; ++Kp)
                if (Kp > J && Kp < I) f *= dk4[Kp];
            }
          }
          sm.fac[pair_index(I, J)][i] = f;
        }
      if (K == 0) sm.ec[i] = d0 * d1 * d2 * d3;
#pragma unroll
      for (int r = 0; r < SB; ++r) {
        const float qv = __bfloat162float(sm.q[st][(r0 + r) * DKH + i]);
        const float kv = __bfloat162float(sm.k[st][(r0 + r) * DKH + i]);
        const float eq = qfac[r] * rq, ek = kfac[r] * rk;
        const int o = (r0 + r) * KP + i;
        sm.qf[o] = __float2bfloat16_rn(qv * eq);
        sm.kf[o] = __float2bfloat16_rn(kv * ek);
        sm.qi[o] = __float2bfloat16_rn(qv * qfac[r] * eqk);
        sm.ks[o] = __float2bfloat16_rn(kv * kfac[r] * ksk);
        sm.eqf[o] = __float2bfloat16_rn(eq);
        sm.ekf[o] = __float2bfloat16_rn(ek);
      }
      const int w = __syncthreads_or(!tame);
      const int b = __syncthreads_or(bad);
      flags = (w ? 1 : 0) | (b ? 2 : 0);
    }
    const bool scaled = flags & 1, slow = flags & 2;

    float dv[16][4];  // warps 4..7: partial dv of rows I, all 128 value columns
    if (warp < 4) {
      // ================= dq, dk of rows I (this CTA's key dims) =============
      const int I = warp;
      float acc[8][4];
      // ---- B[I][J <= I] with dO rows I as A ---------------------------------
      {
        uint32_t da[8][4];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ldsm_x4(smem_u32(&sm.dO[st][(16 * I + (lane & 15)) * VP + kk * 16 + (lane >> 4) * 8]),
                  da[kk][0], da[kk][1], da[kk][2], da[kk][3]);
        float bs[NSB][2][4];
#pragma unroll
        for (int J = 0; J < NSB; ++J) {
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) bs[J][nt][e] = 0.f;
          if (J > I) continue;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(smem_u32(&sm.v[st][(16 * J + (lane & 7) + ((lane >> 4) << 3)) * VP + kk * 16 +
                                       ((lane >> 3) & 1) * 8]),
                    b0, b1, b2, b3);
            mma_bf16(bs[J][0], da[kk], b0, b1);
            mma_bf16(bs[J][1], da[kk], b2, b3);
          }
          if (J == I) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int t = gr + (e >> 1) * 8, sk = nt * 8 + gc + (e & 1);
                if (sk > t) bs[J][nt][e] = 0.f;
              }
          }
        }
        // ---- dq accumulator: inter (dO S_prev^T, scaled by ci per dim) -----
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
        const float* ciI = sm.ci[I];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
          for (int ntp = 0; ntp < 4; ++ntp) {
            uint32_t b0, b1, b2, b3;
            const int n = ntp * 16 + (lane & 7) + ((lane >> 4) << 3);
            ldsm_x4(smem_u32(&sm.sp[swz(n, kk * 16 + ((lane >> 3) & 1) * 8)]), b0, b1, b2, b3);
            const float f0 = ciI[ntp * 16 + gr], f1 = ciI[ntp * 16 + 8 + gr];
            b0 = scale_bf16x2(b0, f0, f0);
            b1 = scale_bf16x2(b1, f0, f0);
            b2 = scale_bf16x2(b2, f1, f1);
            b3 = scale_bf16x2(b3, f1, f1);
            mma_bf16(acc[2 * ntp], da[kk], b0, b1);
            mma_bf16(acc[2 * ntp + 1], da[kk], b2, b3);
          }
        }
        // ---- seed part: column sums of q * dq_inter over this warp's rows ----
#pragma unroll
        for (int nt = 0; nt < 8; ++nt) {
          const int il = nt * 8 + gc;
          float s0 = 0.f, s1 = 0.f;
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int t = 16 * I + gr + 8 * hh;
            const float2 eq = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.eqf[t * KP + il]));
            const float2 qv = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.q[st][t * DKH + il]));
            s0 += qv.x * acc[nt][2 * hh] * eq.x;
            s1 += qv.y * acc[nt][2 * hh + 1] * eq.y;
          }
#pragma unroll
          for (int o = 4; o < 32; o <<= 1) {
            s0 += __shfl_xor_sync(0xffffffffu, s0, o);
            s1 += __shfl_xor_sync(0xffffffffu, s1, o);
          }
          if (gr == 0) {
            sm.qdqi[I][il] = s0;
            sm.qdqi[I][il + 1] = s1;
          }
        }
        // ---- dq intra: sum_J B[I][J] (Kf_J * F_IJ) --------------------------
#pragma unroll
        for (int J = 0; J < NSB; ++J) {
          if (J > I) continue;
          if (J == I && slow) continue;  // handled elementwise below
          const uint32_t pa[4] = {pack_bf16(bs[J][0][0], bs[J][0][1]), pack_bf16(bs[J][0][2], bs[J][0][3]),
                                  pack_bf16(bs[J][1][0], bs[J][1][1]), pack_bf16(bs[J][1][2], bs[J][1][3])};
          const float* fac = sm.fac[pair_index(I, J)];
#pragma unroll
          for (int ntp = 0; ntp < 4; ++ntp) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(smem_u32(&sm.kf[(16 * J + (lane & 7) + ((lane >> 3) & 1) * 8) * KP + ntp * 16 +
                                      (lane >> 4) * 8]),
                      b0, b1, b2, b3);
            if (scaled) {
              const float f0 = fac[ntp * 16 + gr], f1 = fac[ntp * 16 + 8 + gr];
              b0 = scale_bf16x2(b0, f0, f0);
              b1 = scale_bf16x2(b1, f0, f0);
              b2 = scale_bf16x2(b2, f1, f1);
              b3 = scale_bf16x2(b3, f1, f1);
            }
            mma_bf16(acc[2 * ntp], pa, b0, b1);
            mma_bf16(acc[2 * ntp + 1], pa, b2, b3);
          }
        }
        // ---- dq = Eq * acc (+ slow diagonal term), store, stage q*dq -------
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int t = 16 * I + gr + 8 * hh;
            const int il = nt * 8 + gc;
            const float2 eq = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.eqf[t * KP + il]));
            float x0 = acc[nt][2 * hh] * eq.x, x1 = acc[nt][2 * hh + 1] * eq.y;
            if (slow) {
              // diagonal block: sum_{s in I, s <= t} B[t][s] k_s exp(b_t - b_s)
              for (int s2 = 0; s2 <= gr + 8 * hh; ++s2) {
                const int rs = 16 * I + s2;
                // B[t][s] lives in another lane's registers: rebuild it
                float bts = 0.f;
                for (int j = 0; j < DV; ++j)
                  bts += __bfloat162float(sm.dO[st][t * VP + j]) * __bfloat162float(sm.v[st][rs * VP + j]);
                float e0, e1;
                diag_gate_elementwise(g + (size_t)c0 * DK + i0, rows, I, gr + 8 * hh, s2, il, &e0);
                diag_gate_elementwise(g + (size_t)c0 * DK + i0, rows, I, gr + 8 * hh, s2, il + 1, &e1);
                x0 += bts * __bfloat162float(sm.k[st][rs * DKH + il]) * e0;
                x1 += bts * __bfloat162float(sm.k[st][rs * DKH + il + 1]) * e1;
              }
            }
            if (c0 + t < T) {
              const size_t off = tk + (size_t)(c0 + t) * DK + i0 + il;
              float y0 = x0, y1 = x1;
              if (p.add_dq) {
                const float2 a = *reinterpret_cast<const float2*>(&p.add_dq[off]);
                y0 += a.x;
                y1 += a.y;
              } else if (p.add_in_place) {
                const float2 a = unpack_bf16(*reinterpret_cast<const uint32_t*>(&((const bf16*)p.dq)[off]));
                y0 += a.x;
                y1 += a.y;
              }
              *reinterpret_cast<uint32_t*>(&((bf16*)p.dq)[off]) = pack_bf16(y0, y1);
            }
            const float2 qv = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.q[st][t * DKH + il]));
            sm.red[t * RP + il] = qv.x * x0;
            sm.red[t * RP + il + 1] = qv.y * x1;
          }
      }
      // ---- B^T[I][J >= I] with v rows I as A ---------------------------------
      {
        uint32_t va[8][4];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          ldsm_x4(smem_u32(&sm.v[st][(16 * I + (lane & 15)) * VP + kk * 16 + (lane >> 4) * 8]),
                  va[kk][0], va[kk][1], va[kk][2], va[kk][3]);
        float bt[NSB][2][4];
#pragma unroll
        for (int J = 0; J < NSB; ++J) {
#pragma unroll
          for (int nt = 0; nt < 2; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) bt[J][nt][e] = 0.f;
          if (J < I) continue;
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4(smem_u32(&sm.dO[st][(16 * J + (lane & 7) + ((lane >> 4) << 3)) * VP + kk * 16 +
                                        ((lane >> 3) & 1) * 8]),
                    b0, b1, b2, b3);
            mma_bf16(bt[J][0], va[kk], b0, b1);
            mma_bf16(bt[J][1], va[kk], b2, b3);
          }
          if (J == I) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int t = gr + (e >> 1) * 8, u = nt * 8 + gc + (e & 1);
                if (u < t) bt[J][nt][e] = 0.f;
              }
          }
        }
        // ---- dk accumulator: inter (v G^T, scaled by ck per dim) ------------
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
        const float* ckI = sm.ck[I];
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
#pragma unroll
          for (int ntp = 0; ntp < 4; ++ntp) {
            uint32_t b0, b1, b2, b3;
            const int n = ntp * 16 + (lane & 7) + ((lane >> 4) << 3);
            ldsm_x4(smem_u32(&sm.g16[swz(n, kk * 16 + ((lane >> 3) & 1) * 8)]), b0, b1, b2, b3);
            const float f0 = ckI[ntp * 16 + gr], f1 = ckI[ntp * 16 + 8 + gr];
            b0 = scale_bf16x2(b0, f0, f0);
            b1 = scale_bf16x2(b1, f0, f0);
            b2 = scale_bf16x2(b2, f1, f1);
            b3 = scale_bf16x2(b3, f1, f1);
            mma_bf16(acc[2 * ntp], va[kk], b0, b1);
            mma_bf16(acc[2 * ntp + 1], va[kk], b2, b3);
          }
        }
        // ---- dk intra: sum_{J >= I} B^T[I][J] (Qf_J * F_JI) -----------------
#pragma unroll
        for (int J = 0; J < NSB; ++J) {
          if (J < I) continue;
          if (J == I && slow) continue;
          const uint32_t pa[4] = {pack_bf16(bt[J][0][0], bt[J][0][1]), pack_bf16(bt[J][0][2], bt[J][0][3]),
                                  pack_bf16(bt[J][1][0], bt[J][1][1]), pack_bf16(bt[J][1][2], bt[J][1][3])};
          const float* fac = sm.fac[pair_index(J, I)];
#pragma unroll
          for (int ntp = 0; ntp < 4; ++ntp) {
            uint32_t b0, b1, b2, b3;
            ldsm_x4_t(smem_u32(&sm.qf[(16 * J + (lane & 7) + ((lane >> 3) & 1) * 8) * KP + ntp * 16 +
                                      (lane >> 4) * 8]),
                      b0, b1, b2, b3);
            if (scaled) {
              const float f0 = fac[ntp * 16 + gr], f1 = fac[ntp * 16 + 8 + gr];
              b0 = scale_bf16x2(b0, f0, f0);
              b1 = scale_bf16x2(b1, f0, f0);
              b2 = scale_bf16x2(b2, f1, f1);
              b3 = scale_bf16x2(b3, f1, f1);
            }
            mma_bf16(acc[2 * ntp], pa, b0, b1);
            mma_bf16(acc[2 * ntp + 1], pa, b2, b3);
          }
        }
        // ---- dk = Ek * acc (+ slow diagonal term), store, stage -k*dk -------
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int t = 16 * I + gr + 8 * hh;
            const int il = nt * 8 + gc;
            const float2 ek = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.ekf[t * KP + il]));
            float x0 = acc[nt][2 * hh] * ek.x, x1 = acc[nt][2 * hh + 1] * ek.y;
            if (slow) {
              // diagonal block: sum_{u in I, u >= t} B[u][t] q_u exp(b_u - b_t)
              for (int u2 = gr + 8 * hh; u2 < SB; ++u2) {
                const int ru = 16 * I + u2;
                float but = 0.f;
                for (int j = 0; j < DV; ++j)
                  but += __bfloat162float(sm.dO[st][ru * VP + j]) * __bfloat162float(sm.v[st][t * VP + j]);
                float e0, e1;
                diag_gate_elementwise(g + (size_t)c0 * DK + i0, rows, I, u2, gr + 8 * hh, il, &e0);
                diag_gate_elementwise(g + (size_t)c0 * DK + i0, rows, I, u2, gr + 8 * hh, il + 1, &e1);
                x0 += but * __bfloat162float(sm.q[st][ru * DKH + il]) * e0;
                x1 += but * __bfloat162float(sm.q[st][ru * DKH + il + 1]) * e1;
              }
            }
            if (c0 + t < T) {
              const size_t off = tk + (size_t)(c0 + t) * DK + i0 + il;
              float y0 = x0, y1 = x1;
              if (p.add_dk) {
                const float2 a = *reinterpret_cast<const float2*>(&p.add_dk[off]);
                y0 += a.x;
                y1 += a.y;
              } else if (p.add_in_place) {
                const float2 a = unpack_bf16(*reinterpret_cast<const uint32_t*>(&((const bf16*)p.dk)[off]));
                y0 += a.x;
                y1 += a.y;
              }
              *reinterpret_cast<uint32_t*>(&((bf16*)p.dk)[off]) = pack_bf16(y0, y1);
            }
            const float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.k[st][t * DKH + il]));
            sm.red[t * RP + il] -= kv.x * x0;
            sm.red[t * RP + il + 1] -= kv.y * x1;
          }
      }
    } else {
      // ================= partial dv of rows I over this CTA's key dims ======
      const int I = warp - 4;
      float at[NSB][2][4];
#pragma unroll
      for (int J = 0; J < NSB; ++J) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) at[J][nt][e] = 0.f;
        if (J < I) continue;
        const float* fac = sm.fac[pair_index(J, I)];
#pragma unroll
        for (int kk = 0; kk < DKH / 16; ++kk) {
          uint32_t a[4];
          ldsm_x4(smem_u32(&sm.kf[(16 * I + (lane & 15)) * KP + kk * 16 + (lane >> 4) * 8]), a[0], a[1],
                  a[2], a[3]);
          if (scaled) {
            const float2 f0 = *reinterpret_cast<const float2*>(&fac[kk * 16 + gc]);
            const float2 f1 = *reinterpret_cast<const float2*>(&fac[kk * 16 + 8 + gc]);
            a[0] = scale_bf16x2(a[0], f0.x, f0.y);
            a[1] = scale_bf16x2(a[1], f0.x, f0.y);
            a[2] = scale_bf16x2(a[2], f1.x, f1.y);
            a[3] = scale_bf16x2(a[3], f1.x, f1.y);
          }
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_u32(&sm.qf[(16 * J + (lane & 7) + ((lane >> 4) << 3)) * KP + kk * 16 +
                                  ((lane >> 3) & 1) * 8]),
                  b0, b1, b2, b3);
          mma_bf16(at[J][0], a, b0, b1);
          mma_bf16(at[J][1], a, b2, b3);
        }
        if (J == I) {
          if (slow) {
            diag_at_elementwise(sm.q[st], sm.k[st], g + (size_t)c0 * DK + i0, rows, I, lane, at[J]);
          } else {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int t = gr + (e >> 1) * 8, u = nt * 8 + gc + (e & 1);
                if (u < t) at[J][nt][e] = 0.f;
              }
          }
        }
      }
#pragma unroll
      for (int nt = 0; nt < 16; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) dv[nt][e] = 0.f;
      // inter: (k e^{b_l - b})_I G   (k over this CTA's key dims)
#pragma unroll
      for (int kk = 0; kk < DKH / 16; ++kk) {
        uint32_t a[4];
        ldsm_x4(smem_u32(&sm.ks[(16 * I + (lane & 15)) * KP + kk * 16 + (lane >> 4) * 8]), a[0], a[1],
                a[2], a[3]);
#pragma unroll
        for (int ntp = 0; ntp < 8; ++ntp) {
          uint32_t b0, b1, b2, b3;
          const int kr = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
          ldsm_x4_t(smem_u32(&sm.g16[swz(kr, ntp * 16 + (lane >> 4) * 8)]), b0, b1, b2, b3);
          mma_bf16(dv[2 * ntp], a, b0, b1);
          mma_bf16(dv[2 * ntp + 1], a, b2, b3);
        }
      }
      // intra: sum_{J >= I} A^T[I][J] dO_J
#pragma unroll
      for (int J = 0; J < NSB; ++J) {
        if (J < I) continue;
        const uint32_t pa[4] = {pack_bf16(at[J][0][0], at[J][0][1]), pack_bf16(at[J][0][2], at[J][0][3]),
                                pack_bf16(at[J][1][0], at[J][1][1]), pack_bf16(at[J][1][2], at[J][1][3])};
#pragma unroll
        for (int ntp = 0; ntp < 8; ++ntp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(&sm.dO[st][(16 * J + (lane & 7) + ((lane >> 3) & 1) * 8) * VP + ntp * 16 +
                                        (lane >> 4) * 8]),
                    b0, b1, b2, b3);
          mma_bf16(dv[2 * ntp], pa, b0, b1);
          mma_bf16(dv[2 * ntp + 1], pa, b2, b3);
        }
      }
    }

    // ---- <G, S_prev> per key dim (G still the gradient carried into the chunk)
    {
      float a0 = 0.f, a1 = 0.f;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        const int j = 64 * gnh + nt * 8 + gc;
        const float2 s0 = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.sp[swz(16 * mt + gr, j)]));
        const float2 s1 = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.sp[swz(16 * mt + gr + 8, j)]));
        a0 += G[nt][0] * s0.x + G[nt][1] * s0.y;
        a1 += G[nt][2] * s1.x + G[nt][3] * s1.y;
      }
      a0 += __shfl_xor_sync(0xffffffffu, a0, 1);
      a0 += __shfl_xor_sync(0xffffffffu, a0, 2);
      a1 += __shfl_xor_sync(0xffffffffu, a1, 1);
      a1 += __shfl_xor_sync(0xffffffffu, a1, 2);
      if ((lane & 3) == 0) {
        sm.gsp[gnh][16 * mt + gr] = a0;
        sm.gsp[gnh][16 * mt + gr + 8] = a1;
      }
    }
    // ---- carried gradient: G = diag(e^{b_l}) G + (q e^{b})^T dO --------------
    {
      const float d0 = sm.ec[16 * mt + gr], d1 = sm.ec[16 * mt + gr + 8];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        G[nt][0] *= d0;
        G[nt][1] *= d0;
        G[nt][2] *= d1;
        G[nt][3] *= d1;
      }
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk) {
        uint32_t a[4];
        ldsm_x4_t(smem_u32(&sm.qi[(16 * kk + (lane & 7) + ((lane >> 4) << 3)) * KP + 16 * mt +
                                  ((lane >> 3) & 1) * 8]),
                  a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int ntp = 0; ntp < 4; ++ntp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(&sm.dO[st][(16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8) * VP + 64 * gnh +
                                        ntp * 16 + (lane >> 4) * 8]),
                    b0, b1, b2, b3);
          mma_bf16(G[2 * ntp], a, b0, b1);
          mma_bf16(G[2 * ntp + 1], a, b2, b3);
        }
      }
    }
    __syncthreads();  // red staged; every reader of sp, g16 and the operands is done
    if (c > 0) issue_sp(c - 1);
    write_g16();

    // ---- dg: exact seed at the chunk's first row, then a running sum inside --
    {
      const int col = tid & 63, qq = tid >> 6;
      float loc[SB];
      float run = 0.f;
#pragma unroll
      for (int r = 0; r < SB; ++r) {  // exclusive prefix of q*dq - k*dk
        loc[r] = run;
        run += sm.red[(16 * qq + r) * RP + col];
      }
      sm.tot[qq][col] = run;
      __syncthreads();
      float base = sm.ec[col] * (sm.gsp[0][col] + sm.gsp[1][col]) + sm.qdqi[0][col] +
                   sm.qdqi[1][col] + sm.qdqi[2][col] + sm.qdqi[3][col];
#pragma unroll
      for (int q2 = 0; q2 < NSB; ++q2)
        if (q2 < qq) base -= sm.tot[q2][col];
#pragma unroll
      for (int r = 0; r < SB; ++r) {
        const int t = c0 + 16 * qq + r;
        if (t < T) p.dg[tk + (size_t)t * DK + i0 + col] = base - loc[r];
      }
    }

    // ---- dv: exchange the peer's 64 columns through distributed smem --------
    cluster.sync();  // both CTAs are done with red
    if (warp >= 4) {
      const int I = warp - 4;
      const int pcol = 64 * (half ^ 1);
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int t = 16 * I + gr + 8 * hh, cl = nt * 8 + gc;
          const int ntg = (pcol >> 3) + nt;
          *reinterpret_cast<float2*>(&peer_red[t * RP + cl]) =
              make_float2(dv[ntg][2 * hh], dv[ntg][2 * hh + 1]);
        }
    }
    cluster.sync();  // the peer's share has landed in red
    if (warp >= 4) {
      const int I = warp - 4;
      const int mcol = 64 * half;
#pragma unroll
      for (int nt = 0; nt < 8; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int t = 16 * I + gr + 8 * hh, cl = nt * 8 + gc;
          const int ntg = (mcol >> 3) + nt;
          if (c0 + t >= T) continue;
          const float2 pr = *reinterpret_cast<const float2*>(&sm.red[t * RP + cl]);
          float y0 = dv[ntg][2 * hh] + pr.x, y1 = dv[ntg][2 * hh + 1] + pr.y;
          const size_t off = tv + (size_t)(c0 + t) * DV + mcol + cl;
          if (p.add_dv) {
            const float2 a = *reinterpret_cast<const float2*>(&p.add_dv[off]);
            y0 += a.x;
            y1 += a.y;
          } else if (p.add_in_place) {
            const float2 a = unpack_bf16(*reinterpret_cast<const uint32_t*>(&((const bf16*)p.dv)[off]));
            y0 += a.x;
            y1 += a.y;
          }
          *reinterpret_cast<uint32_t*>(&((bf16*)p.dv)[off]) = pack_bf16(y0, y1);
        }
    }
  }
  // dh0 = G carried to before token 0
  if (p.dh0) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int ii = i0 + 16 * mt + gr + 8 * hh, j = 64 * gnh + nt * 8 + gc;
        *reinterpret_cast<float2*>(&p.dh0[((size_t)bh * DK + ii) * DV + j]) =
            make_float2(G[nt][2 * hh], G[nt][2 * hh + 1]);
      }
  }
  cluster.sync();  // keep this CTA's shared memory alive until the peer is done with it
}

}  // namespace

bool gla_bwd_mma_supported(int dk, int dv, bool bf16) { return bf16 && dk == DK && dv == DV; }

cudaError_t launch_gla_bwd_mma(const GlaBwdParams& p, cudaStream_t s) {
  if (p.B * p.H == 0) return cudaSuccess;
  const size_t bytes = sizeof(BwdSmem);
  cudaError_t e = cudaFuncSetAttribute(gla_bwd_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes);
  if (e != cudaSuccess) return e;
  dim3 grid(2, p.B * p.H);
  {
    ScopedTiming tm("gla_bwd_mma", s);
    gla_bwd_mma_kernel<<<grid, NT, bytes, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace lz
