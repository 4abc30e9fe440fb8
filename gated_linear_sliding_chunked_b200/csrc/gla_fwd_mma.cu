// Chunked gated linear attention forward on the tensor cores (bf16 I/O,
// fp32 accumulation, dk = 128).
//
// Recurrence (Lizard technical summary, section 2a, state update equation):
//   S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T,   o_t = q_t^T S_t.
// One CTA walks one (batch, head) chain over 64-token chunks for a slice of
// DVT value columns; the fp32 state slice S [128 x DVT] stays in registers
// (warp w owns rows 16w..16w+15) for the whole walk.
//
// Gate numerics.  A chunk is four 16-row sub-blocks.  With e_u = exp(g_u),
// D_K the product of e over sub-block K, and for row t in sub-block I
//   Qf_t = q_t * prod_{u = start(I)..t} e_u          (<= 1)
//   Kf_s = k_s * prod_{u = s+1..end(J)} e_u           (<= 1, s in sub-block J)
// the gated score is A[t][s] = sum_i Qf_t,i Kf_s,i F_IJ,i with
//   F_IJ = prod_{J<K<I} D_K  (<= 1) for J < I,   F_II = 1 / D_I,
// the inter-chunk output uses Qf_t * prod_{K<I} D_K  (<= 1) against the
// state, and the state update uses Kf_s * prod_{K>J} D_K (<= 1).  So every
// operand is bounded by 1 except the diagonal factor 1/D_I; when a sub-block
// decays by more than e^-60 in some key dim the chunk's diagonal blocks are
// computed with exp(b_t - b_s) per element instead.  Only one exponential per
// gate element is taken; the rest are products.
//
// Per chunk: warp w handles query sub-block I = w/2 and half of the DVT
// output columns: scores for key sub-blocks J <= I (mma.m16n8k16, the
// per-(I,J) factor applied to the query fragments in registers), P V from
// the score registers, the inter-chunk product with the bf16 copy of the
// state, and the hybrid epilogue o = o_gla + alpha * add.  Then every warp
// updates its 16 state rows: S = diag(e^{b_l}) S + Ks^T V.
#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"

namespace lz {
namespace {

constexpr int C = 64;        // chunk rows
constexpr int SB = 16;       // sub-block rows
constexpr int NSB = C / SB;  // sub-blocks per chunk
constexpr int DK = 128;
constexpr int NT = 256;
constexpr int QKP = DK + 8;  // padded bf16 row of the ldmatrix operands
constexpr int NPAIR = NSB * (NSB + 1) / 2;
constexpr int PTP = C + 8;   // padded row of a query sub-block's score tile
// a sub-block whose decay is below this in some key dim takes the
// elementwise path for its diagonal scores
__device__ constexpr float kMinBlockDecay = 8.75651076e-27f;  // e^-60

template <int DVT>
struct FwdSmem {
  bf16 q[2][C * DK];
  bf16 k[2][C * DK];
  bf16 v[2][C * (DVT + 8)];
  float g[C * DK];          // one buffer: refilled for the next chunk after prep 1
  bf16 qf[C * QKP];         // score query operand
  bf16 kf[C * QKP];         // score key operand
  bf16 qi[C * QKP];         // inter-chunk query operand  q e^{b}
  bf16 ks[C * QKP];         // state-update key operand   k e^{b_l - b}
  bf16 s16[DK * (DVT + 8)];
  float dec[NSB][DK];       // sub-block decays D_K
  float fac[NPAIR][DK];     // score factors F_IJ (1 for tame key dims)
  float ec[DK];             // chunk decay e^{b_l}
  bf16 pt[NSB][SB * PTP];   // bf16 scores of each query sub-block (shared by its warp pair)
};

static_assert(sizeof(FwdSmem<64>) <= 232448, "shared memory per block exceeds 227 KB");

__device__ __forceinline__ int pair_index(int I, int J) { return I * (I + 1) / 2 + J; }

// barrier for the two warps (64 threads) that share query sub-block I
__device__ __forceinline__ void pair_sync(int I) {
  asm volatile("bar.sync %0, 64;\n" ::"r"(1 + I) : "memory");
}

// Diagonal-block score with one exponential per key dim:
// A[t][s] = sum_i q_t,i k_s,i exp(sum_{u=s+1..t} g_u,i) for rows t, s of
// the chunk (s <= t < rows).  Used only when a sub-block's gate decay leaves
// the range of the factorized form; g points at the chunk's first row in
// global memory.  Returns a scalar so that no register array of the caller
// has its address taken.
__device__ __noinline__ float diag_score_elementwise(const bf16* q, const bf16* k, const float* g,
                                                     int rt, int rs) {
  float a = 0.f;
  for (int i = 0; i < DK; ++i) {
    float lg = 0.f;
    for (int u = rs + 1; u <= rt; ++u) lg += g[(size_t)u * DK + i];
    a += __bfloat162float(q[rt * DK + i]) * __bfloat162float(k[rs * DK + i]) * __expf(lg);
  }
  return a;
}

template <int DVT>
__global__ void __launch_bounds__(NT, 1) gla_fwd_mma_kernel(GlaFwdParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  FwdSmem<DVT>& sm = *reinterpret_cast<FwdSmem<DVT>*>(smem_raw);
  constexpr int VP = DVT + 8;
  constexpr int SNT = DVT / 8;   // state n-tiles per warp
  constexpr int ONT = DVT / 16;  // output n-tiles per warp (half the columns)
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, gc = (lane & 3) * 2;
  const int j0 = blockIdx.x * DVT;
  const int bh = blockIdx.y;
  const int T = p.T, DV = p.dv;
  const bf16* q = (const bf16*)p.q + (size_t)bh * T * DK;
  const bf16* k = (const bf16*)p.k + (size_t)bh * T * DK;
  const bf16* v = (const bf16*)p.v + (size_t)bh * T * DV;
  const float* g = p.g + (size_t)bh * T * DK;
  const int nchunks = (T + C - 1) / C;

  auto issue_qkv = [&](int c, int st) {
    const int c0 = c * C;
    for (int x = tid; x < C * DK / 8; x += NT) {
      const int r = x / (DK / 8), cc = x % (DK / 8);
      const bool ok = c0 + r < T;
      const size_t off = (size_t)(ok ? c0 + r : 0) * DK + cc * 8;
      cp_async16(&sm.q[st][r * DK + cc * 8], q + off, ok ? 16 : 0);
      cp_async16(&sm.k[st][r * DK + cc * 8], k + off, ok ? 16 : 0);
    }
    for (int x = tid; x < C * DVT / 8; x += NT) {
      const int r = x / (DVT / 8), cc = x % (DVT / 8);
      const bool ok = c0 + r < T;
      const size_t off = (size_t)(ok ? c0 + r : 0) * DV + j0 + cc * 8;
      cp_async16(&sm.v[st][r * VP + cc * 8], v + off, ok ? 16 : 0);
    }
    cp_async_commit();
  };
  auto issue_g = [&](int c) {
    const int c0 = c * C;
    for (int x = tid; x < C * DK / 4; x += NT) {
      const int r = x / (DK / 4), cc = x % (DK / 4);
      const bool ok = c0 + r < T;
      const size_t off = (size_t)(ok ? c0 + r : 0) * DK + cc * 4;
      cp_async16(&sm.g[r * DK + cc * 4], g + off, ok ? 16 : 0);
    }
    cp_async_commit();
  };

  // ---- state registers and its bf16 copy ----------------------------------
  float s[SNT][4];
#pragma unroll
  for (int nt = 0; nt < SNT; ++nt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = 16 * warp + gr + 8 * hh, j = nt * 8 + gc;
      float a = 0.f, b = 0.f;
      if (p.h0) {
        const float* hp = p.h0 + ((size_t)bh * DK + i) * DV + j0 + j;
        a = hp[0];
        b = hp[1];
      }
      s[nt][2 * hh] = a;
      s[nt][2 * hh + 1] = b;
    }
  auto write_s16 = [&]() {
#pragma unroll
    for (int nt = 0; nt < SNT; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int i = 16 * warp + gr + 8 * hh, j = nt * 8 + gc;
        *reinterpret_cast<uint32_t*>(&sm.s16[i * VP + j]) =
            pack_bf16(s[nt][2 * hh], s[nt][2 * hh + 1]);
      }
  };
  write_s16();

  if (nchunks > 0) {
    issue_qkv(0, 0);
    issue_g(0);
  }
  for (int c = 0; c < nchunks; ++c) {
    const int st = c & 1;
    const int c0 = c * C;
    cp_async_wait<0>();
    __syncthreads();  // chunk c landed; the previous chunk's readers are done
    if (c + 1 < nchunks) issue_qkv(c + 1, st ^ 1);
    if (p.states) {  // state before this chunk, for the backward
      float* dst = p.states + ((size_t)bh * nchunks + c) * DK * DV + j0;
#pragma unroll
      for (int nt = 0; nt < SNT; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int i = 16 * warp + gr + 8 * hh, j = nt * 8 + gc;
          *reinterpret_cast<float2*>(&dst[(size_t)i * DV + j]) =
              make_float2(s[nt][2 * hh], s[nt][2 * hh + 1]);
        }
    }
    if (p.states16) {  // the same in bf16
      bf16* dst = (bf16*)p.states16 + ((size_t)bh * nchunks + c) * DK * DV + j0;
#pragma unroll
      for (int nt = 0; nt < SNT; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int i = 16 * warp + gr + 8 * hh, j = nt * 8 + gc;
          *reinterpret_cast<uint32_t*>(&dst[(size_t)i * DV + j]) =
              pack_bf16(s[nt][2 * hh], s[nt][2 * hh + 1]);
        }
    }

    // ---- prep: thread -> (sub-block K, key dims i, i+1) ----------------------
    const int K = tid >> 6, i2 = (tid & 63) * 2, r0 = K * SB;
    float2 qfac[SB], kfac[SB];
    {
      float2 e[SB];
#pragma unroll
      for (int r = 0; r < SB; ++r) {
        const float2 gg = *reinterpret_cast<const float2*>(&sm.g[(r0 + r) * DK + i2]);
        e[r] = make_float2(__expf(gg.x), __expf(gg.y));
      }
      float2 run = make_float2(1.f, 1.f);
#pragma unroll
      for (int r = SB - 1; r >= 0; --r) {  // k side: prod_{u = r+1 .. end} e_u
        kfac[r] = run;
        run.x *= e[r].x;
        run.y *= e[r].y;
      }
      run = make_float2(1.f, 1.f);
#pragma unroll
      for (int r = 0; r < SB; ++r) {  // q side: prod_{u = start .. r} e_u
        run.x *= e[r].x;
        run.y *= e[r].y;
        qfac[r] = run;
      }
      *reinterpret_cast<float2*>(&sm.dec[K][i2]) = run;
    }
    __syncthreads();
    if (c + 1 < nchunks) issue_g(c + 1);  // sm.g is free until the next chunk's prep
    int flags;
    {
      float2 D[NSB];
#pragma unroll
      for (int J = 0; J < NSB; ++J) D[J] = *reinterpret_cast<const float2*>(&sm.dec[J][i2]);
      // per key dim: "tame" when each 32-row half decays by at most e^-60; then
      // scores use one reference (the end of the first half) for all rows
      bool tame[2], wild_bad = false, any_wild = false;
      float rq[2], rk[2], eqk[2], ksk[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        const float d0 = h2 ? D[0].y : D[0].x, d1 = h2 ? D[1].y : D[1].x;
        const float d2 = h2 ? D[2].y : D[2].x, d3 = h2 ? D[3].y : D[3].x;
        tame[h2] = (d0 * d1 >= kMinBlockDecay) && (d2 * d3 >= kMinBlockDecay);
        any_wild |= !tame[h2];
        if (!tame[h2])
          wild_bad |= !(d0 >= kMinBlockDecay && d1 >= kMinBlockDecay &&
                        d2 >= kMinBlockDecay && d3 >= kMinBlockDecay);
        const float dk[NSB] = {d0, d1, d2, d3};
        float rqK = 1.f, rkK = 1.f;
        if (tame[h2]) {
          rqK = K == 0 ? 1.f / (d0 * d1) : K == 1 ? 1.f / d1 : K == 2 ? 1.f : d2;
          rkK = K == 0 ? d1 : K == 1 ? 1.f : K == 2 ? 1.f / d2 : 1.f / (d2 * d3);
        }
        float eq = 1.f, kk = 1.f;
#pragma unroll
        for (int J = 0; J < NSB; ++J) {
          if (J < K) eq *= dk[J];
          if (J > K) kk *= dk[J];
        }
        rq[h2] = rqK;
        rk[h2] = rkK;
        eqk[h2] = eq;
        ksk[h2] = kk;
        // score factors of this thread's share of the (I, J) pairs
#pragma unroll
        for (int I = 0; I < NSB; ++I)
#pragma unroll
          for (int J = 0; J <= I; ++J) {
            if (pair_index(I, J) % NSB != K) continue;
            float f = 1.f;
            if (!tame[h2]) {
              if (J == I) {
                f = 1.f / fmaxf(dk[I], 1e-30f);
              } else {
#pragma unroll
                for (int Kp = 0; Kp < NSB; ++Kp)
                  if (Kp > J && Kp < I) f *= dk[Kp];
              }
            }
            sm.fac[pair_index(I, J)][i2 + h2] = f;
          }
        if (K == 0) sm.ec[i2 + h2] = d0 * d1 * d2 * d3;
      }
      if (p.o) {
#pragma unroll
        for (int r = 0; r < SB; ++r) {
          const float2 qv = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.q[st][(r0 + r) * DK + i2]));
          const float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.k[st][(r0 + r) * DK + i2]));
          const float qx = qv.x * qfac[r].x, qy = qv.y * qfac[r].y;
          const float kx = kv.x * kfac[r].x, ky = kv.y * kfac[r].y;
          const int o = (r0 + r) * QKP + i2;
          *reinterpret_cast<uint32_t*>(&sm.qf[o]) = pack_bf16(qx * rq[0], qy * rq[1]);
          *reinterpret_cast<uint32_t*>(&sm.qi[o]) = pack_bf16(qx * eqk[0], qy * eqk[1]);
          *reinterpret_cast<uint32_t*>(&sm.kf[o]) = pack_bf16(kx * rk[0], ky * rk[1]);
          *reinterpret_cast<uint32_t*>(&sm.ks[o]) = pack_bf16(kx * ksk[0], ky * ksk[1]);
        }
      } else {  // state pass: only the state-update key operand
#pragma unroll
        for (int r = 0; r < SB; ++r) {
          const float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.k[st][(r0 + r) * DK + i2]));
          *reinterpret_cast<uint32_t*>(&sm.ks[(r0 + r) * QKP + i2]) =
              pack_bf16(kv.x * kfac[r].x * ksk[0], kv.y * kfac[r].y * ksk[1]);
        }
      }
      const int w = __syncthreads_or(any_wild);
      const int b = __syncthreads_or(wild_bad);
      flags = (w ? 1 : 0) | (b ? 2 : 0);
    }
    const bool scaled = flags & 1, slow = flags & 2;

    // ---- outputs: warp -> (query sub-block I, column half nh) --------------
    if (p.o) {
      const int I = warp >> 1, nh = warp & 1;
      float2 addv[ONT][2];
      const bool has_add = p.add || p.add16;
      if (has_add) {
#pragma unroll
        for (int nt = 0; nt < ONT; ++nt)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {
            const int t = c0 + 16 * I + gr + 8 * hh;
            const int j = j0 + nh * (DVT / 2) + nt * 8 + gc;
            const size_t off = ((size_t)bh * T + t) * DV + j;
            addv[nt][hh] = make_float2(0.f, 0.f);
            if (t < T)
              addv[nt][hh] = p.add16 ? unpack_bf16(*reinterpret_cast<const uint32_t*>(&((const bf16*)p.add16)[off]))
                                     : *reinterpret_cast<const float2*>(&p.add[off]);
          }
      }
      uint32_t qa[DK / 16][4];
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk)
        ldsm_x4(smem_u32(&sm.qf[(16 * I + (lane & 15)) * QKP + kk * 16 + (lane >> 4) * 8]),
                qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
      float acc[NSB][2][4];
#pragma unroll
      for (int J = 0; J < NSB; ++J) {
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[J][nt][e] = 0.f;
        if (J > I || (J & 1) != nh) continue;  // the pair splits the score blocks
        const float* fac = sm.fac[pair_index(I, J)];
        float acc2[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};  // odd k steps
#pragma unroll
        for (int kk = 0; kk < DK / 16; ++kk) {
          uint32_t a[4] = {qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]};
          if (scaled) {
            const float2 f0 = *reinterpret_cast<const float2*>(&fac[kk * 16 + gc]);
            const float2 f1 = *reinterpret_cast<const float2*>(&fac[kk * 16 + 8 + gc]);
            a[0] = scale_bf16x2(a[0], f0.x, f0.y);
            a[1] = scale_bf16x2(a[1], f0.x, f0.y);
            a[2] = scale_bf16x2(a[2], f1.x, f1.y);
            a[3] = scale_bf16x2(a[3], f1.x, f1.y);
          }
          uint32_t b0, b1, b2, b3;
          ldsm_x4(smem_u32(&sm.kf[(16 * J + (lane & 7) + ((lane >> 4) << 3)) * QKP + kk * 16 +
                                  ((lane >> 3) & 1) * 8]),
                  b0, b1, b2, b3);
          float (*dst)[4] = (kk & 1) ? acc2 : acc[J];
          mma_bf16(dst[0], a, b0, b1);
          mma_bf16(dst[1], a, b2, b3);
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) acc[J][nt][e] += acc2[nt][e];
        if (J == I) {
          if (slow) {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int t = gr + (e >> 1) * 8, sk = nt * 8 + gc + (e & 1);
                const int rt = 16 * I + t, rs = 16 * I + sk;
                acc[J][nt][e] = (sk <= t && rt < T - c0)
                                    ? diag_score_elementwise(sm.q[st], sm.k[st], g + (size_t)c0 * DK, rt, rs)
                                    : 0.f;
              }
          } else {
#pragma unroll
            for (int nt = 0; nt < 2; ++nt)
#pragma unroll
              for (int e = 0; e < 4; ++e) {
                const int t = gr + (e >> 1) * 8, sk = nt * 8 + gc + (e & 1);
                if (sk > t) acc[J][nt][e] = 0.f;
              }
          }
        }
      }
      float o[ONT][4];
#pragma unroll
      for (int nt = 0; nt < ONT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
      // share this warp's score blocks with its pair through shared memory
      bf16* pt = sm.pt[I];
#pragma unroll
      for (int J = 0; J < NSB; ++J) {
        if (J > I || (J & 1) != nh) continue;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt)
#pragma unroll
          for (int hh = 0; hh < 2; ++hh)
            *reinterpret_cast<uint32_t*>(&pt[(gr + 8 * hh) * PTP + 16 * J + nt * 8 + gc]) =
                pack_bf16(acc[J][nt][2 * hh], acc[J][nt][2 * hh + 1]);
      }
      pair_sync(I);
      // intra: P V over the key sub-blocks J <= I
#pragma unroll
      for (int J = 0; J < NSB; ++J) {
        if (J > I) continue;
        uint32_t pa[4];
        ldsm_x4(smem_u32(&pt[(lane & 15) * PTP + 16 * J + (lane >> 4) * 8]), pa[0], pa[1], pa[2], pa[3]);
#pragma unroll
        for (int ntp = 0; ntp < ONT / 2; ++ntp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(&sm.v[st][(16 * J + (lane & 7) + ((lane >> 3) & 1) * 8) * VP +
                                       nh * (DVT / 2) + ntp * 16 + (lane >> 4) * 8]),
                    b0, b1, b2, b3);
          mma_bf16(o[2 * ntp], pa, b0, b1);
          mma_bf16(o[2 * ntp + 1], pa, b2, b3);
        }
      }
      // inter: (q e^{b}) S_prev
#pragma unroll
      for (int kk = 0; kk < DK / 16; ++kk) {
        uint32_t a[4];
        ldsm_x4(smem_u32(&sm.qi[(16 * I + (lane & 15)) * QKP + kk * 16 + (lane >> 4) * 8]), a[0],
                a[1], a[2], a[3]);
#pragma unroll
        for (int ntp = 0; ntp < ONT / 2; ++ntp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(&sm.s16[(16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8) * VP +
                                     nh * (DVT / 2) + ntp * 16 + (lane >> 4) * 8]),
                    b0, b1, b2, b3);
          mma_bf16(o[2 * ntp], a, b0, b1);
          mma_bf16(o[2 * ntp + 1], a, b2, b3);
        }
      }
      // epilogue: o = o_gla + alpha * add, rounded to bf16
#pragma unroll
      for (int nt = 0; nt < ONT; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int t = c0 + 16 * I + gr + 8 * hh;
          if (t >= T) continue;
          const int j = j0 + nh * (DVT / 2) + nt * 8 + gc;
          const size_t off = ((size_t)bh * T + t) * DV + j;
          float x0 = o[nt][2 * hh], x1 = o[nt][2 * hh + 1];
          if (has_add) {
            x0 += p.alpha * addv[nt][hh].x;
            x1 += p.alpha * addv[nt][hh].y;
          }
          *reinterpret_cast<uint32_t*>(&((bf16*)p.o)[off]) = pack_bf16(x0, x1);
        }
    }

    // ---- state update: S = diag(e^{b_l}) S + Ks^T V -------------------------
    {
      const float d0 = sm.ec[16 * warp + gr], d1 = sm.ec[16 * warp + gr + 8];
#pragma unroll
      for (int nt = 0; nt < SNT; ++nt) {
        s[nt][0] *= d0;
        s[nt][1] *= d0;
        s[nt][2] *= d1;
        s[nt][3] *= d1;
      }
#pragma unroll
      for (int kk = 0; kk < C / 16; ++kk) {
        uint32_t a[4];
        ldsm_x4_t(smem_u32(&sm.ks[(16 * kk + (lane & 7) + ((lane >> 4) << 3)) * QKP + 16 * warp +
                                  ((lane >> 3) & 1) * 8]),
                  a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int ntp = 0; ntp < SNT / 2; ++ntp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(&sm.v[st][(16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8) * VP +
                                       ntp * 16 + (lane >> 4) * 8]),
                    b0, b1, b2, b3);
          mma_bf16(s[2 * ntp], a, b0, b1);
          mma_bf16(s[2 * ntp + 1], a, b2, b3);
        }
      }
    }
    __syncthreads();  // every reader of the old bf16 state is done
    write_s16();
  }
  if (p.hT) {
#pragma unroll
    for (int nt = 0; nt < SNT; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int i = 16 * warp + gr + 8 * hh, j = nt * 8 + gc;
        *reinterpret_cast<float2*>(&p.hT[((size_t)bh * DK + i) * DV + j0 + j]) =
            make_float2(s[nt][2 * hh], s[nt][2 * hh + 1]);
      }
  }
}

template <int DVT>
cudaError_t launch_dvt(const GlaFwdParams& p, cudaStream_t s) {
  const size_t bytes = sizeof(FwdSmem<DVT>);
  auto kern = gla_fwd_mma_kernel<DVT>;
  cudaError_t e =
      cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  dim3 grid(p.dv / DVT, p.B * p.H);
  {
    ScopedTiming tm(p.o ? "gla_fwd_mma" : "gla_state_pass_mma", s);
    kern<<<grid, NT, bytes, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace

bool gla_fwd_mma_supported(int dk, int dv, bool bf16) { return bf16 && dk == 128 && dv % 32 == 0; }

int gla_fwd_mma_chunk() { return C; }

cudaError_t launch_gla_fwd_mma(const GlaFwdParams& p, cudaStream_t s) {
  if (p.B * p.H == 0) return cudaSuccess;
  // enough CTAs to cover the SMs: narrower value slices for few chains
  const long chains = (long)p.B * p.H;
  if (p.dv % 64 == 0 && chains * (p.dv / 64) >= 96) return launch_dvt<64>(p, s);
  return launch_dvt<32>(p, s);
}

}  // namespace lz
