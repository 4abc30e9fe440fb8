// Backward of the window + meta-token softmax on the tensor cores (bf16
// I/O, fp32 accumulation, dk = dv = 128).
//
// With P = exp(logit - lse), dO' = gscale * dO (the window branch's share of
// the output gradient) and D_t = dO_t . o_t (rebuilt as sum_j P_tj dP_tj):
//   dP = dO V^T,  dS = gscale * P * (dP - D)
//   dq = scale * dS K,   dk = scale * dS^T Q,   dv = gscale * P^T dO
//   dmeta_k = scale * sum_t dS_t,m q_t,  dmeta_v = gscale * sum_t P_t,m dO_t
// (Lizard technical summary, section 2a: window keys j in [t-w+1, t] plus M
// always-visible meta tokens in the softmax).
//
// Kernel 1 (query-major): CTA = one (batch, head) and a slab of query rows,
// walked in 64-row tiles by 4 warps x 16 rows.  With the forward output at
// hand D_t = dO_t . o_t comes straight off it and one sweep over the key
// tiles gives dS and dq; without it a first sweep accumulates D.  Meta-token
// gradients accumulate in registers over the slab and are written as one
// partial per CTA; D goes to scratch for kernel 2.
// Kernel 2 (key-major): CTA = 64 keys of one (batch, head), 4 warps x 16
// keys, walking the 32-row query tiles that see them; dk, dv in registers.
// A fixed-order reduction (shared with the SIMT path) sums the partials.
// Split query side (kernel 1 with WINDOW = false, the tcgen05 key side and
// kernel 3): when the forward output is given and the key side runs on
// tcgen05, the key side stores the dS^T tiles it forms anyway, kernel 1 keeps
// only D, the meta tokens' dS and the meta gradients, and kernel 3 forms dq
// from the stored tiles, so the band's scores are formed once.
#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"

namespace lz {
namespace {

constexpr int D = 128;
constexpr int RPAD = D + 8;
constexpr float kLog2e = 1.4426950408889634f;
constexpr int QTILE = 64;   // kernel 1 query rows per tile
constexpr int KT1 = 32;     // kernel 1 keys per tile
constexpr int MT = 16;      // meta tile
constexpr int SLAB = kSwaBwdSlab;  // kernel 1 query rows per CTA (one meta partial each)
constexpr int NT = 128;

template <int N>
struct IntTag {
  static constexpr int value = N;
};

struct QSmem {
  bf16 q[QTILE * RPAD];
  bf16 dO[QTILE * RPAD];
  bf16 mk[MT * RPAD];
  bf16 mv[MT * RPAD];
  bf16 dsm[QTILE * 24];   // meta dS (bf16), rows x 16 (+8 pad)
  bf16 pm[QTILE * 24];    // meta P (bf16)
  float lse2[QTILE];
  float drow[QTILE];      // D_t from the saved forward output
  // last, so that the split pass (no key sweep) launches without them
  bf16 k[2][KT1 * RPAD];
  bf16 v[2][KT1 * RPAD];
};

static_assert(sizeof(QSmem) <= 232448, "shared memory per block exceeds 227 KB");

// the same with the A fragments read from shared memory as they are used
// (arow: this lane's ldmatrix row of the warp's 16 query rows)
template <int NK>
__device__ __forceinline__ void qk_scores_sm(const bf16* arow, const bf16* ks, int lane, float (*s)[4]) {
#pragma unroll
  for (int nt = 0; nt < NK / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk) {
    uint32_t a[4];
    ldsm_x4(smem_u32(arow + kk * 16), a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int ntp = 0; ntp < NK / 16; ++ntp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(smem_u32(&ks[(ntp * 16 + (lane & 7) + ((lane >> 4) << 3)) * RPAD + kk * 16 +
                           ((lane >> 3) & 1) * 8]),
              b0, b1, b2, b3);
      mma_bf16(s[2 * ntp], a, b0, b1);
      mma_bf16(s[2 * ntp + 1], a, b2, b3);
    }
  }
}

// scores of 16 query rows (A fragments qa) against NK keys stored row-major
template <int NK>
__device__ __forceinline__ void qk_scores(const uint32_t (*qa)[4], const bf16* ks, int lane,
                                          float (*s)[4]) {
#pragma unroll
  for (int nt = 0; nt < NK / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[nt][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < D / 16; ++kk)
#pragma unroll
    for (int ntp = 0; ntp < NK / 16; ++ntp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4(smem_u32(&ks[(ntp * 16 + (lane & 7) + ((lane >> 4) << 3)) * RPAD + kk * 16 +
                           ((lane >> 3) & 1) * 8]),
              b0, b1, b2, b3);
      mma_bf16(s[2 * ntp], qa[kk], b0, b1);
      mma_bf16(s[2 * ntp + 1], qa[kk], b2, b3);
    }
}

// WINDOW = false: the split query side (the forward output is given): no key
// sweep and no dq; the meta tokens' dS goes to p.ds_meta for swa_bwd_dq, and
// D and the meta gradients are formed as in the full pass.
template <bool WINDOW>
__global__ void __launch_bounds__(NT, WINDOW ? 2 : 4) swa_bwd_q_mma_kernel(SwaBwdParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  QSmem& sm = *reinterpret_cast<QSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, gc = (lane & 3) * 2;
  const int h = blockIdx.x, b = blockIdx.y, slab = blockIdx.z;
  const int H = p.H, T = p.T, w = p.w, M = p.M;
  const int bh = b * H + h;
  const bf16* q = (const bf16*)p.q + (size_t)bh * T * D;
  const bf16* k = (const bf16*)p.k + (size_t)bh * T * D;
  const bf16* v = (const bf16*)p.v + (size_t)bh * T * D;
  const bf16* dO = (const bf16*)p.dO + (size_t)bh * T * D;
  const float* lse = p.lse + (size_t)bh * T;
  const float c2 = p.scale * kLog2e;
  const int r0 = slab * SLAB, r1 = min(T, r0 + SLAB);

  auto load_rows = [&](bf16* dst, const bf16* src, int row0, int nvalid, int nrows) {
    for (int x = tid; x < nrows * D / 8; x += NT) {
      const int r = x / (D / 8), cc = x % (D / 8);
      const bool ok = r < nvalid;
      cp_async16(&dst[r * RPAD + cc * 8], src + (size_t)(ok ? row0 + r : row0) * D + cc * 8,
                 ok ? 16 : 0);
    }
  };
  if (M > 0) {
    load_rows(sm.mk, (const bf16*)p.mk + (size_t)h * M * D, 0, M, MT);
    if (p.mv) load_rows(sm.mv, (const bf16*)p.mv + (size_t)h * M * D, 0, M, MT);
  }
  // meta gradient partials: warp owns value/key columns [32 warp, 32 warp + 32)
  float gmk[4][4], gmv[4][4];
#pragma unroll
  for (int nt = 0; nt < 4; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) gmk[nt][e] = gmv[nt][e] = 0.f;
  float dsum = 0.f;

  for (int t0 = r0; t0 < r1; t0 += QTILE) {
    const int lo = max(0, t0 - w + 1);
    const int hi = min(T - 1, t0 + QTILE - 1);
    const int ntiles = (hi - lo + KT1) / KT1;
    __syncthreads();  // previous tile's readers are done
    load_rows(sm.q, q, t0, min(QTILE, T - t0), QTILE);
    load_rows(sm.dO, dO, t0, min(QTILE, T - t0), QTILE);
    for (int x = tid; x < QTILE; x += NT)
      sm.lse2[x] = t0 + x < T ? lse[t0 + x] * kLog2e : 0.f;
    cp_async_commit();
    if (p.osw && tid < 2 * QTILE && t0 + (tid >> 1) < T)  // the output rows D reads: into L1 meanwhile
      asm volatile("prefetch.global.L1 [%0];" ::"l"((const bf16*)p.osw + ((size_t)bh * T + t0 + (tid >> 1)) * D +
                                                    (tid & 1) * 64));
    cp_async_wait<0>();
    __syncthreads();
    if (p.osw) {  // D_t = dO_t . o_t, two threads per row
      const int r = tid >> 1, c0 = (tid & 1) * (D / 2);
      float acc = 0.f;
      if (t0 + r < T) {
        const uint4* op = reinterpret_cast<const uint4*>((const bf16*)p.osw + ((size_t)bh * T + t0 + r) * D + c0);
#pragma unroll
        for (int x = 0; x < D / 16; ++x) {
          const uint4 ov = __ldg(op + x);
          const uint4 dv4 = *reinterpret_cast<const uint4*>(&sm.dO[r * RPAD + c0 + 8 * x]);
          const uint32_t ow[4] = {ov.x, ov.y, ov.z, ov.w}, dw[4] = {dv4.x, dv4.y, dv4.z, dv4.w};
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            const float2 a = unpack_bf16(ow[y]), bb = unpack_bf16(dw[y]);
            acc = fmaf(a.x, bb.x, acc);
            acc = fmaf(a.y, bb.y, acc);
          }
        }
      }
      acc += __shfl_xor_sync(0xffffffffu, acc, 1);
      if ((tid & 1) == 0) sm.drow[r] = acc;
      __syncthreads();
    }
    const int row0 = t0 + 16 * warp + gr;
    // the key sweep keeps the warp's q / dO fragments in registers; the split
    // pass (one 16-key meta tile) reads them from shared memory instead
    uint32_t qa[WINDOW ? D / 16 : 1][4], da[WINDOW ? D / 16 : 1][4];
    const bf16* qrow = &sm.q[(16 * warp + (lane & 15)) * RPAD + (lane >> 4) * 8];
    const bf16* drow_a = &sm.dO[(16 * warp + (lane & 15)) * RPAD + (lane >> 4) * 8];
    if constexpr (WINDOW) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk) {
        ldsm_x4(smem_u32(qrow + kk * 16), qa[kk][0], qa[kk][1], qa[kk][2], qa[kk][3]);
        ldsm_x4(smem_u32(drow_a + kk * 16), da[kk][0], da[kk][1], da[kk][2], da[kk][3]);
      }
    }
    const float l2[2] = {sm.lse2[16 * warp + gr], sm.lse2[16 * warp + gr + 8]};
    float Drow[2] = {0.f, 0.f};
    if (p.osw) {
      Drow[0] = sm.drow[16 * warp + gr];
      Drow[1] = sm.drow[16 * warp + gr + 8];
    }
    float dq[D / 8][4];
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) dq[nt][e] = 0.f;

    // P and dP of one key tile; returns them in s / dp (masked entries 0)
    auto tile_pdp = [&](const bf16* ks, const bf16* vs, auto nk_tag, auto valid, float (*s)[4],
                        float (*dp)[4]) {
      constexpr int NK = decltype(nk_tag)::value;
      if constexpr (WINDOW) qk_scores<NK>(qa, ks, lane, s);
      else qk_scores_sm<NK>(qrow, ks, lane, s);
      if (vs) {
        if constexpr (WINDOW) qk_scores<NK>(da, vs, lane, dp);
        else qk_scores_sm<NK>(drow_a, vs, lane, dp);
      } else {
#pragma unroll
        for (int nt = 0; nt < NK / 8; ++nt)
#pragma unroll
          for (int e = 0; e < 4; ++e) dp[nt][e] = 0.f;
      }
#pragma unroll
      for (int nt = 0; nt < NK / 8; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int hh = e >> 1, j = nt * 8 + gc + (e & 1);
          s[nt][e] = valid(hh, j) ? exp2f(s[nt][e] * c2 - l2[hh]) : 0.f;
        }
    };
    auto window_valid = [&](int kb) {
      return [=](int hh, int j) {
        const int t = row0 + 8 * hh, key = kb + j;
        return t < T && key <= t && key >= t - w + 1 && key <= hi;
      };
    };
    auto meta_valid = [=](int hh, int j) { return j < M && row0 + 8 * hh < T; };
    const bf16* mvs = p.mv ? sm.mv : nullptr;

    for (int sweep = p.osw ? 1 : 0; sweep < 2; ++sweep) {
      if (M > 0) {  // meta tile
        float s[MT / 8][4], dp[MT / 8][4];
        tile_pdp(sm.mk, mvs, IntTag<MT>{}, meta_valid, s, dp);
        if (sweep == 0) {
#pragma unroll
          for (int nt = 0; nt < MT / 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) Drow[e >> 1] += s[nt][e] * dp[nt][e];
        } else {
          float ds[MT / 8][4];
#pragma unroll
          for (int nt = 0; nt < MT / 8; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) ds[nt][e] = p.gscale * s[nt][e] * (dp[nt][e] - Drow[e >> 1]);
          if constexpr (WINDOW) {  // dq += dS_meta mk
            const uint32_t pa[4] = {pack_bf16(ds[0][0], ds[0][1]), pack_bf16(ds[0][2], ds[0][3]),
                                    pack_bf16(ds[1][0], ds[1][1]), pack_bf16(ds[1][2], ds[1][3])};
#pragma unroll
            for (int ntp = 0; ntp < D / 16; ++ntp) {
              uint32_t b0, b1, b2, b3;
              ldsm_x4_t(smem_u32(&sm.mk[((lane & 7) + ((lane >> 3) & 1) * 8) * RPAD + ntp * 16 +
                                        (lane >> 4) * 8]),
                        b0, b1, b2, b3);
              mma_bf16(dq[2 * ntp], pa, b0, b1);
              mma_bf16(dq[2 * ntp + 1], pa, b2, b3);
            }
          } else {  // the meta tokens' dS without the gscale factor, for swa_bwd_dq
#pragma unroll
            for (int nt = 0; nt < MT / 8; ++nt)
#pragma unroll
              for (int hh = 0; hh < 2; ++hh) {
                const int t = row0 + 8 * hh, j = nt * 8 + gc;
                if (t < T)
                  *reinterpret_cast<uint32_t*>(&((bf16*)p.ds_meta)[((size_t)bh * T + t) * MT + j]) =
                      pack_bf16(s[nt][2 * hh] * (dp[nt][2 * hh] - Drow[hh]),
                                s[nt][2 * hh + 1] * (dp[nt][2 * hh + 1] - Drow[hh]));
              }
          }
          // stage dS_meta and P_meta for the meta-gradient products
#pragma unroll
          for (int nt = 0; nt < MT / 8; ++nt)
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              const int r = 16 * warp + gr + 8 * hh, j = nt * 8 + gc;
              *reinterpret_cast<uint32_t*>(&sm.dsm[r * 24 + j]) = pack_bf16(ds[nt][2 * hh], ds[nt][2 * hh + 1]);
              *reinterpret_cast<uint32_t*>(&sm.pm[r * 24 + j]) = pack_bf16(s[nt][2 * hh], s[nt][2 * hh + 1]);
            }
        }
      }
      if constexpr (WINDOW) {
        // window tiles, double-buffered
        load_rows(sm.k[0], k, lo, hi - lo + 1, KT1);
        load_rows(sm.v[0], v, lo, hi - lo + 1, KT1);
        cp_async_commit();
        for (int it = 0; it < ntiles; ++it) {
          const int stg = it & 1, kb = lo + it * KT1;
          cp_async_wait<0>();
          __syncthreads();
          if (it + 1 < ntiles) {
            const int nb = kb + KT1;
            load_rows(sm.k[stg ^ 1], k, nb, hi - nb + 1, KT1);
            load_rows(sm.v[stg ^ 1], v, nb, hi - nb + 1, KT1);
            cp_async_commit();
          }
          float s[KT1 / 8][4], dp[KT1 / 8][4];
          tile_pdp(sm.k[stg], sm.v[stg], IntTag<KT1>{}, window_valid(kb), s, dp);
          if (sweep == 0) {
  #pragma unroll
            for (int nt = 0; nt < KT1 / 8; ++nt)
  #pragma unroll
              for (int e = 0; e < 4; ++e) Drow[e >> 1] += s[nt][e] * dp[nt][e];
          } else {
  #pragma unroll
            for (int kk = 0; kk < KT1 / 16; ++kk) {
              float d0[4], d1[4];
  #pragma unroll
              for (int e = 0; e < 4; ++e) {
                d0[e] = p.gscale * s[2 * kk][e] * (dp[2 * kk][e] - Drow[e >> 1]);
                d1[e] = p.gscale * s[2 * kk + 1][e] * (dp[2 * kk + 1][e] - Drow[e >> 1]);
              }
              const uint32_t pa[4] = {pack_bf16(d0[0], d0[1]), pack_bf16(d0[2], d0[3]),
                                      pack_bf16(d1[0], d1[1]), pack_bf16(d1[2], d1[3])};
  #pragma unroll
              for (int ntp = 0; ntp < D / 16; ++ntp) {
                uint32_t b0, b1, b2, b3;
                ldsm_x4_t(smem_u32(&sm.k[stg][(kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * RPAD +
                                              ntp * 16 + (lane >> 4) * 8]),
                          b0, b1, b2, b3);
                mma_bf16(dq[2 * ntp], pa, b0, b1);
                mma_bf16(dq[2 * ntp + 1], pa, b2, b3);
              }
            }
          }
        }
      }
      __syncthreads();  // key buffers free for the next sweep
      if (sweep == 0) {
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          Drow[hh] += __shfl_xor_sync(0xffffffffu, Drow[hh], 1);
          Drow[hh] += __shfl_xor_sync(0xffffffffu, Drow[hh], 2);
        }
      }
    }
    // ---- dq, D ---------------------------------------------------------------
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int t = row0 + 8 * hh;
      if (t >= T) continue;
      const size_t off = ((size_t)bh * T + t) * D;
      if constexpr (WINDOW) {
#pragma unroll
        for (int nt = 0; nt < D / 8; ++nt) {
          const int j = nt * 8 + gc;
          const float x0 = dq[nt][2 * hh] * p.scale, x1 = dq[nt][2 * hh + 1] * p.scale;
          if (p.dq_f32) *reinterpret_cast<float2*>(&p.dq_f32[off + j]) = make_float2(x0, x1);
          else *reinterpret_cast<uint32_t*>(&((bf16*)p.dq)[off + j]) = pack_bf16(x0, x1);
        }
      }
      if ((lane & 3) == 0) {
        p.Dbuf[(size_t)bh * T + t] = Drow[hh];
        dsum += Drow[hh];
      }
    }
    // ---- meta gradients of this tile: dS_meta^T Q and P_meta^T dO ----------
    if (M > 0) {
      __syncthreads();  // dsm / pm staged by every warp
#pragma unroll
      for (int kk = 0; kk < QTILE / 16; ++kk) {
        uint32_t a1[4], a2[4];
        // A = dS_meta^T: [m][t] from the [t][m] tile (transposed load)
        ldsm_x4_t(smem_u32(&sm.dsm[(kk * 16 + (lane & 7) + ((lane >> 4) << 3)) * 24 +
                                   ((lane >> 3) & 1) * 8]),
                  a1[0], a1[1], a1[2], a1[3]);
        ldsm_x4_t(smem_u32(&sm.pm[(kk * 16 + (lane & 7) + ((lane >> 4) << 3)) * 24 +
                                  ((lane >> 3) & 1) * 8]),
                  a2[0], a2[1], a2[2], a2[3]);
#pragma unroll
        for (int ntp = 0; ntp < 2; ++ntp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(&sm.q[(kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * RPAD + 32 * warp +
                                   ntp * 16 + (lane >> 4) * 8]),
                    b0, b1, b2, b3);
          mma_bf16(gmk[2 * ntp], a1, b0, b1);
          mma_bf16(gmk[2 * ntp + 1], a1, b2, b3);
          ldsm_x4_t(smem_u32(&sm.dO[(kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * RPAD + 32 * warp +
                                    ntp * 16 + (lane >> 4) * 8]),
                    b0, b1, b2, b3);
          mma_bf16(gmv[2 * ntp], a2, b0, b1);
          mma_bf16(gmv[2 * ntp + 1], a2, b2, b3);
        }
      }
    }
  }
  // ---- per-CTA partials: meta gradients and sum of D ------------------------
  if (M > 0) {
    const int nslab = gridDim.z;
    float* part = p.meta_part + (((size_t)b * nslab + slab) * H + h) * M * (2 * D);
#pragma unroll
    for (int nt = 0; nt < 4; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int m = gr + 8 * hh;
        if (m >= M) continue;
        const int col = 32 * warp + nt * 8 + gc;
        float* dst = part + (size_t)m * (2 * D);
        dst[col] = gmk[nt][2 * hh] * p.scale;
        dst[col + 1] = gmk[nt][2 * hh + 1] * p.scale;
        dst[D + col] = gmv[nt][2 * hh] * p.gscale;
        dst[D + col + 1] = gmv[nt][2 * hh + 1] * p.gscale;
      }
  }
  __shared__ float red[NT / 32];
  dsum += __shfl_xor_sync(0xffffffffu, dsum, 4);
  dsum += __shfl_xor_sync(0xffffffffu, dsum, 8);
  dsum += __shfl_xor_sync(0xffffffffu, dsum, 16);
  if (lane == 0) red[warp] = dsum;
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
    for (int x = 0; x < NT / 32; ++x) s += red[x];
    p.alpha_part[((size_t)b * gridDim.z + slab) * H + h] = s;
  }
}

// ---------------------------------------------------------------------------
// Kernel 2: dk, dv (key-major)
// ---------------------------------------------------------------------------
constexpr int KT2 = 64;  // keys per CTA
constexpr int QT2 = 32;  // query rows per tile

struct KVSmem {
  bf16 k[KT2 * RPAD];
  bf16 v[KT2 * RPAD];
  bf16 q[2][QT2 * RPAD];
  bf16 dO[2][QT2 * RPAD];
  float lse2[2][QT2];
  float Dt[2][QT2];
};

__global__ void __launch_bounds__(NT, 2) swa_bwd_kv_mma_kernel(SwaBwdParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  KVSmem& sm = *reinterpret_cast<KVSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, gc = (lane & 3) * 2;
  const int bh = blockIdx.y;
  const int T = p.T, w = p.w;
  const int j0 = blockIdx.x * KT2;
  const bf16* q = (const bf16*)p.q + (size_t)bh * T * D;
  const bf16* k = (const bf16*)p.k + (size_t)bh * T * D;
  const bf16* v = (const bf16*)p.v + (size_t)bh * T * D;
  const bf16* dO = (const bf16*)p.dO + (size_t)bh * T * D;
  const float* lse = p.lse + (size_t)bh * T;
  const float* Db = p.Dbuf + (size_t)bh * T;
  const float c2 = p.scale * kLog2e;
  const int tlo = j0;
  const int thi = min(T - 1, j0 + KT2 - 1 + w - 1);
  const int ntiles = (thi - tlo + QT2) / QT2;

  auto load_rows = [&](bf16* dst, const bf16* src, int row0, int nvalid, int nrows) {
    for (int x = tid; x < nrows * D / 8; x += NT) {
      const int r = x / (D / 8), cc = x % (D / 8);
      const bool ok = r < nvalid;
      cp_async16(&dst[r * RPAD + cc * 8], src + (size_t)(ok ? row0 + r : row0) * D + cc * 8,
                 ok ? 16 : 0);
    }
  };
  auto load_qtile = [&](int tb, int st) {
    load_rows(sm.q[st], q, tb, thi - tb + 1, QT2);
    load_rows(sm.dO[st], dO, tb, thi - tb + 1, QT2);
    cp_async_commit();
    for (int x = tid; x < QT2; x += NT) {
      const bool ok = tb + x <= thi;
      sm.lse2[st][x] = ok ? lse[tb + x] * kLog2e : 0.f;
      sm.Dt[st][x] = ok ? Db[tb + x] : 0.f;
    }
  };
  load_rows(sm.k, k, j0, min(KT2, T - j0), KT2);
  load_rows(sm.v, v, j0, min(KT2, T - j0), KT2);
  cp_async_commit();
  load_qtile(tlo, 0);

  float dk[D / 8][4], dv[D / 8][4];
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[nt][e] = dv[nt][e] = 0.f;
  const int key0 = j0 + 16 * warp + gr;  // this lane's keys: key0 and key0 + 8

  for (int it = 0; it < ntiles; ++it) {
    const int st = it & 1, tb = tlo + it * QT2;
    cp_async_wait<0>();
    __syncthreads();
    if (it + 1 < ntiles) load_qtile(tb + QT2, st ^ 1);
    // S^T = K Q^T and dP^T = V dO^T for this warp's 16 keys x 32 queries
    float s[QT2 / 8][4], dp[QT2 / 8][4];
#pragma unroll
    for (int nt = 0; nt < QT2 / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) s[nt][e] = dp[nt][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < D / 16; ++kk) {
      uint32_t ka[4], va[4];
      ldsm_x4(smem_u32(&sm.k[(16 * warp + (lane & 15)) * RPAD + kk * 16 + (lane >> 4) * 8]), ka[0], ka[1],
              ka[2], ka[3]);
      ldsm_x4(smem_u32(&sm.v[(16 * warp + (lane & 15)) * RPAD + kk * 16 + (lane >> 4) * 8]), va[0], va[1],
              va[2], va[3]);
#pragma unroll
      for (int ntp = 0; ntp < QT2 / 16; ++ntp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4(smem_u32(&sm.q[st][(ntp * 16 + (lane & 7) + ((lane >> 4) << 3)) * RPAD + kk * 16 +
                                   ((lane >> 3) & 1) * 8]),
                b0, b1, b2, b3);
        mma_bf16(s[2 * ntp], ka, b0, b1);
        mma_bf16(s[2 * ntp + 1], ka, b2, b3);
        ldsm_x4(smem_u32(&sm.dO[st][(ntp * 16 + (lane & 7) + ((lane >> 4) << 3)) * RPAD + kk * 16 +
                                    ((lane >> 3) & 1) * 8]),
                b0, b1, b2, b3);
        mma_bf16(dp[2 * ntp], va, b0, b1);
        mma_bf16(dp[2 * ntp + 1], va, b2, b3);
      }
    }
    // P^T, dS^T
#pragma unroll
    for (int nt = 0; nt < QT2 / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int j = key0 + 8 * (e >> 1), tl = nt * 8 + gc + (e & 1), t = tb + tl;
        const bool ok = j < T && t <= thi && t >= j && t <= j + w - 1;
        const float P = ok ? exp2f(s[nt][e] * c2 - sm.lse2[st][tl]) : 0.f;
        s[nt][e] = P;
        dp[nt][e] = P * (dp[nt][e] - sm.Dt[st][tl]);
      }
    // dv += P^T dO, dk += dS^T Q
#pragma unroll
    for (int kk = 0; kk < QT2 / 16; ++kk) {
      const uint32_t pa[4] = {pack_bf16(s[2 * kk][0], s[2 * kk][1]), pack_bf16(s[2 * kk][2], s[2 * kk][3]),
                              pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]),
                              pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3])};
      const uint32_t da[4] = {pack_bf16(dp[2 * kk][0], dp[2 * kk][1]), pack_bf16(dp[2 * kk][2], dp[2 * kk][3]),
                              pack_bf16(dp[2 * kk + 1][0], dp[2 * kk + 1][1]),
                              pack_bf16(dp[2 * kk + 1][2], dp[2 * kk + 1][3])};
#pragma unroll
      for (int ntp = 0; ntp < D / 16; ++ntp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(&sm.dO[st][(kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * RPAD + ntp * 16 +
                                      (lane >> 4) * 8]),
                  b0, b1, b2, b3);
        mma_bf16(dv[2 * ntp], pa, b0, b1);
        mma_bf16(dv[2 * ntp + 1], pa, b2, b3);
        ldsm_x4_t(smem_u32(&sm.q[st][(kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * RPAD + ntp * 16 +
                                     (lane >> 4) * 8]),
                  b0, b1, b2, b3);
        mma_bf16(dk[2 * ntp], da, b0, b1);
        mma_bf16(dk[2 * ntp + 1], da, b2, b3);
      }
    }
  }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int j = key0 + 8 * hh;
    if (j >= T) continue;
    const size_t off = ((size_t)bh * T + j) * D;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      const int c = nt * 8 + gc;
      const float k0 = dk[nt][2 * hh] * p.scale * p.gscale, k1 = dk[nt][2 * hh + 1] * p.scale * p.gscale;
      const float v0 = dv[nt][2 * hh] * p.gscale, v1 = dv[nt][2 * hh + 1] * p.gscale;
      if (p.dk_f32) *reinterpret_cast<float2*>(&p.dk_f32[off + c]) = make_float2(k0, k1);
      else *reinterpret_cast<uint32_t*>(&((bf16*)p.dk)[off + c]) = pack_bf16(k0, k1);
      if (p.dv_f32) *reinterpret_cast<float2*>(&p.dv_f32[off + c]) = make_float2(v0, v1);
      else *reinterpret_cast<uint32_t*>(&((bf16*)p.dv)[off + c]) = pack_bf16(v0, v1);
    }
  }
}

// ---------------------------------------------------------------------------
// Kernel 3 (split query side): dq from the key side's dS tiles
// ---------------------------------------------------------------------------
// The tcgen05 key side forms, for every 128-key block b and every 64-query
// tile i that sees it, dS^T = P^T (dP^T - D) without the gscale factor and
// stores it in bf16: ds_tiles[bh][b][i][key][query].  A query tile q0 takes
// those of the blocks its window reaches and the meta tokens' dS:
//   dq = scale * gscale * (sum_b dS_b K_b + dS_meta MK)
// (Lizard technical summary, section 2a: the window keys and the always-visible
// meta tokens share one softmax, so they share its Jacobian).
constexpr int QT3 = 64;        // query rows per dS tile
constexpr int QR3 = 128;       // query rows per CTA (8 warps x 16): two tiles that see the same key blocks
constexpr int NT3 = 256;
constexpr int KB3 = 128;       // keys per block of the key side
constexpr int KU3 = 64;        // keys per streamed unit (half a block)
constexpr int DSP = QT3 + 8;   // padded row of a [key][query] dS tile

struct DqSmem {
  bf16 ds[2][2][KU3 * DSP];    // [stage][query tile]: a unit's rows of the CTA's two dS tiles
  bf16 k[2][KU3 * RPAD];       // [stage]: the unit's keys
  bf16 mk[MT * RPAD];
  bf16 dsm[QR3 * 24];          // the meta tokens' dS, [query][16] (+8 pad)
};
static_assert(sizeof(DqSmem) <= 232448 / 2, "two dq CTAs must fit one SM");

// one CTA = 128 query rows q0 .. q0 + 127 (q0 a multiple of 128, so its two
// 64-row tiles see the same key blocks); warp wq takes rows 16 wq .. 16 wq + 15
__global__ void __launch_bounds__(NT3, 2) swa_bwd_dq_kernel(SwaBwdParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  DqSmem& sm = *reinterpret_cast<DqSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, gc = (lane & 3) * 2;
  // batch-heads in reverse: the key side wrote the last ones' tiles last, so
  // they are still in L2 when this pass starts
  const int q0 = blockIdx.x * QR3, bh = gridDim.y - 1 - blockIdx.y, h = bh % p.H;
  const int T = p.T, w = p.w, M = p.M;
  const int nblk = (T + KB3 - 1) / KB3;
  const int half = warp >> 2, rw = 16 * (warp & 3);  // the warp's tile and its rows in it
  // the key blocks whose window reaches the CTA's rows: keys >= q0 - w + 1, <= q0 + 127
  const int b_lo = max(0, q0 - w + 1) / KB3, b_hi = min(q0 / KB3, nblk - 1);
  // tiles the key side formed for block b (the same count as its own loop)
  auto tiles_of = [&](int b) { return (min(T - 1, b * KB3 + KB3 - 1 + w - 1) - b * KB3 + QT3) / QT3; };
  // the blocks stream through two stages in units of 64 keys: unit u = block
  // b_lo + u / 2, keys [64 (u % 2), 64 (u % 2) + 64) of it
  const int nu = 2 * (b_hi - b_lo + 1);
  auto load_unit = [&](int u) {
    const int b = b_lo + u / 2, st = u & 1, ko = KU3 * (u % 2);
    const int j0 = b * KB3, nq = tiles_of(b);
    for (int hf = 0; hf < 2; ++hf) {
      const int i = (q0 - j0) / QT3 + hf;
      if (i >= nq) continue;  // no query of this tile sees the block: its warps skip it below
      const bf16* ds = (const bf16*)p.ds_tiles + (((size_t)bh * nblk + b) * p.ds_nq + i) * KB3 * QT3 +
                       (size_t)ko * QT3;
      for (int x = tid; x < KU3 * QT3 / 8; x += NT3) {
        const int r = x / (QT3 / 8), cc = x % (QT3 / 8);
        cp_async16(&sm.ds[st][hf][r * DSP + cc * 8], ds + (size_t)r * QT3 + cc * 8, 16);
      }
    }
    const bf16* k = (const bf16*)p.k + (size_t)bh * T * D;
    const int rows = min(KU3, T - j0 - ko);  // may be <= 0: all zeros
    for (int x = tid; x < KU3 * D / 8; x += NT3) {
      const int r = x / (D / 8), cc = x % (D / 8);
      const bool ok = r < rows;  // zero-filled rows still name an in-bounds source row
      cp_async16(&sm.k[st][r * RPAD + cc * 8], k + (size_t)(ok ? j0 + ko + r : j0) * D + cc * 8, ok ? 16 : 0);
    }
  };

  float dq[D / 8][4];
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) dq[nt][e] = 0.f;

  if (M > 0) {  // the meta tokens' dS and MK ride with the first unit's copies
    const bf16* dsm = (const bf16*)p.ds_meta + ((size_t)bh * T + q0) * MT;
    for (int x = tid; x < QR3 * MT / 8; x += NT3) {
      const int r = x / (MT / 8), cc = x % (MT / 8);
      const bool ok = q0 + r < T;
      cp_async16(&sm.dsm[r * 24 + cc * 8], dsm + (size_t)(ok ? r : 0) * MT + cc * 8, ok ? 16 : 0);
    }
    const bf16* mk = (const bf16*)p.mk + (size_t)h * M * D;
    for (int x = tid; x < MT * D / 8; x += NT3) {
      const int r = x / (D / 8), cc = x % (D / 8);
      const bool ok = r < M;
      cp_async16(&sm.mk[r * RPAD + cc * 8], mk + (size_t)(ok ? r : 0) * D + cc * 8, ok ? 16 : 0);
    }
  }
  load_unit(0);
  cp_async_commit();
  if (nu > 1) load_unit(1);
  cp_async_commit();
  for (int u = 0; u < nu; ++u) {
    cp_async_wait<1>();  // unit u's group (one group is committed per unit, empty past the end)
    __syncthreads();
    if (M > 0 && u == 0) {  // dq += dS_meta MK
      uint32_t a[4];
      ldsm_x4(smem_u32(&sm.dsm[(16 * warp + (lane & 15)) * 24 + (lane >> 4) * 8]), a[0], a[1], a[2], a[3]);
#pragma unroll
      for (int ntp = 0; ntp < D / 16; ++ntp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(&sm.mk[((lane & 7) + ((lane >> 3) & 1) * 8) * RPAD + ntp * 16 + (lane >> 4) * 8]),
                  b0, b1, b2, b3);
        mma_bf16(dq[2 * ntp], a, b0, b1);
        mma_bf16(dq[2 * ntp + 1], a, b2, b3);
      }
    }
    const int b = b_lo + u / 2, st = u & 1;
    if ((q0 - b * KB3) / QT3 + half < tiles_of(b)) {  // this warp's tile sees the block
      const bf16* dsb = sm.ds[st][half];
      const bf16* kb = sm.k[st];
#pragma unroll
      for (int kk = 0; kk < KU3 / 16; ++kk) {
        uint32_t a[4];  // A = dS (queries x keys) from the [key][query] tile, transposed
        ldsm_x4_t(smem_u32(&dsb[(kk * 16 + (lane & 7) + ((lane >> 4) << 3)) * DSP + rw + ((lane >> 3) & 1) * 8]),
                  a[0], a[1], a[2], a[3]);
#pragma unroll
        for (int ntp = 0; ntp < D / 16; ++ntp) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(smem_u32(&kb[(kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * RPAD + ntp * 16 +
                                 (lane >> 4) * 8]),
                    b0, b1, b2, b3);
          mma_bf16(dq[2 * ntp], a, b0, b1);
          mma_bf16(dq[2 * ntp + 1], a, b2, b3);
        }
      }
    }
    __syncthreads();  // stage st is free
    if (u + 2 < nu) load_unit(u + 2);
    cp_async_commit();
  }
  const float sc = p.scale * p.gscale;
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int t = q0 + 16 * warp + gr + 8 * hh;
    if (t >= T) continue;
    const size_t off = ((size_t)bh * T + t) * D;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt)
      *reinterpret_cast<uint32_t*>(&((bf16*)p.dq)[off + nt * 8 + gc]) =
          pack_bf16(dq[nt][2 * hh] * sc, dq[nt][2 * hh + 1] * sc);
  }
}

}  // namespace

bool swa_bwd_mma_supported(int dk, int dv, bool bf16) { return bf16 && dk == D && dv == D; }

cudaError_t launch_swa_bwd_mma(const SwaBwdParams& p, cudaStream_t s) {
  const bool empty = p.T == 0 || p.B * p.H == 0;
  const int nslab = (p.T + SLAB - 1) / SLAB;
  cudaError_t e = cudaSuccess;
  const bool kv_tc = p.tc && swa_bwd_kv_tc_supported(p.dkd, p.dvd, true);
  const bool q_tc = p.tc_q && swa_bwd_q_tc_supported(p);
  // split query side: D and the meta terms here, dq from the key side's dS tiles
  const bool split = p.ds_tiles && p.ds_meta && p.osw && p.dq && !p.dq_f32 && kv_tc && !q_tc;
  SwaBwdParams pp = p;
  if (split) pp.ds_nq = swa_bwd_ds_nq(p.w);
  else pp.ds_tiles = nullptr;
  if (!empty) {
    if (q_tc) {
      e = launch_swa_bwd_q_tc(pp, s);
    } else {
      const auto kern = split ? swa_bwd_q_mma_kernel<false> : swa_bwd_q_mma_kernel<true>;
      const size_t b1 = split ? offsetof(QSmem, k) : sizeof(QSmem);
      e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)b1);
      if (e != cudaSuccess) return e;
      {
        ScopedTiming tm(split ? "swa_bwd_meta" : "swa_bwd_q_mma", s);
        kern<<<dim3(p.H, p.B, nslab), NT, b1, s>>>(pp);
      }
      e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    if (p.query_done) e = cudaEventRecord((cudaEvent_t)p.query_done, s);
    if (e != cudaSuccess) return e;
    if (kv_tc) {
      e = launch_swa_bwd_kv_tc(pp, s);
    } else {
      const size_t b2 = sizeof(KVSmem);
      e = cudaFuncSetAttribute(swa_bwd_kv_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)b2);
      if (e != cudaSuccess) return e;
      {
        ScopedTiming tm("swa_bwd_kv_mma", s);
        swa_bwd_kv_mma_kernel<<<dim3((p.T + KT2 - 1) / KT2, p.B * p.H), NT, b2, s>>>(pp);
      }
      e = cudaGetLastError();
    }
    if (e != cudaSuccess) return e;
    if (split) {
      const size_t b3 = sizeof(DqSmem);
      e = cudaFuncSetAttribute(swa_bwd_dq_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)b3);
      if (e != cudaSuccess) return e;
      {
        ScopedTiming tm("swa_bwd_dq", s);
        swa_bwd_dq_kernel<<<dim3((p.T + QR3 - 1) / QR3, p.B * p.H), NT3, b3, s>>>(pp);
      }
      e = cudaGetLastError();
      if (e != cudaSuccess) return e;
    }
  }
  if (empty && p.query_done) e = cudaEventRecord((cudaEvent_t)p.query_done, s);
  if (e != cudaSuccess || p.defer_reduce) return e;
  return launch_swa_bwd_mma_reduce(p, s);
}

cudaError_t launch_swa_bwd_mma_reduce(const SwaBwdParams& p, cudaStream_t s) {
  const bool empty = p.T == 0 || p.B * p.H == 0;
  const int nslab = (p.T + SLAB - 1) / SLAB;
  const int nparts = (p.M > 0 && !empty) ? p.B * nslab : 0;
  const int nalpha = empty ? 0 : p.B * p.H * nslab;
  return launch_swa_bwd_reduce(p, nparts, nalpha, s);
}

}  // namespace lz
