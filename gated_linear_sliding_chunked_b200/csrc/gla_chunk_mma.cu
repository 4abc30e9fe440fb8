// Two-pass chunked gated linear attention forward on the tensor cores (bf16
// I/O, fp32 accumulation, dk = dv = 128).
//
// Recurrence (Lizard technical summary, section 2a, state update equation):
//   S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T,   o_t = q_t^T S_t.
// Over 64-token chunks with b_t the running log-gate inside the chunk and b_l
// its last value:
//   S_next = diag(e^{b_l}) S_prev + sum_s (k_s e^{b_l - b_s}) v_s^T
//   o_t    = (q_t e^{b_t})^T S_prev + sum_{s<=t} A[t][s] v_s,
//   A[t][s] = sum_i q_t,i k_s,i e^{b_t,i - b_s,i}.
// Only the state carries a dependence between chunks, and its recurrence
// over chunks is linear, so the work is split:
//   pass 1, two levels: gla_delta_kernel<0> forms every chunk's increment
//     (k e^{b_l - b})^T v and decay e^{b_l} at once; gla_scan_kernel<0> walks
//     the chunks elementwise and writes the bf16 state before every chunk
//     (and the final fp32 state).  gla_states_kernel, one CTA per (batch,
//     head, 32 value columns) walking the chunks with the state in
//     registers, serves one-chunk sequences;
//   pass 2 (gla_out_kernel): one CTA per (chunk, batch, head) computes the
//     chunk's outputs from its incoming state, all chunks in parallel.
// The backward's first level reuses the pass-1 kernels on the query side
// (gla_delta_kernel<1>, gla_scan_kernel<1>, launch_gla_bwd_scan).
// Gate factors are the bounded ones of the single-pass kernel: per key dim
// one reference row when each 32-row half decays by at most e^-60 ("tame"),
// else 16-row sub-block references with per-pair factors F_IJ; diagonal
// blocks that decay past e^-60 take exp(b_t - b_s) per element.
#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"

namespace lz {
namespace {

constexpr int C = 64;
constexpr int SB = 16;
constexpr int NSB = C / SB;
constexpr int DK = 128;
constexpr int DV = 128;
constexpr int NT = 256;
constexpr int QKP = DK + 8;
constexpr int VP = DV + 8;
constexpr int NPAIR = NSB * (NSB + 1) / 2;
__device__ constexpr float kMinBlockDecay = 8.75651076e-27f;  // e^-60

__device__ __forceinline__ int pair_index(int I, int J) { return I * (I + 1) / 2 + J; }

// ===========================================================================
// Pass 1: the state walk
// ===========================================================================
constexpr int DVS = 32;          // value columns per CTA
constexpr int SVP = DVS + 8;     // padded row of the v slice

struct StateSmem {
  bf16 k[2][C * DK];
  bf16 v[2][C * SVP];
  float g[C * DK];
  bf16 ks[C * QKP];              // k e^{b_l - b}
  float dec[NSB][DK];
  float ec[DK];
};
static_assert(sizeof(StateSmem) <= 115712, "two state-pass CTAs must fit one SM");

__global__ void __launch_bounds__(NT, 2) gla_states_kernel(GlaFwdParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  StateSmem& sm = *reinterpret_cast<StateSmem*>(smem_raw);
  constexpr int SNT = DVS / 8;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, gc = (lane & 3) * 2;
  const int j0 = blockIdx.x * DVS;
  const int bh = blockIdx.y;
  const int T = p.T;
  const bf16* k = (const bf16*)p.k + (size_t)bh * T * DK;
  const bf16* v = (const bf16*)p.v + (size_t)bh * T * DV;
  const float* g = p.g + (size_t)bh * T * DK;
  const int nchunks = (T + C - 1) / C;

  auto issue_kv = [&](int c, int st) {
    const int c0 = c * C;
    for (int x = tid; x < C * DK / 8; x += NT) {
      const int r = x / (DK / 8), cc = x % (DK / 8);
      const bool ok = c0 + r < T;
      cp_async16(&sm.k[st][r * DK + cc * 8], k + (size_t)(ok ? c0 + r : 0) * DK + cc * 8, ok ? 16 : 0);
    }
    for (int x = tid; x < C * DVS / 8; x += NT) {
      const int r = x / (DVS / 8), cc = x % (DVS / 8);
      const bool ok = c0 + r < T;
      cp_async16(&sm.v[st][r * SVP + cc * 8], v + (size_t)(ok ? c0 + r : 0) * DV + j0 + cc * 8,
                 ok ? 16 : 0);
    }
    cp_async_commit();
  };
  auto issue_g = [&](int c) {
    const int c0 = c * C;
    for (int x = tid; x < C * DK / 4; x += NT) {
      const int r = x / (DK / 4), cc = x % (DK / 4);
      const bool ok = c0 + r < T;
      cp_async16(&sm.g[r * DK + cc * 4], g + (size_t)(ok ? c0 + r : 0) * DK + cc * 4, ok ? 16 : 0);
    }
    cp_async_commit();
  };

  // state rows 16w .. 16w+15, this CTA's 32 value columns, fp32 in registers
  float s[SNT][4];
#pragma unroll
  for (int nt = 0; nt < SNT; ++nt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = 16 * warp + gr + 8 * hh, j = j0 + nt * 8 + gc;
      float a = 0.f, b = 0.f;
      if (p.h0) {
        const float* hp = p.h0 + ((size_t)bh * DK + i) * DV + j;
        a = hp[0];
        b = hp[1];
      }
      s[nt][2 * hh] = a;
      s[nt][2 * hh + 1] = b;
    }

  if (nchunks > 0) {
    issue_kv(0, 0);
    issue_g(0);
  }
  for (int c = 0; c < nchunks; ++c) {
    const int st = c & 1;
    cp_async_wait<0>();
    __syncthreads();
    if (c + 1 < nchunks) issue_kv(c + 1, st ^ 1);
    {  // state before this chunk
      bf16* dst = (bf16*)p.states16 + ((size_t)bh * nchunks + c) * DK * DV + j0;
#pragma unroll
      for (int nt = 0; nt < SNT; ++nt)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int i = 16 * warp + gr + 8 * hh, j = nt * 8 + gc;
          *reinterpret_cast<uint32_t*>(&dst[(size_t)i * DV + j]) = pack_bf16(s[nt][2 * hh], s[nt][2 * hh + 1]);
        }
    }
    // prep: thread -> (sub-block K, key dims i2, i2+1); k side only
    const int K = tid >> 6, i2 = (tid & 63) * 2, r0 = K * SB;
    float2 kfac[SB];
    {
      float2 run = make_float2(1.f, 1.f);
#pragma unroll
      for (int r = SB - 1; r >= 0; --r) {  // prod_{u = r+1 .. end} e_u
        kfac[r] = run;
        const float2 gg = *reinterpret_cast<const float2*>(&sm.g[(r0 + r) * DK + i2]);
        run.x *= __expf(gg.x);
        run.y *= __expf(gg.y);
      }
      *reinterpret_cast<float2*>(&sm.dec[K][i2]) = run;
    }
    __syncthreads();
    if (c + 1 < nchunks) issue_g(c + 1);
    {
      float2 f = make_float2(1.f, 1.f);
#pragma unroll
      for (int J = 0; J < NSB; ++J)
        if (J > K) {
          const float2 d = *reinterpret_cast<const float2*>(&sm.dec[J][i2]);
          f.x *= d.x;
          f.y *= d.y;
        }
      if (K == 0) {
        float2 e = make_float2(1.f, 1.f);
#pragma unroll
        for (int J = 0; J < NSB; ++J) {
          const float2 d = *reinterpret_cast<const float2*>(&sm.dec[J][i2]);
          e.x *= d.x;
          e.y *= d.y;
        }
        *reinterpret_cast<float2*>(&sm.ec[i2]) = e;
      }
#pragma unroll
      for (int r = 0; r < SB; ++r) {
        const float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.k[st][(r0 + r) * DK + i2]));
        *reinterpret_cast<uint32_t*>(&sm.ks[(r0 + r) * QKP + i2]) =
            pack_bf16(kv.x * kfac[r].x * f.x, kv.y * kfac[r].y * f.y);
      }
    }
    __syncthreads();
    // S = diag(e^{b_l}) S + Ks^T V
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
          ldsm_x4_t(smem_u32(&sm.v[st][(16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8) * SVP + ntp * 16 +
                                       (lane >> 4) * 8]),
                    b0, b1, b2, b3);
          mma_bf16(s[2 * ntp], a, b0, b1);
          mma_bf16(s[2 * ntp + 1], a, b2, b3);
        }
      }
    }
  }
  if (p.hT) {
#pragma unroll
    for (int nt = 0; nt < SNT; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int i = 16 * warp + gr + 8 * hh, j = j0 + nt * 8 + gc;
        *reinterpret_cast<float2*>(&p.hT[((size_t)bh * DK + i) * DV + j]) =
            make_float2(s[nt][2 * hh], s[nt][2 * hh + 1]);
      }
  }
}

// ===========================================================================
// Pass 1, two-level variant for long sequences: every chunk's own state
// increment in parallel, then an elementwise scan over the chunks
// ===========================================================================
//   dS_c = (k e^{b_l - b})^T v over the chunk,  E_c = e^{b_l} per key dim,
//   S_{c+1} = diag(E_c) S_c + dS_c.
// dS_c goes through memory in bf16 (the states the output pass reads are
// bf16 as well); the scan keeps S in fp32.
// Measured on B200 it beats the sequential pass at 32 chunks x 64 heads
// (0.079 vs 0.096 ms), 128 x 64 (0.276 vs 0.363 ms) and 1024 x 32 (1.14 vs
// 1.81 ms); a single chunk has nothing to scan.
constexpr int kScanMinChunks = 2;

// the CTA's threads request the 128-byte lines of [base, base + bytes) into L2
__device__ __forceinline__ void prefetch_l2_lines(const void* base, size_t bytes, int tid) {
  const char* b = static_cast<const char*>(base);
  for (size_t off = (size_t)tid * 128; off < bytes; off += (size_t)NT * 128)
    asm volatile("prefetch.global.L2 [%0];" ::"l"(b + off));
}

struct DeltaSmem {
  bf16 k[C * QKP];
  bf16 v[C * VP];
  float g[C * DK];
  bf16 ks[C * QKP];
  float dec[NSB][DK];
};
static_assert(sizeof(DeltaSmem) <= 115712, "two delta CTAs must fit one SM");

// One chunk's increment of a carried [dk][dv] matrix, X^T Y over the chunk
// with X the key-side or query-side operand scaled by its in-chunk decay:
//   forward (key side):   dS_c = (k e^{b_l - b})^T v,   S_{c+1} = diag(E_c) S_c + dS_c
//   backward (query side): dG_c = (q e^{b})^T dO,       G_{c-1} = diag(E_c) G_c + dG_c
// with b the running log-gate from the chunk's start (inclusive) and E_c =
// e^{b_l} per key dim.  Every factor is a product of per-row gates, so <= 1.
struct DeltaArgs {
  const bf16* x;   // k or q  [BH][T][DK]
  const bf16* y;   // v or dO [BH][T][DV]
  const float* g;  // [BH][T][DK] log-gates, or NULL with
  const bf16* gz;  //   the gate logits [BH][T][DK]
  float gs;        //   and their scale
  bf16* delta;     // [BH][nchunks][DK][DV]
  float* decay;    // [BH][nchunks][DK]
  int T;
  int wave = 0;    // resident CTAs: the inputs of the CTA this far ahead go to L2
};

template <bool QSIDE>
__global__ void __launch_bounds__(NT, 2) gla_delta_kernel(DeltaArgs p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  DeltaSmem& sm = *reinterpret_cast<DeltaSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, gc = (lane & 3) * 2;
  const int c = blockIdx.x, bh = blockIdx.y;
  const int T = p.T, nchunks = gridDim.x;
  const int c0 = c * C, rows = min(C, T - c0);
  const bf16* k = p.x + ((size_t)bh * T + c0) * DK;
  const bf16* v = p.y + ((size_t)bh * T + c0) * DV;
  for (int x = tid; x < C * DK / 8; x += NT) {
    const int r = x / (DK / 8), cc = x % (DK / 8);
    const bool ok = r < rows;
    cp_async16(&sm.k[r * QKP + cc * 8], k + (size_t)(ok ? r : 0) * DK + cc * 8, ok ? 16 : 0);
    cp_async16(&sm.v[r * VP + cc * 8], v + (size_t)(ok ? r : 0) * DV + cc * 8, ok ? 16 : 0);
  }
  if (p.gz) {  // logits go through ks (written only after the prep's first barrier)
    const bf16* z = p.gz + ((size_t)bh * T + c0) * DK;
    for (int x = tid; x < C * DK / 8; x += NT) {
      const int r = x / (DK / 8), cc = x % (DK / 8);
      const bool ok = r < rows;
      cp_async16(&sm.ks[r * QKP + cc * 8], z + (size_t)(ok ? r : 0) * DK + cc * 8, ok ? 16 : 0);
    }
  } else {
    const float* g = p.g + ((size_t)bh * T + c0) * DK;
    for (int x = tid; x < C * DK / 4; x += NT) {
      const int r = x / (DK / 4), cc = x % (DK / 4);
      const bool ok = r < rows;
      cp_async16(&sm.g[r * DK + cc * 4], g + (size_t)(ok ? r : 0) * DK + cc * 4, ok ? 16 : 0);
    }
  }
  cp_async_commit();
  if (p.wave > 0) {  // the inputs of the CTA one wave later, into L2 (as in the output pass)
    const size_t L = (size_t)blockIdx.y * gridDim.x + blockIdx.x + (size_t)p.wave;
    if (L < (size_t)gridDim.x * gridDim.y) {
      const int cn = (int)(L % gridDim.x), bhn = (int)(L / gridDim.x);
      const int rn = min(C, T - cn * C);
      const size_t row = (size_t)bhn * T + (size_t)cn * C;
      prefetch_l2_lines(p.x + row * DK, (size_t)rn * DK * 2, tid);
      prefetch_l2_lines(p.y + row * DV, (size_t)rn * DV * 2, tid);
      if (p.gz) prefetch_l2_lines(p.gz + row * DK, (size_t)rn * DK * 2, tid);
      else prefetch_l2_lines(p.g + row * DK, (size_t)rn * DK * 4, tid);
    }
  }
  cp_async_wait<0>();
  __syncthreads();
  if (p.gz) {  // log-gates from the logits; rows past the end: g = 0
    for (int x = tid; x < C * DK; x += NT) {
      const int r = x / DK, c = x % DK;
      sm.g[r * DK + c] = r < rows ? gate_from_logit(__bfloat162float(sm.ks[r * QKP + c]), p.gs) : 0.f;
    }
    __syncthreads();
  }
  // prep: thread -> (sub-block K, key dims i2, i2+1); rows past the end have
  // g = 0 (no decay) and x = 0.  fac[r]: the in-sub-block part of the row's
  // factor (key side: gates after the row; query side: gates up to it)
  const int K = tid >> 6, i2 = (tid & 63) * 2, r0 = K * SB;
  float2 fac[SB];
  {
    float2 run = make_float2(1.f, 1.f);
#pragma unroll
    for (int rr = 0; rr < SB; ++rr) {
      const int r = QSIDE ? rr : SB - 1 - rr;
      if (!QSIDE) fac[r] = run;
      const float2 gg = *reinterpret_cast<const float2*>(&sm.g[(r0 + r) * DK + i2]);
      run.x *= __expf(gg.x);
      run.y *= __expf(gg.y);
      if (QSIDE) fac[r] = run;
    }
    *reinterpret_cast<float2*>(&sm.dec[K][i2]) = run;
  }
  __syncthreads();
  {
    // f: the other sub-blocks' part (key side: later ones; query side: earlier)
    float2 f = make_float2(1.f, 1.f), e = make_float2(1.f, 1.f);
#pragma unroll
    for (int J = 0; J < NSB; ++J) {
      const float2 d = *reinterpret_cast<const float2*>(&sm.dec[J][i2]);
      if (QSIDE ? (J < K) : (J > K)) {
        f.x *= d.x;
        f.y *= d.y;
      }
      e.x *= d.x;
      e.y *= d.y;
    }
    if (K == 0)
      *reinterpret_cast<float2*>(&p.decay[((size_t)bh * nchunks + c) * DK + i2]) = e;
#pragma unroll
    for (int r = 0; r < SB; ++r) {
      const float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.k[(r0 + r) * QKP + i2]));
      *reinterpret_cast<uint32_t*>(&sm.ks[(r0 + r) * QKP + i2]) =
          pack_bf16(kv.x * fac[r].x * f.x, kv.y * fac[r].y * f.y);
    }
  }
  __syncthreads();
  // increment rows 16w .. 16w+15, all 128 value columns
  float acc[DV / 8][4];
#pragma unroll
  for (int nt = 0; nt < DV / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
#pragma unroll
  for (int kk = 0; kk < C / 16; ++kk) {
    uint32_t a[4];
    ldsm_x4_t(smem_u32(&sm.ks[(16 * kk + (lane & 7) + ((lane >> 4) << 3)) * QKP + 16 * warp +
                              ((lane >> 3) & 1) * 8]),
              a[0], a[1], a[2], a[3]);
#pragma unroll
    for (int ntp = 0; ntp < DV / 16; ++ntp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(&sm.v[(16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8) * VP + ntp * 16 + (lane >> 4) * 8]),
                b0, b1, b2, b3);
      mma_bf16(acc[2 * ntp], a, b0, b1);
      mma_bf16(acc[2 * ntp + 1], a, b2, b3);
    }
  }
  bf16* dst = p.delta + ((size_t)bh * nchunks + c) * DK * DV;
#pragma unroll
  for (int nt = 0; nt < DV / 8; ++nt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int i = 16 * warp + gr + 8 * hh, j = nt * 8 + gc;
      *reinterpret_cast<uint32_t*>(&dst[(size_t)i * DV + j]) = pack_bf16(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
    }
}

// Elementwise scan over the chunks; thread -> (batch-head, key dim i, 8 value
// columns).  Forward: out[c] = S before chunk c, S <- E_c S + dS_c, fin = S
// after the last chunk.  Reverse: out[c] = G entering chunk c from the later
// chunks, G <- E_c G + dG_c, gsp[c][i] = <G, S_prev[c]> over the value
// columns with the updated G (the gate gradient at the chunk's first row),
// fin = G before token 0.
struct ScanArgs {
  const bf16* delta;   // [BH][nchunks][DK][DV]
  const float* decay;  // [BH][nchunks][DK]
  const float* init;   // nullable [BH][DK][DV]
  bf16* out;           // [BH][nchunks][DK][DV]
  float* fin;          // nullable [BH][DK][DV]
  const bf16* sprev;   // reverse only: the forward states [BH][nchunks][DK][DV]
  float* gsp;          // reverse only: [BH][nchunks][DK]
  int BH, nchunks;
};
constexpr int SCAN_NT = 128;
constexpr int SCAN_U = 4;  // chunks whose loads are in flight together

template <bool REV>
__global__ void __launch_bounds__(SCAN_NT) gla_scan_kernel(ScanArgs p) {
  const size_t id = (size_t)blockIdx.x * SCAN_NT + threadIdx.x;
  const size_t per_bh = (size_t)DK * (DV / 8);
  // whole warps only: the thread count is a multiple of DK * DV / 8
  if (id >= (size_t)p.BH * per_bh) return;
  const int nchunks = p.nchunks;
  const size_t bh = id / per_bh;
  const int i = (int)((id / (DV / 8)) % DK), j8 = (int)(id % (DV / 8)) * 8;
  float s[8];
  if (p.init) {
    const float4* hp = reinterpret_cast<const float4*>(p.init + (bh * DK + i) * DV + j8);
    const float4 a = hp[0], b = hp[1];
    s[0] = a.x; s[1] = a.y; s[2] = a.z; s[3] = a.w; s[4] = b.x; s[5] = b.y; s[6] = b.z; s[7] = b.w;
  } else {
#pragma unroll
    for (int x = 0; x < 8; ++x) s[x] = 0.f;
  }
  const size_t stride = (size_t)DK * DV;  // one chunk's matrix
  const size_t base = bh * nchunks * stride + (size_t)i * DV + j8;
  const bf16* dl = p.delta + base;
  bf16* out = p.out + base;
  const float* ec = p.decay + bh * nchunks * DK + i;
  for (int it0 = 0; it0 < nchunks; it0 += SCAN_U) {
    uint4 d[SCAN_U], sv[SCAN_U];
    float e[SCAN_U];
#pragma unroll
    for (int u = 0; u < SCAN_U; ++u) {
      const int it = it0 + u;
      const int c = REV ? nchunks - 1 - it : it;
      const bool ok = it < nchunks;
      d[u] = ok ? __ldcs(reinterpret_cast<const uint4*>(dl + c * stride)) : make_uint4(0, 0, 0, 0);
      e[u] = ok ? __ldcs(ec + (size_t)c * DK) : 1.f;
      if (REV) sv[u] = ok ? __ldcs(reinterpret_cast<const uint4*>(p.sprev + base + c * stride)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < SCAN_U; ++u) {
      const int it = it0 + u;
      if (it >= nchunks) break;
      const int c = REV ? nchunks - 1 - it : it;
      *reinterpret_cast<uint4*>(out + c * stride) =
          make_uint4(pack_bf16(s[0], s[1]), pack_bf16(s[2], s[3]), pack_bf16(s[4], s[5]), pack_bf16(s[6], s[7]));
      const uint32_t dw[4] = {d[u].x, d[u].y, d[u].z, d[u].w};
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float2 f = unpack_bf16(dw[x]);
        s[2 * x] = fmaf(e[u], s[2 * x], f.x);
        s[2 * x + 1] = fmaf(e[u], s[2 * x + 1], f.y);
      }
      if (REV) {
        const uint32_t pw[4] = {sv[u].x, sv[u].y, sv[u].z, sv[u].w};
        float dot = 0.f;
#pragma unroll
        for (int x = 0; x < 4; ++x) {
          const float2 f = unpack_bf16(pw[x]);
          dot = fmaf(s[2 * x], f.x, fmaf(s[2 * x + 1], f.y, dot));
        }
        // the 16 threads of key dim i are 16 consecutive lanes
#pragma unroll
        for (int m = 8; m >= 1; m >>= 1) dot += __shfl_xor_sync(0xffffffffu, dot, m);
        if ((threadIdx.x & 15) == 0) p.gsp[(bh * nchunks + c) * DK + i] = dot;
      }
    }
  }
  if (p.fin) {
    float4* hp = reinterpret_cast<float4*>(p.fin + (bh * DK + i) * DV + j8);
    hp[0] = make_float4(s[0], s[1], s[2], s[3]);
    hp[1] = make_float4(s[4], s[5], s[6], s[7]);
  }
}

template <bool QSIDE>
cudaError_t run_delta(const DeltaArgs& a, int nchunks, int BH, const char* name, cudaStream_t s) {
  const size_t bytes = sizeof(DeltaSmem);
  cudaError_t e = cudaFuncSetAttribute(gla_delta_kernel<QSIDE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes);
  if (e != cudaSuccess) return e;
  DeltaArgs aa = a;
  aa.wave = resident_ctas(gla_delta_kernel<QSIDE>, NT, bytes);
  {
    ScopedTiming tm(name, s);
    gla_delta_kernel<QSIDE><<<dim3(nchunks, BH), NT, bytes, s>>>(aa);
  }
  return cudaGetLastError();
}

template <bool REV>
cudaError_t run_scan(const ScanArgs& a, const char* name, cudaStream_t s) {
  const size_t threads = (size_t)a.BH * DK * (DV / 8);
  {
    ScopedTiming tm(name, s);
    gla_scan_kernel<REV><<<(unsigned)((threads + SCAN_NT - 1) / SCAN_NT), SCAN_NT, 0, s>>>(a);
  }
  return cudaGetLastError();
}

// ===========================================================================
// Pass 2: chunk outputs, all chunks in parallel
// ===========================================================================
struct OutSmem {
  bf16 q[C * QKP];     // raw q, then the score operand Qf in place
  bf16 k[C * QKP];     // raw k, then Kf in place
  bf16 qi[C * QKP];    // q e^{b}
  bf16 v[C * VP];
  bf16 sp[DK * VP];    // state before the chunk
  float dec[NSB][DK];
  float fac[NPAIR][DK];
  float lsum[NT / 32];  // per-warp sums of the fused loss
};
static_assert(sizeof(OutSmem) <= 115712, "two output CTAs must fit one SM");

// A[t][s] with one exponential per key dim (strong-decay diagonal blocks);
// q, k, g: global rows of the chunk.
template <class Gates>
__device__ __noinline__ float diag_score_global(const bf16* q, const bf16* k, Gates g, int rt, int rs) {
  float a = 0.f;
  for (int i = 0; i < DK; ++i) {
    float lg = 0.f;
    for (int u = rs + 1; u <= rt; ++u) lg += g.at((size_t)u * DK + i);
    a += __bfloat162float(q[(size_t)rt * DK + i]) * __bfloat162float(k[(size_t)rs * DK + i]) * __expf(lg);
  }
  return a;
}

// LOSS: the stage-1 loss epilogue (p.target set); LOGITS: the gates arrive as
// logits (p.gz set).  Separate instantiations, so that the plain forward keeps
// its registers and schedule.
template <bool LOSS, bool LOGITS>
__global__ void __launch_bounds__(NT, 2) gla_out_kernel(GlaFwdParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  OutSmem& sm = *reinterpret_cast<OutSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, gc = (lane & 3) * 2;
  // batch-heads in reverse: the window forward wrote the last ones' outputs
  // last, so they are still in L2 when this pass starts
  const int c = blockIdx.x, bh = gridDim.y - 1 - blockIdx.y;
  const int T = p.T;
  const int c0 = c * C;
  const int rows = min(C, T - c0);
  const int nchunks = gridDim.x;
  const bf16* q = (const bf16*)p.q + ((size_t)bh * T + c0) * DK;
  const bf16* k = (const bf16*)p.k + ((size_t)bh * T + c0) * DK;
  const bf16* v = (const bf16*)p.v + ((size_t)bh * T + c0) * DV;
  const float* g = LOGITS ? nullptr : p.g + ((size_t)bh * T + c0) * DK;
  const bf16* gz = LOGITS ? (const bf16*)p.gz + ((size_t)bh * T + c0) * DK : nullptr;
  const bf16* sp = (const bf16*)p.states16 + ((size_t)bh * nchunks + c) * DK * DV;

  for (int x = tid; x < C * DK / 8; x += NT) {
    const int r = x / (DK / 8), cc = x % (DK / 8);
    const bool ok = r < rows;
    const size_t off = (size_t)(ok ? r : 0) * DK + cc * 8;
    cp_async16(&sm.q[r * QKP + cc * 8], q + off, ok ? 16 : 0);
    cp_async16(&sm.k[r * QKP + cc * 8], k + off, ok ? 16 : 0);
  }
  for (int x = tid; x < C * DV / 8; x += NT) {
    const int r = x / (DV / 8), cc = x % (DV / 8);
    const bool ok = r < rows;
    cp_async16(&sm.v[r * VP + cc * 8], v + (size_t)(ok ? r : 0) * DV + cc * 8, ok ? 16 : 0);
  }
  for (int x = tid; x < DK * DV / 8; x += NT) {
    const int r = x / (DV / 8), cc = x % (DV / 8);
    cp_async16(&sm.sp[r * VP + cc * 8], sp + (size_t)r * DV + cc * 8, 16);
  }
  cp_async_commit();
  if (p.wave > 0) {
    // CTAs start in linear-index order, so the one `wave` places on starts
    // about when this one ends: its inputs go to L2 now, and its loads find
    // them there instead of waiting on HBM
    const size_t L = (size_t)blockIdx.y * gridDim.x + blockIdx.x + (size_t)p.wave;
    if (L < (size_t)gridDim.x * gridDim.y) {
      const int cn = (int)(L % gridDim.x), bhn = (int)(gridDim.y - 1 - L / gridDim.x);
      const int rn = min(C, T - cn * C);
      const size_t row = (size_t)bhn * T + (size_t)cn * C;
      prefetch_l2_lines((const bf16*)p.q + row * DK, (size_t)rn * DK * 2, tid);
      prefetch_l2_lines((const bf16*)p.k + row * DK, (size_t)rn * DK * 2, tid);
      prefetch_l2_lines((const bf16*)p.v + row * DV, (size_t)rn * DV * 2, tid);
      if (LOGITS) prefetch_l2_lines((const bf16*)p.gz + row * DK, (size_t)rn * DK * 2, tid);
      else prefetch_l2_lines(p.g + row * DK, (size_t)rn * DK * 4, tid);
      if (p.add16) prefetch_l2_lines((const bf16*)p.add16 + row * DV, (size_t)rn * DV * 2, tid);
      prefetch_l2_lines((const bf16*)p.states16 + ((size_t)bhn * nchunks + cn) * DK * DV, (size_t)DK * DV * 2, tid);
    }
  }

  // ---- prep 1 (gates straight from global): thread -> (sub-block K, dims i2, i2+1)
  const int K = tid >> 6, i2 = (tid & 63) * 2, r0 = K * SB;
  float2 qfac[SB], kfac[SB];
  {
    float2 e[SB];
#pragma unroll
    for (int r = 0; r < SB; ++r) {
      float2 gg = make_float2(0.f, 0.f);
      if (r0 + r < rows) {
        if constexpr (LOGITS) {
          const float2 zz = unpack_bf16(*reinterpret_cast<const uint32_t*>(&gz[(size_t)(r0 + r) * DK + i2]));
          gg = make_float2(gate_from_logit(zz.x, p.gs), gate_from_logit(zz.y, p.gs));
        } else {
          gg = *reinterpret_cast<const float2*>(&g[(size_t)(r0 + r) * DK + i2]);
        }
      }
      e[r] = make_float2(__expf(gg.x), __expf(gg.y));
    }
    float2 run = make_float2(1.f, 1.f);
#pragma unroll
    for (int r = SB - 1; r >= 0; --r) {
      kfac[r] = run;
      run.x *= e[r].x;
      run.y *= e[r].y;
    }
    run = make_float2(1.f, 1.f);
#pragma unroll
    for (int r = 0; r < SB; ++r) {
      run.x *= e[r].x;
      run.y *= e[r].y;
      qfac[r] = run;
    }
    *reinterpret_cast<float2*>(&sm.dec[K][i2]) = run;
  }
  cp_async_wait<0>();
  __syncthreads();
  // ---- prep 2: operands and score factors ----------------------------------
  int flags;
  {
    float2 D[NSB];
#pragma unroll
    for (int J = 0; J < NSB; ++J) D[J] = *reinterpret_cast<const float2*>(&sm.dec[J][i2]);
    bool wild_bad = false, any_wild = false;
    float rq[2], rk[2], eqk[2];
#pragma unroll
    for (int h2 = 0; h2 < 2; ++h2) {
      const float d0 = h2 ? D[0].y : D[0].x, d1 = h2 ? D[1].y : D[1].x;
      const float d2 = h2 ? D[2].y : D[2].x, d3 = h2 ? D[3].y : D[3].x;
      const bool tame = (d0 * d1 >= kMinBlockDecay) && (d2 * d3 >= kMinBlockDecay);
      any_wild |= !tame;
      if (!tame)
        wild_bad |= !(d0 >= kMinBlockDecay && d1 >= kMinBlockDecay && d2 >= kMinBlockDecay &&
                      d3 >= kMinBlockDecay);
      const float dk[NSB] = {d0, d1, d2, d3};
      float rqK = 1.f, rkK = 1.f;
      if (tame) {
        rqK = K == 0 ? 1.f / (d0 * d1) : K == 1 ? 1.f / d1 : K == 2 ? 1.f : d2;
        rkK = K == 0 ? d1 : K == 1 ? 1.f : K == 2 ? 1.f / d2 : 1.f / (d2 * d3);
      }
      float eq = 1.f;
#pragma unroll
      for (int J = 0; J < NSB; ++J)
        if (J < K) eq *= dk[J];
      rq[h2] = rqK;
      rk[h2] = rkK;
      eqk[h2] = eq;
#pragma unroll
      for (int I = 0; I < NSB; ++I)
#pragma unroll
        for (int J = 0; J <= I; ++J) {
          if (pair_index(I, J) % NSB != K) continue;
          float f = 1.f;
          if (!tame) {
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
    }
#pragma unroll
    for (int r = 0; r < SB; ++r) {
      const int o = (r0 + r) * QKP + i2;
      const float2 qv = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.q[o]));
      const float2 kv = unpack_bf16(*reinterpret_cast<const uint32_t*>(&sm.k[o]));
      const float qx = qv.x * qfac[r].x, qy = qv.y * qfac[r].y;
      const float kx = kv.x * kfac[r].x, ky = kv.y * kfac[r].y;
      *reinterpret_cast<uint32_t*>(&sm.q[o]) = pack_bf16(qx * rq[0], qy * rq[1]);
      *reinterpret_cast<uint32_t*>(&sm.qi[o]) = pack_bf16(qx * eqk[0], qy * eqk[1]);
      *reinterpret_cast<uint32_t*>(&sm.k[o]) = pack_bf16(kx * rk[0], ky * rk[1]);
    }
    const int w = __syncthreads_or(any_wild);
    const int b = __syncthreads_or(wild_bad);
    flags = (w ? 1 : 0) | (b ? 2 : 0);
  }
  const bool scaled = flags & 1, slow = flags & 2;

  // ---- outputs: warp -> (query sub-block I, value half nh) --------------------
  const int I = warp >> 1, nh = warp & 1;
  float2 addv[8][2];
  if (p.add16) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = 16 * I + gr + 8 * hh;
        addv[nt][hh] = t < rows ? unpack_bf16(*reinterpret_cast<const uint32_t*>(
                                      &((const bf16*)p.add16)[((size_t)bh * T + c0 + t) * DV + 64 * nh + nt * 8 + gc]))
                                : make_float2(0.f, 0.f);
      }
  }
  float o[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
  // inter: (q e^{b}) S_prev
#pragma unroll 2
  for (int kk = 0; kk < DK / 16; ++kk) {
    uint32_t a[4];
    ldsm_x4(smem_u32(&sm.qi[(16 * I + (lane & 15)) * QKP + kk * 16 + (lane >> 4) * 8]), a[0], a[1], a[2],
            a[3]);
#pragma unroll
    for (int ntp = 0; ntp < 4; ++ntp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(&sm.sp[(16 * kk + (lane & 7) + ((lane >> 3) & 1) * 8) * VP + 64 * nh + ntp * 16 +
                                (lane >> 4) * 8]),
                b0, b1, b2, b3);
      mma_bf16(o[2 * ntp], a, b0, b1);
      mma_bf16(o[2 * ntp + 1], a, b2, b3);
    }
  }
  // intra: one score block at a time (J <= I), P V right away
  for (int J = 0; J <= I; ++J) {
    float sc[2][4], sc2[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] = sc2[nt][e] = 0.f;
    const float* fac = sm.fac[pair_index(I, J)];
#pragma unroll
    for (int kk = 0; kk < DK / 16; ++kk) {
      uint32_t a[4];
      ldsm_x4(smem_u32(&sm.q[(16 * I + (lane & 15)) * QKP + kk * 16 + (lane >> 4) * 8]), a[0], a[1], a[2],
              a[3]);
      if (scaled) {
        const float2 f0 = *reinterpret_cast<const float2*>(&fac[kk * 16 + gc]);
        const float2 f1 = *reinterpret_cast<const float2*>(&fac[kk * 16 + 8 + gc]);
        a[0] = scale_bf16x2(a[0], f0.x, f0.y);
        a[1] = scale_bf16x2(a[1], f0.x, f0.y);
        a[2] = scale_bf16x2(a[2], f1.x, f1.y);
        a[3] = scale_bf16x2(a[3], f1.x, f1.y);
      }
      uint32_t b0, b1, b2, b3;
      ldsm_x4(smem_u32(&sm.k[(16 * J + (lane & 7) + ((lane >> 4) << 3)) * QKP + kk * 16 +
                             ((lane >> 3) & 1) * 8]),
              b0, b1, b2, b3);
      float (*dst)[4] = (kk & 1) ? sc2 : sc;
      mma_bf16(dst[0], a, b0, b1);
      mma_bf16(dst[1], a, b2, b3);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int t = gr + (e >> 1) * 8, sk = nt * 8 + gc + (e & 1);
        float x = sc[nt][e] + sc2[nt][e];
        if (J == I) {
          if (sk > t) x = 0.f;
          else if (slow) {
            if (16 * I + t >= rows) x = 0.f;
            else if constexpr (LOGITS) x = diag_score_global(q, k, LogitGates{gz, p.gs}, 16 * I + t, 16 * I + sk);
            else x = diag_score_global(q, k, LogGates{g}, 16 * I + t, 16 * I + sk);
          }
        }
        sc[nt][e] = x;
      }
    const uint32_t pa[4] = {pack_bf16(sc[0][0], sc[0][1]), pack_bf16(sc[0][2], sc[0][3]),
                            pack_bf16(sc[1][0], sc[1][1]), pack_bf16(sc[1][2], sc[1][3])};
#pragma unroll
    for (int ntp = 0; ntp < 4; ++ntp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(&sm.v[(16 * J + (lane & 7) + ((lane >> 3) & 1) * 8) * VP + 64 * nh + ntp * 16 +
                               (lane >> 4) * 8]),
                b0, b1, b2, b3);
      mma_bf16(o[2 * ntp], pa, b0, b1);
      mma_bf16(o[2 * ntp + 1], pa, b2, b3);
    }
  }
  // epilogue: o = o_gla + alpha * add
  if (p.add16) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        o[nt][2 * hh] += p.alpha * addv[nt][hh].x;
        o[nt][2 * hh + 1] += p.alpha * addv[nt][hh].y;
      }
  }
  float lsq = 0.f;
  uint32_t tg[8][2];
  if constexpr (LOSS) {  // all target loads in flight before the first store
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = 16 * I + gr + 8 * hh;
        const size_t off = ((size_t)bh * T + c0 + t) * DV + 64 * nh + nt * 8 + gc;
        tg[nt][hh] = t < rows ? __ldg(reinterpret_cast<const unsigned int*>(&((const bf16*)p.target)[off])) : 0u;
      }
  }
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      const int t = 16 * I + gr + 8 * hh;
      if (t >= rows) continue;
      const size_t off = ((size_t)bh * T + c0 + t) * DV + 64 * nh + nt * 8 + gc;
      const float x0 = o[nt][2 * hh], x1 = o[nt][2 * hh + 1];
      if constexpr (LOSS) {  // stage-1 loss on the fp32 output, before its rounding
        const float2 tv = unpack_bf16(tg[nt][hh]);
        const float e0 = x0 - tv.x, e1 = x1 - tv.y;
        lsq = fmaf(e0, e0, fmaf(e1, e1, lsq));
        if (p.dO_loss)
          *reinterpret_cast<uint32_t*>(&((bf16*)p.dO_loss)[off]) = pack_bf16(p.loss_scale * e0, p.loss_scale * e1);
      }
      *reinterpret_cast<uint32_t*>(&((bf16*)p.o)[off]) = pack_bf16(x0, x1);
    }
  if constexpr (LOSS) {  // fixed-order reduction: lanes, then warps
#pragma unroll
    for (int m = 16; m >= 1; m >>= 1) lsq += __shfl_xor_sync(0xffffffffu, lsq, m);
    if (lane == 0) sm.lsum[warp] = lsq;
    __syncthreads();
    if (tid == 0) {
      float tot = 0.f;
#pragma unroll
      for (int w = 0; w < NT / 32; ++w) tot += sm.lsum[w];
      p.loss_part[(size_t)bh * nchunks + c] = tot;
    }
  }
}

}  // namespace

bool gla_chunk_mma_supported(int dk, int dv, bool bf16) { return bf16 && dk == DK && dv == DV; }

bool gla_states_scan_wanted(int T) { return (T + C - 1) / C >= kScanMinChunks; }

cudaError_t launch_gla_states(const GlaFwdParams& p, cudaStream_t s) {
  if (p.B * p.H == 0) return cudaSuccess;
  const int nchunks = (p.T + C - 1) / C;
  // gate logits take the two-level path for every non-empty sequence (the
  // sequential pass reads log-gates); an empty one only passes h0 to hT
  if (p.gz && nchunks > 0 && !(p.delta16 && p.decay)) return cudaErrorInvalidValue;
  if (p.delta16 && p.decay && nchunks > 0 && (nchunks >= kScanMinChunks || p.gz)) {
    DeltaArgs da{(const bf16*)p.k, (const bf16*)p.v, p.g, (const bf16*)p.gz, p.gs, (bf16*)p.delta16,
                 p.decay, p.T};
    cudaError_t e = run_delta<false>(da, nchunks, p.B * p.H, "gla_delta_mma", s);
    if (e != cudaSuccess) return e;
    ScanArgs sa{(const bf16*)p.delta16, p.decay, p.h0, (bf16*)p.states16, p.hT, nullptr, nullptr,
                p.B * p.H, nchunks};
    return run_scan<false>(sa, "gla_scan", s);
  }
  const size_t bytes = sizeof(StateSmem);
  cudaError_t e = cudaFuncSetAttribute(gla_states_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes);
  if (e != cudaSuccess) return e;
  {
    ScopedTiming tm("gla_states_mma", s);
    gla_states_kernel<<<dim3(DV / DVS, p.B * p.H), NT, bytes, s>>>(p);
  }
  return cudaGetLastError();
}

// ---------------------------------------------------------------------------
// Gates given as logits (Gamma = sigma(z)): one pass maps them to fp32
// log-gates g = scale * log sigma(z) for the log-gate kernels, and one maps
// those kernels' dL/dg to dL/dz = dL/dg * scale * sigma(-z) (the same
// gate_from_logit / dlogit as the kernels that map them on the fly).
// Eight elements a thread, one thread per eight elements (grid-stride past
// 2^31 - 1 blocks), so that every load of the stream is in flight at once.
__global__ void __launch_bounds__(256) gate_logits_to_log_kernel(const bf16* __restrict__ z, float* __restrict__ g,
                                                                 size_t n8, float gs) {
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n8; i += (size_t)gridDim.x * 256) {
    const uint4 zz = __ldcs(reinterpret_cast<const uint4*>(z) + i);
    const uint32_t zw[4] = {zz.x, zz.y, zz.z, zz.w};
    float o[8];
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float2 f = unpack_bf16(zw[x]);
      o[2 * x] = gate_from_logit(f.x, gs);
      o[2 * x + 1] = gate_from_logit(f.y, gs);
    }
    float4* dst = reinterpret_cast<float4*>(g) + 2 * i;
    dst[0] = make_float4(o[0], o[1], o[2], o[3]);
    dst[1] = make_float4(o[4], o[5], o[6], o[7]);
  }
}

__global__ void __launch_bounds__(256) gate_dlogit_kernel(float* __restrict__ dg, const bf16* __restrict__ z,
                                                          size_t n8, float gs) {
  for (size_t i = (size_t)blockIdx.x * 256 + threadIdx.x; i < n8; i += (size_t)gridDim.x * 256) {
    const uint4 zz = __ldcs(reinterpret_cast<const uint4*>(z) + i);
    const uint32_t zw[4] = {zz.x, zz.y, zz.z, zz.w};
    float4* d = reinterpret_cast<float4*>(dg) + 2 * i;
    const float4 a = d[0], b = d[1];
    float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const float2 f = unpack_bf16(zw[x]);
      v[2 * x] = dlogit(v[2 * x], f.x, gs);
      v[2 * x + 1] = dlogit(v[2 * x + 1], f.y, gs);
    }
    d[0] = make_float4(v[0], v[1], v[2], v[3]);
    d[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

static unsigned gate_pass_grid(size_t n8) {
  const size_t want = (n8 + 255) / 256;
  return (unsigned)(want < 0x7fffffffu ? (want > 0 ? want : 1) : 0x7fffffffu);
}

cudaError_t launch_gate_logits_to_log(const void* z, float* g, size_t n, float gs, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (n % 8) return cudaErrorInvalidValue;
  {
    ScopedTiming tm("gate_logits_to_log", s);
    gate_logits_to_log_kernel<<<gate_pass_grid(n / 8), 256, 0, s>>>((const bf16*)z, g, n / 8, gs);
  }
  return cudaGetLastError();
}

cudaError_t launch_gate_dlogit(float* dg, const void* z, size_t n, float gs, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  if (n % 8) return cudaErrorInvalidValue;
  {
    ScopedTiming tm("gate_dlogit", s);
    gate_dlogit_kernel<<<gate_pass_grid(n / 8), 256, 0, s>>>(dg, (const bf16*)z, n / 8, gs);
  }
  return cudaGetLastError();
}

size_t gla_out_loss_parts(int B, int H, int T) { return (size_t)B * H * ((T + C - 1) / C); }

cudaError_t launch_gla_bwd_scan(const GlaBwdScanParams& p, cudaStream_t s) {
  const int nchunks = (p.T + C - 1) / C;
  const int BH = p.B * p.H;
  if (BH == 0) return cudaSuccess;
  if (nchunks > 0) {
    DeltaArgs da{(const bf16*)p.q, (const bf16*)p.dO, p.g, (const bf16*)p.gz, p.gs, (bf16*)p.delta16,
                 p.decay, p.T};
    cudaError_t e = run_delta<true>(da, nchunks, BH, "gla_bwd_delta", s);
    if (e != cudaSuccess) return e;
  }
  ScanArgs sa{(const bf16*)p.delta16, p.decay, p.dhT, (bf16*)p.gin16, p.dh0, (const bf16*)p.states16,
              p.gsp, BH, nchunks};
  return run_scan<true>(sa, "gla_bwd_scan", s);
}

cudaError_t launch_gla_out(const GlaFwdParams& p, cudaStream_t s) {
  const int nchunks = (p.T + C - 1) / C;
  if (p.B * p.H == 0 || nchunks == 0) return cudaSuccess;
  const size_t bytes = sizeof(OutSmem);
  const auto kern = p.target ? (p.gz ? gla_out_kernel<true, true> : gla_out_kernel<true, false>)
                             : (p.gz ? gla_out_kernel<false, true> : gla_out_kernel<false, false>);
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  GlaFwdParams pp = p;
  pp.wave = resident_ctas(kern, NT, bytes);
  {
    ScopedTiming tm(p.target ? "gla_out_mma_loss" : "gla_out_mma", s);
    kern<<<dim3(nchunks, p.B * p.H), NT, bytes, s>>>(pp);
  }
  return cudaGetLastError();
}

}  // namespace lz
