// Chunked gated linear attention backward on the tensor cores (bf16 I/O,
// fp32 accumulation, dk = dv = 128).
//
// Gradient of S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T, o_t = q_t^T S_t (the
// attention-output regression of the first training stage, Lizard technical
// summary section 2b, needs it).  Per 64-token chunk, with b_t the running
// log-gate inside the chunk, b_l its last value, G the state gradient entering
// the chunk from the later chunks (dL/dhT after the last one), S_prev the
// state before the chunk, B[t][s] = dO_t . v_s and A[t][s] = sum_i q_t k_s
// e^{b_t-b_s} (both for s <= t):
//   dq_t = e^{b_t} (S_prev dO_t) + sum_{s<=t} B[t][s] k_s e^{b_t - b_s}
//   dk_t = e^{b_l - b_t} (G v_t) + sum_{u>=t} B[u][t] q_u e^{b_u - b_t}
//   dv_t = (k_t e^{b_l - b_t})^T G + sum_{u>=t} A[u][t] dO_u
//   G_new = diag(e^{b_l}) G + sum_u (q_u e^{b_u})^T dO_u  (G of the previous chunk)
//   dg   : the gate's direct gradient is dg_t = e^{g_t} <dS_t, S_{t-1}> per key
//          dim; at the chunk's first row that is <G_new, S_prev>, and inside
//          the chunk dg_t = dg_first - sum_{u<t} (q_u dq_u - k_u dk_u), so
//          rounding errors add up over one chunk, not the whole sequence.
//
// The running sum cancels: every intra-chunk pair (u, s) enters q_u dq_u and
// k_s dk_s with the same value, and only the pairs that straddle t survive.
// Under fast forgetting the surviving part is small, so the two copies of a
// pair must round identically.  Hence (a) the diagonal pairs (s = u, whose
// copies cancel exactly) stay out of the MMAs and are added to dq and dk in
// fp32 only, and (b) the products entering the sum are taken from the bf16
// MMA operands themselves, Qf_u * acc_q,u and Kf_s * acc_k,s, in which a pair
// is the same product Qf_u B[u][s] Kf_s on both sides, instead of q * dq and
// k * dk, whose output scales round differently on the two sides.
//
// Two levels: launch_gla_bwd_scan (gla_chunk_mma.cu) forms every chunk's
// increment of G in parallel and scans them in reverse, giving G and
// <G_new, S_prev> for every chunk; the kernel here then takes all chunks at
// once.  Work split: a cluster of two CTAs per (chunk, batch-head); CTA r owns
// key dims [64r, 64r+64).  dq, dk and dg are complete inside the CTA; dv is a
// sum over key dims, so each CTA sends the partial dv of the peer's 64 value
// columns through distributed shared memory and adds the peer's share to its
// own before storing.  Staging tiles reuse buffers that are dead by then, so
// that two CTAs fit one SM.
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
#include <type_traits>

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
constexpr int RP = DKH;        // dg staging row (64 floats, see rsw)
constexpr int NPAIR = NSB * (NSB + 1) / 2;
__device__ constexpr float kMinBlockDecay = 8.75651076e-27f;  // e^-60

// [rows][128] bf16 tile with its 16-byte chunks XOR-swizzled by row
__device__ __forceinline__ int swz(int row, int col) {
  return row * 128 + ((((col >> 3) ^ row) & 15) << 3) + (col & 7);
}
// [rows][64] bf16 tile, same idea (8 chunks per row)
__device__ __forceinline__ int swz64(int row, int col) {
  return row * 64 + ((((col >> 3) ^ row) & 7) << 3) + (col & 7);
}
// [rows][64] fp32 staging tile: 8-float groups XOR-swizzled by row % 4, so
// that the float2 accesses of an MMA fragment (rows g, columns 2c) and the
// column scans (one row, consecutive columns) are both free of bank conflicts
__device__ __forceinline__ int rsw(int row, int col) {
  return row * RP + (col ^ ((row & 3) << 3));
}

__device__ __forceinline__ int pair_index(int I, int J) { return I * (I + 1) / 2 + J; }

// exp(sum_{x = s+1 .. t} g_x,i) for chunk rows s <= t (g, or the logits gz:
// global, the chunk's first row, already offset to this CTA's key dims).
// Used only by the strong-decay fallback of the diagonal blocks; it returns a
// scalar so that no register array of the caller has its address taken.
template <class Gates>
__device__ __noinline__ float gate_ratio(Gates g, int rows, int t, int s, int i) {
  float lg = 0.f;
  for (int x = s + 1; x <= t && x < rows; ++x) lg += g.at((size_t)x * DK + i);
  return __expf(lg);
}

struct ChunkSmem {
  bf16 v[C * VP];       // then the k-side dg products (fp32, rsw layout)
  bf16 dO[C * VP];
  bf16 sp[DKH * DV];    // S_prev (swizzled); then the q-side dg products (fp32, rsw)
  bf16 g16[DKH * DV];   // G entering the chunk (swizzled)
  bf16 qf[C * KP];      // qf and kf: then the peer's dv share (fp32, rsw layout)
  bf16 kf[C * KP];
  bf16 eqf[C * KP];
  bf16 ekf[C * KP];
  float dec[NSB][DKH];
  float fac[NPAIR][DKH];
  float ci[NSB][DKH];
  float ck[NSB][DKH];
  float ksr[NSB][DKH];  // (k e^{b_l - b}) / kf per (sub-block, key dim)
  float tot[NSB][DKH];
  float bdg[2][C];      // fp32 dO_t . v_t (the diagonal pairs), per role
};
static_assert(sizeof(ChunkSmem) + 1024 <= 232448 / 2, "two chunk CTAs must fit one SM");
static_assert(sizeof(float) * C * RP <= sizeof(bf16) * C * VP, "dg staging must fit the v tile");
static_assert(sizeof(float) * C * RP <= sizeof(bf16) * DKH * DV, "dg staging must fit the state tile");
static_assert(sizeof(float) * C * RP <= 2 * sizeof(bf16) * C * KP, "dv share must fit qf + kf");

// Diagonal-block intra term of a strong-decay chunk at (row t, key dim il),
// without the pair s = u = t (added separately, in fp32, for every chunk):
// role 0 (dq): sum_{s in block, s < t} (dO_t . v_s) k_s,il exp(b_t - b_s)
// role 1 (dk): sum_{u in block, u > t} (dO_u . v_t) q_u,il exp(b_u - b_t)
// (dO, v: shared tiles; kq, g: global, the chunk's first row, offset to this
// CTA's key dims)
template <class Gates>
__device__ __noinline__ float diag_intra_term(const bf16* dO, const bf16* v, const bf16* kq, Gates g,
                                              int rows, int I, int t, int il, int role) {
  float x = 0.f;
  const int lo = role == 0 ? SB * I : t + 1, hi = role == 0 ? t - 1 : SB * I + SB - 1;
  for (int r = lo; r <= hi && r < rows; ++r) {
    const int rq = role == 0 ? t : r, rv = role == 0 ? r : t;
    float b = 0.f;
    for (int j = 0; j < DV; ++j) b += __bfloat162float(dO[rq * VP + j]) * __bfloat162float(v[rv * VP + j]);
    x += b * __bfloat162float(kq[(size_t)r * DK + il]) *
         (role == 0 ? gate_ratio(g, rows, t, r, il) : gate_ratio(g, rows, r, t, il));
  }
  return x;
}

// A^T[t][u] = sum_i q_u,i k_t,i exp(b_u,i - b_t,i) over this CTA's key dims,
// chunk rows t <= u < rows (strong-decay fallback of the diagonal blocks)
template <class Gates>
__device__ __noinline__ float diag_at_entry(const bf16* q, const bf16* k, Gates g, int rows, int t,
                                            int u) {
  float a = 0.f;
  for (int i = 0; i < DKH; ++i) {
    float lg = 0.f;
    for (int x = t + 1; x <= u && x < rows; ++x) lg += g.at((size_t)x * DK + i);
    a += __bfloat162float(q[(size_t)u * DK + i]) * __bfloat162float(k[(size_t)t * DK + i]) * __expf(lg);
  }
  return a;
}

// LOGITS: the gates arrive as logits (p.gz set) and dg receives dL/dz; a
// separate instantiation, so that the log-gate path keeps its schedule.
template <bool LOGITS>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NT, 2)
    gla_bwd_chunk_kernel(GlaBwdParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  ChunkSmem& sm = *reinterpret_cast<ChunkSmem*>(smem_raw);
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, gc = (lane & 3) * 2;
  const int half = blockIdx.x & 1;  // == rank in the cluster
  const int i0 = half * DKH;        // first key dim of this CTA
  const int T = p.T, nchunks = (T + C - 1) / C;
  const int c = (int)((blockIdx.x >> 1) % (unsigned)nchunks), bh = (int)((blockIdx.x >> 1) / (unsigned)nchunks);
  // chunks the tcgen05 kernel has computed (both CTAs of the cluster leave)
  if (p.tc_flags && p.tc_flags[(size_t)bh * ((T + 2 * C - 1) / (2 * C)) + c / 2] == 0) return;
  const int c0 = c * C;
  const int rows = min(C, T - c0);
  const size_t tk = (size_t)bh * T * DK, tv = (size_t)bh * T * DV;
  // this chunk's first row, this CTA's key dims
  const bf16* qc = (const bf16*)p.q + tk + (size_t)c0 * DK + i0;
  const bf16* kc = (const bf16*)p.k + tk + (size_t)c0 * DK + i0;
  // log-gates, or the gate logits (then dg receives dL/dz)
  const float* gch = LOGITS ? nullptr : p.g + tk + (size_t)c0 * DK + i0;
  const bf16* gzc = LOGITS ? (const bf16*)p.gz + tk + (size_t)c0 * DK + i0 : nullptr;
  using Gates = typename std::conditional<LOGITS, LogitGates, LogGates>::type;
  Gates gsrc;
  if constexpr (LOGITS) gsrc = LogitGates{gzc, p.gs};
  else gsrc = LogGates{gch};
  float* stq = reinterpret_cast<float*>(sm.sp);   // Qf * acc_q (q dq without the diagonal pairs)
  float* stk = reinterpret_cast<float*>(sm.v);    // Kf * acc_k
  float* xch = reinterpret_cast<float*>(sm.qf);   // the peer's dv share
  float* peer_xch = cluster.map_shared_rank(xch, half ^ 1);

  // raw g, q, k of this CTA's key dims, staged where qf / kf and eqf / ekf go
  // once the prep has read them (rows past the end read as zeros)
  float* gs = reinterpret_cast<float*>(sm.qf);  // [C][DKH] fp32
  bf16* qs = sm.eqf;                            // [C][DKH] bf16 (swz64)
  bf16* ks = sm.ekf;
  // logits: staged in the upper half of the log-gate tile, converted below
  bf16* zs = reinterpret_cast<bf16*>(reinterpret_cast<unsigned char*>(gs) + sizeof(bf16) * C * DKH);
  {
    if constexpr (LOGITS) {
      for (int x = tid; x < C * DKH / 8; x += NT) {
        const int r = x / (DKH / 8), cc = x % (DKH / 8);
        const bool ok = r < rows;
        cp_async16(&zs[r * DKH + cc * 8], gzc + (size_t)(ok ? r : 0) * DK + cc * 8, ok ? 16 : 0);
      }
    } else {
      for (int x = tid; x < C * DKH / 4; x += NT) {
        const int r = x / (DKH / 4), cc = x % (DKH / 4);
        const bool ok = r < rows;
        cp_async16(&gs[r * DKH + cc * 4], gch + (size_t)(ok ? r : 0) * DK + cc * 4, ok ? 16 : 0);
      }
    }
    for (int x = tid; x < C * DKH / 8; x += NT) {
      const int r = x / (DKH / 8), cc = x % (DKH / 8);
      const bool ok = r < rows;
      const size_t off = (size_t)(ok ? r : 0) * DK + cc * 8;
      cp_async16(&qs[swz64(r, cc * 8)], qc + off, ok ? 16 : 0);
      cp_async16(&ks[swz64(r, cc * 8)], kc + off, ok ? 16 : 0);
    }
    cp_async_commit();
  }
  if (p.add_in_place && !p.add_dq) {
    // the window branch's gradients, added in the epilogue, were written long
    // before this kernel and have left L2: start bringing them back now (one
    // 128-byte line per row: this CTA's 64 dims of dq and dk, its 64 value
    // columns of dv)
    const int r = tid & 63, which = tid >> 6;  // 4 x 64 threads: dq, dk, dv
    if (which < 3 && r < rows) {
      const bf16* base = which == 0 ? (const bf16*)p.dq : which == 1 ? (const bf16*)p.dk : (const bf16*)p.dv;
      const size_t off = which < 2 ? tk + (size_t)(c0 + r) * DK + i0 : tv + (size_t)(c0 + r) * DV + 64 * half;
      asm volatile("prefetch.global.L2 [%0];" ::"l"(base + off));
    }
  }
  {  // tiles: v, dO, S_prev and G rows of this CTA's key dims
    const bf16* v = (const bf16*)p.v + tv + (size_t)c0 * DV;
    const bf16* dO = (const bf16*)p.dO + tv + (size_t)c0 * DV;
    for (int x = tid; x < C * DV / 8; x += NT) {
      const int r = x / (DV / 8), cc = x % (DV / 8);
      const bool ok = r < rows;
      const size_t off = (size_t)(ok ? r : 0) * DV + cc * 8;
      cp_async16(&sm.v[r * VP + cc * 8], v + off, ok ? 16 : 0);
      cp_async16(&sm.dO[r * VP + cc * 8], dO + off, ok ? 16 : 0);
    }
    const size_t so = ((size_t)bh * nchunks + c) * DK * DV + (size_t)i0 * DV;
    const bf16* sp = (const bf16*)p.states16 + so;
    const bf16* gi = (const bf16*)p.gin16 + so;
    for (int x = tid; x < DKH * DV / 8; x += NT) {
      const int r = x / (DV / 8), cc = x % (DV / 8);
      cp_async16(&sm.sp[swz(r, cc * 8)], sp + (size_t)r * DV + cc * 8, 16);
      cp_async16(&sm.g16[swz(r, cc * 8)], gi + (size_t)r * DV + cc * 8, 16);
    }
    cp_async_commit();
  }
  cp_async_wait<1>();
  __syncthreads();
  if constexpr (LOGITS) {  // log-gates from the logits (each thread 16 consecutive elements);
              // rows past the end: g = 0
    const uint4 za = *reinterpret_cast<const uint4*>(&zs[tid * 16]);
    const uint4 zb = *reinterpret_cast<const uint4*>(&zs[tid * 16 + 8]);
    __syncthreads();  // every logit is read before the log-gates overwrite them
    const bool ok = (tid * 16) / DKH < rows;
    const uint32_t zw[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
    float gv[16];
#pragma unroll
    for (int x = 0; x < 8; ++x) {
      const float2 f = unpack_bf16(zw[x]);
      gv[2 * x] = ok ? gate_from_logit(f.x, p.gs) : 0.f;
      gv[2 * x + 1] = ok ? gate_from_logit(f.y, p.gs) : 0.f;
    }
    float4* gd = reinterpret_cast<float4*>(&gs[tid * 16]);
#pragma unroll
    for (int x = 0; x < 4; ++x) gd[x] = make_float4(gv[4 * x], gv[4 * x + 1], gv[4 * x + 2], gv[4 * x + 3]);
    __syncthreads();
  }

  // ---- prep 1: per key dim cumulative gate products ------------------------
  const int K = tid >> 6, i = tid & 63, r0 = K * SB;
  float qfac[SB], kfac[SB];
  {
    float e[SB];
#pragma unroll
    for (int r = 0; r < SB; ++r) e[r] = __expf(gs[(r0 + r) * DKH + i]);
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
    sm.ksr[K][i] = ksk / rk;
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
    // qf / kf go over the staged gates (read before the last barrier); the
    // output scales go over the raw q / k once every thread has read them
#pragma unroll
    for (int r = 0; r < SB; ++r) {
      const int o = (r0 + r) * KP + i;
      sm.qf[o] = __float2bfloat16_rn(__bfloat162float(qs[swz64(r0 + r, i)]) * (qfac[r] * rq));
      sm.kf[o] = __float2bfloat16_rn(__bfloat162float(ks[swz64(r0 + r, i)]) * (kfac[r] * rk));
    }
    const int w = __syncthreads_or(!tame);
#pragma unroll
    for (int r = 0; r < SB; ++r) {
      const int o = (r0 + r) * KP + i;
      sm.eqf[o] = __float2bfloat16_rn(qfac[r] * rq);
      sm.ekf[o] = __float2bfloat16_rn(kfac[r] * rk);
    }
    cp_async_wait<0>();
    const int b = __syncthreads_or(bad);
    flags = (w ? 1 : 0) | (b ? 2 : 0);
  }
  const bool scaled = flags & 1, slow = flags & 2;

  // warp -> (row block I, role): role 0 computes dq and dv of value columns
  // [0, 64); role 1 computes dk and dv of value columns [64, 128)
  const int I = warp & 3, role = warp >> 2;
  const bf16* arows = role == 0 ? sm.dO : sm.v;
  const bf16* prows = role == 0 ? sm.v : sm.dO;
  const bf16* inter_b = role == 0 ? sm.sp : sm.g16;
  const bf16* intra_b = role == 0 ? sm.kf : sm.qf;
  const float* colf = role == 0 ? sm.ci[I] : sm.ck[I];
  const bf16* oscale = role == 0 ? sm.eqf : sm.ekf;
  float acc[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.f;
  // ---- inter: (dO S_prev^T | v G^T), then per-dim factor (ci | ck) --------
#pragma unroll 2
  for (int kk = 0; kk < 8; ++kk) {
    uint32_t a[4];
    ldsm_x4(smem_u32(&arows[(16 * I + (lane & 15)) * VP + kk * 16 + (lane >> 4) * 8]), a[0], a[1], a[2],
            a[3]);
#pragma unroll
    for (int ntp = 0; ntp < 4; ++ntp) {
      uint32_t b0, b1, b2, b3;
      const int n = ntp * 16 + (lane & 7) + ((lane >> 4) << 3);
      ldsm_x4(smem_u32(&inter_b[swz(n, kk * 16 + ((lane >> 3) & 1) * 8)]), b0, b1, b2, b3);
      mma_bf16(acc[2 * ntp], a, b0, b1);
      mma_bf16(acc[2 * ntp + 1], a, b2, b3);
    }
  }
#pragma unroll
  for (int nt = 0; nt < 8; ++nt) {
    const float2 f = *reinterpret_cast<const float2*>(&colf[nt * 8 + gc]);
    acc[nt][0] *= f.x;
    acc[nt][1] *= f.y;
    acc[nt][2] *= f.x;
    acc[nt][3] *= f.y;
  }
  {  // the finalize's lines (raw operand and previous gradient, rows t and t + 8), into L1
    const int tr = 16 * I + gr + ((lane & 2) ? 8 : 0);
    if (tr < rows) {
      if ((lane & 1) == 0)
        asm volatile("prefetch.global.L1 [%0];" ::"l"((role == 0 ? kc : qc) + (size_t)tr * DK));
      else if (p.add_in_place && !(role == 0 ? p.add_dq : p.add_dk))
        asm volatile("prefetch.global.L1 [%0];" ::"l"((const bf16*)(role == 0 ? p.dq : p.dk) + tk +
                                                      (size_t)(c0 + tr) * DK + i0));
    }
  }
  // ---- intra: one 16x16 score block at a time, consumed right away -------
  const int jlo = role == 0 ? 0 : I, jhi = role == 0 ? I : NSB - 1;

  for (int J = jlo; J <= jhi; ++J) {
    float sc[2][4], sc2[2][4];  // two partial sums over k for independent MMA chains
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] = sc2[nt][e] = 0.f;
#pragma unroll
    for (int kk = 0; kk < 8; kk += 2) {
      uint32_t a[4], b0, b1, b2, b3, cc[4], d0, d1, d2, d3;
      ldsm_x4(smem_u32(&arows[(16 * I + (lane & 15)) * VP + kk * 16 + (lane >> 4) * 8]), a[0], a[1], a[2],
              a[3]);
      ldsm_x4(smem_u32(&prows[(16 * J + (lane & 7) + ((lane >> 4) << 3)) * VP + kk * 16 +
                              ((lane >> 3) & 1) * 8]),
              b0, b1, b2, b3);
      ldsm_x4(smem_u32(&arows[(16 * I + (lane & 15)) * VP + kk * 16 + 16 + (lane >> 4) * 8]), cc[0], cc[1],
              cc[2], cc[3]);
      ldsm_x4(smem_u32(&prows[(16 * J + (lane & 7) + ((lane >> 4) << 3)) * VP + kk * 16 + 16 +
                              ((lane >> 3) & 1) * 8]),
              d0, d1, d2, d3);
      mma_bf16(sc[0], a, b0, b1);
      mma_bf16(sc[1], a, b2, b3);
      mma_bf16(sc2[0], cc, d0, d1);
      mma_bf16(sc2[1], cc, d2, d3);
    }
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) sc[nt][e] += sc2[nt][e];
    if (J == I) {
      // the diagonal (t, t) of row gr (gr + 8) sits in lane 4 gr + gr / 2,
      // fragment element (gr & 1) of column tile 0 (1)
      if ((lane & 3) == (gr >> 1)) {
        sm.bdg[role][16 * I + gr] = (gr & 1) ? sc[0][1] : sc[0][0];
        sm.bdg[role][16 * I + gr + 8] = (gr & 1) ? sc[1][3] : sc[1][2];
      }
      if (slow) continue;  // the diagonal block of a strong-decay chunk: below
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = gr + (e >> 1) * 8, u = nt * 8 + gc + (e & 1);
          if (role == 0 ? (u >= t) : (u <= t)) sc[nt][e] = 0.f;
        }
    }
    const uint32_t pa[4] = {pack_bf16(sc[0][0], sc[0][1]), pack_bf16(sc[0][2], sc[0][3]),
                            pack_bf16(sc[1][0], sc[1][1]), pack_bf16(sc[1][2], sc[1][3])};
    const float* fac = sm.fac[role == 0 ? pair_index(I, J) : pair_index(J, I)];
#pragma unroll
    for (int ntp = 0; ntp < 4; ++ntp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(&intra_b[(16 * J + (lane & 7) + ((lane >> 3) & 1) * 8) * KP + ntp * 16 +
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
  __syncwarp();
  // ---- finalize (dq | dk) = (Eq | Ek) * acc + diagonal, store; keep the
  // products (Qf acc_q | Kf acc_k) for dg -----------------------------------
  {
    const bf16* raw = role == 0 ? kc : qc;  // the other factor of the diagonal pair
    const bf16* same = role == 0 ? qc : kc;
    const bf16* fop = role == 0 ? sm.qf : sm.kf;
    bf16* outp = (bf16*)(role == 0 ? p.dq : p.dk);
    const float* addf = role == 0 ? p.add_dq : p.add_dk;
    // two rounds of four column tiles; each round issues its global loads
    // before its first store
#pragma unroll
    for (int n0 = 0; n0 < 8; n0 += 4) {
      uint32_t rv[4][2], inp[4][2];
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int t = 16 * I + gr + 8 * hh;
          const int il = (n0 + n) * 8 + gc;
          const bool ok = t < rows;
          rv[n][hh] = ok ? __ldg(reinterpret_cast<const unsigned int*>(&raw[(size_t)t * DK + il])) : 0u;
          inp[n][hh] = ok && p.add_in_place && !addf
                           ? *reinterpret_cast<const uint32_t*>(&outp[tk + (size_t)(c0 + t) * DK + i0 + il])
                           : 0u;
        }
#pragma unroll
      for (int n = 0; n < 4; ++n)
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {
          const int nt = n0 + n;
          const int t = 16 * I + gr + 8 * hh;
          const int il = nt * 8 + gc;
          const float2 os = unpack_bf16(*reinterpret_cast<const uint32_t*>(&oscale[t * KP + il]));
          const float2 fq = unpack_bf16(*reinterpret_cast<const uint32_t*>(&fop[t * KP + il]));
          const float2 xo = unpack_bf16(rv[n][hh]);
          const float a0 = acc[nt][2 * hh], a1 = acc[nt][2 * hh + 1];
          float p0 = fq.x * a0, p1 = fq.y * a1;
          const float bd = sm.bdg[role][t];
          float x0 = a0 * os.x + bd * xo.x, x1 = a1 * os.y + bd * xo.y;
          if (slow) {
            const float d0 = diag_intra_term(sm.dO, sm.v, raw, gsrc, rows, I, t, il, role);
            const float d1 = diag_intra_term(sm.dO, sm.v, raw, gsrc, rows, I, t, il + 1, role);
            x0 += d0;
            x1 += d1;
            if (t < rows) {
              const float2 sv =
                  unpack_bf16(__ldg(reinterpret_cast<const unsigned int*>(&same[(size_t)t * DK + il])));
              p0 += sv.x * d0;
              p1 += sv.y * d1;
            }
          }
          if (t < rows) {
            const size_t off = tk + (size_t)(c0 + t) * DK + i0 + il;
            float y0 = x0, y1 = x1;
            if (addf) {
              const float2 a = *reinterpret_cast<const float2*>(&addf[off]);
              y0 += a.x;
              y1 += a.y;
            } else {
              const float2 a = unpack_bf16(inp[n][hh]);
              y0 += a.x;
              y1 += a.y;
            }
            *reinterpret_cast<uint32_t*>(&outp[off]) = pack_bf16(y0, y1);
          }
          acc[nt][2 * hh] = p0;
          acc[nt][2 * hh + 1] = p1;
        }
    }
  }
  __syncthreads();  // every reader of S_prev and v is done
  {
    float* st = role == 0 ? stq : stk;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = 16 * I + gr + 8 * hh, il = nt * 8 + gc;
        *reinterpret_cast<float2*>(&st[rsw(t, il)]) = make_float2(acc[nt][2 * hh], acc[nt][2 * hh + 1]);
      }
  }

  // ---- partial dv of row block Iv, value columns [64 role, 64 role + 64) ---
  // (role 1 takes the mirrored row block so that every warp multiplies
  // 5 score blocks)
  const int Iv = role == 0 ? I : NSB - 1 - I;
  float dvh[8][4];
#pragma unroll
  for (int nt = 0; nt < 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) dvh[nt][e] = 0.f;
  // inter: (k e^{b_l - b})_Iv G[:, this role's columns], the k operand as kf
  // rescaled per key dim
  {
    const float* ksr = sm.ksr[Iv];
#pragma unroll
    for (int kk = 0; kk < DKH / 16; ++kk) {
      uint32_t a[4];
      ldsm_x4(smem_u32(&sm.kf[(16 * Iv + (lane & 15)) * KP + kk * 16 + (lane >> 4) * 8]), a[0], a[1], a[2],
              a[3]);
      const float2 f0 = *reinterpret_cast<const float2*>(&ksr[kk * 16 + gc]);
      const float2 f1 = *reinterpret_cast<const float2*>(&ksr[kk * 16 + 8 + gc]);
      a[0] = scale_bf16x2(a[0], f0.x, f0.y);
      a[1] = scale_bf16x2(a[1], f0.x, f0.y);
      a[2] = scale_bf16x2(a[2], f1.x, f1.y);
      a[3] = scale_bf16x2(a[3], f1.x, f1.y);
#pragma unroll
      for (int ntp = 0; ntp < 4; ++ntp) {
        uint32_t b0, b1, b2, b3;
        const int kr = kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
        ldsm_x4_t(smem_u32(&sm.g16[swz(kr, 64 * role + ntp * 16 + (lane >> 4) * 8)]), b0, b1, b2, b3);
        mma_bf16(dvh[2 * ntp], a, b0, b1);
        mma_bf16(dvh[2 * ntp + 1], a, b2, b3);
      }
    }
  }
  // intra: A^T[Iv][J] dO_J for J >= Iv, one score block at a time
  for (int J = Iv; J < NSB; ++J) {
    float at[2][4];
#pragma unroll
    for (int nt = 0; nt < 2; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) at[nt][e] = 0.f;
    const float* fac = sm.fac[pair_index(J, Iv)];
#pragma unroll
    for (int kk = 0; kk < DKH / 16; ++kk) {
      uint32_t a[4];
      ldsm_x4(smem_u32(&sm.kf[(16 * Iv + (lane & 15)) * KP + kk * 16 + (lane >> 4) * 8]), a[0], a[1], a[2],
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
      ldsm_x4(smem_u32(&sm.qf[(16 * J + (lane & 7) + ((lane >> 4) << 3)) * KP + kk * 16 +
                              ((lane >> 3) & 1) * 8]),
              b0, b1, b2, b3);
      mma_bf16(at[0], a, b0, b1);
      mma_bf16(at[1], a, b2, b3);
    }
    if (J == Iv) {
#pragma unroll
      for (int nt = 0; nt < 2; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int t = gr + (e >> 1) * 8, u = nt * 8 + gc + (e & 1);
          const int rt = 16 * Iv + t, ru = 16 * Iv + u;
          if (u < t) at[nt][e] = 0.f;
          else if (slow) at[nt][e] = ru < rows ? diag_at_entry(qc, kc, gsrc, rows, rt, ru) : 0.f;
        }
    }
    const uint32_t pa[4] = {pack_bf16(at[0][0], at[0][1]), pack_bf16(at[0][2], at[0][3]),
                            pack_bf16(at[1][0], at[1][1]), pack_bf16(at[1][2], at[1][3])};
#pragma unroll
    for (int ntp = 0; ntp < 4; ++ntp) {
      uint32_t b0, b1, b2, b3;
      ldsm_x4_t(smem_u32(&sm.dO[(16 * J + (lane & 7) + ((lane >> 3) & 1) * 8) * VP + 64 * role + ntp * 16 +
                                (lane >> 4) * 8]),
                b0, b1, b2, b3);
      mma_bf16(dvh[2 * ntp], pa, b0, b1);
      mma_bf16(dvh[2 * ntp + 1], pa, b2, b3);
    }
  }
  // the gate gradient at the chunk's first row, from the reverse scan (loaded
  // here so that the load overlaps the cluster barrier)
  const float dg_first = p.gsp[((size_t)bh * nchunks + c) * DK + i0 + (tid & 63)];
  // this CTA no longer reads qf / kf (the peer's dv share lands over them):
  // arrive now, and compute dg before waiting for the peer to do the same
  auto done_reading = cluster.barrier_arrive();
  __syncthreads();  // the dg products staged by every warp
  // ---- dg: the scan's value at the chunk's first row, then a running sum ---
  {
    const int col = tid & 63, qq = tid >> 6;
    float loc[SB];
    float run = 0.f;
#pragma unroll
    for (int r = 0; r < SB; ++r) {  // exclusive prefix of the q-side minus the k-side products
      loc[r] = run;
      run += stq[rsw(16 * qq + r, col)] - stk[rsw(16 * qq + r, col)];
    }
    sm.tot[qq][col] = run;
    __syncthreads();
    float base = dg_first;
#pragma unroll
    for (int q2 = 0; q2 < NSB; ++q2)
      if (q2 < qq) base -= sm.tot[q2][col];
#pragma unroll
    for (int r = 0; r < SB; ++r) {
      const int t = 16 * qq + r;
      if (t < rows) {
        float x = base - loc[r];
        if constexpr (LOGITS) x = dlogit(x, __bfloat162float(__ldg(&gzc[(size_t)t * DK + col])), p.gs);
        p.dg[tk + (size_t)(c0 + t) * DK + i0 + col] = x;
      }
    }
  }
  cluster.barrier_wait(std::move(done_reading));
  // ---- dv: the peer's 64 columns go to its exchange tile -------------------
  if (role != half) {
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = 16 * Iv + gr + 8 * hh, cl = nt * 8 + gc;
        *reinterpret_cast<float2*>(&peer_xch[rsw(t, cl)]) = make_float2(dvh[nt][2 * hh], dvh[nt][2 * hh + 1]);
      }
  }
  auto share_sent = cluster.barrier_arrive();
  if (role == half && p.add_in_place && !p.add_dv) {  // loads ahead of the stores below
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = 16 * Iv + gr + 8 * hh, cl = nt * 8 + gc;
        const uint32_t a = t < rows ? *reinterpret_cast<const uint32_t*>(
                                          &((const bf16*)p.dv)[tv + (size_t)(c0 + t) * DV + 64 * half + cl])
                                    : 0u;
        const float2 f = unpack_bf16(a);
        dvh[nt][2 * hh] += f.x;
        dvh[nt][2 * hh + 1] += f.y;
      }
  }
  cluster.barrier_wait(std::move(share_sent));  // the peer's share has landed
  if (role == half) {
    const int mcol = 64 * half;
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        const int t = 16 * Iv + gr + 8 * hh, cl = nt * 8 + gc;
        if (t >= rows) continue;
        const float2 pr = *reinterpret_cast<const float2*>(&xch[rsw(t, cl)]);
        float y0 = dvh[nt][2 * hh] + pr.x, y1 = dvh[nt][2 * hh + 1] + pr.y;
        const size_t off = tv + (size_t)(c0 + t) * DV + mcol + cl;
        if (p.add_dv) {
          const float2 a = *reinterpret_cast<const float2*>(&p.add_dv[off]);
          y0 += a.x;
          y1 += a.y;
        }
        *reinterpret_cast<uint32_t*>(&((bf16*)p.dv)[off]) = pack_bf16(y0, y1);
      }
  }
}

}  // namespace

bool gla_bwd_mma_supported(int dk, int dv, bool bf16) { return bf16 && dk == DK && dv == DV; }


cudaError_t launch_gla_bwd_chunks(const GlaBwdParams& p, cudaStream_t s) {
  const int nchunks = (p.T + C - 1) / C;
  if (p.B * p.H == 0 || nchunks == 0) return cudaSuccess;
  if (2 * (size_t)nchunks * p.B * p.H > 0x7fffffffu) return cudaErrorInvalidConfiguration;
  const size_t bytes = sizeof(ChunkSmem);
  const auto kern = p.gz ? gla_bwd_chunk_kernel<true> : gla_bwd_chunk_kernel<false>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e != cudaSuccess) return e;
  {
    ScopedTiming tm("gla_bwd_chunks", s);
    kern<<<(unsigned)(2 * (size_t)nchunks * p.B * p.H), NT, bytes, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace lz
