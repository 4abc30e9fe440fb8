// Chunked gated linear attention backward on the Blackwell tensor cores:
// every contraction is a tcgen05.mma (M = 128) with its accumulator in tensor
// memory, the operands brought in by TMA (bf16 I/O, fp32 accumulation,
// dk = dv = 128).
//
// Gradient of S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T, o_t = q_t^T S_t (the
// attention-output regression of the first training stage, Lizard technical
// summary section 2b, needs it).  Per 128-token chunk with b_t the running
// log-gate inside the chunk, r = 63 (the end of its first half) the
// reference row, S_prev the state
// before the chunk, G the state gradient entering it from the later chunks
// (launch_gla_bwd_scan), and the bounded factors
//   Eq_t = e^{b_t - b_r},  Qf = q Eq,  Kf = k / Eq,  ci = e^{b_r},  ck = e^{b_l - b_r},
// B[t][s] = dO_t . v_s (masked to s < t), A[t][s] = Qf_t . Kf_s (s <= t):
//   dq = Eq * (ci * (dO S_prev^T) + B Kf)          + B[t][t] k_t
//   dk = (ck * (V G^T) + B^T Qf) / Eq                + B[t][t] q_t
//   dv = Kf (diag(ck) G) + A^T dO
//   dg_t = <G_new, S_prev> - sum_{u<t} (Qf_u acc_q,u - Kf_u acc_k,u),
// acc_q / acc_k the brackets of dq / dk.  The diagonal pairs (s = t) stay out
// of the MMAs: their two copies in the running sum of dg cancel exactly, and
// every other pair enters both sides as the same product Qf_u B[u][s] Kf_s,
// so under fast forgetting the running sum leaves only the pairs that
// straddle t, with the rounding of one product each.
//
// The factors stay within e^{+-60} when each 64-row half of the chunk decays
// by at most e^-60 in every key dim; a chunk where some dim decays faster is
// flagged in `flags` and left to launch_gla_bwd_chunks (per 64-row sub-block
// references and elementwise diagonal blocks), which then runs only the
// flagged chunks.
//
// Work split: a cluster of two CTAs per (chunk, batch-head); CTA r owns key
// dims [64r, 64r + 64) (its q, k, g columns and S_prev / G rows).  Both
// compute B (over all value dims) and keep it once, masked, in shared memory:
// dq reads it as a K-major operand, dk the same tile transposed (MN-major).
// dq, dk and dg are complete inside the CTA; dv is a sum over key dims, so
// each CTA sends its partial dv of the peer's 64 value columns through
// distributed shared memory.  One thread issues the TMA copies and the MMAs;
// all 8 warps read the accumulators.
//
// Tensor memory (512 columns): [0,128) B, then A^T; [128,256) dv;
// [256,320) dO S^T; [320,384) B Kf; [384,448) V G^T; [448,512) B^T Qf.
#include <cooperative_groups.h>

#include <cstddef>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"
#include "tc05.cuh"
#include "tma_host.h"

namespace cg = cooperative_groups;

namespace lz {
namespace {

constexpr int C = 128;       // tokens per chunk (MMA M)
constexpr int D = 128;       // dk = dv
constexpr int DH = 64;       // key dims per CTA
constexpr int NTH = 256;
constexpr uint32_t kRowB = 128;                  // bytes of one swizzled 64-wide row
constexpr uint32_t kBox128 = C * kRowB;          // [128 rows][64] bf16, 128-byte swizzle
constexpr uint32_t kBox64 = DH * kRowB;          // [64 rows][64] bf16
constexpr float kMaxHalfDecay = -60.f;           // log-decay bound of a 64-row half
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColB = 0, kColDV = 128, kColXq = 256, kColYq = 320, kColXk = 384, kColYk = 448;
constexpr uint32_t kLoadBytes1 = 2 * 2 * kBox128 + 2 * 2 * kBox64;  // dO, V, S_prev, G
constexpr uint32_t kLoadBytes2 = 2 * kBox128;                       // q, k

struct TcSmem {
  uint8_t dO[2][kBox128];  // [t][j], j halves (TMA); dv exchange at the end (fp32 [128][64])
  uint8_t v[2][kBox128];   // [s][j]
  uint8_t qf[kBox128];     // [t][i] of this CTA's dims: raw q (TMA), then Qf in place
  uint8_t kf[kBox128];     // raw k, then Kf
  uint8_t sp[2][kBox64];   // S_prev rows i of this CTA, j halves; then dg's quarter totals
  uint8_t gg[2][kBox64];   // G rows i; scaled by ck once V G^T is done
  uint8_t bm[2][kBox128];  // the gates' quarter totals; B masked [t][s] (s halves, swizzled
                           // like the TMA tiles); then A^T masked [s][t]; then the dg
                           // products (fp32 [128][64])
  float eq[C][DH + 4];     // Eq (rows padded: a warp reads 32 rows at one column)
  float btt[C];            // fp32 dO_t . v_t
  float ci[DH], ck[DH];
  uint64_t bar_ld, bar_lq, bar_a, bar_b, bar_c;
  uint32_t tmem_base;
  int wild;       // some dim of this CTA decays past the bound in a 64-row half
  int peer_wild;  // the same for the peer (written by the peer)
};
static_assert(sizeof(TcSmem) + 1024 <= 232448, "shared memory per block exceeds 227 KB");
static_assert(offsetof(TcSmem, v) % 1024 == 0 && offsetof(TcSmem, qf) % 1024 == 0 &&
                  offsetof(TcSmem, kf) % 1024 == 0 && offsetof(TcSmem, sp) % 1024 == 0 &&
                  offsetof(TcSmem, gg) % 1024 == 0 && offsetof(TcSmem, bm) % 1024 == 0,
              "swizzled tiles must be 1024-byte aligned");

// byte offset of 16-byte chunk `chunk` (8 bf16) of row `row` of a [rows][64]
// bf16 tile with the 128-byte swizzle (chunks XOR-permuted by row % 8)
__device__ __forceinline__ uint32_t sw_chunk(int row, int chunk) {
  return (uint32_t)row * kRowB + ((((uint32_t)chunk) ^ ((uint32_t)row & 7u)) << 4);
}

__device__ __forceinline__ float4 ld4(const float* p) { return *reinterpret_cast<const float4*>(p); }

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(NTH, 1)
    gla_bwd_tc_kernel(GlaBwdParams p, int* flags, const __grid_constant__ CUtensorMap tq,
                      const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                      const __grid_constant__ CUtensorMap tdo, const __grid_constant__ CUtensorMap tsp,
                      const __grid_constant__ CUtensorMap tgi) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  TcSmem& sm = *reinterpret_cast<TcSmem*>(smem_raw + ((1024u - (raw & 1023u)) & 1023u));
  cg::cluster_group cluster = cg::this_cluster();
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int half = (int)(blockIdx.x & 1);  // == rank in the cluster
  const int i0 = half * DH;
  const int T = p.T, n128 = (T + C - 1) / C, n64 = (T + 63) / 64;
  const int c = (int)((blockIdx.x >> 1) % (unsigned)n128), bh = (int)((blockIdx.x >> 1) / (unsigned)n128);
  const int c0 = c * C, rows = min(C, T - c0);
  const size_t tk0 = (size_t)bh * T * D;  // first element of this (batch, head) in q, k, v, dO

  const uint32_t s_do = smem_u32(sm.dO), s_v = smem_u32(sm.v), s_qf = smem_u32(sm.qf);
  const uint32_t s_kf = smem_u32(sm.kf), s_sp = smem_u32(sm.sp), s_gg = smem_u32(sm.gg);
  const uint32_t s_bm = smem_u32(sm.bm);
  const uint32_t bar_ld = smem_u32(&sm.bar_ld), bar_lq = smem_u32(&sm.bar_lq);
  const uint32_t bar_a = smem_u32(&sm.bar_a), bar_b = smem_u32(&sm.bar_b), bar_c = smem_u32(&sm.bar_c);

  if (warp == 0) tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
  if (tid == 0) {
    mbar_init(bar_ld, 1);
    mbar_init(bar_lq, 1);
    mbar_init(bar_a, 1);
    mbar_init(bar_b, 1);
    mbar_init(bar_c, 1);
    mbar_init_fence();
    // the operands of the first products, then q and k; rows past the
    // sequence read as zeros
    mbar_expect_tx(bar_ld, kLoadBytes1);
    const int cs = 2 * c, cg_ = min(2 * c + 1, n64 - 1);  // 64-token chunks: state before, G after
    for (int hf = 0; hf < 2; ++hf) {
      tma_load_3d(s_do + hf * kBox128, &tdo, bar_ld, hf * 64, c0, bh);
      tma_load_3d(s_v + hf * kBox128, &tv, bar_ld, hf * 64, c0, bh);
      tma_load_3d(s_sp + hf * kBox64, &tsp, bar_ld, hf * 64, cs * D + i0, bh);
      tma_load_3d(s_gg + hf * kBox64, &tgi, bar_ld, hf * 64, cg_ * D + i0, bh);
    }
    mbar_expect_tx(bar_lq, kLoadBytes2);
    tma_load_3d(s_qf, &tq, bar_lq, i0, c0, bh);
    tma_load_3d(s_kf, &tk, bar_lq, i0, c0, bh);
  }

  // ---- gates: running log-gate per key dim, its bound, the factors --------
  const int i = tid & (DH - 1), qt = tid >> 6;  // key dim, quarter of the rows
  float bl[32];
  {
    const float* gc = p.g + tk0 + (size_t)c0 * D + i0 + i;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const int t = qt * 32 + r;
      bl[r] = t < rows ? __ldg(gc + (size_t)t * D) : 0.f;
    }
    float run = 0.f;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      run += bl[r];
      bl[r] = run;
    }
    reinterpret_cast<float*>(sm.bm)[qt * DH + i] = run;  // (B is written much later)
  }
  tc_fence_before();
  __syncthreads();  // barriers, TMEM address, quarter totals
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;
  const float* gtot = reinterpret_cast<const float*>(sm.bm);
  const float t0 = gtot[i], t1 = gtot[DH + i], t2 = gtot[2 * DH + i], t3 = gtot[3 * DH + i];
  const float bref = t0 + t1, blast = bref + t2 + t3;
  {
    const bool w = (t0 + t1 < kMaxHalfDecay) || (t2 + t3 < kMaxHalfDecay);
    const int anyw = __syncthreads_or(w);
    if (tid == 0) {
      sm.wild = anyw;
      *cluster.map_shared_rank(&sm.peer_wild, half ^ 1) = anyw;
    }
  }
  cluster.sync();
  bool alive = true;
  if (sm.wild || sm.peer_wild) {
    // left to the per-64-row kernel: flag the chunk, let the copies land, leave
    if (tid == 0 && half == 0) flags[(size_t)bh * n128 + c] = 1;
    if (tid == 0) {
      mbar_wait(bar_ld, 0, p.status);
      mbar_wait(bar_lq, 0, p.status);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
      tc_fence_after();
      tmem_dealloc(tmem, kTmemCols);
    }
    return;
  }
  if (tid == 0 && half == 0) flags[(size_t)bh * n128 + c] = 0;

  // thread 0: the products that need no gate factors start at once
  if (tid == 0) {
    alive = mbar_wait(bar_ld, 0, p.status);
    if (alive) {
      tc_fence_after();
      constexpr uint32_t idBB = idesc_bf16(C, C, false), idX = idesc_bf16(C, DH, false);
#pragma unroll 1
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t ko = (kk >> 2) * kBox128 + (kk & 3) * 32, k64 = (kk >> 2) * kBox64 + (kk & 3) * 32;
        const uint32_t acc = kk > 0;
        const uint64_t ado = sdesc_sw128(s_do + ko, 16, 1024), av = sdesc_sw128(s_v + ko, 16, 1024);
        mma_bf16_ss(tmem + kColB, ado, av, idBB, acc);                                  // B
        mma_bf16_ss(tmem + kColXq, ado, sdesc_sw128(s_sp + k64, 16, 1024), idX, acc);   // dO S^T
        mma_bf16_ss(tmem + kColXk, av, sdesc_sw128(s_gg + k64, 16, 1024), idX, acc);    // V G^T
      }
      mma_commit(bar_a);
    }
  }
  // Eq per (row, dim); ci, ck per dim
  {
    const float off = (qt > 0 ? t0 : 0.f) + (qt > 1 ? t1 : 0.f) + (qt > 2 ? t2 : 0.f);
#pragma unroll
    for (int r = 0; r < 32; ++r) sm.eq[qt * 32 + r][i] = __expf(off + bl[r] - bref);
    if (qt == 0) {
      sm.ci[i] = __expf(bref);
      sm.ck[i] = __expf(blast - bref);
    }
  }
  alive = mbar_wait(bar_lq, 0, p.status) && alive;
  __syncthreads();  // every Eq written
  // Qf = q Eq and Kf = k / Eq in place: row tid / 2, 32 dims per thread
  {
    const int t = tid >> 1, cb = (tid & 1) * 4;
#pragma unroll
    for (int x = 0; x < 4; ++x) {
      const int ch8 = cb + x;
      const float4 e0 = ld4(&sm.eq[t][ch8 * 8]), e1 = ld4(&sm.eq[t][ch8 * 8 + 4]);
      const float e[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
      uint4* pq = reinterpret_cast<uint4*>(sm.qf + sw_chunk(t, ch8));
      uint4* pk = reinterpret_cast<uint4*>(sm.kf + sw_chunk(t, ch8));
      uint4 uq = *pq, uk = *pk;
      uint32_t* wq = reinterpret_cast<uint32_t*>(&uq);
      uint32_t* wk = reinterpret_cast<uint32_t*>(&uk);
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const float2 a = unpack_bf16(wq[u]), b = unpack_bf16(wk[u]);
        wq[u] = pack_bf16(a.x * e[2 * u], a.y * e[2 * u + 1]);
        wk[u] = pack_bf16(__fdividef(b.x, e[2 * u]), __fdividef(b.y, e[2 * u + 1]));
      }
      *pq = uq;
      *pk = uk;
    }
  }

  // ---- B out of tensor memory, masked, into shared memory -----------------
  const int lq = warp & 3, ch = warp >> 2;  // lane quarter, column half
  const int row = lq * 32 + lane;           // TMEM lane = accumulator row
  const uint32_t lrow = tmem + ((uint32_t)(lq * 32) << 16);
  if (tid == 0 && alive) alive = mbar_wait(bar_a, 0, p.status);
  alive = __syncthreads_and(alive);  // also: every Qf, Kf, ci, ck written
  tc_fence_after();
#pragma unroll 1
  for (int cb = 0; cb < 2; ++cb) {  // B rows t, keep s < t; columns [64 ch + 32 cb, +32)
    const int col0 = ch * 64 + cb * 32;
    uint32_t x[32];
    tmem_ld32(lrow + kColB + col0, x);
    tmem_ld_wait();
    uint32_t pk[16];
    float dval = 0.f;
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int cc = col0 + e;
      if (cc == row) dval = __uint_as_float(x[e]);
      if (cc + 1 == row) dval = __uint_as_float(x[e + 1]);
      pk[e / 2] = pack_bf16(cc < row ? __uint_as_float(x[e]) : 0.f,
                            cc + 1 < row ? __uint_as_float(x[e + 1]) : 0.f);
    }
    if (row >= col0 && row < col0 + 32) sm.btt[row] = dval;
#pragma unroll
    for (int x4 = 0; x4 < 4; ++x4)
      *reinterpret_cast<uint4*>(sm.bm[ch] + sw_chunk(row, cb * 4 + x4)) =
          make_uint4(pk[4 * x4], pk[4 * x4 + 1], pk[4 * x4 + 2], pk[4 * x4 + 3]);
  }
  // G' = diag(ck) G (V G^T is done): rows i, 32 of the 128 columns per thread
  {
    const int gi = tid >> 2, gc0 = (tid & 3) * 32;
    const float f = sm.ck[gi];
#pragma unroll
    for (int x8 = 0; x8 < 4; ++x8) {
      const int col = gc0 + x8 * 8;
      uint4* pv = reinterpret_cast<uint4*>(sm.gg[col >> 6] + sw_chunk(gi, (col & 63) >> 3));
      uint4 u = *pv;
      u.x = scale_bf16x2(u.x, f, f);
      u.y = scale_bf16x2(u.y, f, f);
      u.z = scale_bf16x2(u.z, f, f);
      u.w = scale_bf16x2(u.w, f, f);
      *pv = u;
    }
  }
  fence_async_smem();
  tc_fence_before();
  alive = __syncthreads_and(alive);
  if (tid == 0 && alive) {
    tc_fence_after();
    constexpr uint32_t idBB = idesc_bf16(C, C, false), idMN64 = idesc_bf16(C, DH, true);
    constexpr uint32_t idMN128 = idesc_bf16(C, D, true), idTT64 = idesc_bf16_at(C, DH, true);
#pragma unroll 1
    for (int kk = 0; kk < DH / 16; ++kk) {  // K = this CTA's 64 key dims
      const uint64_t akf = sdesc_sw128(s_kf + kk * 32, 16, 1024);
      mma_bf16_ss(tmem + kColB, akf, sdesc_sw128(s_qf + kk * 32, 16, 1024), idBB, kk > 0);  // A^T
      mma_bf16_ss(tmem + kColDV, akf, sdesc_sw128(s_gg + kk * 2048, kBox64, 1024), idMN128,
                  kk > 0);  // dv = Kf G'
    }
#pragma unroll 1
    for (int kk = 0; kk < C / 16; ++kk) {  // K = the chunk's 128 tokens
      const uint32_t ko = (kk >> 2) * kBox128 + (kk & 3) * 32;
      mma_bf16_ss(tmem + kColYq, sdesc_sw128(s_bm + ko, 16, 1024),
                  sdesc_sw128(s_kf + kk * 2048, kBox128, 1024), idMN64, kk > 0);  // B Kf
      mma_bf16_ss(tmem + kColYk, sdesc_sw128(s_bm + kk * 2048, kBox128, 1024),
                  sdesc_sw128(s_qf + kk * 2048, kBox128, 1024), idTT64, kk > 0);  // B^T Qf
    }
    mma_commit(bar_b);
  }
  if (tid == 0 && alive) alive = mbar_wait(bar_b, 0, p.status);
  alive = __syncthreads_and(alive);
  tc_fence_after();
  // A^T rows s (keep t >= s) over the spent B tile, then dv += A^T dO
#pragma unroll 1
  for (int cb = 0; cb < 2; ++cb) {
    const int col0 = ch * 64 + cb * 32;
    uint32_t x[32];
    tmem_ld32(lrow + kColB + col0, x);
    tmem_ld_wait();
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int cc = col0 + e;
      pk[e / 2] = pack_bf16(cc >= row ? __uint_as_float(x[e]) : 0.f,
                            cc + 1 >= row ? __uint_as_float(x[e + 1]) : 0.f);
    }
#pragma unroll
    for (int x4 = 0; x4 < 4; ++x4)
      *reinterpret_cast<uint4*>(sm.bm[ch] + sw_chunk(row, cb * 4 + x4)) =
          make_uint4(pk[4 * x4], pk[4 * x4 + 1], pk[4 * x4 + 2], pk[4 * x4 + 3]);
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  if (tid == 0 && alive) {
    tc_fence_after();
    constexpr uint32_t idMN128 = idesc_bf16(C, D, true);
#pragma unroll 1
    for (int kk = 0; kk < C / 16; ++kk)
      mma_bf16_ss(tmem + kColDV, sdesc_sw128(s_bm + (kk >> 2) * kBox128 + (kk & 3) * 32, 16, 1024),
                  sdesc_sw128(s_do + kk * 2048, kBox128, 1024), idMN128, 1u);
    mma_commit(bar_c);
  }

  // ---- dq, dk of row `row`, dims [32 ch, 32 ch + 32) (overlaps the dv MMA) --
  float* prod = reinterpret_cast<float*>(sm.sp);  // [128][64] fp32: S_prev and G' are spent
  {
    const int t = row;
    const float btt = sm.btt[t];
    const size_t go = tk0 + (size_t)(c0 + t) * D + i0;
    const bf16* qr = (const bf16*)p.q + go;
    const bf16* kr = (const bf16*)p.k + go;
    const bool ok = t < rows;
#pragma unroll 1
    for (int cb = 0; cb < 2; ++cb) {
      const int d0 = ch * 32 + cb * 16;  // first dim (within this CTA's 64)
      uint32_t xq[16], yq[16], xk[16], yk[16];
      tmem_ld16(lrow + kColXq + d0, xq);
      tmem_ld16(lrow + kColYq + d0, yq);
      tmem_ld16(lrow + kColXk + d0, xk);
      tmem_ld16(lrow + kColYk + d0, yk);
      uint4 qraw[2], kraw[2], inq[2], ink[2];
      const bool inp = ok && p.add_in_place && !p.add_dq;
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        qraw[h2] = ok ? __ldg(reinterpret_cast<const uint4*>(qr + d0) + h2) : make_uint4(0, 0, 0, 0);
        kraw[h2] = ok ? __ldg(reinterpret_cast<const uint4*>(kr + d0) + h2) : make_uint4(0, 0, 0, 0);
        inq[h2] = inp ? *(reinterpret_cast<const uint4*>((const bf16*)p.dq + go + d0) + h2)
                      : make_uint4(0, 0, 0, 0);
        ink[h2] = inp ? *(reinterpret_cast<const uint4*>((const bf16*)p.dk + go + d0) + h2)
                      : make_uint4(0, 0, 0, 0);
      }
      float cif[16], ckf[16], eqf[16];
#pragma unroll
      for (int x = 0; x < 4; ++x) {
        const float4 a = ld4(&sm.ci[d0 + 4 * x]), b = ld4(&sm.ck[d0 + 4 * x]), e = ld4(&sm.eq[t][d0 + 4 * x]);
        cif[4 * x] = a.x; cif[4 * x + 1] = a.y; cif[4 * x + 2] = a.z; cif[4 * x + 3] = a.w;
        ckf[4 * x] = b.x; ckf[4 * x + 1] = b.y; ckf[4 * x + 2] = b.z; ckf[4 * x + 3] = b.w;
        eqf[4 * x] = e.x; eqf[4 * x + 1] = e.y; eqf[4 * x + 2] = e.z; eqf[4 * x + 3] = e.w;
      }
      uint4 qfu[2], kfu[2];
#pragma unroll
      for (int h2 = 0; h2 < 2; ++h2) {
        qfu[h2] = *reinterpret_cast<const uint4*>(sm.qf + sw_chunk(t, d0 / 8 + h2));
        kfu[h2] = *reinterpret_cast<const uint4*>(sm.kf + sw_chunk(t, d0 / 8 + h2));
      }
      tmem_ld_wait();
      const uint32_t* qw = reinterpret_cast<const uint32_t*>(qraw);
      const uint32_t* kw = reinterpret_cast<const uint32_t*>(kraw);
      const uint32_t* iqw = reinterpret_cast<const uint32_t*>(inq);
      const uint32_t* ikw = reinterpret_cast<const uint32_t*>(ink);
      const uint32_t* qfw = reinterpret_cast<const uint32_t*>(qfu);
      const uint32_t* kfw = reinterpret_cast<const uint32_t*>(kfu);
      uint32_t oq[8], ok2[8];
      float pr[16];
#pragma unroll
      for (int e = 0; e < 16; e += 2) {
        const float2 qv = unpack_bf16(qw[e / 2]), kv = unpack_bf16(kw[e / 2]);
        const float2 qf2 = unpack_bf16(qfw[e / 2]), kf2 = unpack_bf16(kfw[e / 2]);
        float dqv[2], dkv[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const float aq = fmaf(cif[e + u], __uint_as_float(xq[e + u]), __uint_as_float(yq[e + u]));
          const float ak = fmaf(ckf[e + u], __uint_as_float(xk[e + u]), __uint_as_float(yk[e + u]));
          pr[e + u] = (u ? qf2.y : qf2.x) * aq - (u ? kf2.y : kf2.x) * ak;
          dqv[u] = fmaf(eqf[e + u], aq, btt * (u ? kv.y : kv.x));
          dkv[u] = __fdividef(ak, eqf[e + u]) + btt * (u ? qv.y : qv.x);
        }
        float2 aq2 = unpack_bf16(iqw[e / 2]), ak2 = unpack_bf16(ikw[e / 2]);
        if (p.add_dq && ok) {
          const float2 a = *reinterpret_cast<const float2*>(&p.add_dq[go + d0 + e]);
          const float2 b = *reinterpret_cast<const float2*>(&p.add_dk[go + d0 + e]);
          aq2.x += a.x; aq2.y += a.y; ak2.x += b.x; ak2.y += b.y;
        }
        oq[e / 2] = pack_bf16(dqv[0] + aq2.x, dqv[1] + aq2.y);
        ok2[e / 2] = pack_bf16(dkv[0] + ak2.x, dkv[1] + ak2.y);
      }
      if (ok && alive) {
        uint4* dq = reinterpret_cast<uint4*>((bf16*)p.dq + go + d0);
        uint4* dk = reinterpret_cast<uint4*>((bf16*)p.dk + go + d0);
        dq[0] = make_uint4(oq[0], oq[1], oq[2], oq[3]);
        dq[1] = make_uint4(oq[4], oq[5], oq[6], oq[7]);
        dk[0] = make_uint4(ok2[0], ok2[1], ok2[2], ok2[3]);
        dk[1] = make_uint4(ok2[4], ok2[5], ok2[6], ok2[7]);
      }
#pragma unroll
      for (int e = 0; e < 16; e += 4)  // row-major [128][64], float4 groups rotated by row
        *reinterpret_cast<float4*>(&prod[t * DH + (((d0 + e) >> 2) ^ (t & 15)) * 4]) =
            make_float4(pr[e], pr[e + 1], pr[e + 2], pr[e + 3]);
    }
  }
  __syncthreads();  // every product staged
  // ---- dg: the reverse scan's value at the chunk's first row, minus the
  // running sum of the products over the rows before t --------------------
  {
    const float* gsp = p.gsp + ((size_t)bh * n64 + 2 * c) * D + i0;
    float loc[32];
    float run = 0.f;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const int t = qt * 32 + r;
      loc[r] = run;
      run += prod[t * DH + ((i >> 2) ^ (t & 15)) * 4 + (i & 3)];
    }
    float* qtot = reinterpret_cast<float*>(sm.eq);  // [4][64] totals (Eq is spent)
    qtot[qt * DH + i] = run;
    __syncthreads();
    float base = __ldg(gsp + i);
#pragma unroll
    for (int q2 = 0; q2 < 4; ++q2)
      if (q2 < qt) base -= qtot[q2 * DH + i];
    float* dg = p.dg + tk0 + (size_t)c0 * D + i0 + i;
#pragma unroll
    for (int r = 0; r < 32; ++r) {
      const int t = qt * 32 + r;
      if (t < rows && alive) dg[(size_t)t * D] = base - loc[r];
    }
  }

  // ---- dv: row s, value columns [64 ch, 64 ch + 64); the peer's half goes to
  // its exchange tile, this CTA's half waits for the peer's share ------------
  if (tid == 0 && alive) alive = mbar_wait(bar_c, 0, p.status);
  alive = __syncthreads_and(alive);
  tc_fence_after();
  // both CTAs' last MMA (which reads dO) is done before either writes into the
  // other's dO tile
  cluster.sync();
  float* xch = reinterpret_cast<float*>(sm.dO);  // [128][64] fp32 (dO is spent)
  if (ch != half) {
    float* peer = cluster.map_shared_rank(xch, half ^ 1);
#pragma unroll 1
    for (int cb = 0; cb < 2; ++cb) {
      uint32_t x[32];
      tmem_ld32(lrow + kColDV + ch * 64 + cb * 32, x);
      tmem_ld_wait();
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const int cl = cb * 32 + e;
        *reinterpret_cast<float4*>(&peer[row * DH + ((cl >> 2) ^ (row & 15)) * 4]) =
            make_float4(__uint_as_float(x[e]), __uint_as_float(x[e + 1]), __uint_as_float(x[e + 2]),
                        __uint_as_float(x[e + 3]));
      }
    }
  }
  cluster.sync();  // the peer's share has landed
  if (ch == half) {
    const int s = row;
    const size_t go = tk0 + (size_t)(c0 + s) * D + half * 64;
#pragma unroll 1
    for (int cb = 0; cb < 2; ++cb) {
      uint32_t x[32];
      tmem_ld32(lrow + kColDV + ch * 64 + cb * 32, x);
      tmem_ld_wait();
      if (!alive || s >= rows) continue;
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 32; e += 4) {
        const int cl = cb * 32 + e;
        const float4 pr = *reinterpret_cast<const float4*>(&xch[s * DH + ((cl >> 2) ^ (s & 15)) * 4]);
        float y[4] = {__uint_as_float(x[e]) + pr.x, __uint_as_float(x[e + 1]) + pr.y,
                      __uint_as_float(x[e + 2]) + pr.z, __uint_as_float(x[e + 3]) + pr.w};
        if (p.add_dv) {
          const float4 a = *reinterpret_cast<const float4*>(&p.add_dv[go + cl]);
          y[0] += a.x; y[1] += a.y; y[2] += a.z; y[3] += a.w;
        } else if (p.add_in_place) {
          const uint2 a = *reinterpret_cast<const uint2*>((const bf16*)p.dv + go + cl);
          const float2 a0 = unpack_bf16(a.x), a1 = unpack_bf16(a.y);
          y[0] += a0.x; y[1] += a0.y; y[2] += a1.x; y[3] += a1.y;
        }
        pk[e / 2] = pack_bf16(y[0], y[1]);
        pk[e / 2 + 1] = pack_bf16(y[2], y[3]);
      }
      uint4* dst = reinterpret_cast<uint4*>((bf16*)p.dv + go + cb * 32);
#pragma unroll
      for (int x4 = 0; x4 < 4; ++x4) dst[x4] = make_uint4(pk[4 * x4], pk[4 * x4 + 1], pk[4 * x4 + 2], pk[4 * x4 + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool gla_bwd_tc_supported(const GlaBwdParams& p) {
  return p.dkd == D && p.dvd == D && p.gz == nullptr && p.g != nullptr && p.gin16 && p.gsp;
}

int gla_bwd_tc_nchunks(int T) { return (T + C - 1) / C; }

cudaError_t launch_gla_bwd_tc(const GlaBwdParams& p, int* flags, cudaStream_t s) {
  const int n128 = (p.T + C - 1) / C, n64 = (p.T + 63) / 64;
  if (p.B * p.H == 0 || n128 == 0) return cudaSuccess;
  if (2 * (size_t)n128 * p.B * p.H > 0x7fffffffu) return cudaErrorInvalidConfiguration;
  const size_t bytes = sizeof(TcSmem) + 1024;  // + room to align the base to 1024
  cudaError_t e = cudaFuncSetAttribute(gla_bwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes);
  if (e != cudaSuccess) return e;
  GlaBwdParams pp = p;
  pp.status = device_status_word();
  if (pp.status == nullptr) return cudaErrorInvalidDevicePointer;
  const uint64_t bh = (uint64_t)p.B * p.H;
  CUtensorMap tq, tk, tv, tdo, tsp, tgi;
  if (!tma_map_rows128(&tq, p.q, p.T, bh, C) || !tma_map_rows128(&tk, p.k, p.T, bh, C) ||
      !tma_map_rows128(&tv, p.v, p.T, bh, C) || !tma_map_rows128(&tdo, p.dO, p.T, bh, C) ||
      !tma_map_rows128(&tsp, p.states16, (uint64_t)n64 * D, bh, DH) ||
      !tma_map_rows128(&tgi, p.gin16, (uint64_t)n64 * D, bh, DH))
    return cudaErrorInvalidValue;
  {
    ScopedTiming tm("gla_bwd_chunks_tc", s);
    gla_bwd_tc_kernel<<<(unsigned)(2 * (size_t)n128 * p.B * p.H), NTH, bytes, s>>>(pp, flags, tq, tk, tv,
                                                                                   tdo, tsp, tgi);
  }
  return cudaGetLastError();
}

}  // namespace lz
