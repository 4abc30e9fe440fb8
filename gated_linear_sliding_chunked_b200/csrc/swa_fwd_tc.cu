// Sliding-window softmax attention with meta-memory sinks on the Blackwell
// tensor cores: tcgen05.mma with the accumulators in tensor memory (bf16
// I/O, fp32 accumulation, dk = dv = 128).
//
// Lizard technical summary, section 2a ("anchor window attention"): query t
// attends to keys j in [t-w+1, t] and to the M meta tokens, which always sit
// in the softmax denominator (and add p_m mv_m to the numerator when meta
// values are given).
//
// One CTA = 128 query rows of one (batch, head); 8 warps, two threads per
// query row (each takes half of every key tile's columns).  With w <= 129 the rows' key band spans at most 255 keys, so
// the scores of the whole band (four 64-key tiles) and of the meta tile fit
// in TMEM next to the output accumulator:
//   columns [0,128) O,  [128,144) S_meta,  [192 + 64 j, 256 + 64 j) S_j.
// The row maximum is therefore exact before any exponent is taken and O is
// never rescaled:
//   1. TMA (one thread, 128-byte swizzled boxes of 64 dims): Q, meta K and
//      the K tiles on one mbarrier; V tiles and meta V on a second
//   2. thread 0: S_meta = Q MK^T, S_j = Q K_j^T (K = 16 per MMA), commit
//   3. per row: max over S read from TMEM, then P = exp2(S - max) as bf16
//      into shared memory over the spent K tiles, row sum l
//   4. thread 0: O = P_meta MV + sum_j P_j V_j, commit
//   5. O / l -> bf16 rows, lse = (max + log2 l) ln 2.
// Q, K, MK (K-major) and V, MV (MN-major: their rows are keys, the reduction
// dim) sit in shared memory as the TMA writes them, 128-byte swizzled; P is
// written by the threads in the no-swizzle K-major layout (tc05.cuh).
#include <cstddef>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"
#include "tc05.cuh"
#include "tma_host.h"

namespace lz {
namespace {

constexpr int QR = 128;    // query rows per CTA
constexpr int KT = 64;     // keys per tile
constexpr int MAXT = 4;    // key tiles held at once
constexpr int MTT = 16;    // meta tile (M <= 16)
constexpr int D = 128;
constexpr int NTH = 256;
constexpr int kMaxWindow = MAXT * KT - QR + 1;  // 129
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColO = 0, kColSM = 128, kColS0 = 192;
constexpr uint32_t kTileBytes = KT * D * 2;  // 16 KB
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

constexpr uint32_t kHalf = 64 * 2;  // bytes of one swizzled row (64 dims)

// Every array starts 1024-byte aligned (the 128-byte swizzle atom).
struct TcSmem {
  uint8_t q[2][QR * kHalf];        // dims [0,64), [64,128): 128 rows each
  uint8_t k[MAXT][2][KT * kHalf];  // K_j halves; then P_j (16 KB, no swizzle)
  uint8_t v[MAXT][2][KT * kHalf];
  uint8_t mk[2][MTT * kHalf];      // meta K halves; then P_meta (4 KB)
  uint8_t mv[2][MTT * kHalf];
  float rmax[2][QR];               // the two column halves' row max ...
  float rsum[2][QR];               // ... and row sum
  uint64_t bar_ld0;                // Q, meta K, K tiles landed
  uint64_t bar_ld1;                // V tiles, meta V landed
  uint64_t bar_s;
  uint64_t bar_o;
  uint32_t tmem_base;
};
static_assert(sizeof(TcSmem) + 1024 <= 232448, "shared memory per block exceeds 227 KB");
static_assert(kColS0 + MAXT * KT <= kTmemCols, "score tiles exceed the TMEM allocation");
static_assert(offsetof(TcSmem, k) % 1024 == 0 && offsetof(TcSmem, v) % 1024 == 0 &&
                  offsetof(TcSmem, mk) % 1024 == 0 && offsetof(TcSmem, mv) % 1024 == 0,
              "swizzled tiles must be 1024-byte aligned");

__global__ void __launch_bounds__(NTH, 1)
    swa_fwd_tc_kernel(SwaFwdParams p, const __grid_constant__ CUtensorMap tq,
                      const __grid_constant__ CUtensorMap tk, const __grid_constant__ CUtensorMap tv,
                      const __grid_constant__ CUtensorMap tmk, const __grid_constant__ CUtensorMap tmv) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  TcSmem& sm = *reinterpret_cast<TcSmem*>(smem_raw + ((1024u - (raw & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5;
  const int bh = blockIdx.y, h = bh % p.H;
  const int T = p.T, w = p.w, M = p.M;
  const int t0 = blockIdx.x * QR;
  const int lo = max(0, t0 - w + 1);
  const int hi = min(T - 1, t0 + QR - 1);
  const int ntiles = (hi - lo + KT) / KT;  // 1..MAXT (w <= kMaxWindow)
  const bool has_meta = M > 0;
  const bool meta_v = has_meta && p.mv != nullptr;

  const uint32_t s_q = smem_u32(sm.q), s_k = smem_u32(sm.k), s_v = smem_u32(sm.v);
  const uint32_t s_mk = smem_u32(sm.mk), s_mv = smem_u32(sm.mv);
  const uint32_t bar_ld0 = smem_u32(&sm.bar_ld0), bar_ld1 = smem_u32(&sm.bar_ld1);
  const uint32_t bar_s = smem_u32(&sm.bar_s), bar_o = smem_u32(&sm.bar_o);

  if (warp == 0) tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
  if (tid == 0) {
    mbar_init(bar_ld0, 1);
    mbar_init(bar_ld1, 1);
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    mbar_init_fence();
  }
  tc_fence_before();
  __syncthreads();  // barriers and the TMEM address are visible
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // ---- loads: one thread issues the tensor copies (x = 0 or 64 dims) -------
  if (tid == 0) {
    mbar_expect_tx(bar_ld0, 2 * QR * kHalf + ntiles * 2 * KT * kHalf + (has_meta ? 2 * MTT * kHalf : 0));
    for (int hf = 0; hf < 2; ++hf) {
      tma_load_3d(s_q + hf * QR * kHalf, &tq, bar_ld0, hf * 64, t0, bh);
      if (has_meta) tma_load_3d(s_mk + hf * MTT * kHalf, &tmk, bar_ld0, hf * 64, 0, h);
      for (int j = 0; j < ntiles; ++j)
        tma_load_3d(s_k + (2 * j + hf) * KT * kHalf, &tk, bar_ld0, hf * 64, lo + j * KT, bh);
    }
    mbar_expect_tx(bar_ld1, ntiles * 2 * KT * kHalf + (meta_v ? 2 * MTT * kHalf : 0));
    for (int hf = 0; hf < 2; ++hf) {
      if (meta_v) tma_load_3d(s_mv + hf * MTT * kHalf, &tmv, bar_ld1, hf * 64, 0, h);
      for (int j = 0; j < ntiles; ++j)
        tma_load_3d(s_v + (2 * j + hf) * KT * kHalf, &tv, bar_ld1, hf * 64, lo + j * KT, bh);
    }
  }
  bool alive = mbar_wait(bar_ld0, 0, p.status);

  // ---- scores ----------------------------------------------------------------
  if (tid == 0 && alive) {
    constexpr uint32_t idS = idesc_bf16(QR, KT, false), idM = idesc_bf16(QR, MTT, false);
#pragma unroll 1
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t hf = kk >> 2, ko = (kk & 3) * 32;  // dim half, byte offset in the row
      const uint64_t a = sdesc_sw128(s_q + hf * QR * kHalf + ko, 16, 1024);
      if (has_meta)
        mma_bf16_ss(tmem + kColSM, a, sdesc_sw128(s_mk + hf * MTT * kHalf + ko, 16, 1024), idM, kk > 0);
      for (int j = 0; j < ntiles; ++j)
        mma_bf16_ss(tmem + kColS0 + j * KT, a, sdesc_sw128(s_k + (2 * j + hf) * KT * kHalf + ko, 16, 1024),
                    idS, kk > 0);
    }
    mma_commit(bar_s);
  }

  // ---- softmax: row m = tid % 128, column half hf = tid / 128 ---------------
  // Warps w and w + 4 read the same TMEM lanes (32 (w % 4) ..), each half of
  // every 64-key tile; the row's two threads combine max and sum in shared
  // memory.
  const int m = tid & (QR - 1), hf = tid >> 7;
  const int t = t0 + m;
  const bool row_ok = t < T;
  // visible window keys of row t: [t - w + 1, t] (meta tokens separately)
  const int kmin = max(0, t - w + 1);
  const unsigned span = row_ok ? (unsigned)(t - kmin + 1) : 0u;
  const float c2 = p.scale * kLog2e;  // logits in log2 units
  const uint32_t lrow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  alive = alive && mbar_wait(bar_s, 0, p.status);
  tc_fence_after();

  // this thread's scores: 32 columns of every key tile (and the meta tile),
  // read from TMEM once and kept in registers for both passes
  uint32_t sr[MAXT][32], smr[16];
  if (has_meta && hf == 0) tmem_ld16(lrow + kColSM, smr);
#pragma unroll
  for (int j = 0; j < MAXT; ++j)
    if (j < ntiles) tmem_ld32(lrow + kColS0 + j * KT + hf * 32, sr[j]);
  tmem_ld_wait();

  float mx = -INFINITY;
  if (has_meta && hf == 0) {
#pragma unroll
    for (int c = 0; c < MTT; ++c)
      if (c < M && row_ok) mx = fmaxf(mx, __uint_as_float(smr[c]) * c2);
  }
#pragma unroll
  for (int j = 0; j < MAXT; ++j) {
    if (j >= ntiles) break;
    const int kb = lo + j * KT + hf * 32 - kmin;
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if ((unsigned)(kb + c) < span) mx = fmaxf(mx, __uint_as_float(sr[j][c]) * c2);
  }
  sm.rmax[hf][m] = mx;
  __syncthreads();
  mx = fmaxf(sm.rmax[0][m], sm.rmax[1][m]);
  const float base = mx == -INFINITY ? 0.f : mx;

  float l = 0.f;
  if (has_meta && hf == 0) {
    uint32_t pk[8];
#pragma unroll
    for (int c = 0; c < MTT; c += 2) {
      const float p0 = (c < M && row_ok) ? exp2f(fmaf(__uint_as_float(smr[c]), c2, -base)) : 0.f;
      const float p1 = (c + 1 < M && row_ok) ? exp2f(fmaf(__uint_as_float(smr[c + 1]), c2, -base)) : 0.f;
      l += p0 + p1;
      pk[c / 2] = pack_bf16(p0, p1);
    }
    // P_meta: K-major [128 rows][16], 8-row groups 256 bytes apart
#pragma unroll
    for (int kc = 0; kc < 2; ++kc)
      *reinterpret_cast<uint4*>(&sm.mk[0][0] + (m >> 3) * 256 + kc * 128 + (m & 7) * 16) =
          make_uint4(pk[4 * kc], pk[4 * kc + 1], pk[4 * kc + 2], pk[4 * kc + 3]);
  }
#pragma unroll
  for (int j = 0; j < MAXT; ++j) {
    if (j >= ntiles) break;
    const int kb = lo + j * KT + hf * 32 - kmin;
    uint32_t pk[16];
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
      const float p0 = (unsigned)(kb + c) < span ? exp2f(fmaf(__uint_as_float(sr[j][c]), c2, -base)) : 0.f;
      const float p1 =
          (unsigned)(kb + c + 1) < span ? exp2f(fmaf(__uint_as_float(sr[j][c + 1]), c2, -base)) : 0.f;
      l += p0 + p1;
      pk[c / 2] = pack_bf16(p0, p1);
    }
    // P_j: K-major [128 rows][64 keys], 8-row groups 1024 bytes apart
#pragma unroll
    for (int kc = 0; kc < 4; ++kc)
      *reinterpret_cast<uint4*>(&sm.k[j][0][0] + (m >> 3) * 1024 + (hf * 4 + kc) * 128 + (m & 7) * 16) =
          make_uint4(pk[4 * kc], pk[4 * kc + 1], pk[4 * kc + 2], pk[4 * kc + 3]);
  }
  sm.rsum[hf][m] = l;
  fence_async_smem();
  tc_fence_before();
  alive = __syncthreads_and(alive);
  l = sm.rsum[0][m] + sm.rsum[1][m];

  // ---- O = P_meta MV + sum_j P_j V_j ------------------------------------------
  if (tid == 0 && alive) alive = mbar_wait(bar_ld1, 0, p.status);
  if (tid == 0 && alive) {
    tc_fence_after();
    constexpr uint32_t idO = idesc_bf16(QR, D, true);
    uint32_t acc = 0;
    if (meta_v) {  // B = MV, MN-major: 16 meta rows, the dim halves 2 KB apart
      mma_bf16_ss(tmem + kColO, sdesc(s_mk, 128, 256), sdesc_sw128(s_mv, MTT * kHalf, 1024), idO, 0);
      acc = 1;
    }
    for (int j = 0; j < ntiles; ++j)
#pragma unroll
      for (int kk = 0; kk < KT / 16; ++kk) {  // B = V_j, MN-major: 16 keys = 2048 bytes per step
        mma_bf16_ss(tmem + kColO, sdesc(s_k + j * kTileBytes + kk * 256, 128, 1024),
                    sdesc_sw128(s_v + j * kTileBytes + kk * 2048, KT * kHalf, 1024), idO, acc);
        acc = 1;
      }
    mma_commit(bar_o);
  }
  alive = __syncthreads_and(alive);
  if (alive) alive = mbar_wait(bar_o, 0, p.status);
  tc_fence_after();

  // ---- epilogue: O / l, this thread's 64 columns --------------------------------
  const float inv = l > 0.f ? 1.f / l : 0.f;
  const size_t off = ((size_t)bh * T + t) * D;
#pragma unroll 1
  for (int c0 = hf * 64; c0 < hf * 64 + 64; c0 += 32) {
    uint32_t r[32];
    tmem_ld32(lrow + kColO + c0, r);
    tmem_ld_wait();
    if (!row_ok || !alive) continue;
    if (p.o) {
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2)
        pk[c / 2] = pack_bf16(__uint_as_float(r[c]) * inv, __uint_as_float(r[c + 1]) * inv);
      uint4* dst = reinterpret_cast<uint4*>((bf16*)p.o + off + c0);
#pragma unroll
      for (int x = 0; x < 4; ++x) dst[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
    }
    if (p.o_f32) {
      float4* dst = reinterpret_cast<float4*>(p.o_f32 + off + c0);
#pragma unroll
      for (int x = 0; x < 8; ++x)
        dst[x] = make_float4(__uint_as_float(r[4 * x]) * inv, __uint_as_float(r[4 * x + 1]) * inv,
                             __uint_as_float(r[4 * x + 2]) * inv, __uint_as_float(r[4 * x + 3]) * inv);
    }
  }
  if (hf == 0 && row_ok && alive && p.lse) p.lse[(size_t)bh * T + t] = (mx + log2f(l)) * kLn2;

  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool swa_fwd_tc_supported(int dk, int dv, bool bf16, int w) {
  return bf16 && dk == D && dv == D && w <= kMaxWindow;
}

cudaError_t launch_swa_fwd_tc(const SwaFwdParams& p, cudaStream_t s) {
  if (p.B * p.H == 0 || p.T == 0) return cudaSuccess;
  const size_t bytes = sizeof(TcSmem) + 1024;  // + room to align the base to 1024
  cudaError_t e = cudaFuncSetAttribute(swa_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes);
  if (e != cudaSuccess) return e;
  SwaFwdParams pp = p;
  pp.status = device_status_word();
  if (pp.status == nullptr) return cudaErrorInvalidDevicePointer;
  const uint64_t bh = (uint64_t)p.B * p.H;
  CUtensorMap tq, tk, tv, tmk, tmv;
  if (!tma_map_rows128(&tq, p.q, p.T, bh, QR) || !tma_map_rows128(&tk, p.k, p.T, bh, KT) ||
      !tma_map_rows128(&tv, p.v, p.T, bh, KT))
    return cudaErrorInvalidValue;
  tmk = tq;
  tmv = tq;
  if (p.M > 0 && !tma_map_rows128(&tmk, p.mk, p.M, p.H, MTT)) return cudaErrorInvalidValue;
  if (p.M > 0 && p.mv && !tma_map_rows128(&tmv, p.mv, p.M, p.H, MTT)) return cudaErrorInvalidValue;
  dim3 grid((p.T + QR - 1) / QR, p.B * p.H);
  {
    ScopedTiming tm("swa_fwd_tc", s);
    swa_fwd_tc_kernel<<<grid, NTH, bytes, s>>>(pp, tq, tk, tv, tmk, tmv);
  }
  return cudaGetLastError();
}

}  // namespace lz
