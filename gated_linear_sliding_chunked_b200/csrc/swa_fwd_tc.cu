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
//   1. cp.async: Q, meta K and the K tiles (group 0); V tiles, meta V (1)
//   2. thread 0: S_meta = Q MK^T, S_j = Q K_j^T (K = 16 per MMA), commit
//   3. per row: max over S read from TMEM, then P = exp2(S - max) as bf16
//      into shared memory over the spent K tiles, row sum l
//   4. thread 0: O = P_meta MV + sum_j P_j V_j, commit
//   5. O / l -> bf16 rows, lse = (max + log2 l) ln 2.
// Operands use the no-swizzle canonical layouts of tc05.cuh: Q, K, MK, P
// K-major; V and MV MN-major (their rows are keys, the reduction dim).
#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"
#include "tc05.cuh"

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

struct TcSmem {
  uint8_t q[QR * D * 2];
  uint8_t k[MAXT][kTileBytes];  // K_j, then P_j
  uint8_t v[MAXT][kTileBytes];
  uint8_t mk[MTT * D * 2];      // meta K, then P_meta
  uint8_t mv[MTT * D * 2];
  float rmax[2][QR];             // the two column halves' row max ...
  float rsum[2][QR];             // ... and row sum
  uint64_t bar_s;
  uint64_t bar_o;
  uint32_t tmem_base;
};
static_assert(sizeof(TcSmem) <= 232448, "shared memory per block exceeds 227 KB");
static_assert(kColS0 + MAXT * KT <= kTmemCols, "score tiles exceed the TMEM allocation");

// byte offset of 16-byte chunk kc of row `row` in a K-major [rows][128] tile
__device__ __forceinline__ uint32_t kmaj(int row, int kc) {
  return (uint32_t)((row >> 3) * 2048 + kc * 128 + (row & 7) * 16);
}
// byte offset of chunk dc of key row kr in an MN-major [keys][128] tile whose
// 8-element column groups are `sbo` bytes apart
__device__ __forceinline__ uint32_t mnmaj(int kr, int dc, int sbo) {
  return (uint32_t)(dc * sbo + (kr >> 3) * 128 + (kr & 7) * 16);
}

__global__ void __launch_bounds__(NTH, 1) swa_fwd_tc_kernel(SwaFwdParams p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  TcSmem& sm = *reinterpret_cast<TcSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int bh = blockIdx.y, h = bh % p.H;
  const int T = p.T, w = p.w, M = p.M;
  const int t0 = blockIdx.x * QR;
  const bf16* q = (const bf16*)p.q + (size_t)bh * T * D;
  const bf16* k = (const bf16*)p.k + (size_t)bh * T * D;
  const bf16* v = (const bf16*)p.v + (size_t)bh * T * D;
  const int lo = max(0, t0 - w + 1);
  const int hi = min(T - 1, t0 + QR - 1);
  const int ntiles = (hi - lo + KT) / KT;  // 1..MAXT (w <= kMaxWindow)
  const bool has_meta = M > 0;
  const bool meta_v = has_meta && p.mv != nullptr;

  const uint32_t s_q = smem_u32(sm.q), s_k = smem_u32(sm.k[0]), s_v = smem_u32(sm.v[0]);
  const uint32_t s_mk = smem_u32(sm.mk), s_mv = smem_u32(sm.mv);
  const uint32_t bar_s = smem_u32(&sm.bar_s), bar_o = smem_u32(&sm.bar_o);

  if (warp == 0) tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
  if (tid == 0) {
    mbar_init(bar_s, 1);
    mbar_init(bar_o, 1);
    mbar_init_fence();
  }

  // ---- loads: 8 consecutive threads fill the 8 rows of one core matrix ----
  for (int x = tid; x < QR * 16; x += NTH) {
    const int row = ((x >> 7) << 3) | (x & 7), kc = (x >> 3) & 15;
    const bool ok = t0 + row < T;
    cp_async16(sm.q + kmaj(row, kc), q + (size_t)(ok ? t0 + row : 0) * D + kc * 8, ok ? 16 : 0);
  }
  if (has_meta) {
    const bf16* mk = (const bf16*)p.mk + (size_t)h * M * D;
    for (int x = tid; x < MTT * 16; x += NTH) {
      const int row = ((x >> 7) << 3) | (x & 7), kc = (x >> 3) & 15;
      const bool ok = row < M;
      cp_async16(sm.mk + kmaj(row, kc), mk + (size_t)(ok ? row : 0) * D + kc * 8, ok ? 16 : 0);
    }
  }
  for (int j = 0; j < ntiles; ++j)
    for (int x = tid; x < KT * 16; x += NTH) {
      const int row = ((x >> 7) << 3) | (x & 7), kc = (x >> 3) & 15;
      const int key = lo + j * KT + row;
      const bool ok = key <= hi;
      cp_async16(sm.k[j] + kmaj(row, kc), k + (size_t)(ok ? key : 0) * D + kc * 8, ok ? 16 : 0);
    }
  cp_async_commit();
  for (int j = 0; j < ntiles; ++j)
    for (int x = tid; x < KT * 16; x += NTH) {
      const int dc = ((x >> 7) << 1) | (x & 1), kr = (((x >> 4) & 7) << 3) | ((x >> 1) & 7);
      const int key = lo + j * KT + kr;
      const bool ok = key <= hi;
      cp_async16(sm.v[j] + mnmaj(kr, dc, 1024), v + (size_t)(ok ? key : 0) * D + dc * 8, ok ? 16 : 0);
    }
  if (meta_v) {
    const bf16* mv = (const bf16*)p.mv + (size_t)h * M * D;
    for (int x = tid; x < MTT * 16; x += NTH) {
      const int dc = ((x >> 5) << 1) | (x & 1), kr = (((x >> 4) & 1) << 3) | ((x >> 1) & 7);
      const bool ok = kr < M;
      cp_async16(sm.mv + mnmaj(kr, dc, 256), mv + (size_t)(ok ? kr : 0) * D + dc * 8, ok ? 16 : 0);
    }
  }
  cp_async_commit();

  cp_async_wait<1>();
  fence_async_smem();
  tc_fence_before();
  __syncthreads();  // Q, K tiles, meta K, barriers and the TMEM address are visible
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // ---- scores ----------------------------------------------------------------
  if (tid == 0) {
    constexpr uint32_t idS = idesc_bf16(QR, KT, false), idM = idesc_bf16(QR, MTT, false);
#pragma unroll 1
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint64_t a = sdesc(s_q + kk * 256, 128, 2048);
      if (has_meta) mma_bf16_ss(tmem + kColSM, a, sdesc(s_mk + kk * 256, 128, 2048), idM, kk > 0);
      for (int j = 0; j < ntiles; ++j)
        mma_bf16_ss(tmem + kColS0 + j * KT, a, sdesc(s_k + j * kTileBytes + kk * 256, 128, 2048), idS,
                    kk > 0);
    }
    mma_commit(bar_s);
  }
  cp_async_wait<0>();
  fence_async_smem();  // V tiles and meta V, for the second set of MMAs

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
  bool alive = mbar_wait(bar_s, 0, p.status);
  tc_fence_after();

  float mx = -INFINITY;
  if (has_meta && hf == 0) {
    uint32_t r[16];
    tmem_ld16(lrow + kColSM, r);
    tmem_ld_wait();
#pragma unroll
    for (int c = 0; c < MTT; ++c)
      if (c < M && row_ok) mx = fmaxf(mx, __uint_as_float(r[c]) * c2);
  }
  for (int j = 0; j < ntiles; ++j) {
    uint32_t r[32];
    tmem_ld32(lrow + kColS0 + j * KT + hf * 32, r);
    tmem_ld_wait();
    const int kb = lo + j * KT + hf * 32 - kmin;
#pragma unroll
    for (int c = 0; c < 32; ++c)
      if ((unsigned)(kb + c) < span) mx = fmaxf(mx, __uint_as_float(r[c]) * c2);
  }
  sm.rmax[hf][m] = mx;
  __syncthreads();
  mx = fmaxf(sm.rmax[0][m], sm.rmax[1][m]);
  const float base = mx == -INFINITY ? 0.f : mx;

  float l = 0.f;
  if (has_meta && hf == 0) {
    uint32_t r[16];
    tmem_ld16(lrow + kColSM, r);
    tmem_ld_wait();
    uint32_t pk[8];
#pragma unroll
    for (int c = 0; c < MTT; c += 2) {
      const float p0 = (c < M && row_ok) ? exp2f(fmaf(__uint_as_float(r[c]), c2, -base)) : 0.f;
      const float p1 = (c + 1 < M && row_ok) ? exp2f(fmaf(__uint_as_float(r[c + 1]), c2, -base)) : 0.f;
      l += p0 + p1;
      pk[c / 2] = pack_bf16(p0, p1);
    }
    // P_meta: K-major [128 rows][16], 8-row groups 256 bytes apart
#pragma unroll
    for (int kc = 0; kc < 2; ++kc)
      *reinterpret_cast<uint4*>(sm.mk + (m >> 3) * 256 + kc * 128 + (m & 7) * 16) =
          make_uint4(pk[4 * kc], pk[4 * kc + 1], pk[4 * kc + 2], pk[4 * kc + 3]);
  }
  for (int j = 0; j < ntiles; ++j) {
    uint32_t r[32];
    tmem_ld32(lrow + kColS0 + j * KT + hf * 32, r);
    tmem_ld_wait();
    const int kb = lo + j * KT + hf * 32 - kmin;
    uint32_t pk[16];
#pragma unroll
    for (int c = 0; c < 32; c += 2) {
      const float p0 = (unsigned)(kb + c) < span ? exp2f(fmaf(__uint_as_float(r[c]), c2, -base)) : 0.f;
      const float p1 =
          (unsigned)(kb + c + 1) < span ? exp2f(fmaf(__uint_as_float(r[c + 1]), c2, -base)) : 0.f;
      l += p0 + p1;
      pk[c / 2] = pack_bf16(p0, p1);
    }
    // P_j: K-major [128 rows][64 keys], 8-row groups 1024 bytes apart
#pragma unroll
    for (int kc = 0; kc < 4; ++kc)
      *reinterpret_cast<uint4*>(sm.k[j] + (m >> 3) * 1024 + (hf * 4 + kc) * 128 + (m & 7) * 16) =
          make_uint4(pk[4 * kc], pk[4 * kc + 1], pk[4 * kc + 2], pk[4 * kc + 3]);
  }
  sm.rsum[hf][m] = l;
  fence_async_smem();
  tc_fence_before();
  alive = __syncthreads_and(alive);
  l = sm.rsum[0][m] + sm.rsum[1][m];

  // ---- O = P_meta MV + sum_j P_j V_j ------------------------------------------
  if (tid == 0 && alive) {
    tc_fence_after();
    constexpr uint32_t idO = idesc_bf16(QR, D, true);
    uint32_t acc = 0;
    if (meta_v) {
      mma_bf16_ss(tmem + kColO, sdesc(s_mk, 128, 256), sdesc(s_mv, 128, 256), idO, 0);
      acc = 1;
    }
    for (int j = 0; j < ntiles; ++j)
#pragma unroll
      for (int kk = 0; kk < KT / 16; ++kk) {
        mma_bf16_ss(tmem + kColO, sdesc(s_k + j * kTileBytes + kk * 256, 128, 1024),
                    sdesc(s_v + j * kTileBytes + kk * 256, 128, 1024), idO, acc);
        acc = 1;
      }
    mma_commit(bar_o);
  }
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
  const size_t bytes = sizeof(TcSmem);
  cudaError_t e = cudaFuncSetAttribute(swa_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes);
  if (e != cudaSuccess) return e;
  SwaFwdParams pp = p;
  pp.status = device_status_word();
  if (pp.status == nullptr) return cudaErrorInvalidDevicePointer;
  dim3 grid((p.T + QR - 1) / QR, p.B * p.H);
  {
    ScopedTiming tm("swa_fwd_tc", s);
    swa_fwd_tc_kernel<<<grid, NTH, bytes, s>>>(pp);
  }
  return cudaGetLastError();
}

}  // namespace lz
