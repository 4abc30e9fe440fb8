// Query side of the window + meta softmax backward on the Blackwell tensor
// cores: tcgen05.mma with dq and the meta-token gradients accumulated in
// tensor memory, operands brought in by TMA (bf16 I/O, fp32 accumulation,
// dk = dv = 128, w <= 129, the forward's window output given).
//
// Lizard technical summary, section 2a: query t sees keys j in [t-w+1, t] and
// the M meta tokens.  With P = exp(logit - lse), the window branch's share
// gscale * dO of the output gradient and D_t = dO_t . o_t (o the forward's
// window output):
//   dS = gscale * P * (dO V^T - D),   dq = scale * (dS K + dS_meta MK),
//   dmeta_k = scale * dS_meta^T Q,    dmeta_v = gscale * P_meta^T dO.
// One CTA = one slab of 256 query rows of one (batch, head), walked as two
// 128-row tiles (the meta-gradient and dalpha partials are per slab, summed
// by the fixed-order reduction).  Per tile, the rows' key band spans at most
// 255 keys (four 64-key tiles):
//   TMA (one thread): Q, dO, the K tiles and the meta K / V on one barrier,
//                     the V tiles on a second
//   thread 0: S_meta = Q MK^T, dP_meta = dO MV^T, then for key tiles 0 and 1
//             S_j = Q K_j^T, dP_j = dO V_j^T into a double-buffered TMEM pair
//   per key tile j: each row's two threads read 32 columns of S_j and dP_j,
//             form dS_j (bf16) over the spent V_j tile; thread 0 issues
//             dq += dS_j K_j and the scores of tile j + 2 into the freed pair
//   after the band: dq += dS_meta MK; dmeta_k^T += Q^T dS_meta and
//             dmeta_v^T += dO^T P_meta (Q, dO read transposed as MN-major A)
// Tensor memory: [0,128) dq, [128,384) two (S_j, dP_j) pairs, [384,400)
// S_meta, [400,416) dP_meta, [416,432) dmeta_k^T, [432,448) dmeta_v^T.
#include <cstddef>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"
#include "tc05.cuh"
#include "tma_host.h"

namespace lz {
namespace {

constexpr int QR = 128;    // query rows per tile
constexpr int KT = 64;     // keys per tile
constexpr int MAXT = 4;    // key tiles of one query tile's band
constexpr int MTT = 16;    // meta tile (M <= 16)
constexpr int D = 128;
constexpr int NTH = 256;
constexpr int kMaxWindow = MAXT * KT - QR + 1;  // 129
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDQ = 0, kColS = 128, kColSM = 384, kColDPM = 400, kColGK = 416, kColGV = 432;
constexpr uint32_t kHalf = 64 * 2;              // bytes of one swizzled row (64 dims)
constexpr uint32_t kQBox = QR * kHalf;          // [128 rows][64] bf16
constexpr uint32_t kKBox = KT * kHalf;          // [64 rows][64]
constexpr uint32_t kMBox = MTT * kHalf;         // [16 rows][64]
constexpr float kLog2e = 1.4426950408889634f;

struct QtcSmem {
  uint8_t q[2][kQBox];              // dim halves
  uint8_t dO[2][kQBox];
  uint8_t k[MAXT][2][kKBox];
  uint8_t v[MAXT][2][kKBox];        // V_j; then dS_j (bf16, K-major no swizzle [128][64])
  uint8_t mk[2][kMBox];
  uint8_t mv[2][kMBox];
  uint8_t dsm[QR * MTT * 2];        // dS_meta, K-major [128 rows][16]
  uint8_t dsmT[MTT * QR * 2];       // dS_meta^T, K-major [16 rows][128]
  uint8_t pmT[MTT * QR * 2];        // P_meta^T
  float lse2[QR];
  float drow[QR];
  float dsum[NTH / 32];
  uint64_t bar_ld0, bar_ld1, bar_s[2], bar_f;
  uint32_t tmem_base;
};
static_assert(sizeof(QtcSmem) + 1024 <= 232448, "shared memory per block exceeds 227 KB");
static_assert(offsetof(QtcSmem, dO) % 1024 == 0 && offsetof(QtcSmem, k) % 1024 == 0 &&
                  offsetof(QtcSmem, v) % 1024 == 0 && offsetof(QtcSmem, mk) % 1024 == 0 &&
                  offsetof(QtcSmem, mv) % 1024 == 0 && offsetof(QtcSmem, dsm) % 1024 == 0,
              "swizzled tiles must be 1024-byte aligned");

__global__ void __launch_bounds__(NTH, 1)
    swa_bwd_q_tc_kernel(SwaBwdParams p, const __grid_constant__ CUtensorMap tq,
                        const __grid_constant__ CUtensorMap tdo, const __grid_constant__ CUtensorMap tk,
                        const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tmk,
                        const __grid_constant__ CUtensorMap tmv) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  QtcSmem& sm = *reinterpret_cast<QtcSmem*>(smem_raw + ((1024u - (raw & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int h = blockIdx.x, b = blockIdx.y, slab = blockIdx.z;
  const int H = p.H, T = p.T, w = p.w, M = p.M;
  const int bh = b * H + h;
  const bool has_meta = M > 0, meta_v = has_meta && p.mv != nullptr;
  const float c2 = p.scale * kLog2e;

  const uint32_t s_q = smem_u32(sm.q), s_do = smem_u32(sm.dO), s_k = smem_u32(sm.k);
  const uint32_t s_v = smem_u32(sm.v), s_mk = smem_u32(sm.mk), s_mv = smem_u32(sm.mv);
  const uint32_t s_dsm = smem_u32(sm.dsm), s_dsmT = smem_u32(sm.dsmT), s_pmT = smem_u32(sm.pmT);
  const uint32_t bar_ld0 = smem_u32(&sm.bar_ld0), bar_ld1 = smem_u32(&sm.bar_ld1);
  const uint32_t bar_s0 = smem_u32(&sm.bar_s[0]), bar_f = smem_u32(&sm.bar_f);

  if (warp == 0) tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
  if (tid == 0) {
    mbar_init(bar_ld0, 1);
    mbar_init(bar_ld1, 1);
    mbar_init(bar_s0, 1);
    mbar_init(bar_s0 + 8, 1);
    mbar_init(bar_f, 1);
    mbar_init_fence();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // this thread: row m (TMEM lane), 32 columns of each 64-key tile (half hf)
  const int m = tid & (QR - 1), hf = tid >> 7;
  const uint32_t lrow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
  bool alive = true;
  float dsum = 0.f;
  uint32_t ph_s = 0;  // phase bits of the two score barriers
  uint32_t ph_ld = 0, ph_f = 0;

#pragma unroll 1
  for (int tile = 0; tile < kSwaBwdSlab / QR; ++tile) {
    const int t0 = slab * kSwaBwdSlab + tile * QR;
    if (t0 >= T) break;
    const int lo = max(0, t0 - w + 1), hi = min(T - 1, t0 + QR - 1);
    const int ntiles = (hi - lo + KT) / KT;  // 1..MAXT
    // ---- loads ----------------------------------------------------------------
    if (tid == 0) {
      mbar_expect_tx(bar_ld0, 4 * kQBox + ntiles * 2 * kKBox + (has_meta ? 2 * kMBox : 0) +
                                  (meta_v ? 2 * kMBox : 0));
      for (int hh = 0; hh < 2; ++hh) {
        tma_load_3d(s_q + hh * kQBox, &tq, bar_ld0, hh * 64, t0, bh);
        tma_load_3d(s_do + hh * kQBox, &tdo, bar_ld0, hh * 64, t0, bh);
        if (has_meta) tma_load_3d(s_mk + hh * kMBox, &tmk, bar_ld0, hh * 64, 0, h);
        if (meta_v) tma_load_3d(s_mv + hh * kMBox, &tmv, bar_ld0, hh * 64, 0, h);
        for (int j = 0; j < ntiles; ++j)
          tma_load_3d(s_k + (2 * j + hh) * kKBox, &tk, bar_ld0, hh * 64, lo + j * KT, bh);
      }
      mbar_expect_tx(bar_ld1, ntiles * 2 * kKBox);
      for (int hh = 0; hh < 2; ++hh)
        for (int j = 0; j < ntiles; ++j)
          tma_load_3d(s_v + (2 * j + hh) * kKBox, &tv, bar_ld1, hh * 64, lo + j * KT, bh);
    }
    // lse (log2 units) and D_t = dO_t . o_t from the forward output (two
    // threads per row, 64 dims each), kept for the key side in Dbuf
    {
      const int t = t0 + m;
      float acc = 0.f;
      if (t < T) {
        const size_t off = ((size_t)bh * T + t) * D + hf * 64;
        const uint4* op = reinterpret_cast<const uint4*>((const bf16*)p.osw + off);
        const uint4* dp = reinterpret_cast<const uint4*>((const bf16*)p.dO + off);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          const uint4 a = __ldg(op + x), c = __ldg(dp + x);
          const uint32_t aw[4] = {a.x, a.y, a.z, a.w}, cw[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
          for (int y = 0; y < 4; ++y) {
            const float2 f = unpack_bf16(aw[y]), g = unpack_bf16(cw[y]);
            acc = fmaf(f.x, g.x, acc);
            acc = fmaf(f.y, g.y, acc);
          }
        }
      }
      if (hf == 1) sm.drow[m] = acc;
      __syncthreads();
      if (hf == 0) {
        acc += sm.drow[m];
        sm.lse2[m] = t < T ? p.lse[(size_t)bh * T + t] * kLog2e : 0.f;
        if (t < T) {
          p.Dbuf[(size_t)bh * T + t] = acc;
          dsum += acc;
        }
      }
      __syncthreads();
      if (hf == 0) sm.drow[m] = acc;
      __syncthreads();
    }
    // ---- scores of the meta tile and of key tiles 0 and 1 --------------------
    auto issue_scores = [&](int j) {  // S_j, dP_j into TMEM pair j & 1
      constexpr uint32_t idS = idesc_bf16(QR, KT, false);
      const uint32_t col = kColS + 128 * (j & 1);
#pragma unroll 1
      for (int kk = 0; kk < D / 16; ++kk) {
        const uint32_t hh = kk >> 2, ko = (kk & 3) * 32;
        mma_bf16_ss(tmem + col, sdesc_sw128(s_q + hh * kQBox + ko, 16, 1024),
                    sdesc_sw128(s_k + (2 * j + hh) * kKBox + ko, 16, 1024), idS, kk > 0);
        mma_bf16_ss(tmem + col + 64, sdesc_sw128(s_do + hh * kQBox + ko, 16, 1024),
                    sdesc_sw128(s_v + (2 * j + hh) * kKBox + ko, 16, 1024), idS, kk > 0);
      }
      mma_commit(bar_s0 + 8 * (j & 1));
    };
    if (tid == 0) {
      alive = alive && mbar_wait(bar_ld0, ph_ld, p.status) && mbar_wait(bar_ld1, ph_ld, p.status);
      if (alive) {
        tc_fence_after();
        if (has_meta) {
          constexpr uint32_t idM = idesc_bf16(QR, MTT, false);
#pragma unroll 1
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t hh = kk >> 2, ko = (kk & 3) * 32;
            mma_bf16_ss(tmem + kColSM, sdesc_sw128(s_q + hh * kQBox + ko, 16, 1024),
                        sdesc_sw128(s_mk + hh * kMBox + ko, 16, 1024), idM, kk > 0);
            if (meta_v)
              mma_bf16_ss(tmem + kColDPM, sdesc_sw128(s_do + hh * kQBox + ko, 16, 1024),
                          sdesc_sw128(s_mv + hh * kMBox + ko, 16, 1024), idM, kk > 0);
          }
        }
        issue_scores(0);  // the meta products complete with it
        if (ntiles > 1) issue_scores(1);
      }
    }
    ph_ld ^= 1;
    const int t = t0 + m;
    const bool row_ok = t < T;
    const float l2 = sm.lse2[m], Dr = sm.drow[m];
    // ---- key tiles ---------------------------------------------------------------
#pragma unroll 1
    for (int j = 0; j < ntiles; ++j) {
      const int pb = j & 1;
      if (alive) alive = mbar_wait(bar_s0 + 8 * pb, (ph_s >> pb) & 1u, p.status);
      ph_s ^= 1u << pb;
      tc_fence_after();
      uint32_t s[32], dp[32];
      tmem_ld32(lrow + kColS + 128 * pb + hf * 32, s);
      tmem_ld32(lrow + kColS + 128 * pb + 64 + hf * 32, dp);
      uint32_t sm16[16], dpm16[16];
      const bool do_meta = j == 0 && has_meta && hf == 0;
      if (do_meta) {
        tmem_ld16(lrow + kColSM, sm16);
        tmem_ld16(lrow + kColDPM, dpm16);
      }
      tmem_ld_wait();
      const int kb = lo + j * KT + hf * 32;  // first key of this thread's columns
      uint32_t pk[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float ds[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = kb + c + e;
          const bool ok = row_ok && key <= t && key >= t - w + 1;
          const float P = ok ? exp2f(fmaf(__uint_as_float(s[c + e]), c2, -l2)) : 0.f;
          ds[e] = p.gscale * P * (__uint_as_float(dp[c + e]) - Dr);
        }
        pk[c / 2] = pack_bf16(ds[0], ds[1]);
      }
      // dS_j over the spent V_j: K-major [128 rows][64 keys], 8-row groups 1024 B apart
      uint8_t* dst = &sm.v[j][0][0];
#pragma unroll
      for (int kc = 0; kc < 4; ++kc)
        *reinterpret_cast<uint4*>(dst + (m >> 3) * 1024 + (hf * 4 + kc) * 128 + (m & 7) * 16) =
            make_uint4(pk[4 * kc], pk[4 * kc + 1], pk[4 * kc + 2], pk[4 * kc + 3]);
      if (do_meta) {  // dS_meta and P_meta of row m: [128][16] and the transposes [16][128]
        uint32_t dk8[8];
#pragma unroll
        for (int c = 0; c < MTT; c += 2) {
          float dsv[2], pv[2];
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int mm = c + e;
            const float P = (mm < M && row_ok) ? exp2f(fmaf(__uint_as_float(sm16[mm]), c2, -l2)) : 0.f;
            const float dpv = meta_v ? __uint_as_float(dpm16[mm]) : 0.f;
            dsv[e] = p.gscale * P * (dpv - Dr);
            pv[e] = P;
          }
          dk8[c / 2] = pack_bf16(dsv[0], dsv[1]);
          const bf16 d0 = __float2bfloat16_rn(dsv[0]), d1 = __float2bfloat16_rn(dsv[1]);
          const bf16 p0 = __float2bfloat16_rn(pv[0]), p1 = __float2bfloat16_rn(pv[1]);
          // element (mm, m) of a K-major [16][128] tile: 8-row groups 2048 B apart
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const int mm = c + e;
            const uint32_t o = (mm >> 3) * 2048 + (m >> 3) * 128 + (mm & 7) * 16 + (m & 7) * 2;
            *reinterpret_cast<bf16*>(sm.dsmT + o) = e ? d1 : d0;
            *reinterpret_cast<bf16*>(sm.pmT + o) = e ? p1 : p0;
          }
        }
#pragma unroll
        for (int kc = 0; kc < 2; ++kc)  // K-major [128][16]: 8-row groups 256 B apart
          *reinterpret_cast<uint4*>(sm.dsm + (m >> 3) * 256 + kc * 128 + (m & 7) * 16) =
              make_uint4(dk8[4 * kc], dk8[4 * kc + 1], dk8[4 * kc + 2], dk8[4 * kc + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      alive = __syncthreads_and(alive);
      if (tid == 0 && alive) {
        tc_fence_after();
        constexpr uint32_t idQ = idesc_bf16(QR, D, true);
#pragma unroll
        for (int kk = 0; kk < KT / 16; ++kk)  // B = K_j, MN-major: 16 keys = 2048 bytes per step
          mma_bf16_ss(tmem + kColDQ, sdesc(smem_u32(dst) + kk * 256, 128, 1024),
                      sdesc_sw128(s_k + 2 * j * kKBox + kk * 2048, kKBox, 1024), idQ, (j > 0 || kk > 0));
        if (j + 2 < ntiles) issue_scores(j + 2);  // into the pair this tile freed
      }
    }
    // ---- meta: dq += dS_meta MK; the meta gradients --------------------------------
    if (tid == 0 && alive) {
      if (has_meta) {
        constexpr uint32_t idQ = idesc_bf16(QR, D, true), idG = idesc_bf16_at(QR, MTT, false);
        mma_bf16_ss(tmem + kColDQ, sdesc(s_dsm, 128, 256), sdesc_sw128(s_mk, kMBox, 1024), idQ, 1u);
        const uint32_t acc0 = tile > 0 ? 1u : 0u;
#pragma unroll
        for (int kk = 0; kk < QR / 16; ++kk) {  // A = Q / dO transposed (rows = K = queries)
          mma_bf16_ss(tmem + kColGK, sdesc_sw128(s_q + kk * 2048, kQBox, 1024),
                      sdesc(s_dsmT + kk * 256, 128, 2048), idG, (acc0 || kk > 0) ? 1u : 0u);
          mma_bf16_ss(tmem + kColGV, sdesc_sw128(s_do + kk * 2048, kQBox, 1024),
                      sdesc(s_pmT + kk * 256, 128, 2048), idG, (acc0 || kk > 0) ? 1u : 0u);
        }
      }
      mma_commit(bar_f);
    }
    if (alive) alive = mbar_wait(bar_f, ph_f, p.status);
    ph_f ^= 1;
    tc_fence_after();
    // ---- dq of row m, this thread's 64 columns ----------------------------------
#pragma unroll 1
    for (int c0 = hf * 64; c0 < hf * 64 + 64; c0 += 32) {
      uint32_t r[32];
      tmem_ld32(lrow + kColDQ + c0, r);
      tmem_ld_wait();
      if (!row_ok || !alive) continue;
      const size_t off = ((size_t)bh * T + t) * D + c0;
      if (p.dq_f32) {
        float4* d4 = reinterpret_cast<float4*>(p.dq_f32 + off);
#pragma unroll
        for (int x = 0; x < 8; ++x)
          d4[x] = make_float4(__uint_as_float(r[4 * x]) * p.scale, __uint_as_float(r[4 * x + 1]) * p.scale,
                              __uint_as_float(r[4 * x + 2]) * p.scale, __uint_as_float(r[4 * x + 3]) * p.scale);
      } else {
        uint32_t pk[16];
#pragma unroll
        for (int c = 0; c < 32; c += 2)
          pk[c / 2] = pack_bf16(__uint_as_float(r[c]) * p.scale, __uint_as_float(r[c + 1]) * p.scale);
        uint4* d4 = reinterpret_cast<uint4*>((bf16*)p.dq + off);
#pragma unroll
        for (int x = 0; x < 4; ++x) d4[x] = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
      }
    }
    tc_fence_before();
    __syncthreads();  // every TMEM read of this tile done before the next tile's products
    tc_fence_after();
  }

  // ---- per-slab partials: meta gradients (TMEM lane = dim) and the sum of D ----
  if (has_meta) {
    const int nslab = gridDim.z;
    float* part = p.meta_part + (((size_t)b * nslab + slab) * H + h) * M * (2 * D);
    if (hf == 0) {  // warps 0..3: lane m = dim m
      uint32_t gk[16], gv[16];
      tmem_ld16(lrow + kColGK, gk);
      tmem_ld16(lrow + kColGV, gv);
      tmem_ld_wait();
      if (alive) {
        for (int mm = 0; mm < M; ++mm) {
          part[(size_t)mm * (2 * D) + m] = __uint_as_float(gk[mm]) * p.scale;
          part[(size_t)mm * (2 * D) + D + m] = __uint_as_float(gv[mm]) * p.gscale;
        }
      }
    }
  }
  dsum = warp_sum(dsum);
  if (lane == 0) sm.dsum[warp] = dsum;
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
    for (int x = 0; x < NTH / 32; ++x) s += sm.dsum[x];
    p.alpha_part[((size_t)b * gridDim.z + slab) * H + h] = s;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

}  // namespace

bool swa_bwd_q_tc_supported(const SwaBwdParams& p) {
  return p.dkd == D && p.dvd == D && p.w <= kMaxWindow && p.M <= MTT && p.osw != nullptr;
}

cudaError_t launch_swa_bwd_q_tc(const SwaBwdParams& p, cudaStream_t s) {
  if (p.B * p.H == 0 || p.T == 0) return cudaSuccess;
  const size_t bytes = sizeof(QtcSmem) + 1024;  // + room to align the base to 1024
  cudaError_t e = cudaFuncSetAttribute(swa_bwd_q_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes);
  if (e != cudaSuccess) return e;
  SwaBwdParams pp = p;
  pp.status = device_status_word();
  if (pp.status == nullptr) return cudaErrorInvalidDevicePointer;
  const uint64_t bh = (uint64_t)p.B * p.H;
  CUtensorMap tq, tdo, tk, tv, tmk, tmv;
  if (!tma_map_rows128(&tq, p.q, p.T, bh, QR) || !tma_map_rows128(&tdo, p.dO, p.T, bh, QR) ||
      !tma_map_rows128(&tk, p.k, p.T, bh, KT) || !tma_map_rows128(&tv, p.v, p.T, bh, KT))
    return cudaErrorInvalidValue;
  tmk = tq;
  tmv = tq;
  if (p.M > 0 && !tma_map_rows128(&tmk, p.mk, p.M, p.H, MTT)) return cudaErrorInvalidValue;
  if (p.M > 0 && p.mv && !tma_map_rows128(&tmv, p.mv, p.M, p.H, MTT)) return cudaErrorInvalidValue;
  const int nslab = (p.T + kSwaBwdSlab - 1) / kSwaBwdSlab;
  {
    ScopedTiming tm("swa_bwd_q_tc", s);
    swa_bwd_q_tc_kernel<<<dim3(p.H, p.B, nslab), NTH, bytes, s>>>(pp, tq, tdo, tk, tv, tmk, tmv);
  }
  return cudaGetLastError();
}

}  // namespace lz
