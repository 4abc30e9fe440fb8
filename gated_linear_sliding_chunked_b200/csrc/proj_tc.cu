// The projections in front of the hybrid operator on the Blackwell tensor
// cores: from the hidden states x [B][T][Dm] (bf16) and weights W [H*dk][Dm]
// (bf16, one row per output feature) one launch computes
//   q = x Wq^T,  k = phi(x Wk^T) with phi the identity,
//   g = scale * log sigma(x Wg^T)
// (Lizard technical summary, section 2a: the gate is Gamma_i =
// sigma(W_gamma x_i) and the state update takes phi(k_i); the pages do not
// define phi), writing q, k (bf16) and the fp32 log-gates g straight into the
// operator's [B][H][T][dk] layout, so the gate's logit never leaves the chip.
//
// One CTA computes a 128-token x 256-feature tile (two heads of 128 or four of
// 64) of one of the three outputs; consecutive CTAs take consecutive feature
// tiles of the same 128 tokens, so the x rows they share come from L2.  Warp
// roles: warp 0 lane 0 issues TMA copies into a 2-stage ring of
// (x, W) k-tiles (64 hidden dims each, 128-byte swizzle; two CTAs share an
// SM, so one's epilogue overlaps the other's main loop); warp 1 lane 0
// issues tcgen05.mma (M = 128, N = 256, K = 16) into a 256-column tensor-memory
// accumulator and frees each stage with tcgen05.commit; warps 2..5 (one TMEM
// lane quarter each) read the accumulator and store the tile.  Every wait is
// bounded (tc05.cuh).
#include <cstdio>

#include "../../include/lizard.h"
#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"
#include "tc05.cuh"
#include "tma_host.h"

namespace lz {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 2;
constexpr int NTH = 192;                   // 6 warps
constexpr uint32_t kA = BM * BK * 2;       // bytes of one x k-tile
constexpr uint32_t kB = BN * BK * 2;       // bytes of one W k-tile
constexpr uint32_t kTmemCols = 256;

struct ProjSmem {
  uint8_t a[STAGES][kA];
  uint8_t b[STAGES][kB];
  uint64_t full[STAGES], empty[STAGES], acc;
  uint32_t tmem_base;
};
static_assert(sizeof(ProjSmem) + 1024 <= 232448, "shared memory per block exceeds 227 KB");

struct ProjParams {
  int B, T, Dm, H, dk;
  int nk;          // k-tiles of 64 hidden dims
  int ntile;       // feature tiles per output (H * dk / 256)
  int which[3];    // output of feature-tile group y: 0 = q, 1 = k, 2 = g
  void* out[3];
  float scale;
  unsigned int* status;
};

__global__ void __launch_bounds__(NTH, 2)
    proj_tc_kernel(ProjParams p, const __grid_constant__ CUtensorMap tx,
                   const __grid_constant__ CUtensorMap tw0, const __grid_constant__ CUtensorMap tw1,
                   const __grid_constant__ CUtensorMap tw2) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  ProjSmem& sm = *reinterpret_cast<ProjSmem*>(smem_raw + ((1024u - (raw & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int grp = blockIdx.x / p.ntile;
  const int which = grp == 0 ? p.which[0] : grp == 1 ? p.which[1] : p.which[2];
  void* outp = which == 0 ? p.out[0] : which == 1 ? p.out[1] : p.out[2];
  const int n0 = (blockIdx.x % p.ntile) * BN;  // first feature of the tile within its output
  const int m0 = blockIdx.y * BM;              // first token (b * T + t)
  const int ntok = p.B * p.T;
  const CUtensorMap* tw = which == 0 ? &tw0 : which == 1 ? &tw1 : &tw2;

  if (warp == 0) tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
  if (tid == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(smem_u32(&sm.full[s]), 1);
      mbar_init(smem_u32(&sm.empty[s]), 1);
    }
    mbar_init(smem_u32(&sm.acc), 1);
    mbar_init_fence();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  if (warp == 0 && lane == 0) {  // ---- producer
    for (int kt = 0; kt < p.nk; ++kt) {
      const int s = kt % STAGES;
      if (kt >= STAGES && !mbar_wait(smem_u32(&sm.empty[s]), ((kt / STAGES) - 1) & 1, p.status)) break;
      const uint32_t bar = smem_u32(&sm.full[s]);
      mbar_expect_tx(bar, kA + kB);
      tma_load_2d(smem_u32(sm.a[s]), &tx, bar, kt * BK, m0);
      tma_load_2d(smem_u32(sm.b[s]), tw, bar, kt * BK, n0);
    }
  } else if (warp == 1 && lane == 0) {  // ---- MMA issuer
    constexpr uint32_t idesc = idesc_bf16(BM, BN, false);
    bool ok = true;
    for (int kt = 0; kt < p.nk && ok; ++kt) {
      const int s = kt % STAGES;
      ok = mbar_wait(smem_u32(&sm.full[s]), (kt / STAGES) & 1, p.status);
      if (!ok) break;
      tc_fence_after();
      const uint32_t sa = smem_u32(sm.a[s]), sb = smem_u32(sm.b[s]);
#pragma unroll
      for (int kk = 0; kk < BK / 16; ++kk)
        mma_bf16_ss(tmem, sdesc_sw128(sa + kk * 32, 16, 1024), sdesc_sw128(sb + kk * 32, 16, 1024), idesc,
                    (kt > 0 || kk > 0) ? 1u : 0u);
      mma_commit(smem_u32(&sm.empty[s]));  // the stage is free once these MMAs are done
    }
    if (ok) mma_commit(smem_u32(&sm.acc));
  } else if (warp >= 2) {  // ---- epilogue: TMEM lane quarter warp % 4 = rows of the tile
    const int q4 = warp & 3, row = q4 * 32 + lane, m = m0 + row;
    const bool ok = mbar_wait(smem_u32(&sm.acc), 0, p.status);
    tc_fence_after();
    const int b = m / p.T, t = m - b * p.T;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(tmem + ((uint32_t)(q4 * 32) << 16) + c * 32, r);
      tmem_ld_wait();
      if (!ok || m >= ntok) continue;
      const int n = n0 + c * 32, h = n / p.dk, i = n - h * p.dk;  // 32 features of one head
      const size_t off = (((size_t)b * p.H + h) * p.T + t) * p.dk + i;
      if (which == 2) {
        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(outp) + off);
#pragma unroll
        for (int x = 0; x < 8; ++x) {
          float y[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float z = __uint_as_float(r[4 * x + e]);
            y[e] = p.scale * (fminf(z, 0.f) - log1pf(__expf(-fabsf(z))));
          }
          dst[x] = make_float4(y[0], y[1], y[2], y[3]);
        }
      } else {
        uint4* dst = reinterpret_cast<uint4*>(static_cast<bf16*>(outp) + off);
#pragma unroll
        for (int x = 0; x < 4; ++x)
          dst[x] = make_uint4(pack_bf16(__uint_as_float(r[8 * x]), __uint_as_float(r[8 * x + 1])),
                              pack_bf16(__uint_as_float(r[8 * x + 2]), __uint_as_float(r[8 * x + 3])),
                              pack_bf16(__uint_as_float(r[8 * x + 4]), __uint_as_float(r[8 * x + 5])),
                              pack_bf16(__uint_as_float(r[8 * x + 6]), __uint_as_float(r[8 * x + 7])));
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

lz_status fail(lz_status st, const char* what) { return (lz_status)set_last_error(st, what); }
bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace
}  // namespace lz

extern "C" lz_status lz_qkg_projection(int B, int T, int Dm, int H, int dk, const void* x,
                                       const void* Wq, const void* Wk, const void* Wg,
                                       float gate_scale, void* q, void* k, float* g,
                                       lz_stream stream) {
  using namespace lz;
  if (B < 0 || T < 0 || H < 1) return fail(LZ_ERR_INVALID_ARG, "lz_qkg_projection: B, T >= 0, H >= 1");
  if (Dm < 8 || Dm % 8) return fail(LZ_ERR_UNSUPPORTED, "lz_qkg_projection: Dm must be a multiple of 8");
  if ((dk != 64 && dk != 128) || ((size_t)H * dk) % BN)
    return fail(LZ_ERR_UNSUPPORTED, "lz_qkg_projection: dk must be 64 or 128 and H * dk a multiple of 256");
  if (!(gate_scale > 0.f)) return fail(LZ_ERR_INVALID_ARG, "lz_qkg_projection: gate_scale must be > 0");
  const void* W[3] = {Wq, Wk, Wg};
  void* out[3] = {q, k, g};
  const size_t ntok = (size_t)B * T;
  ProjParams p{};
  int nw = 0;
  for (int w = 0; w < 3; ++w) {
    if ((W[w] == nullptr) != (out[w] == nullptr))
      return fail(LZ_ERR_INVALID_ARG, "lz_qkg_projection: a weight and its output must both be given or both NULL");
    if (W[w] && (!aligned16(W[w]) || !aligned16(out[w])))
      return fail(LZ_ERR_INVALID_ARG, "lz_qkg_projection: pointers must be 16-byte aligned");
    if (W[w]) p.which[nw++] = w;
  }
  if (nw == 0 || ntok == 0) {
    set_last_error(LZ_OK, "");
    return LZ_OK;
  }
  if (!x || !aligned16(x)) return fail(LZ_ERR_INVALID_ARG, "lz_qkg_projection: x must be non-NULL and 16-byte aligned");
  if ((ntok + BM - 1) / BM > 65535) return fail(LZ_ERR_UNSUPPORTED, "lz_qkg_projection: B * T too large");
  p.B = B; p.T = T; p.Dm = Dm; p.H = H; p.dk = dk;
  p.nk = (Dm + BK - 1) / BK;
  p.ntile = H * dk / BN;
  for (int w = 0; w < 3; ++w) p.out[w] = out[w];
  p.scale = gate_scale;
  p.status = device_status_word();
  if (p.status == nullptr) return fail(LZ_ERR_CUDA, "lz_qkg_projection: device status word unavailable");
  CUtensorMap tx, tw[3];
  if (!tma_map_2d(&tx, x, Dm, ntok, BM)) return fail(LZ_ERR_CUDA, "lz_qkg_projection: tensor map of x");
  for (int w = 0; w < 3; ++w)
    if (!tma_map_2d(&tw[w], W[w] ? W[w] : W[p.which[0]], Dm, (uint64_t)H * dk, BN))
      return fail(LZ_ERR_CUDA, "lz_qkg_projection: tensor map of a weight");
  const size_t bytes = sizeof(ProjSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(proj_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) {
    dim3 grid((unsigned)(nw * p.ntile), (unsigned)((ntok + BM - 1) / BM));
    ScopedTiming tm("qkg_projection_tc", (cudaStream_t)stream);
    proj_tc_kernel<<<grid, NTH, bytes, (cudaStream_t)stream>>>(p, tx, tw[0], tw[1], tw[2]);
    e = cudaGetLastError();
  }
  if (e != cudaSuccess) {
    char msg[256];
    std::snprintf(msg, sizeof(msg), "lz_qkg_projection: %s", cudaGetErrorString(e));
    return fail(LZ_ERR_CUDA, msg);
  }
  set_last_error(LZ_OK, "");
  return LZ_OK;
}
