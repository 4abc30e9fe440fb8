// Sliding-window softmax attention with meta-memory sinks on the tensor
// cores (bf16 I/O, fp32 accumulation, dk = dv = 128).
//
// Lizard technical summary, section 2a ("anchor window attention"): for
// query t the keys are j in [t-w+1, t] plus the M meta tokens, which stay in
// the softmax denominator as sinks (and add p_m mv_m to the numerator when
// meta values are given).  One CTA owns 64 query rows of one (batch, head);
// each of its 4 warps owns 16 rows.  Scores S = Q K^T and the products P V
// run on mma.m16n8k16; the running max and sum stay in registers (online
// softmax in the log2 domain); K/V tiles of 64 keys are double-buffered with
// cp.async.  The meta tokens form one extra tile of 16 keys.
#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"

namespace lz {
namespace {

constexpr int QT = 64;       // query rows per CTA
constexpr int KT = 64;       // keys per tile
constexpr int MT = 16;       // meta tile (M <= 16)
constexpr int D = 128;
constexpr int NT = 128;
constexpr int RPAD = D + 8;  // padded bf16 row
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

template <int N>
struct IntC {
  static constexpr int value = N;
};

struct SwaSmem {
  bf16 q[QT * RPAD];
  bf16 k[2][KT * RPAD];
  bf16 v[2][KT * RPAD];
  bf16 mk[MT * RPAD];
  bf16 mv[MT * RPAD];
};

static_assert(sizeof(SwaSmem) <= 232448, "shared memory per block exceeds 227 KB");

__global__ void __launch_bounds__(NT, 2) swa_fwd_mma_kernel(SwaFwdParams p) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SwaSmem& sm = *reinterpret_cast<SwaSmem*>(smem_raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gr = lane >> 2, gc = (lane & 3) * 2;
  const int bh = blockIdx.y, h = bh % p.H;
  const int T = p.T, w = p.w, M = p.M;
  const int t0 = blockIdx.x * QT;
  const bf16* q = (const bf16*)p.q + (size_t)bh * T * D;
  const bf16* k = (const bf16*)p.k + (size_t)bh * T * D;
  const bf16* v = (const bf16*)p.v + (size_t)bh * T * D;
  const float c2 = p.scale * kLog2e;  // logits in log2 units

  const int lo = max(0, t0 - w + 1);
  const int hi = min(T - 1, t0 + QT - 1);
  const int ntiles = (hi - lo + KT) / KT;

  auto load_rows = [&](bf16* dst, const bf16* src, int r0, int nvalid, int nrows) {
    for (int x = tid; x < nrows * D / 8; x += NT) {
      const int r = x / (D / 8), cc = x % (D / 8);
      const bool ok = r < nvalid;
      cp_async16(&dst[r * RPAD + cc * 8], src + (size_t)(ok ? r0 + r : r0) * D + cc * 8, ok ? 16 : 0);
    }
  };
  // query tile + meta tokens + first key tile
  load_rows(sm.q, q, t0, min(QT, T - t0), QT);
  if (M > 0) {
    load_rows(sm.mk, (const bf16*)p.mk + (size_t)h * M * D, 0, M, MT);
    if (p.mv) load_rows(sm.mv, (const bf16*)p.mv + (size_t)h * M * D, 0, M, MT);
  }
  load_rows(sm.k[0], k, lo, hi - lo + 1, KT);
  load_rows(sm.v[0], v, lo, hi - lo + 1, KT);
  cp_async_commit();

  float o[D / 8][4];
#pragma unroll
  for (int nt = 0; nt < D / 8; ++nt)
#pragma unroll
    for (int e = 0; e < 4; ++e) o[nt][e] = 0.f;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.f, 0.f};
  const int row0 = t0 + 16 * warp + gr;  // rows row0 and row0 + 8
  uint32_t qa[D / 16][4];

  // One tile of keys: scores, online softmax update, P V.  `valid(r, j)`
  // tells whether key column j (0..NK-1) is visible from row hh.
  auto process = [&](const bf16* ks, const bf16* vs, auto nk_tag, auto valid) {
    constexpr int NK = decltype(nk_tag)::value;
    float s[NK / 8][4];
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
    float mx[2] = {-INFINITY, -INFINITY};
#pragma unroll
    for (int nt = 0; nt < NK / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hh = e >> 1, j = nt * 8 + gc + (e & 1);
        const float x = valid(hh, j) ? s[nt][e] * c2 : -INFINITY;
        s[nt][e] = x;
        mx[hh] = fmaxf(mx[hh], x);
      }
    float corr[2], base[2];
#pragma unroll
    for (int hh = 0; hh < 2; ++hh) {
      mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 1));
      mx[hh] = fmaxf(mx[hh], __shfl_xor_sync(0xffffffffu, mx[hh], 2));
      const float mn = fmaxf(m[hh], mx[hh]);
      base[hh] = mn == -INFINITY ? 0.f : mn;
      corr[hh] = exp2f(m[hh] - base[hh]);  // 0 when m was -inf
      m[hh] = mn;
      l[hh] *= corr[hh];
    }
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      o[nt][0] *= corr[0];
      o[nt][1] *= corr[0];
      o[nt][2] *= corr[1];
      o[nt][3] *= corr[1];
    }
#pragma unroll
    for (int nt = 0; nt < NK / 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float pe = exp2f(s[nt][e] - base[e >> 1]);  // exp2(-inf) = 0
        s[nt][e] = pe;
        l[e >> 1] += pe;
      }
    if (vs == nullptr) return;  // sink-only meta tokens: denominator only
#pragma unroll
    for (int kk = 0; kk < NK / 16; ++kk) {
      const uint32_t pa[4] = {pack_bf16(s[2 * kk][0], s[2 * kk][1]), pack_bf16(s[2 * kk][2], s[2 * kk][3]),
                              pack_bf16(s[2 * kk + 1][0], s[2 * kk + 1][1]),
                              pack_bf16(s[2 * kk + 1][2], s[2 * kk + 1][3])};
#pragma unroll
      for (int ntp = 0; ntp < D / 16; ++ntp) {
        uint32_t b0, b1, b2, b3;
        ldsm_x4_t(smem_u32(&vs[(kk * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * RPAD + ntp * 16 +
                               (lane >> 4) * 8]),
                  b0, b1, b2, b3);
        mma_bf16(o[2 * ntp], pa, b0, b1);
        mma_bf16(o[2 * ntp + 1], pa, b2, b3);
      }
    }
  };

  for (int it = 0; it < ntiles; ++it) {
    const int st = it & 1;
    const int kb = lo + it * KT;
    cp_async_wait<0>();
    __syncthreads();
    if (it + 1 < ntiles) {
      const int nb = kb + KT;
      load_rows(sm.k[st ^ 1], k, nb, hi - nb + 1, KT);
      load_rows(sm.v[st ^ 1], v, nb, hi - nb + 1, KT);
      cp_async_commit();
    }
    if (it == 0) {
#pragma unroll
      for (int kk = 0; kk < D / 16; ++kk)
        ldsm_x4(smem_u32(&sm.q[(16 * warp + (lane & 15)) * RPAD + kk * 16 + (lane >> 4) * 8]), qa[kk][0],
                qa[kk][1], qa[kk][2], qa[kk][3]);
      if (M > 0)
        process(sm.mk, p.mv ? sm.mv : nullptr, IntC<MT>{},
                [&](int hh, int j) { return j < M && row0 + 8 * hh < T; });
    }
    process(sm.k[st], sm.v[st], IntC<KT>{}, [&](int hh, int j) {
      const int t = row0 + 8 * hh, key = kb + j;
      return t < T && key <= t && key >= t - w + 1 && key <= hi;
    });
  }
  // normalize, store o and lse
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], 1);
    l[hh] += __shfl_xor_sync(0xffffffffu, l[hh], 2);
  }
#pragma unroll
  for (int hh = 0; hh < 2; ++hh) {
    const int t = row0 + 8 * hh;
    if (t >= T) continue;
    const float inv = 1.f / l[hh];
    const size_t off = ((size_t)bh * T + t) * D;
#pragma unroll
    for (int nt = 0; nt < D / 8; ++nt) {
      const int j = nt * 8 + gc;
      const float x0 = o[nt][2 * hh] * inv, x1 = o[nt][2 * hh + 1] * inv;
      if (p.o) *reinterpret_cast<uint32_t*>(&((bf16*)p.o)[off + j]) = pack_bf16(x0, x1);
      if (p.o_f32) *reinterpret_cast<float2*>(&p.o_f32[off + j]) = make_float2(x0, x1);
    }
    if (p.lse && (lane & 3) == 0) p.lse[(size_t)bh * T + t] = m[hh] * kLn2 + logf(l[hh]);
  }
}

}  // namespace

bool swa_fwd_mma_supported(int dk, int dv, bool bf16) { return bf16 && dk == D && dv == D; }

cudaError_t launch_swa_fwd_mma(const SwaFwdParams& p, cudaStream_t s) {
  if (p.B * p.H == 0 || p.T == 0) return cudaSuccess;
  const size_t bytes = sizeof(SwaSmem);
  cudaError_t e = cudaFuncSetAttribute(swa_fwd_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes);
  if (e != cudaSuccess) return e;
  dim3 grid((p.T + QT - 1) / QT, p.B * p.H);
  {
    ScopedTiming tm("swa_fwd_mma", s);
    swa_fwd_mma_kernel<<<grid, NT, bytes, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace lz
