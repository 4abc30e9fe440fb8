// Key side of the window + meta softmax backward on the Blackwell tensor
// cores: tcgen05.mma with dK, dV accumulated in tensor memory, operands
// brought in by TMA (bf16 I/O, fp32 accumulation, dk = dv = 128).
//
// Lizard technical summary, section 2a: key j is seen by queries
// t in [j, j + w - 1].  With P = exp(logit - lse), the window branch's share
// gscale * dO of the output gradient and D_t = dO_t . o_t:
//   dV_j = gscale * sum_t P_tj dO_t,   dK_j = scale * gscale * sum_t dS_tj q_t,
//   dS_tj = P_tj (dO_t . v_j - D_t).
// One CTA = kBlocksPerCta consecutive blocks of 128 keys of one (batch,
// head); it walks the (key block, 64-query tile) pairs in which a tile sees a
// block as one sequence, so that the next block's K / V copy and first scores
// overlap the current block's last tiles, and the dK / dV of a block are read
// out of tensor memory by the softmax warps after its last tile.  Nine warps:
//   warp 8, the producer (one lane): the TMA copies, and per pair g the NEXT
//             pair's S^T = K Q^T and dP^T = V dO^T (M = 128 keys, N = 64
//             queries) into the other half of a double-buffered TMEM pair,
//             then, once pair g's P^T and dS^T are in shared memory,
//             dV += P^T dO and dK += dS^T Q (M = 128, N = 128, K = 64) and a
//             commit;
//   warps 0-7: each key row's two threads read 32 query columns of pair g's
//             scores and form P^T and dS^T (bf16) in one of two shared-memory
//             buffers, so that they wait for the gradient MMAs of pair g - 2,
//             not of pair g - 1.
// Q / dO tiles rotate through three shared-memory buffers, loaded by TMA
// two pairs ahead.  With p.ds_tiles set the threads also store their bf16
// dS^T rows of every tile to global memory, from which swa_bwd_dq forms dq
// (so that the query side does not form the band's scores a second time).
// K, V (K-major) and the Q / dO tiles sit in shared memory 128-byte
// swizzled as TMA writes them; the gradient MMAs read Q / dO as MN-major B
// operands (rows = queries, the reduction dim) from the same tiles.
#include <cstddef>

#include "common.cuh"
#include "kernels.h"
#include "mma.cuh"
#include "tc05.cuh"
#include "tma_host.h"

namespace lz {
namespace {

constexpr int KR = 128;   // keys per CTA (MMA M)
constexpr int QT = 64;    // queries per tile
constexpr int D = 128;
constexpr int NSW = 256;  // softmax threads (warps 0-7)
constexpr int kBlocksPerCta = 2;  // consecutive key blocks one CTA walks (3: 0.410, 4: 0.392, 8: 0.462 ms alone)
constexpr int NTH = NSW + 32;  // + the producer warp
constexpr uint32_t kHalf = 64 * 2;  // bytes of one swizzled row (64 dims)
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kColDK = 0, kColDV = 128, kColS = 256, kColDP = 384;  // S^T, dP^T: + 64 * buffer
constexpr float kLog2e = 1.4426950408889634f;

struct KvSmem {
  uint8_t k[2][KR * kHalf];       // dims [0,64), [64,128): 128 key rows each
  uint8_t v[2][KR * kHalf];
  uint8_t q[3][2][QT * kHalf];    // [buffer][dim half]: 64 query rows
  uint8_t dO[3][2][QT * kHalf];
  uint8_t pt[2][KR * QT * 2];     // P^T of tile i in buffer i & 1, bf16, no-swizzle K-major
  uint8_t dst[2][KR * QT * 2];    // dS^T
  float lse2[3][QT];              // lse * log2(e) of the tile's queries
  float dq[3][QT];                // D of the tile's queries
  uint64_t bar_kv;
  uint64_t bar_ld[3];             // Q / dO buffer landed
  uint64_t bar_s[2];              // tile i's scores in TMEM buffer i & 1
  uint64_t bar_o[2];              // tile i's gradient MMAs done: P^T / dS^T buffer i & 1 free
  uint64_t bar_p[2];              // tile i's P^T / dS^T written (one arrival per softmax warp)
  uint32_t tmem_base;
};
static_assert(sizeof(KvSmem) + 1024 <= 232448, "shared memory per block exceeds 227 KB");
static_assert(offsetof(KvSmem, v) % 1024 == 0 && offsetof(KvSmem, q) % 1024 == 0 &&
                  offsetof(KvSmem, dO) % 1024 == 0 && offsetof(KvSmem, pt) % 1024 == 0,
              "swizzled tiles must be 1024-byte aligned");

__global__ void __launch_bounds__(NTH, 1)
    swa_bwd_kv_tc_kernel(SwaBwdParams p, const __grid_constant__ CUtensorMap tk,
                         const __grid_constant__ CUtensorMap tv, const __grid_constant__ CUtensorMap tq,
                         const __grid_constant__ CUtensorMap tdo) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  KvSmem& sm = *reinterpret_cast<KvSmem*>(smem_raw + ((1024u - (raw & 1023u)) & 1023u));
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int T = p.T, w = p.w;
  const int nblk = (T + KR - 1) / KR;
  const int blk0 = blockIdx.x * kBlocksPerCta, blk1 = min(nblk, blk0 + kBlocksPerCta);
  // query tiles that see key block b (at least one)
  auto nq_of = [&](int b) {
    const int j0 = b * KR;
    return (min(T - 1, j0 + KR - 1 + w - 1) - j0 + QT) / QT;
  };
  // the CTA walks the (key block, query tile) pairs of its blocks as one
  // sequence g = 0 .. npair - 1
  int npair = 0;
  for (int b = blk0; b < blk1; ++b) npair += nq_of(b);
  auto pair_of = [&](int g, int& b, int& i) {
    b = blk0;
    i = g;
    while (b + 1 < blk1) {
      const int n = nq_of(b);
      if (i < n) break;
      i -= n;
      ++b;
    }
  };
  const float* lse = p.lse + (size_t)bh * T;
  const float* Db = p.Dbuf + (size_t)bh * T;
  const float c2 = p.scale * kLog2e;

  const uint32_t s_k = smem_u32(sm.k), s_v = smem_u32(sm.v), s_q = smem_u32(sm.q);
  const uint32_t s_do = smem_u32(sm.dO), s_pt = smem_u32(sm.pt), s_dst = smem_u32(sm.dst);
  const uint32_t bar_kv = smem_u32(&sm.bar_kv);
  const uint32_t bar_ld0 = smem_u32(&sm.bar_ld[0]), bar_s0 = smem_u32(&sm.bar_s[0]);  // + 8 per buffer
  const uint32_t bar_o0 = smem_u32(&sm.bar_o[0]), bar_p0 = smem_u32(&sm.bar_p[0]);
  constexpr uint32_t kTileBytes = 2 * 2 * QT * kHalf;                               // Q and dO, both halves
  constexpr uint32_t kPBytes = KR * QT * 2;                                         // one P^T / dS^T buffer

  // K, V of key block b (the producer)
  auto issue_kv = [&](int b) {
    mbar_expect_tx(bar_kv, 2 * 2 * KR * kHalf);
    for (int hf = 0; hf < 2; ++hf) {
      tma_load_3d(s_k + hf * KR * kHalf, &tk, bar_kv, hf * 64, b * KR, bh);
      tma_load_3d(s_v + hf * KR * kHalf, &tv, bar_kv, hf * 64, b * KR, bh);
    }
  };
  // pair g's query tile -> buffer g % 3: Q / dO by TMA (the producer), lse and
  // D by softmax threads
  auto issue_tile = [&](int g) {
    int b, i;
    pair_of(g, b, i);
    const int buf = g % 3, t = b * KR + i * QT;
    mbar_expect_tx(bar_ld0 + 8 * buf, kTileBytes);
    for (int hf = 0; hf < 2; ++hf) {
      tma_load_3d(s_q + (2 * buf + hf) * QT * kHalf, &tq, bar_ld0 + 8 * buf, hf * 64, t, bh);
      tma_load_3d(s_do + (2 * buf + hf) * QT * kHalf, &tdo, bar_ld0 + 8 * buf, hf * 64, t, bh);
    }
  };
  auto load_stats = [&](int g) {
    int b, i;
    pair_of(g, b, i);
    const int buf = g % 3, t = b * KR + i * QT;
    if (tid < QT) sm.lse2[buf][tid] = t + tid < T ? lse[t + tid] * kLog2e : 0.f;
    else if (tid < 2 * QT) sm.dq[buf][tid - QT] = t + tid - QT < T ? Db[t + tid - QT] : 0.f;
  };
  // S^T and dP^T of pair g (shared-memory buffer g % 3, the K / V in shared
  // memory) into TMEM buffer g & 1
  auto issue_scores = [&](int g, uint32_t tmem) {
    const int buf = g % 3, tb = g & 1;
    constexpr uint32_t idS = idesc_bf16(KR, QT, false);
#pragma unroll 1
    for (int kk = 0; kk < D / 16; ++kk) {
      const uint32_t hf = kk >> 2, ko = (kk & 3) * 32;
      mma_bf16_ss(tmem + kColS + QT * tb, sdesc_sw128(s_k + hf * KR * kHalf + ko, 16, 1024),
                  sdesc_sw128(s_q + (2 * buf + hf) * QT * kHalf + ko, 16, 1024), idS, kk > 0);
      mma_bf16_ss(tmem + kColDP + QT * tb, sdesc_sw128(s_v + hf * KR * kHalf + ko, 16, 1024),
                  sdesc_sw128(s_do + (2 * buf + hf) * QT * kHalf + ko, 16, 1024), idS, kk > 0);
    }
    mma_commit(bar_s0 + 8 * tb);
  };
  // dV += P^T dO, dK += dS^T Q of pair g (first: the block's first pair, which
  // starts the accumulators): P^T / dS^T buffer g & 1, Q / dO buffer g % 3 as
  // MN-major B operands (16 queries = 2048 bytes per step)
  auto issue_grads = [&](int g, bool first, uint32_t tmem) {
    const int buf = g % 3, pb = g & 1;
    constexpr uint32_t idG = idesc_bf16(KR, D, true);
#pragma unroll
    for (int kk = 0; kk < QT / 16; ++kk) {
      const uint32_t acc = (!first || kk > 0) ? 1u : 0u;
      mma_bf16_ss(tmem + kColDV, sdesc(s_pt + pb * kPBytes + kk * 256, 128, 1024),
                  sdesc_sw128(s_do + 2 * buf * QT * kHalf + kk * 2048, QT * kHalf, 1024), idG, acc);
      mma_bf16_ss(tmem + kColDK, sdesc(s_dst + pb * kPBytes + kk * 256, 128, 1024),
                  sdesc_sw128(s_q + 2 * buf * QT * kHalf + kk * 2048, QT * kHalf, 1024), idG, acc);
    }
    mma_commit(bar_o0 + 8 * pb);
  };

  if (warp == 0) tmem_alloc(smem_u32(&sm.tmem_base), kTmemCols);
  if (tid == 0) {
    mbar_init(bar_kv, 1);
    for (int b = 0; b < 3; ++b) mbar_init(bar_ld0 + 8 * b, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(bar_s0 + 8 * b, 1);
      mbar_init(bar_o0 + 8 * b, 1);
      mbar_init(bar_p0 + 8 * b, NSW / 32);
    }
    mbar_init_fence();
  }
  for (int g = 0; g < 3 && g < npair; ++g) load_stats(g);
  tc_fence_before();
  __syncthreads();  // barriers, TMEM address, first statistics
  tc_fence_after();
  const uint32_t tmem = sm.tmem_base;

  // Every wait below is on a barrier whose next phase cannot complete before
  // the wait is satisfied (each ring of barriers is indexed by the pair's
  // parity and advanced only through the other role; bar_kv only by the
  // producer itself), so parity waits never see a phase ahead of the one
  // they wait for.
  bool alive = true;
  if (warp == NSW / 32) {
    // ---- producer ---------------------------------------------------------
    if (lane == 0) {
      issue_kv(blk0);
      for (int g = 0; g < 3 && g < npair; ++g) issue_tile(g);
      alive = mbar_wait(bar_kv, 0, p.status) && mbar_wait(bar_ld0, 0, p.status);
      if (alive) issue_scores(0, tmem);
      int kvb = blk0, kvn = 0;  // the block whose K / V are loaded, and its load count - 1
#pragma unroll 1
      for (int g = 0; g < npair; ++g) {
        int b, i;
        pair_of(g, b, i);
        // the next pair's scores run on the tensor cores during this softmax
        // (TMEM buffer (g + 1) & 1 was last read before pair g - 1's arrival)
        if (g + 1 < npair) {
          int b1, i1;
          pair_of(g + 1, b1, i1);
          if (b1 != kvb) {  // a new key block: pair g's scores were the last to read K / V
            if (alive) alive = mbar_wait(bar_s0 + 8 * (g & 1), (g >> 1) & 1, p.status);
            if (alive) issue_kv(b1);
            kvb = b1;
            ++kvn;
            if (alive) alive = mbar_wait(bar_kv, kvn & 1, p.status);
          }
          if (alive) alive = mbar_wait(bar_ld0 + 8 * ((g + 1) % 3), ((g + 1) / 3) & 1, p.status);
          if (alive) issue_scores(g + 1, tmem);
        }
        if (g > 0 && g + 2 < npair) {  // Q / dO buffer (g + 2) % 3: read by pair g - 1's gradient MMAs
          if (alive) alive = mbar_wait(bar_o0 + 8 * ((g - 1) & 1), ((g - 1) >> 1) & 1, p.status);
          if (alive) issue_tile(g + 2);
        }
        // pair g's P^T / dS^T written; at a block's first pair this also
        // means the previous block's dK / dV were read out of TMEM (the same
        // warps read them before this pair's softmax)
        if (alive) alive = mbar_wait(bar_p0 + 8 * (g & 1), (g >> 1) & 1, p.status);
        tc_fence_after();
        if (alive) issue_grads(g, i == 0, tmem);
      }
    }
    __syncwarp();
  } else {
    // ---- softmax warps: key row kr (TMEM lane), query columns [32 hf, 32 hf + 32)
    const int kr = tid & (KR - 1), hf = tid >> 7;
    const uint32_t lrow = tmem + ((uint32_t)((warp & 3) * 32) << 16);
    const float sk = p.scale * p.gscale, sv = p.gscale;
#pragma unroll 1
    for (int g = 0; g < npair; ++g) {
      int b, i;
      pair_of(g, b, i);
      const int buf = g % 3, tb = g & 1;
      const int j = b * KR + kr;
      const int t0c = b * KR + i * QT + hf * 32;  // first query column of this thread
      // statistics buffer (g + 2) % 3 was last read for pair g - 1, before
      // the softmax warps' barrier that ended the previous iteration
      if (g > 0 && g + 2 < npair) load_stats(g + 2);
      if (alive) alive = mbar_wait(bar_s0 + 8 * tb, (g >> 1) & 1, p.status);
      tc_fence_after();
      uint32_t s[32], dp[32];
      tmem_ld32(lrow + kColS + QT * tb + hf * 32, s);
      tmem_ld32(lrow + kColDP + QT * tb + hf * 32, dp);
      tmem_ld_wait();
      // P^T, dS^T of this thread's 32 columns
      uint32_t pk[16], dk2[16];
#pragma unroll
      for (int c = 0; c < 32; c += 2) {
        float pr[2], ds[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int t = t0c + c + e, cl = hf * 32 + c + e;
          const bool ok = j < T && t < T && (unsigned)(t - j) < (unsigned)w;
          const float P = ok ? exp2f(fmaf(__uint_as_float(s[c + e]), c2, -sm.lse2[buf][cl])) : 0.f;
          pr[e] = P;
          ds[e] = P * (__uint_as_float(dp[c + e]) - sm.dq[buf][cl]);
        }
        pk[c / 2] = pack_bf16(pr[0], pr[1]);
        dk2[c / 2] = pack_bf16(ds[0], ds[1]);
      }
      if (p.ds_tiles) {  // dS^T of this pair for the split query side: [bh][block][tile][key][query]
        uint4* dst = reinterpret_cast<uint4*>((bf16*)p.ds_tiles +
                                              ((((size_t)bh * nblk + b) * p.ds_nq + i) * KR + kr) * QT + hf * 32);
#pragma unroll
        for (int x = 0; x < 4; ++x) dst[x] = make_uint4(dk2[4 * x], dk2[4 * x + 1], dk2[4 * x + 2], dk2[4 * x + 3]);
      }
      // buffer tb was read by pair g - 2's gradient MMAs
      if (g >= 2 && alive) alive = mbar_wait(bar_o0 + 8 * tb, ((g - 2) >> 1) & 1, p.status);
      uint8_t* ptb = sm.pt[tb];
      uint8_t* dsb = sm.dst[tb];
#pragma unroll
      for (int x = 0; x < 4; ++x) {  // K-major [128 keys][64 queries], 8-row groups 1024 bytes apart
        const uint32_t off = (kr >> 3) * 1024 + (hf * 4 + x) * 128 + (kr & 7) * 16;
        *reinterpret_cast<uint4*>(ptb + off) = make_uint4(pk[4 * x], pk[4 * x + 1], pk[4 * x + 2], pk[4 * x + 3]);
        *reinterpret_cast<uint4*>(dsb + off) = make_uint4(dk2[4 * x], dk2[4 * x + 1], dk2[4 * x + 2], dk2[4 * x + 3]);
      }
      fence_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar_p0 + 8 * tb);
      if (i == nq_of(b) - 1) {
        // ---- the block's last pair: dK, dV rows of its keys, 64 columns per thread
        if (alive) alive = mbar_wait(bar_o0 + 8 * tb, (g >> 1) & 1, p.status);
        tc_fence_after();
        const size_t off = ((size_t)bh * T + j) * D;
#pragma unroll 1
        for (int gi = 0; gi < 2; ++gi) {  // 0: dK, 1: dV
#pragma unroll 1
          for (int c0 = hf * 64; c0 < hf * 64 + 64; c0 += 32) {
            uint32_t r[32];
            tmem_ld32(lrow + (gi == 0 ? kColDK : kColDV) + c0, r);
            tmem_ld_wait();
            if (!alive || j >= T) continue;
            const float sc = gi == 0 ? sk : sv;
            float* f32 = gi == 0 ? p.dk_f32 : p.dv_f32;
            if (f32) {
              float4* dst = reinterpret_cast<float4*>(f32 + off + c0);
#pragma unroll
              for (int x = 0; x < 8; ++x)
                dst[x] = make_float4(__uint_as_float(r[4 * x]) * sc, __uint_as_float(r[4 * x + 1]) * sc,
                                     __uint_as_float(r[4 * x + 2]) * sc, __uint_as_float(r[4 * x + 3]) * sc);
            } else {
              uint32_t pk2[16];
#pragma unroll
              for (int c = 0; c < 32; c += 2)
                pk2[c / 2] = pack_bf16(__uint_as_float(r[c]) * sc, __uint_as_float(r[c + 1]) * sc);
              uint4* dst = reinterpret_cast<uint4*>((bf16*)(gi == 0 ? p.dk : p.dv) + off + c0);
#pragma unroll
              for (int x = 0; x < 4; ++x)
                dst[x] = make_uint4(pk2[4 * x], pk2[4 * x + 1], pk2[4 * x + 2], pk2[4 * x + 3]);
            }
          }
        }
        tc_fence_before();  // these TMEM reads precede the next arrival
      }
      asm volatile("bar.sync 1, %0;" ::"n"(NSW) : "memory");  // softmax warps only
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

bool swa_bwd_kv_tc_supported(int dk, int dv, bool bf16) { return bf16 && dk == D && dv == D; }

cudaError_t launch_swa_bwd_kv_tc(const SwaBwdParams& p, cudaStream_t s) {
  if (p.B * p.H == 0 || p.T == 0) return cudaSuccess;
  const size_t bytes = sizeof(KvSmem) + 1024;  // + room to align the base to 1024
  cudaError_t e = cudaFuncSetAttribute(swa_bwd_kv_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)bytes);
  if (e != cudaSuccess) return e;
  SwaBwdParams pp = p;
  pp.status = device_status_word();
  if (pp.status == nullptr) return cudaErrorInvalidDevicePointer;
  const uint64_t bh = (uint64_t)p.B * p.H;
  CUtensorMap tk, tv, tq, tdo;
  if (!tma_map_rows128(&tk, p.k, p.T, bh, KR) || !tma_map_rows128(&tv, p.v, p.T, bh, KR) ||
      !tma_map_rows128(&tq, p.q, p.T, bh, QT) || !tma_map_rows128(&tdo, p.dO, p.T, bh, QT))
    return cudaErrorInvalidValue;
  dim3 grid(((p.T + KR - 1) / KR + kBlocksPerCta - 1) / kBlocksPerCta, p.B * p.H);
  {
    ScopedTiming tm("swa_bwd_kv_tc", s);
    swa_bwd_kv_tc_kernel<<<grid, NTH, bytes, s>>>(pp, tk, tv, tq, tdo);
  }
  return cudaGetLastError();
}

}  // namespace lz
