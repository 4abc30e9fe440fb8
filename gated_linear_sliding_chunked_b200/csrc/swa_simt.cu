// Sliding-window softmax attention with meta-memory sinks, SIMT path.
//
// Lizard technical summary, section 2a ("anchor window attention"): exact
// softmax over a local window of recent keys, with learnable meta-memory
// tokens that act as attention sinks in the softmax denominator.  For query
// t the keys are j in [t-w+1, t] plus the M meta keys (always visible):
//   logit_j = scale q_t . k_j,  logit_m = scale q_t . mk_m
//   o_t = (sum_j e^{logit_j} v_j + sum_m e^{logit_m} mv_m) / sum(all e^{logit})
// (mv = 0 in the sink-only reading).  Online max / sum over 32-key tiles.
//
// Backward (textbook softmax Jacobian, dO' = gscale * dO):
//   P = e^{logit - lse},  D_t = dO_t . o_t,  dS = P (dO' . v - gscale D_t)
//   dq_t = scale sum_j dS_tj k_j (+ meta),  dk_j = scale sum_t dS_tj q_t,
//   dv_j = sum_t P_tj dO'_t,  dmk/dmv summed over batch and sequence.
#include "common.cuh"
#include "kernels.h"

namespace lz {
namespace {

constexpr int QR = 16;   // query rows per CTA
constexpr int KT = 32;   // keys per tile (one per lane)
constexpr int NW = 4;    // warps per CTA
constexpr int RPW = QR / NW;
constexpr int KVW = 8;   // warps in the key-major backward kernel

template <typename IO>
__device__ __forceinline__ float ld_or0(const IO* base, size_t off, bool ok) {
  return ok ? ldf(base + off) : 0.f;
}

template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(NW * 32) swa_fwd_simt_kernel(SwaFwdParams p) {
  constexpr int DKP = DK + 1;
  constexpr int NC = DV / 32;
  __shared__ float qs[QR][DK];
  __shared__ float Ks[KT][DKP];
  __shared__ float Vs[KT][DV];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int bh = blockIdx.y, h = bh % p.H;
  const int T = p.T, w = p.w, M = p.M;
  const int t0 = blockIdx.x * QR;
  const IO* q = (const IO*)p.q + (size_t)bh * T * DK;
  const IO* k = (const IO*)p.k + (size_t)bh * T * DK;
  const IO* v = (const IO*)p.v + (size_t)bh * T * DV;
  const IO* mk = (const IO*)p.mk + (size_t)h * M * DK;
  const IO* mv = p.mv ? (const IO*)p.mv + (size_t)h * M * DV : nullptr;

  for (int x = tid; x < QR * DK; x += NW * 32) {
    int r = x / DK, i = x % DK;
    qs[r][i] = ld_or0(q, (size_t)(t0 + r) * DK + i, t0 + r < T) * p.scale;
  }
  float m[RPW], l[RPW], acc[RPW][NC];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    m[rr] = -INFINITY;
    l[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < NC; ++c) acc[rr][c] = 0.f;
  }
  const int lo = max(0, t0 - w + 1);
  const int hi = min(T - 1, t0 + QR - 1);
  const int nmeta = M > 0 ? 1 : 0;
  const int nwt = (hi - lo + KT) / KT;
  for (int tile = 0; tile < nmeta + nwt; ++tile) {
    const bool is_meta = tile < nmeta;
    const int kbase = is_meta ? 0 : lo + (tile - nmeta) * KT;
    __syncthreads();
    for (int x = tid; x < KT * DK; x += NW * 32) {
      int r = x / DK, i = x % DK;
      Ks[r][i] = is_meta ? ld_or0(mk, (size_t)r * DK + i, r < M)
                         : ld_or0(k, (size_t)(kbase + r) * DK + i, kbase + r <= hi);
    }
    for (int x = tid; x < KT * DV; x += NW * 32) {
      int r = x / DV, j = x % DV;
      Vs[r][j] = is_meta ? (mv ? ld_or0(mv, (size_t)r * DV + j, r < M) : 0.f)
                         : ld_or0(v, (size_t)(kbase + r) * DV + j, kbase + r <= hi);
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < RPW; ++rr) {
      const int r = warp * RPW + rr, t = t0 + r;
      const int key = kbase + lane;
      bool valid = is_meta ? (lane < M) : (key <= t && key >= t - w + 1 && key <= hi);
      valid = valid && t < T;
      float s = -INFINITY;
      if (valid) {
        float a = 0.f;
#pragma unroll 8
        for (int i = 0; i < DK; ++i) a += qs[r][i] * Ks[lane][i];
        s = a;
      }
      const float mn = fmaxf(m[rr], warp_max(s));
      if (mn == -INFINITY) continue;
      const float pe = valid ? expf(s - mn) : 0.f;
      const float corr = expf(m[rr] - mn);
      l[rr] = l[rr] * corr + warp_sum(pe);
#pragma unroll
      for (int c = 0; c < NC; ++c) acc[rr][c] *= corr;
#pragma unroll 4
      for (int jj = 0; jj < KT; ++jj) {
        const float pj = __shfl_sync(0xffffffffu, pe, jj);
#pragma unroll
        for (int c = 0; c < NC; ++c) acc[rr][c] += pj * Vs[jj][lane + 32 * c];
      }
      m[rr] = mn;
    }
  }
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int t = t0 + warp * RPW + rr;
    if (t >= T) continue;
    const float inv = 1.f / l[rr];
    const size_t off = ((size_t)bh * T + t) * DV;
#pragma unroll
    for (int c = 0; c < NC; ++c) {
      const float val = acc[rr][c] * inv;
      if (p.o) ((IO*)p.o)[off + lane + 32 * c] = from_f<IO>(val);
      if (p.o_f32) p.o_f32[off + lane + 32 * c] = val;
    }
    if (p.lse && lane == 0) p.lse[(size_t)bh * T + t] = m[rr] + logf(l[rr]);
  }
}

// ---------------------------------------------------------------------------
// Backward, query-major: D_t = dO_t . o_t (rebuilt from lse), dq, and the
// per-block sum of D for dalpha.
// ---------------------------------------------------------------------------
template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(NW * 32) swa_bwd_q_kernel(SwaBwdParams p) {
  constexpr int DKP = DK + 1, DVP = DV + 1;
  constexpr int NCK = DK / 32;
  extern __shared__ float smem_q[];
  float (*qs)[DK] = reinterpret_cast<float (*)[DK]>(smem_q);
  float (*dos)[DV] = reinterpret_cast<float (*)[DV]>(smem_q + QR * DK);
  float (*Ks)[DKP] = reinterpret_cast<float (*)[DKP]>(smem_q + QR * (DK + DV));
  float (*Vs)[DVP] = reinterpret_cast<float (*)[DVP]>(smem_q + QR * (DK + DV) + KT * DKP);
  __shared__ float dsum[NW];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int bh = blockIdx.y, h = bh % p.H;
  const int T = p.T, w = p.w, M = p.M;
  const int t0 = blockIdx.x * QR;
  const IO* q = (const IO*)p.q + (size_t)bh * T * DK;
  const IO* k = (const IO*)p.k + (size_t)bh * T * DK;
  const IO* v = (const IO*)p.v + (size_t)bh * T * DV;
  const IO* dO = (const IO*)p.dO + (size_t)bh * T * DV;
  const IO* mk = (const IO*)p.mk + (size_t)h * M * DK;
  const IO* mv = p.mv ? (const IO*)p.mv + (size_t)h * M * DV : nullptr;
  const float* lse = p.lse + (size_t)bh * T;

  for (int x = tid; x < QR * DK; x += NW * 32) {
    int r = x / DK, i = x % DK;
    qs[r][i] = ld_or0(q, (size_t)(t0 + r) * DK + i, t0 + r < T);
  }
  for (int x = tid; x < QR * DV; x += NW * 32) {
    int r = x / DV, j = x % DV;
    dos[r][j] = ld_or0(dO, (size_t)(t0 + r) * DV + j, t0 + r < T);
  }
  float lrow[RPW], D[RPW], dq[RPW][NCK];
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int t = t0 + warp * RPW + rr;
    lrow[rr] = t < T ? lse[t] : 0.f;
    D[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < NCK; ++c) dq[rr][c] = 0.f;
  }
  const int lo = max(0, t0 - w + 1);
  const int hi = min(T - 1, t0 + QR - 1);
  const int nmeta = M > 0 ? 1 : 0;
  const int nwt = (hi - lo + KT) / KT;
  for (int sweep = 0; sweep < 2; ++sweep) {
    for (int tile = 0; tile < nmeta + nwt; ++tile) {
      const bool is_meta = tile < nmeta;
      const int kbase = is_meta ? 0 : lo + (tile - nmeta) * KT;
      __syncthreads();
      for (int x = tid; x < KT * DK; x += NW * 32) {
        int r = x / DK, i = x % DK;
        Ks[r][i] = is_meta ? ld_or0(mk, (size_t)r * DK + i, r < M)
                           : ld_or0(k, (size_t)(kbase + r) * DK + i, kbase + r <= hi);
      }
      for (int x = tid; x < KT * DV; x += NW * 32) {
        int r = x / DV, j = x % DV;
        Vs[r][j] = is_meta ? (mv ? ld_or0(mv, (size_t)r * DV + j, r < M) : 0.f)
                           : ld_or0(v, (size_t)(kbase + r) * DV + j, kbase + r <= hi);
      }
      __syncthreads();
#pragma unroll
      for (int rr = 0; rr < RPW; ++rr) {
        const int r = warp * RPW + rr, t = t0 + r;
        const int key = kbase + lane;
        bool valid = is_meta ? (lane < M) : (key <= t && key >= t - w + 1 && key <= hi);
        valid = valid && t < T;
        float P = 0.f, dp = 0.f;
        if (valid) {
          float a = 0.f;
#pragma unroll 8
          for (int i = 0; i < DK; ++i) a += qs[r][i] * Ks[lane][i];
          P = expf(a * p.scale - lrow[rr]);
#pragma unroll 8
          for (int j = 0; j < DV; ++j) dp += dos[r][j] * Vs[lane][j];
        }
        if (sweep == 0) {
          D[rr] += warp_sum(P * dp);
        } else {
          const float ds = p.gscale * P * (dp - D[rr]);
#pragma unroll 4
          for (int jj = 0; jj < KT; ++jj) {
            const float dj = __shfl_sync(0xffffffffu, ds, jj);
#pragma unroll
            for (int c = 0; c < NCK; ++c) dq[rr][c] += dj * Ks[jj][lane + 32 * c];
          }
        }
      }
    }
  }
  float blocksum = 0.f;
#pragma unroll
  for (int rr = 0; rr < RPW; ++rr) {
    const int t = t0 + warp * RPW + rr;
    if (t >= T) continue;
    const size_t off = ((size_t)bh * T + t) * DK;
#pragma unroll
    for (int c = 0; c < NCK; ++c) {
      const float val = dq[rr][c] * p.scale;
      if (p.dq_f32) p.dq_f32[off + lane + 32 * c] = val;
      else ((IO*)p.dq)[off + lane + 32 * c] = from_f<IO>(val);
    }
    if (lane == 0) p.Dbuf[(size_t)bh * T + t] = D[rr];
    blocksum += D[rr];
  }
  if (lane == 0) dsum[warp] = blocksum;
  __syncthreads();
  if (tid == 0) {
    float s = 0.f;
    for (int x = 0; x < NW; ++x) s += dsum[x];
    p.alpha_part[(size_t)blockIdx.y * gridDim.x + blockIdx.x] = s;
  }
}

// ---------------------------------------------------------------------------
// Backward, key-major: dk_j, dv_j over the queries t in [j, j+w-1].
// ---------------------------------------------------------------------------
template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(KVW * 32) swa_bwd_kv_kernel(SwaBwdParams p) {
  constexpr int DKP = DK + 1, DVP = DV + 1;
  constexpr int NCK = DK / 32, NCV = DV / 32;
  constexpr int KR = QR;   // keys per CTA
  constexpr int KPW = KR / KVW;  // keys per warp
  extern __shared__ float smem_kv[];
  float (*kj)[DK] = reinterpret_cast<float (*)[DK]>(smem_kv);
  float (*vj)[DV] = reinterpret_cast<float (*)[DV]>(smem_kv + KR * DK);
  float (*Qs)[DKP] = reinterpret_cast<float (*)[DKP]>(smem_kv + KR * (DK + DV));
  float (*dOs)[DVP] = reinterpret_cast<float (*)[DVP]>(smem_kv + KR * (DK + DV) + KT * DKP);
  __shared__ float ls[KT], Ds[KT];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int bh = blockIdx.y;
  const int T = p.T, w = p.w;
  const int j0 = blockIdx.x * KR;
  const IO* q = (const IO*)p.q + (size_t)bh * T * DK;
  const IO* k = (const IO*)p.k + (size_t)bh * T * DK;
  const IO* v = (const IO*)p.v + (size_t)bh * T * DV;
  const IO* dO = (const IO*)p.dO + (size_t)bh * T * DV;
  const float* lse = p.lse + (size_t)bh * T;
  const float* Db = p.Dbuf + (size_t)bh * T;

  for (int x = tid; x < KR * DK; x += KVW * 32) {
    int r = x / DK, i = x % DK;
    kj[r][i] = ld_or0(k, (size_t)(j0 + r) * DK + i, j0 + r < T);
  }
  for (int x = tid; x < KR * DV; x += KVW * 32) {
    int r = x / DV, c = x % DV;
    vj[r][c] = ld_or0(v, (size_t)(j0 + r) * DV + c, j0 + r < T);
  }
  float dk[KPW][NCK], dv[KPW][NCV];
#pragma unroll
  for (int rr = 0; rr < KPW; ++rr) {
#pragma unroll
    for (int c = 0; c < NCK; ++c) dk[rr][c] = 0.f;
#pragma unroll
    for (int c = 0; c < NCV; ++c) dv[rr][c] = 0.f;
  }
  const int tlo = j0;
  const int thi = min(T - 1, j0 + KR - 1 + w - 1);
  for (int tb = tlo; tb <= thi; tb += KT) {
    __syncthreads();
    for (int x = tid; x < KT * DK; x += KVW * 32) {
      int r = x / DK, i = x % DK;
      Qs[r][i] = ld_or0(q, (size_t)(tb + r) * DK + i, tb + r <= thi);
    }
    for (int x = tid; x < KT * DV; x += KVW * 32) {
      int r = x / DV, c = x % DV;
      dOs[r][c] = ld_or0(dO, (size_t)(tb + r) * DV + c, tb + r <= thi);
    }
    if (tid < KT) {
      ls[tid] = tb + tid <= thi ? lse[tb + tid] : 0.f;
      Ds[tid] = tb + tid <= thi ? Db[tb + tid] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < KPW; ++rr) {
      const int r = warp * KPW + rr, j = j0 + r;
      const int t = tb + lane;
      const bool valid = j < T && t <= thi && t >= j && t <= j + w - 1;
      float P = 0.f, ds = 0.f;
      if (valid) {
        float a = 0.f, dp = 0.f;
#pragma unroll 8
        for (int i = 0; i < DK; ++i) a += Qs[lane][i] * kj[r][i];
        P = expf(a * p.scale - ls[lane]);
#pragma unroll 8
        for (int c = 0; c < DV; ++c) dp += dOs[lane][c] * vj[r][c];
        ds = p.gscale * P * (dp - Ds[lane]);
      }
#pragma unroll 4
      for (int tt = 0; tt < KT; ++tt) {
        const float dst = __shfl_sync(0xffffffffu, ds, tt);
        const float pt = __shfl_sync(0xffffffffu, P, tt);
#pragma unroll
        for (int c = 0; c < NCK; ++c) dk[rr][c] += dst * Qs[tt][lane + 32 * c];
#pragma unroll
        for (int c = 0; c < NCV; ++c) dv[rr][c] += pt * dOs[tt][lane + 32 * c];
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < KPW; ++rr) {
    const int j = j0 + warp * KPW + rr;
    if (j >= T) continue;
    const size_t ok = ((size_t)bh * T + j) * DK, ov = ((size_t)bh * T + j) * DV;
#pragma unroll
    for (int c = 0; c < NCK; ++c) {
      const float val = dk[rr][c] * p.scale;
      if (p.dk_f32) p.dk_f32[ok + lane + 32 * c] = val;
      else ((IO*)p.dk)[ok + lane + 32 * c] = from_f<IO>(val);
    }
#pragma unroll
    for (int c = 0; c < NCV; ++c) {
      const float val = dv[rr][c] * p.gscale;
      if (p.dv_f32) p.dv_f32[ov + lane + 32 * c] = val;
      else ((IO*)p.dv)[ov + lane + 32 * c] = from_f<IO>(val);
    }
  }
}

// ---------------------------------------------------------------------------
// Meta gradients: per (batch, head, slab of rows) partial sums, written to
// scratch; one warp per meta token (M <= 16, 8 warps, two tokens each).
// ---------------------------------------------------------------------------
constexpr int SLAB = kSwaBwdSlab;
constexpr int MW = 8;  // warps in the meta kernel

template <typename IO, int DK, int DV>
__global__ void __launch_bounds__(MW * 32) swa_bwd_meta_kernel(SwaBwdParams p) {
  constexpr int NCK = DK / 32, NCV = DV / 32;
  constexpr int RT = 16;
  __shared__ float Qs[RT][DK];
  __shared__ float dOs[RT][DV];
  __shared__ float ls[RT], Ds[RT];
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int h = blockIdx.x, b = blockIdx.y, slab = blockIdx.z;
  const int H = p.H, T = p.T, M = p.M;
  const int bh = b * H + h;
  const IO* q = (const IO*)p.q + (size_t)bh * T * DK;
  const IO* dO = (const IO*)p.dO + (size_t)bh * T * DV;
  const IO* mk = (const IO*)p.mk + (size_t)h * M * DK;
  const IO* mv = p.mv ? (const IO*)p.mv + (size_t)h * M * DV : nullptr;
  const float* lse = p.lse + (size_t)bh * T;
  const float* Db = p.Dbuf + (size_t)bh * T;
  const int r0 = slab * SLAB, r1 = min(T, r0 + SLAB);

  float mkr[2][NCK], mvr[2][NCV], gk[2][NCK], gv[2][NCV];
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int m = warp + MW * e;
#pragma unroll
    for (int c = 0; c < NCK; ++c) {
      mkr[e][c] = m < M ? ldf(mk + (size_t)m * DK + lane + 32 * c) : 0.f;
      gk[e][c] = 0.f;
    }
#pragma unroll
    for (int c = 0; c < NCV; ++c) {
      mvr[e][c] = (m < M && mv) ? ldf(mv + (size_t)m * DV + lane + 32 * c) : 0.f;
      gv[e][c] = 0.f;
    }
  }
  for (int rb = r0; rb < r1; rb += RT) {
    __syncthreads();
    for (int x = tid; x < RT * DK; x += MW * 32) {
      int r = x / DK, i = x % DK;
      Qs[r][i] = ld_or0(q, (size_t)(rb + r) * DK + i, rb + r < r1);
    }
    for (int x = tid; x < RT * DV; x += MW * 32) {
      int r = x / DV, c = x % DV;
      dOs[r][c] = ld_or0(dO, (size_t)(rb + r) * DV + c, rb + r < r1);
    }
    if (tid < RT) {
      ls[tid] = rb + tid < r1 ? lse[rb + tid] : 0.f;
      Ds[tid] = rb + tid < r1 ? Db[rb + tid] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int m = warp + MW * e;
      if (m >= M) continue;
      for (int r = 0; r < RT; ++r) {
        if (rb + r >= r1) break;
        float a = 0.f, dp = 0.f;
#pragma unroll
        for (int c = 0; c < NCK; ++c) a += Qs[r][lane + 32 * c] * mkr[e][c];
#pragma unroll
        for (int c = 0; c < NCV; ++c) dp += dOs[r][lane + 32 * c] * mvr[e][c];
        a = warp_sum(a);
        dp = warp_sum(dp);
        const float P = expf(a * p.scale - ls[r]);
        const float ds = p.gscale * P * (dp - Ds[r]);
#pragma unroll
        for (int c = 0; c < NCK; ++c) gk[e][c] += ds * Qs[r][lane + 32 * c];
#pragma unroll
        for (int c = 0; c < NCV; ++c) gv[e][c] += P * dOs[r][lane + 32 * c];
      }
    }
  }
  const int nslab = gridDim.z;
  float* part = p.meta_part + ((((size_t)b * nslab + slab) * H + h) * M) * (DK + DV);
#pragma unroll
  for (int e = 0; e < 2; ++e) {
    const int m = warp + MW * e;
    if (m >= M) continue;
    float* dst = part + (size_t)m * (DK + DV);
#pragma unroll
    for (int c = 0; c < NCK; ++c) dst[lane + 32 * c] = gk[e][c] * p.scale;
#pragma unroll
    for (int c = 0; c < NCV; ++c) dst[DK + lane + 32 * c] = gv[e][c] * p.gscale;
  }
}

// Fixed-order sums of the partials: meta gradients and dalpha.
__global__ void swa_bwd_reduce_kernel(SwaBwdParams p, int nparts, int nalpha) {
  const int DK = p.dkd, DV = p.dvd, H = p.H, M = p.M;
  const int per = M * (DK + DV);
  const int total = H * per;
  const int gid = blockIdx.x * blockDim.x + threadIdx.x;
  if (gid < total) {
    const int h = gid / per, rem = gid % per;
    const int m = rem / (DK + DV), col = rem % (DK + DV);
    float s = 0.f;
    for (int x = 0; x < nparts; ++x) s += p.meta_part[((size_t)x * H + h) * per + rem];
    if (col < DK) {
      if (p.dmk) p.dmk[((size_t)h * M + m) * DK + col] = s;
    } else {
      if (p.dmv && p.mv) p.dmv[((size_t)h * M + m) * DV + col - DK] = s;
    }
  }
  if (blockIdx.x == 0 && p.dalpha) {
    __shared__ float red[256];
    float s = 0.f;
    for (int x = threadIdx.x; x < nalpha; x += blockDim.x) s += p.alpha_part[x];
    red[threadIdx.x] = s;
    __syncthreads();
    for (int st = blockDim.x / 2; st > 0; st >>= 1) {
      if ((int)threadIdx.x < st) red[threadIdx.x] += red[threadIdx.x + st];
      __syncthreads();
    }
    if (threadIdx.x == 0) p.dalpha[0] = red[0];
  }
}

template <typename IO, int DK, int DV>
cudaError_t fwd_launch(const SwaFwdParams& p, cudaStream_t s) {
  dim3 grid((p.T + QR - 1) / QR, p.B * p.H);
  {
    ScopedTiming tm("swa_fwd_simt", s);
    swa_fwd_simt_kernel<IO, DK, DV><<<grid, NW * 32, 0, s>>>(p);
  }
  return cudaGetLastError();
}

template <typename IO, int DK, int DV>
cudaError_t bwd_launch(const SwaBwdParams& p, cudaStream_t s) {
  dim3 gq((p.T + QR - 1) / QR, p.B * p.H);
  const bool empty = p.T == 0 || p.B * p.H == 0;
  cudaError_t e = cudaSuccess;
  if (!empty) {
    const size_t sq = sizeof(float) * (QR * (DK + DV) + KT * (DK + 1) + KT * (DV + 1));
    e = cudaFuncSetAttribute(swa_bwd_q_kernel<IO, DK, DV>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sq);
    if (e != cudaSuccess) return e;
    {
      ScopedTiming tm("swa_bwd_q_simt", s);
      swa_bwd_q_kernel<IO, DK, DV><<<gq, NW * 32, sq, s>>>(p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    e = cudaFuncSetAttribute(swa_bwd_kv_kernel<IO, DK, DV>,
                             cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sq);
    if (e != cudaSuccess) return e;
    {
      ScopedTiming tm("swa_bwd_kv_simt", s);
      swa_bwd_kv_kernel<IO, DK, DV><<<gq, KVW * 32, sq, s>>>(p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  int nparts = 0;
  if (p.M > 0 && !empty) {
    dim3 gm(p.H, p.B, (p.T + SLAB - 1) / SLAB);
    {
      ScopedTiming tm("swa_bwd_meta_simt", s);
      swa_bwd_meta_kernel<IO, DK, DV><<<gm, MW * 32, 0, s>>>(p);
    }
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    nparts = p.B * ((p.T + SLAB - 1) / SLAB);
  }
  const int total = p.H * p.M * (DK + DV);
  const int blocks = max(1, (total + 255) / 256);
  {
    ScopedTiming tm("swa_bwd_reduce", s);
    swa_bwd_reduce_kernel<<<blocks, 256, 0, s>>>(p, nparts, empty ? 0 : (int)(gq.x * gq.y));
  }
  return cudaGetLastError();
}

}  // namespace

int swa_bwd_n_qblocks(int B, int H, int T) { return ((T + QR - 1) / QR) * B * H; }

cudaError_t launch_swa_bwd_reduce(const SwaBwdParams& p, int nparts, int nalpha, cudaStream_t s) {
  const int total = p.H * p.M * (p.dkd + p.dvd);
  const int blocks = max(1, (total + 255) / 256);
  {
    ScopedTiming tm("swa_bwd_reduce", s);
    swa_bwd_reduce_kernel<<<blocks, 256, 0, s>>>(p, nparts, nalpha);
  }
  return cudaGetLastError();
}
int swa_bwd_n_meta_parts(int B, int T) { return B * ((T + SLAB - 1) / SLAB); }

cudaError_t launch_swa_fwd_simt(const SwaFwdParams& p, bool bf16, cudaStream_t s) {
  if (p.B * p.H == 0 || p.T == 0) return cudaSuccess;
  if (p.dk == 64 && p.dv == 64) return bf16 ? fwd_launch<lz::bf16, 64, 64>(p, s) : fwd_launch<float, 64, 64>(p, s);
  if (p.dk == 64 && p.dv == 128) return bf16 ? fwd_launch<lz::bf16, 64, 128>(p, s) : fwd_launch<float, 64, 128>(p, s);
  if (p.dk == 128 && p.dv == 64) return bf16 ? fwd_launch<lz::bf16, 128, 64>(p, s) : fwd_launch<float, 128, 64>(p, s);
  if (p.dk == 128 && p.dv == 128) return bf16 ? fwd_launch<lz::bf16, 128, 128>(p, s) : fwd_launch<float, 128, 128>(p, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_swa_bwd_simt(const SwaBwdParams& p, bool bf16, cudaStream_t s) {
  if (p.dkd == 64 && p.dvd == 64) return bf16 ? bwd_launch<lz::bf16, 64, 64>(p, s) : bwd_launch<float, 64, 64>(p, s);
  if (p.dkd == 64 && p.dvd == 128) return bf16 ? bwd_launch<lz::bf16, 64, 128>(p, s) : bwd_launch<float, 64, 128>(p, s);
  if (p.dkd == 128 && p.dvd == 64) return bf16 ? bwd_launch<lz::bf16, 128, 64>(p, s) : bwd_launch<float, 128, 64>(p, s);
  if (p.dkd == 128 && p.dvd == 128) return bf16 ? bwd_launch<lz::bf16, 128, 128>(p, s) : bwd_launch<float, 128, 128>(p, s);
  return cudaErrorInvalidValue;
}

}  // namespace lz
