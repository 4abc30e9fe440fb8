// Context parallelism of the hybrid operator: one long sequence split into R
// contiguous segments, one per GPU.
//
// The gated branch's state obeys S_t = diag(exp(g_t)) S_{t-1} + k_t v_t^T
// (Lizard technical summary, section 2a, the state update), a linear
// recurrence, so a whole segment acts on the state it receives as
// h -> diag(E_seg) h + S_seg, with E_seg the product of the segment's gates
// per key dim and S_seg the segment's final state from a zero start.  The
// state entering segment r is therefore a fold of the earlier segments'
// pairs, and the state gradient leaving segment r a reverse fold of the later
// segments' (E, G) pairs; the window branch needs only the last w - 1 keys and
// values of the previous segment (a halo).  The pages describe no
// multi-device split; these kernels are the arithmetic of that exchange
// (segment decays, the folds, and the row copies that assemble halos and sum
// the branches), while the host moves the data between ranks.
#include <algorithm>
#include <cstdio>

#include "../../include/lizard.h"
#include "common.cuh"
#include "kernels.h"

namespace {

constexpr int NT = 256;

// E[bh][i] = exp(sum_t g[bh][t][i]): one block per (batch, head); threads
// cover (row phase, key dim) so that a warp reads consecutive dims of a row;
// the phases' partial sums are added in a fixed order.
__global__ void __launch_bounds__(NT) cp_segment_decay_kernel(int T, int dk, const float* g,
                                                              float* E) {
  __shared__ float part[NT];
  const int bh = blockIdx.x, tid = threadIdx.x;
  const int nph = NT / dk, ph = tid / dk, i = tid % dk;
  const float* gb = g + (size_t)bh * T * dk;
  float s = 0.f;
  if (ph < nph) {
#pragma unroll 8
    for (int t = ph; t < T; t += nph) s += gb[(size_t)t * dk + i];
  }
  part[tid] = s;
  __syncthreads();
  if (tid < dk) {
    float tot = 0.f;
    for (int x = 0; x < nph; ++x) tot += part[x * dk + tid];
    E[(size_t)bh * dk + tid] = expf(tot);
  }
}

// Forward fold (dir 0): h = init; for q = 0 .. r-1: h = diag(E_q) h + X_q.
// Reverse fold (dir 1): h = init; for q = R-1 down to r+1: h = X_q + diag(E_q) h.
// One thread per 4 consecutive value columns of one (batch-head, key dim).
__global__ void __launch_bounds__(NT) cp_fold_kernel(int R, int r, int dir, int BH, int dk, int dv,
                                                     const float* E, const float* X,
                                                     const float* init, float* out) {
  const size_t n4 = (size_t)BH * dk * dv / 4;
  const size_t x = (size_t)blockIdx.x * NT + threadIdx.x;
  if (x >= n4) return;
  const size_t e = x * 4;                 // element index in [BH][dk][dv]
  const size_t row = e / dv;              // bh * dk + i
  const size_t seg = (size_t)BH * dk * dv;
  float4 h = init ? reinterpret_cast<const float4*>(init)[x] : make_float4(0.f, 0.f, 0.f, 0.f);
  const int lo = dir == 0 ? 0 : r + 1, hi = dir == 0 ? r : R;  // segments [lo, hi)
  for (int s = 0; s < hi - lo; ++s) {
    const int q = dir == 0 ? lo + s : hi - 1 - s;
    const float d = E[(size_t)q * BH * dk + row];
    const float4 a = reinterpret_cast<const float4*>(X + (size_t)q * seg)[x];
    h = make_float4(d * h.x + a.x, d * h.y + a.y, d * h.z + a.z, d * h.w + a.w);
  }
  reinterpret_cast<float4*>(out)[x] = h;
}

// dst[bh][dst_off + t][:] = a_scale * A[bh][a_off + t][:] + B[bh][b_off + t][:]
// for t < n (A, B nullable = zeros; fp32 sum, one rounding to IO on store).
template <typename IO>
__global__ void __launch_bounds__(NT) cp_rows_kernel(int n, int d, const IO* A, int aT, int aoff,
                                                     float as, const IO* B, int bT, int boff,
                                                     IO* dst, int dT, int doff) {
  const int bh = blockIdx.y;
  const size_t per = (size_t)n * d;
  for (size_t x = (size_t)blockIdx.x * NT + threadIdx.x; x < per; x += (size_t)gridDim.x * NT) {
    const size_t t = x / d, c = x % d;
    float y = 0.f;
    if (A) y = as * lz::to_f(A[((size_t)bh * aT + aoff + t) * d + c]);
    if (B) y += lz::to_f(B[((size_t)bh * bT + boff + t) * d + c]);
    dst[((size_t)bh * dT + doff + t) * d + c] = lz::from_f<IO>(y);
  }
}

lz_status fail(lz_status st, const char* what) {
  return (lz_status)lz::set_last_error(st, what);
}

lz_status done(cudaError_t e, const char* what) {
  if (e == cudaSuccess) {
    lz::set_last_error(LZ_OK, "");
    return LZ_OK;
  }
  char msg[256];
  std::snprintf(msg, sizeof(msg), "%s: %s", what, cudaGetErrorString(e));
  return fail(LZ_ERR_CUDA, msg);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" {

lz_status lz_cp_segment_decay(int BH, int T, int dk, const float* g, float* E, lz_stream stream) {
  if (BH < 0 || T < 0) return fail(LZ_ERR_INVALID_ARG, "lz_cp_segment_decay: BH, T must be >= 0");
  if (dk != 64 && dk != 128) return fail(LZ_ERR_UNSUPPORTED, "lz_cp_segment_decay: dk must be 64 or 128");
  if (BH == 0) return done(cudaSuccess, "");
  if (!E || (T > 0 && !g)) return fail(LZ_ERR_INVALID_ARG, "lz_cp_segment_decay: NULL g or E");
  if (!aligned16(g) || !aligned16(E))
    return fail(LZ_ERR_INVALID_ARG, "lz_cp_segment_decay: g and E must be 16-byte aligned");
  cp_segment_decay_kernel<<<BH, NT, 0, (cudaStream_t)stream>>>(T, dk, g, E);
  return done(cudaGetLastError(), "lz_cp_segment_decay");
}

lz_status lz_cp_fold(int R, int r, int dir, int BH, int dk, int dv, const float* E, const float* X,
                     const float* init, float* out, lz_stream stream) {
  if (R < 1 || r < 0 || r >= R || (dir != 0 && dir != 1) || BH < 0 || dk < 1 || dv < 1)
    return fail(LZ_ERR_INVALID_ARG, "lz_cp_fold: need R >= 1, 0 <= r < R, dir 0 or 1, BH >= 0");
  if (dv % 4) return fail(LZ_ERR_UNSUPPORTED, "lz_cp_fold: dv must be a multiple of 4");
  if (BH == 0) return done(cudaSuccess, "");
  if (!E || !X || !out) return fail(LZ_ERR_INVALID_ARG, "lz_cp_fold: NULL E, X or out");
  if (!aligned16(X) || !aligned16(out) || (init && !aligned16(init)) || !aligned16(E))
    return fail(LZ_ERR_INVALID_ARG, "lz_cp_fold: pointers must be 16-byte aligned");
  const size_t n4 = (size_t)BH * dk * dv / 4;
  const unsigned blocks = (unsigned)((n4 + NT - 1) / NT);
  cp_fold_kernel<<<blocks, NT, 0, (cudaStream_t)stream>>>(R, r, dir, BH, dk, dv, E, X, init, out);
  return done(cudaGetLastError(), "lz_cp_fold");
}

lz_status lz_cp_rows(int BH, int d, lz_dtype io, int n, const void* A, int a_T, int a_off,
                     float a_scale, const void* B, int b_T, int b_off, void* dst, int dst_T,
                     int dst_off, lz_stream stream) {
  if (BH < 0 || d < 1 || n < 0) return fail(LZ_ERR_INVALID_ARG, "lz_cp_rows: BH, n >= 0, d >= 1");
  if (io != LZ_F32 && io != LZ_BF16) return fail(LZ_ERR_UNSUPPORTED, "lz_cp_rows: io must be LZ_F32 or LZ_BF16");
  if (a_off < 0 || b_off < 0 || dst_off < 0 || (A && a_off + n > a_T) || (B && b_off + n > b_T) ||
      dst_off + n > dst_T)
    return fail(LZ_ERR_INVALID_ARG, "lz_cp_rows: a row range lies outside its tensor");
  if (BH == 0 || n == 0) return done(cudaSuccess, "");
  if (!dst) return fail(LZ_ERR_INVALID_ARG, "lz_cp_rows: dst must not be NULL");
  if (BH > 65535) return fail(LZ_ERR_UNSUPPORTED, "lz_cp_rows: BH must be <= 65535");
  const size_t per = (size_t)n * d;
  const unsigned gx = (unsigned)std::min<size_t>((per + NT - 1) / NT, 1024);
  const dim3 grid(gx, BH);
  if (io == LZ_BF16)
    cp_rows_kernel<lz::bf16><<<grid, NT, 0, (cudaStream_t)stream>>>(
        n, d, (const lz::bf16*)A, a_T, a_off, a_scale, (const lz::bf16*)B, b_T, b_off,
        (lz::bf16*)dst, dst_T, dst_off);
  else
    cp_rows_kernel<float><<<grid, NT, 0, (cudaStream_t)stream>>>(
        n, d, (const float*)A, a_T, a_off, a_scale, (const float*)B, b_T, b_off, (float*)dst,
        dst_T, dst_off);
  return done(cudaGetLastError(), "lz_cp_rows");
}

}  // extern "C"
