// Constant-memory generation step (Lizard technical summary, section 2a: the
// gated branch keeps a fixed-size state instead of a growing KV cache; the
// window branch keeps only the last w keys/values in a ring).
//
// One CTA per (sequence, head).  Per step and head the kernel streams the
// 128x128 fp32 state once in and once out (128-bit loads/stores, 16 rows x 4
// columns per thread), reads the w-slot K/V ring and the M meta tokens once,
// and writes one output row.  It is bound by HBM bandwidth.  The ring rows
// are prefetched into L2 at entry so that their reads overlap the state pass.
//
// The step is one launch: the H CTAs of a sequence read and advance its
// position through one 64-bit atomic on pos[b], whose bits 48 and up count
// the CTAs of the current step that have read it.  A CTA adds 2^48 and takes
// the position from the low bits of the old value; the H-th arrival writes
// position + 1 with a clear count.  Between steps the word is the plain
// position.
#include "common.cuh"
#include "kernels.h"

namespace lz {
namespace {

constexpr int D = 128;
constexpr int NT = 256;
constexpr int WMAX = 1024;
constexpr int MMAX = 16;
constexpr int kPosBits = 48;  // position bits of pos[b]; the arrival count sits above
constexpr unsigned long long kPosMask = (1ull << kPosBits) - 1;

__device__ __forceinline__ void load8(const float* p, float* x) {
  const float4 a = *reinterpret_cast<const float4*>(p);
  const float4 b = *reinterpret_cast<const float4*>(p + 4);
  x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
  x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
}

__device__ __forceinline__ void load8(const bf16* p, float* x) {
  const uint4 u = *reinterpret_cast<const uint4*>(p);
  const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __bfloat1622float2(h[e]);
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
}

template <typename IO>
__global__ void __launch_bounds__(NT, 5) decode_kernel(DecodeParams p) {
  __shared__ float qs[D], ks[D], vs[D], eg[D];
  __shared__ float red[16][D];
  __shared__ float sc[WMAX + MMAX];
  __shared__ float stat[2];
  __shared__ long long spos;
  const int tid = threadIdx.x, warp = tid / 32, lane = tid % 32;
  const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
  const int w = p.w, M = p.M;
  {  // the ring rows the window reads after the state pass: into L2 now, so that
     // they stream from HBM beside the state instead of after it
    constexpr int kLines = D * (int)sizeof(IO) / 128;  // 128-byte lines per ring row
    const int n = 2 * w * kLines;
    for (int x = tid; x < n; x += NT) {
      const int which = x / (w * kLines), r = (x / kLines) % w, ln = x % kLines;
      const IO* ring = (const IO*)(which ? p.vring : p.kring) + ((size_t)bh * w + r) * D;
      asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char*>(ring) + ln * 128));
    }
  }
  if (tid == 0) {  // read the position and count this CTA in (one atomic)
    unsigned long long* pw = reinterpret_cast<unsigned long long*>(p.pos + b);
    const unsigned long long old = atomicAdd(pw, 1ull << kPosBits);
    const unsigned long long cur = old & kPosMask;
    if ((old >> kPosBits) == (unsigned long long)(p.H - 1)) atomicExch(pw, cur + 1);  // last of the H
    spos = (long long)cur;
  }
  if (tid < D) {
    const size_t off = (size_t)bh * D + tid;
    qs[tid] = ldf((const IO*)p.q + off);
    ks[tid] = ldf((const IO*)p.k + off);
    vs[tid] = ldf((const IO*)p.v + off);
    eg[tid] = expf(p.g[off]);
  }
  __syncthreads();
  const long long pos = spos;
  const int slot = (int)(pos % w);
  const int nwin = (int)((pos + 1) < (long long)w ? (pos + 1) : (long long)w);

  // ---- gated state: S <- diag(e^g) S + k v^T ; o_gla = q^T S -------------
  {
    const int rg = warp, cg = lane;  // rows 16*rg .. 16*rg+15, cols 4*cg .. 4*cg+3
    float4* S4 = reinterpret_cast<float4*>(p.state + (size_t)bh * D * D);
    float4 s[16];
#pragma unroll
    for (int r = 0; r < 16; ++r) s[r] = __ldcs(&S4[(rg * 16 + r) * (D / 4) + cg]);
    const float4 vv = reinterpret_cast<const float4*>(vs)[cg];
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
    for (int r = 0; r < 16; ++r) {
      const int i = rg * 16 + r;
      const float e = eg[i], kk = ks[i], qq = qs[i];
      float4 x = s[r];
      x.x = e * x.x + kk * vv.x;
      x.y = e * x.y + kk * vv.y;
      x.z = e * x.z + kk * vv.z;
      x.w = e * x.w + kk * vv.w;
      __stcs(&S4[(rg * 16 + r) * (D / 4) + cg], x);
      o.x += qq * x.x;
      o.y += qq * x.y;
      o.z += qq * x.z;
      o.w += qq * x.w;
    }
    reinterpret_cast<float4*>(red[rg])[cg] = o;
  }

  // ---- window + meta logits: half a warp per key, 8 dims per lane ---------
  const IO* kring = (const IO*)p.kring + (size_t)bh * w * D;
  const IO* vring = (const IO*)p.vring + (size_t)bh * w * D;
  const IO* mk = (const IO*)p.mk + (size_t)h * M * D;
  const IO* mv = p.mv ? (const IO*)p.mv + (size_t)h * M * D : nullptr;
  const int nkeys = nwin + M;
  const int half = lane >> 4, l16 = lane & 15;
  // The trip count depends on the warp only (both half-warps iterate together)
  // because the full-mask shuffles below need all 32 lanes every iteration.
  for (int base = warp * 2; base < nkeys; base += 2 * (NT / 32)) {
    const int key = base + half;
    const bool have = key < nkeys;
    float x[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = 0.f;
    if (!have) {
      // second half-warp past the last key: contributes zeros
    } else if (key == 0) {
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = ks[l16 * 8 + e];
    } else if (key < nwin) {
      const int sl = slot >= key ? slot - key : slot - key + w;  // (pos - key) mod w, 0 < key < w
      load8(kring + (size_t)sl * D + l16 * 8, x);
    } else {
      load8(mk + (size_t)(key - nwin) * D + l16 * 8, x);
    }
    float a = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) a += qs[l16 * 8 + e] * x[e];
    a += __shfl_xor_sync(0xffffffffu, a, 8);
    a += __shfl_xor_sync(0xffffffffu, a, 4);
    a += __shfl_xor_sync(0xffffffffu, a, 2);
    a += __shfl_xor_sync(0xffffffffu, a, 1);
    if (have && l16 == 0) sc[key] = a * p.scale;
  }
  __syncthreads();
  if (warp == 0) {
    float mx = -INFINITY;
    for (int x = lane; x < nkeys; x += 32) mx = fmaxf(mx, sc[x]);
    mx = warp_max(mx);
    float sum = 0.f;
    for (int x = lane; x < nkeys; x += 32) {
      const float e = expf(sc[x] - mx);
      sc[x] = e;
      sum += e;
    }
    sum = warp_sum(sum);
    if (lane == 0) stat[0] = sum;
  }
  __syncthreads();
  // o_gla partials are in red[0..7]; fold them before red is reused
  float og = 0.f;
  if (tid < D) {
#pragma unroll
    for (int r = 0; r < 8; ++r) og += red[r][tid];
  }
  __syncthreads();

  // ---- o_swa numerator: 16 key groups x 16 lanes of 8 dims ----------------
  {
    const int kg = tid / 16, l = tid % 16;
    float acc[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[e] = 0.f;
    for (int key = kg; key < nkeys; key += 16) {
      const float pr = sc[key];
      float x[8];
      if (key == 0) {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = vs[l * 8 + e];
      } else if (key < nwin) {
        const int sl = slot >= key ? slot - key : slot - key + w;  // (pos - key) mod w
        load8(vring + (size_t)sl * D + l * 8, x);
      } else {
        if (!mv) continue;
        load8(mv + (size_t)(key - nwin) * D + l * 8, x);
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e] += pr * x[e];
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) red[kg][l * 8 + e] = acc[e];
  }
  __syncthreads();
  if (tid < D) {
    float osw = 0.f;
#pragma unroll
    for (int r = 0; r < 16; ++r) osw += red[r][tid];
    const float val = og + p.alpha * osw / stat[0];
    ((IO*)p.o)[(size_t)bh * D + tid] = from_f<IO>(val);
    // the new token enters the ring (its slot held a token now out of window)
    ((IO*)p.kring)[((size_t)bh * w + slot) * D + tid] = from_f<IO>(ks[tid]);
    ((IO*)p.vring)[((size_t)bh * w + slot) * D + tid] = from_f<IO>(vs[tid]);
  }
}

// Prefill -> decode hand-off: the state becomes the prefill's final state,
// the ring slot t mod w holds token t of the last min(L, w) prompt tokens,
// pos = L, with L = T or the sequence's own prompt length (lens[b], clamped
// to [0, T]).  One CTA per (sequence, head).
template <typename IO>
__global__ void __launch_bounds__(NT) decode_prefill_kernel(DecodePrefillParams p) {
  const int tid = threadIdx.x;
  const int bh = blockIdx.x, b = bh / p.H, h = bh % p.H;
  const int T = p.T, w = p.w;
  int L = T;
  if (p.lens) {
    const long long l = p.lens[b];
    L = l < 0 ? 0 : (l > T ? T : (int)l);
  }
  float4* st = reinterpret_cast<float4*>(p.state + (size_t)bh * D * D);
  const float4* src = p.hT ? reinterpret_cast<const float4*>(p.hT + (size_t)bh * D * D) : nullptr;
  for (int x = tid; x < D * D / 4; x += NT) st[x] = src ? src[x] : make_float4(0.f, 0.f, 0.f, 0.f);
  const int t0 = L > w ? L - w : 0;
  constexpr int CH = D * (int)sizeof(IO) / 16;  // 16-byte chunks per row
  const uint4* ks = reinterpret_cast<const uint4*>((const IO*)p.k + (size_t)bh * T * D);
  const uint4* vs = reinterpret_cast<const uint4*>((const IO*)p.v + (size_t)bh * T * D);
  uint4* kr = reinterpret_cast<uint4*>((IO*)p.kring + (size_t)bh * w * D);
  uint4* vr = reinterpret_cast<uint4*>((IO*)p.vring + (size_t)bh * w * D);
  for (int x = tid; x < (L - t0) * CH; x += NT) {
    const int t = t0 + x / CH, c = x % CH, slot = t % w;
    kr[(size_t)slot * CH + c] = ks[(size_t)t * CH + c];
    vr[(size_t)slot * CH + c] = vs[(size_t)t * CH + c];
  }
  if (h == 0 && tid == 0) p.pos[b] = L;
}

}  // namespace

cudaError_t launch_decode_prefill(const DecodePrefillParams& p, bool bf16, cudaStream_t s) {
  if (p.Bd == 0 || p.H == 0) return cudaSuccess;
  {
    ScopedTiming tm("decode_prefill", s);
    if (bf16) decode_prefill_kernel<lz::bf16><<<p.Bd * p.H, NT, 0, s>>>(p);
    else decode_prefill_kernel<float><<<p.Bd * p.H, NT, 0, s>>>(p);
  }
  return cudaGetLastError();
}

cudaError_t launch_decode(const DecodeParams& p, bool bf16, cudaStream_t s) {
  if (p.Bd == 0 || p.H == 0) return cudaSuccess;
  {
    ScopedTiming tm("decode_step", s);
    if (bf16) decode_kernel<lz::bf16><<<p.Bd * p.H, NT, 0, s>>>(p);
    else decode_kernel<float><<<p.Bd * p.H, NT, 0, s>>>(p);
  }
  return cudaGetLastError();
}

}  // namespace lz
