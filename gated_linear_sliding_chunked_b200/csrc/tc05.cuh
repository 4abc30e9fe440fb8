// Blackwell (sm_100a) tensor-core primitives, written as inline PTX:
// tensor-memory (TMEM) allocation, shared-memory matrix descriptors, the
// single-thread tcgen05.mma issue with completion on an mbarrier, and the
// TMEM -> register loads of the accumulators.
//
// Shared-memory operands written by threads use the canonical no-swizzle
// ("interleaved") layout: the unit is a core matrix of 8 rows x 16 bytes
// stored as 128 contiguous bytes.
//   K-major operand (rows = M or N, 16-byte chunks along K):
//     byte(row, kc) = (row / 8) * SBO + kc * LBO + (row % 8) * 16
//   MN-major operand (16-byte chunks along M/N, rows along K):
//     byte(kr, nc)  = nc * SBO + (kr / 8) * LBO + (kr % 8) * 16
// One kind::f16 MMA consumes K = 16 (two core matrices along K), so the next
// K step starts 2 * LBO bytes further.  Operands loaded by TMA use the
// 128-byte swizzle instead (sdesc_sw128): a [rows][64] bf16 box is rows of
// 128 bytes; K-major, a K step of 16 moves the start 32 bytes along the row
// and SBO = 1024 steps 8 rows; MN-major (rows = K), a K step of 16 moves 2048
// bytes, SBO = 1024 steps 8 K-rows and LBO steps to the next 64-wide block.
//
// The accumulator D of an M = 128, cta_group::1 MMA sits in TMEM lanes
// 0..127 (lane = row), one fp32 column per output column.  Warp w of the CTA
// may only read lanes [32 (w % 4), 32 (w % 4) + 32).
//
// Every wait is bounded: after kWaitLimitNs of wall time it gives up,
// adds one to the library's device status word (read and cleared by
// lz_device_check) and returns false, so a kernel never spins forever.
#pragma once

#include <stdint.h>

namespace lz {

constexpr unsigned long long kWaitLimitNs = 200ull * 1000 * 1000;  // 0.2 s

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
  return t;
}

// ---- mbarrier ---------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_init_fence() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n.reg .pred p;\n"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(bar), "r"(parity)
      : "memory");
  return done != 0;
}
// One arrival on the barrier's current phase (release at CTA scope).
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
// Waits for the phase with the given parity to complete; false on timeout
// (counted in *status).
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, unsigned int* status) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (uint32_t it = 0; it < (1u << 28); ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) break;
  }
  atomicAdd(status, 1u);
  return false;
}

// ---- TMA (tensor copies global -> shared, no multicast) --------------------
// The issuing thread announces the bytes the barrier's current phase waits
// for (and arrives once); every tensor copy then completes part of them.
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
               : "memory");
}
// Box at (c0, c1, c2) of the 3-D tensor map `map` (a __grid_constant__
// kernel parameter) into shared memory at dst; rows outside the tensor read
// as zeros.  c0 * element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void* map, uint32_t bar, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// Box at (c0, c1) of the 2-D tensor map `map`; same rules.
__device__ __forceinline__ void tma_load_2d(uint32_t dst, const void* map, uint32_t bar, int c0, int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];" ::"r"(
          dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1)
      : "memory");
}

// ---- proxies and ordering -------------------------------------------------
// Makes this thread's generic-proxy shared-memory writes (st.shared,
// cp.async) visible to the tensor core's async proxy.
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// ---- TMEM allocation (one warp, .sync.aligned) ----------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols));
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::);
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

// ---- descriptors ------------------------------------------------------------
// Shared-memory matrix descriptor, no swizzle: start address, leading and
// stride byte offsets (all >> 4), descriptor version 1 (bit 46).
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46);
}
// The same with the 128-byte swizzle of TMA tiles: 8 rows of 128 bytes form
// a 1024-byte atom whose 16-byte chunks are XOR-permuted by row % 8; atoms
// must start 1024-byte aligned.
__device__ __forceinline__ uint64_t sdesc_sw128(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return sdesc(saddr, lbo, sbo) | (2ull << 61);
}
// Instruction descriptor of kind::f16 with bf16 A and B, fp32 accumulation,
// K-major A (bit 15 clear); B K-major (b_mn = false) or MN-major (b_mn =
// true, bit 16).
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool b_mn) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((b_mn ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// The same with A MN-major as well (A read transposed from a tile whose rows
// run along K).
__host__ __device__ constexpr uint32_t idesc_bf16_at(int M, int N, bool b_mn) {
  return idesc_bf16(M, N, b_mn) | (1u << 15);
}

// D[tmem] (+)= A[smem] * B[smem]; issued by one thread.
__device__ __forceinline__ void mma_bf16_ss(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\n"
      "setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n}\n" ::"r"(d_tmem),
      "l"(a), "l"(b), "r"(idesc), "r"(accumulate), "r"(0u));
}
// The mbarrier gets one arrival once every MMA this thread issued before is
// complete.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar)
               : "memory");
}

// ---- TMEM -> registers ----------------------------------------------------
// 32 lanes x 32 consecutive 32-bit columns: thread l of the warp gets lane
// (base lane + l), columns col .. col+31.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// 32 lanes x 16 columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_ld_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

}  // namespace lz
