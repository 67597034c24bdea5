// Device helpers shared by the TileQ kernels (sm_100a).
#pragma once
#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include "tileq.h"

namespace tileq {

constexpr int kMaxExperts = 64;
constexpr int kMaxTopK = 8;

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ldmatrix of four / two 8x8 fp16 tiles from a shared-window address.
__device__ __forceinline__ void ldmatrix_x4_a(uint32_t (&r)[4], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(saddr));
}
__device__ __forceinline__ void ldmatrix_x2_a(uint32_t (&r)[2], uint32_t saddr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.shared.b16 {%0,%1}, [%2];\n" : "=r"(r[0]), "=r"(r[1]) : "r"(saddr));
}

// D = A(16x16, row) * B(16x8, col) + D, fp16 inputs, fp32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                              uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// (a & b) | c in one LOP3.
__device__ __forceinline__ uint32_t and_or(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("lop3.b32 %0, %1, %2, %3, 0xEA;\n" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

__device__ __forceinline__ uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t *>(&h); }
__device__ __forceinline__ __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2 *>(&u); }

// Exact q - z of one k16 step of an m16 A fragment from a packed code word
// (the group scale is applied to the fp32 partial sums instead).  Bits 2i and
// 16+2i of `w` hold the (lo, hi) codes of register i; OR-ing the fp16 exponent
// of 1024 turns a masked field into 1024 + 4^i*q exactly, and one FMA by 4^-i
// with nz[i] = -(1024 * 4^-i + z_row(i)) leaves q - z, also exactly.
__device__ __forceinline__ void dequant_qz_k16(uint32_t w, const __half2 (&nz)[4], uint32_t (&a)[4]) {
  const uint32_t kMagic = 0x64006400u;
  const __half2 v0 = u32_as_h2(and_or(w, 0x00030003u, kMagic));
  const __half2 v1 = u32_as_h2(and_or(w, 0x000C000Cu, kMagic));
  const __half2 v2 = u32_as_h2(and_or(w, 0x00300030u, kMagic));
  const __half2 v3 = u32_as_h2(and_or(w, 0x00C000C0u, kMagic));
  a[0] = h2_as_u32(__hfma2(v0, u32_as_h2(0x3C003C00u), nz[0]));
  a[1] = h2_as_u32(__hfma2(v1, u32_as_h2(0x34003400u), nz[1]));
  a[2] = h2_as_u32(__hfma2(v2, u32_as_h2(0x2C002C00u), nz[2]));
  a[3] = h2_as_u32(__hfma2(v3, u32_as_h2(0x24002400u), nz[3]));
}

// 3-bit codes: as dequant_qz_k16, with the high bit of register i's codes at
// bits 2i+2 and 18+2i of `h` (just above the 2-bit field, which is masked to
// zero there): one more AND-OR places it, and the fp16 value becomes
// 1024 + 4^i*(q_lo + 4*q_hi) = 1024 + 4^i*q, still exact (q <= 7).
__device__ __forceinline__ void dequant_qz3_k16(uint32_t w, uint32_t h, const __half2 (&nz)[4],
                                                uint32_t (&a)[4]) {
  const uint32_t kMagic = 0x64006400u;
  const __half2 v0 = u32_as_h2(and_or(w, 0x00030003u, and_or(h, 0x00040004u, kMagic)));
  const __half2 v1 = u32_as_h2(and_or(w, 0x000C000Cu, and_or(h, 0x00100010u, kMagic)));
  const __half2 v2 = u32_as_h2(and_or(w, 0x00300030u, and_or(h, 0x00400040u, kMagic)));
  const __half2 v3 = u32_as_h2(and_or(w, 0x00C000C0u, and_or(h, 0x01000100u, kMagic)));
  a[0] = h2_as_u32(__hfma2(v0, u32_as_h2(0x3C003C00u), nz[0]));
  a[1] = h2_as_u32(__hfma2(v1, u32_as_h2(0x34003400u), nz[1]));
  a[2] = h2_as_u32(__hfma2(v2, u32_as_h2(0x2C002C00u), nz[2]));
  a[3] = h2_as_u32(__hfma2(v3, u32_as_h2(0x24002400u), nz[3]));
}

// D = A * B (C = 0), fp16 inputs, fp32 result.
__device__ __forceinline__ void mma_f16_16816_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0,
                                                uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%10,%10,%10,%10};\n"
      : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.f));
}

__device__ __forceinline__ void set_status(int *status, int code) {
  if (status) atomicCAS(status, 0, code);
}

__device__ __forceinline__ float silu_f(float a) { return a / (1.0f + __expf(-a)); }

// fp16 of an internal activation (x, z, z', h); a value outside fp16's finite
// range, NaN included, records TILEQ_ERR_RANGE in the device status word.
__device__ __forceinline__ __half half_checked(float v, int *status) {
  if (!(fabsf(v) <= 65504.f)) set_status(status, TILEQ_ERR_RANGE);
  return __float2half_rn(v);
}
__device__ __forceinline__ __half2 half2_checked(float a, float b, int *status) {
  if (!(fmaxf(fabsf(a), fabsf(b)) <= 65504.f) || a != a || b != b) set_status(status, TILEQ_ERR_RANGE);
  return __floats2half2_rn(a, b);
}

// ------------------------------------------------------------------ mbarrier / bulk copy
__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_addr(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_addr(bar)) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_addr(bar)),
               "r"(bytes)
               : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_addr(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Bounded wait: gives up after about 2^31 SM clock cycles (around a second)
// and records TILEQ_ERR_TIMEOUT in *status; a pipeline wait that long means
// the producer or consumer on the other side has stopped.
constexpr long long kWaitLimitCycles = 1ll << 31;
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, int *status) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity)) {
    if (clock64() - t0 > kWaitLimitCycles) {
      set_status(status, TILEQ_ERR_TIMEOUT);
      return false;
    }
  }
  return true;
}
// 1-D bulk copy global -> shared, completion counted in bytes on `bar`.
__device__ __forceinline__ void bulk_g2s(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::"r"(
          smem_addr(dst)),
      "l"(src), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}
// Programmatic dependent launch (the forward's kernels are launched with the
// programmatic stream serialization attribute): wait until the previous kernel
// in the stream has completed and its writes are visible, then let the next one
// start its prologue.  Every CTA calls this before its first global memory
// access, so a kernel never completes before its predecessor.
__device__ __forceinline__ void pdl_wait_and_release() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}
// Hint: bring the line holding `p` into L2.
__device__ __forceinline__ void prefetch_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];\n" ::"l"(p));
}
// Named barrier over `count` threads (count a multiple of 32).
__device__ __forceinline__ void named_sync(int id, int count) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(count) : "memory");
}


}  // namespace tileq
