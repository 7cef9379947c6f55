// Device helpers shared by the libcsa2 kernels: bf16/E4M3/E2M1 codecs,
// shared-memory swizzle, mbarrier + TMA wrappers (inline PTX, sm_100a).
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

// ------------------------------------------------------------------ scalars

__device__ __forceinline__ float bf16_to_f32(uint16_t h) { return __uint_as_float((uint32_t)h << 16); }

// E4M3 byte -> binary32 (exact).  E4M3: sign | 4-bit exponent (bias 7) | 3-bit
// mantissa; exponent 0 is subnormal (m * 2^-9).  0x7F/0xFF (NaN) never occur
// in data this library writes.
__device__ __forceinline__ float e4m3_to_f32(uint32_t b) {
  uint32_t e = (b >> 3) & 15u, m = b & 7u;
  float mag = e ? __uint_as_float(((e + 120u) << 23) | (m << 20)) : (float)m * 0.001953125f;
  return (b & 0x80u) ? -mag : mag;
}

// binary32 -> E4M3, round to nearest even on the 3-bit mantissa, saturating at
// +-448, sign kept (-0 and negative values rounding to zero give 0x80).
__device__ __forceinline__ uint32_t f32_to_e4m3(float x) {
  uint32_t u = __float_as_uint(x);
  uint32_t sign = (u >> 24) & 0x80u;
  float a = fabsf(x);
  if (!(a < 464.0f)) return (x != x) ? 0x7Fu : (sign | 0x7Eu);
  if (a < 0.015625f) {                       // below 2^-6: multiples of 2^-9
    return sign | (uint32_t)rintf(a * 512.0f);   // exact scaling, rint = ties-to-even
  }
  uint32_t ua = __float_as_uint(a);
  int e = (int)(ua >> 23) - 127 + 7;         // biased E4M3 exponent, 1..15
  uint32_t keep = (ua >> 20) & 7u, rest = ua & 0xFFFFFu;
  if (rest > 0x80000u || (rest == 0x80000u && (keep & 1u))) keep += 1u;
  if (keep == 8u) { keep = 0u; e += 1; }
  uint32_t code = ((uint32_t)e << 3) | keep;
  return sign | (code > 0x7Eu ? 0x7Eu : code);
}

// binary32 -> E2M1 code: nearest of {0,.5,1,1.5,2,3,4,6}, ties to the even
// code, saturating at 6, sign kept.  Each threshold is a midpoint; whether it
// is inclusive follows from which neighbour has the even code.
__device__ __forceinline__ uint32_t f32_to_e2m1(float y) {
  float a = fabsf(y);
  uint32_t c = (uint32_t)(a > 0.25f) + (uint32_t)(a >= 0.75f) + (uint32_t)(a > 1.25f) +
               (uint32_t)(a >= 1.75f) + (uint32_t)(a > 2.5f) + (uint32_t)(a >= 3.5f) +
               (uint32_t)(a > 5.0f);
  return c | ((__float_as_uint(y) >> 28) & 8u);
}

// E2M1 code -> binary32 magnitude table evaluated arithmetically (exact).
__device__ __forceinline__ float e2m1_to_f32(uint32_t c) {
  uint32_t e = (c >> 1) & 3u, m = c & 1u;
  float mag = e ? __uint_as_float(((e + 126u) << 23) | (m << 22)) : 0.5f * (float)m;
  return (c & 8u) ? -mag : mag;
}

// ------------------------------------------------------------------ status

__device__ __forceinline__ void flag(unsigned int *status, unsigned int bit) {
  if (status) atomicOr(status, bit);
}

// ------------------------------------------------------------------ swizzle
// Physical offset of logical byte offset o inside a tile written by TMA with
// the 128B (mask 7) or 64B (mask 3) swizzle: 16-byte chunk bits [4,7) are
// XORed with bits [7,10).
template <int MASK>
__device__ __forceinline__ uint32_t swz(uint32_t o) { return o ^ (((o >> 7) & MASK) << 4); }

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

// ------------------------------------------------------------------ mbarrier

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait: returns false (and the caller flags a timeout) after
// `limit` polls; try_wait itself suspends for a hardware-defined interval.
__device__ __forceinline__ bool mbar_wait_bounded(uint64_t *bar, uint32_t parity, uint32_t limit) {
  for (uint32_t i = 0; i < limit; ++i)
    if (mbar_try_wait(bar, parity)) return true;
  return false;
}

// 2D TMA tile load (no multicast) into shared memory, completing on `bar`.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, int x, int y, uint64_t *bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"((uint64_t)map), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map) : "memory");
}

// ------------------------------------------------------------------ ldmatrix / mma

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t &r0, uint32_t &r1, uint32_t &r2, uint32_t &r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

// D += A(16x32 e4m3, row) * B(32x8 e4m3, col), fp32 accumulate.
__device__ __forceinline__ void mma_e4m3_16832(float *d, const uint32_t *a, const uint32_t *b) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.f32.e4m3.e4m3.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// D += A(16x16 f16, row) * B(16x8 f16, col), fp32 accumulate.
__device__ __forceinline__ void mma_f16_16816(float *d, const uint32_t *a, const uint32_t *b) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// ------------------------------------------------------------------ launch helpers (host)

struct DevInfo {
  int sms;
  size_t max_smem_optin;
};

}  // namespace csa2
