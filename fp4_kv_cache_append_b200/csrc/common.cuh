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

// ------------------------------------------------------------------ hardware converts (exact)

// Eight E2M1 codes (one 32-bit word; each byte holds a channel pair, low
// nibble = even channel) -> four f16x2 (low half = even channel).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t *h) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\tmov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\tcvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\tcvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
      : "r"(w));
}
// Four E4M3 bytes (one 32-bit word, low byte first) -> two f16x2.
__device__ __forceinline__ void e4m3x4_to_f16x2(uint32_t w, uint32_t *h) {
  asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
      "cvt.rn.f16x2.e4m3x2 %0, lo;\n\tcvt.rn.f16x2.e4m3x2 %1, hi;\n\t}"
      : "=r"(h[0]), "=r"(h[1])
      : "r"(w));
}
// Two E4M3 bytes (low 16 bits) -> one f16x2.
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t w) {
  uint32_t h;
  asm("{\n\t.reg .b16 lo;\n\tcvt.u16.u32 lo, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, lo;\n\t}" : "=r"(h) : "r"(w));
  return h;
}

// ------------------------------------------------------------------ programmatic dependent launch
// Kernels launched with programmatic stream serialisation start while the
// previous kernel of the stream drains: pdl_wait() returns once that grid has
// completed and its memory is visible (a no-op without the attribute), and
// pdl_launch_dependents() lets the next kernel of the stream launch early.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

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

// Non-blocking test of a phase (never suspends).
__device__ __forceinline__ bool mbar_test_wait(uint64_t *bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n selp.u32 %0, 1, 0, p;\n}\n"
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

// L2 prefetch of one box of a 2D tensor map (x 16-byte aligned).  A prefetch
// only warms L2, the point of coherence, so it may run before the data's
// producer has finished: a later load still sees the producer's stores.
__device__ __forceinline__ void tma_prefetch_l2_2d(const CUtensorMap *map, int x, int y) {
  asm volatile("cp.async.bulk.prefetch.tensor.2d.L2.global.tile [%0, {%1, %2}];" ::"l"((uint64_t)map), "r"(x), "r"(y)
               : "memory");
}
// L2 prefetch of a contiguous range (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void prefetch_l2(const void *src, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(src), "r"(bytes) : "memory");
}

// 1D bulk copy global -> shared (both 16-byte aligned, size a multiple of 16),
// completing on `bar`.
__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   smem_u32(dst)),
               "l"((uint64_t)src), "r"(bytes), "r"(smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void prefetch_tmap(const CUtensorMap *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"((uint64_t)map) : "memory");
}

// ------------------------------------------------------------------ tcgen05 (5th-gen tensor cores, TMEM)

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols) {  // one full warp
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {  // the allocating warp
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Arrive on `bar` once every tcgen05 operation this thread issued so far is done.
__device__ __forceinline__ void tc_commit(uint64_t *bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
               : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, FP8 (E4M3 x E4M3) with fp32 accumulation.
__device__ __forceinline__ void tc_mma_f8(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, f16 x f16 with fp32 accumulation.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                           uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem]^T, f16 x f16 with fp32 accumulation (A read
// from tensor memory: 128 lanes = rows, 16-bit elements packed two per column).
__device__ __forceinline__ void tc_mma_f16_ta(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 32 TMEM lanes (this warp's quarter) x 32 consecutive 32-bit columns.
__device__ __forceinline__ void tmem_ld_x32(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
// Load 16 consecutive 32-bit columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}
// 16 TMEM lanes (the lower half of this warp's 32) in two halves: thread t < 16
// gets lane t's 32 columns from taddr, thread t >= 16 lane t - 16's 32 columns
// from taddr + 32 (the 16x32bx2 shape, half-split offset 32 columns).
__device__ __forceinline__ void tmem_ld_16x32bx2_x32(uint32_t taddr, uint32_t *r) {
  asm volatile(
      "tcgen05.ld.sync.aligned.16x32bx2.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32], 32;"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// Store 32 consecutive 32-bit columns of this warp's 32 TMEM lanes.
__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t *r) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]), "r"(r[17]),
      "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]),
      "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Descriptor of an MN-major operand in the 128B-swizzled layout: rows of 64
// 16-bit elements along M (128 B), 8-row groups along K `sbo` bytes apart,
// 64-element M atoms `lbo` bytes apart.
__device__ __forceinline__ uint64_t smem_desc_mnmajor_sw128(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) | ((uint64_t)(sbo >> 4) << 32) |
         (1ull << 46) | (2ull << 61);
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

// One lane of a converged warp (the lowest active one, the same lane on every
// call with the same active set).  tcgen05.mma / tcgen05.commit are issued
// under it from code the whole warp runs: the descriptors then stay warp-
// uniform, which keeps the issue of back-to-back MMAs near the tensor core's
// own rate (a lane-0-only branch issues them several times slower).
__device__ __forceinline__ bool elect_one() {
  uint32_t p;
  asm volatile("{\n .reg .pred e;\n elect.sync _|e, 0xffffffff;\n selp.u32 %0, 1, 0, e;\n}\n" : "=r"(p));
  return p != 0;
}

// Named barrier over `nthreads` threads (whole warps) that also returns
// whether any of them passed a true predicate.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n .reg .pred p, q;\n setp.ne.u32 q, %1, 0;\n bar.red.or.pred p, %2, %3, q;\n selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(r)
      : "r"((uint32_t)pred), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// Named barrier over the first `nthreads` threads of the block (id 1..15).
__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// Shared-memory matrix descriptor of a K-major operand stored in the
// canonical swizzled layout (rows of `row_bytes` = the swizzle width, 8-row
// atoms `8 * row_bytes` apart): start address >> 4 (bits 0-13), leading byte
// offset (unused for swizzled K-major, 1), stride byte offset >> 4 (bits
// 32-45), descriptor version 1 (bits 46-47), layout type (bits 61-63:
// 2 = 128B swizzle, 4 = 64B swizzle).  The operand base must be aligned to
// the swizzle atom; K steps inside the atom advance the start address.
__device__ __forceinline__ uint64_t smem_desc_kmajor(uint32_t addr, int row_bytes) {
  const uint64_t layout = row_bytes == 128 ? 2ull : 4ull;
  const uint64_t sbo = (uint64_t)(8 * row_bytes) >> 4;
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | (1ull << 16) | (sbo << 32) | (1ull << 46) | (layout << 61);
}

// Instruction descriptor (kind::f8f6f4 / kind::f16): D format f32 (bits 4-5
// = 1), A/B formats (bits 7-9 / 10-12), both operands K-major (bits 15, 16 =
// 0), N >> 3 (bits 17-22), M >> 4 (bits 24-28).
__host__ __device__ constexpr uint32_t mma_idesc(int m, int n, uint32_t a_fmt, uint32_t b_fmt) {
  return (1u << 4) | (a_fmt << 7) | (b_fmt << 10) | ((uint32_t)(n >> 3) << 17) | ((uint32_t)(m >> 4) << 24);
}

// ------------------------------------------------------------------ indexer query preparation

// One warp prepares head h of query row `row` (see QueryPrep in kernels.h):
// E4M3 codes of q_h / s_q with s_q = amax(q_h)/448 (binary32 divisions, round
// to nearest even), written into the 128B (dI = 128) or 64B (dI = 64) swizzled
// B operand, and w_h * s_q.  Heads >= H_I are zero.  The query and the head
// weights are inputs that no launch of the library writes; WAIT makes the warp
// wait for the previous launch only before its stores (the buffer they go to
// may still be read by the previous scan).
template <int DI, bool WAIT, typename Prep>
__device__ __forceinline__ void prep_query_head(const Prep &p, int row, int h, int lane) {
  constexpr int MASK = DI == 128 ? 7 : 3;
  const uint16_t *qrow = p.q_idx + (size_t)row * p.H_I * DI;
  uint8_t *q8 = p.q8 + (size_t)row * 64 * DI;
  float v[DI / 32];
  float amax = 0.f;
  if (h < p.H_I) {
#pragma unroll
    for (int i = 0; i < DI / 32; ++i) {
      v[i] = bf16_to_f32(qrow[h * DI + lane + 32 * i]);
      amax = fmaxf(amax, fabsf(v[i]));
    }
    for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  }
  const float sq = __fdiv_rn(amax, 448.0f);
  uint32_t code[DI / 32];
#pragma unroll
  for (int i = 0; i < DI / 32; ++i) code[i] = (h < p.H_I && sq != 0.f) ? f32_to_e4m3(__fdiv_rn(v[i], sq)) : 0u;
  const float wq = (lane == 0 && h < p.H_I) ? p.w[(size_t)row * p.H_I + h] * sq : 0.f;
  if (WAIT) pdl_wait();
#pragma unroll
  for (int i = 0; i < DI / 32; ++i) q8[swz<MASK>(h * DI + lane + 32 * i)] = (uint8_t)code[i];
  if (lane == 0) p.wq[(size_t)row * 64 + h] = wq;
}

}  // namespace csa2
