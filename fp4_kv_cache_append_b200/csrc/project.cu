// CED decoder-KV producer: kv = H W_KV on the tensor cores, quantised to the
// FP4 cache entry in the GEMM's epilogue.
//   DeepSeek-V4.1-Flash (jaehun.me review), section "1) CED: prefill을 절반으로":
//   the decoder's global KV is the final encoder hidden state projected by
//   each decoder layer's W_KV^l (the flowchart edge "project W_KV^l, W_Z^l";
//   the equation itself was lost, so this is the plain linear projection).
//   Section "3) FP4 main KV": E2M1 values with one E4M3 scale per 16 channels.
//
// One block per (128 token rows, 256 channels), 6 warps:
//   warp 0     TMA producer: per 64-wide slice of d_model, one 128 x 64 box of
//              H (K-major, 128B swizzle) and four 64 x 64 boxes of W_KV (the
//              256 channels, MN-major, 128B swizzle) into a 4-stage ring
//   warp 1     allocates 256 TMEM columns and issues tcgen05.mma kind::f16
//              (bf16 x bf16, fp32 accumulation; M = 128 tokens, N = 256
//              channels, K = 16 per instruction)
//   warps 2-5  epilogue: each thread owns one TMEM lane (= one token) and
//              quantises its 256 channels group by group (scale =
//              E4M3(amax/6), codes = E2M1(x/scale), binary32 divisions,
//              round to nearest even), writing the codes and scales straight
//              to the cache: kv never goes to memory
// The indexer keys of the new entries are formed afterwards from the stored
// FP4 bytes (append_keys_kernel), exactly as for a token append.  All waits
// are bounded; a wait that gives up flags the device status, stops every role,
// drains in-flight copies and MMAs and frees TMEM before the block exits.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kThreads = 192;
constexpr int kStages = 4;
constexpr int kRows = 128;          // tokens per block (M)
constexpr int kCols = 256;          // channels per block (N)
constexpr int kSlice = 64;          // d_model per stage (K): 128 bytes of bf16
constexpr uint32_t kTmemCols = 256;
constexpr uint32_t kWaitLimit = 1u << 22;

struct ProjSmem {
  alignas(1024) uint8_t a[kStages][kRows * kSlice * 2];   // H slice, K-major SW128 (16 KB)
  alignas(1024) uint8_t b[kStages][kSlice * kCols * 2];   // W_KV slice: 4 atoms of 64 k x 64 n (32 KB)
  uint64_t full[kStages], empty[kStages], tfull, drain;
  uint32_t tmem_base;
  int abort;
  int n_issued, n_mma;
};

__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u && *abort) return false;
  }
  *abort = 1;
  return false;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) project_kernel(const __grid_constant__ CUtensorMap h_map,
                                                              const __grid_constant__ CUtensorMap w_map,
                                                              const ProjectArgs a) {
  // bf16 A (K-major) x bf16 B (MN-major), fp32 D
  constexpr uint32_t kIdesc = mma_idesc(kRows, kCols, 1u /*bf16*/, 1u /*bf16*/) | (1u << 16);
  extern __shared__ uint8_t smem_raw[];
  ProjSmem &S = *reinterpret_cast<ProjSmem *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  volatile int *abort = &S.abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row0 = blockIdx.x * kRows, col0 = blockIdx.y * kCols;
  const int nk = a.d / kSlice;

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&S.full[s], 1); mbar_init(&S.empty[s], 1); }
    mbar_init(&S.tfull, 1);
    mbar_init(&S.drain, 1);
    S.abort = 0;
    S.n_issued = 0;
    S.n_mma = 0;
    fence_barrier_init();
    prefetch_tmap(&h_map);
    prefetch_tmap(&w_map);
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  pdl_wait();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;

  auto issue = [&](int i) {   // slice i of d_model into stage i % kStages
    const int s = i % kStages, k0 = i * kSlice;
    mbar_arrive_expect_tx(&S.full[s], kRows * kSlice * 2 + kSlice * kCols * 2);
    tma_load_2d(S.a[s], &h_map, k0, row0, &S.full[s]);
#pragma unroll
    for (int at = 0; at < kCols / 64; ++at)
      tma_load_2d(S.b[s] + at * (kSlice * 128), &w_map, col0 + 64 * at, k0, &S.full[s]);
  };

  if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      for (int i = 0; i < nk; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !wait_or_abort(&S.empty[s], ((i / kStages) - 1) & 1, abort)) break;
        issue(i);
        S.n_issued = i + 1;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      for (int i = 0; i < nk; ++i) {
        const int s = i % kStages;
        if (!wait_or_abort(&S.full[s], (i / kStages) & 1, abort)) break;
        tc_fence_after();
        const uint32_t aa = smem_u32(S.a[s]), bb = smem_u32(S.b[s]);
#pragma unroll
        for (int kk = 0; kk < kSlice / 16; ++kk) {
          // A: 16 bf16 = 32 bytes along the swizzled row; B: 16 rows of 128 B
          tc_mma_f16(tmem, smem_desc_kmajor(aa + kk * 32, 128),
                     smem_desc_mnmajor_sw128(bb + kk * 16 * 128, kSlice * 128, 1024), kIdesc,
                     (i > 0 || kk > 0) ? 1u : 0u);
        }
        tc_commit(&S.empty[s]);
        S.n_mma = i + 1;
      }
      if (S.n_mma == nk) tc_commit(&S.tfull);
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;                 // TMEM lane quarter of this warp
    const int r = row0 + 32 * q + lane;     // token row (b * T + t)
    int ok = 1;
    if (lane == 0) ok = wait_or_abort(&S.tfull, 0, abort);
    ok = __shfl_sync(0xffffffffu, ok, 0);
    if (ok) {
      tc_fence_after();
      const int D = a.D;
      bool live = r < a.B * a.T;
      int b = 0, e = 0;
      if (live) {
        b = r / a.T;
        const int p0 = a.pos0[b];
        e = p0 + r % a.T;
        if (p0 < 0) {
          flag(a.status, CSA2_DEV_BAD_POSITION);
          live = false;
        } else {
          if (blockIdx.y == 0 && r % a.T == a.T - 1) a.n_entries[b] = p0 + a.T;
          if (e >= a.cap) {
            flag(a.status, CSA2_DEV_APPEND_RANGE);
            live = false;
          }
        }
      }
      const size_t er = (size_t)b * a.cap + e;
#pragma unroll 1
      for (int c32 = 0; c32 < kCols / 32; ++c32) {   // 32 channels = two scale groups
        uint32_t v[32];
        tmem_ld_x32(tmem + ((uint32_t)(32 * q) << 16) + 32 * c32, v);
        tmem_wait_ld();
        uint32_t code[4] = {0u, 0u, 0u, 0u};
        uint32_t sb2 = 0u;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
          float amax = 0.0f;
#pragma unroll
          for (int j = 0; j < 16; ++j) amax = fmaxf(amax, fabsf(__uint_as_float(v[16 * g + j])));
          uint32_t sb = amax == 0.0f ? 0u : f32_to_e4m3(__fdiv_rn(amax, 6.0f));
          const float sc = e4m3_to_f32(sb);
          if (sc == 0.0f) sb = 0u;
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const uint32_t cj = sc != 0.0f ? f32_to_e2m1(__fdiv_rn(__uint_as_float(v[16 * g + j]), sc)) : 0u;
            code[2 * g + j / 8] |= cj << (4 * (j % 8));   // byte j/2 of the group: ch 2i low nibble
          }
          sb2 |= sb << (8 * g);
        }
        if (live) {
          const int c0 = col0 + 32 * c32;
          *reinterpret_cast<uint4 *>(a.codes + er * (D / 2) + c0 / 2) = make_uint4(code[0], code[1], code[2], code[3]);
          *reinterpret_cast<uint16_t *>(a.scales + er * (D / 16) + c0 / 16) = (uint16_t)sb2;
        }
      }
    }
  }

  pdl_launch_dependents();
  tc_fence_before();
  __syncthreads();
  if (S.abort) {
    if (tid == 0) {
      flag(a.status, CSA2_DEV_TIMEOUT);
      for (int j = S.n_mma; j < S.n_issued; ++j)
        mbar_wait_bounded(&S.full[j % kStages], (j / kStages) & 1, kWaitLimit);
    }
    if (tid == 32) {
      tc_commit(&S.drain);   // arrives when every MMA issued by this thread is done
      mbar_wait_bounded(&S.drain, 0, kWaitLimit);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }
}

cudaError_t launch_project(const CUtensorMap &h_map, const CUtensorMap &w_map, const ProjectArgs &a, cudaStream_t s) {
  const size_t smem = sizeof(ProjSmem) + 1024;
  cudaError_t e = cudaFuncSetAttribute(project_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  const int rows = a.B * a.T;
  dim3 grid((rows + kRows - 1) / kRows, a.D / kCols);
  return launch_pdl(project_kernel, grid, dim3(kThreads), smem, s, dim3(1, 1, 1), h_map, w_map, a);
}

}  // namespace csa2
