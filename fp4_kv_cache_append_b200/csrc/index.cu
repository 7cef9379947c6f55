// Indexer scoring: score_j = sum_h w_h ReLU(s_q,h s_k,j <q8_h, k8_j>) over the
// FP8 indexer keys (Full: every visible entry; Reindex: the 8-entry blocks of
// the candidate pool).
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2": each Full layer
//   scores the whole context with its own indexer; the Hierarchical Sparse
//   Indexer lets later Reindex layers rescore only the <= 2,048 x 8 pool.
//
// Work layout: entries on M (128-entry tiles), indexer heads on N (64, zero
// padded), d_I on K.  Per block (one query row, a run of tiles), 6 warps:
//   warp 0     TMA producer: a Full tile is one box of 128 rows x d_I bytes,
//              a Reindex tile 16 boxes of 8 rows at the pool's block rows;
//              hardware 128B/64B swizzle, into a STAGES ring
//   warp 1     allocates 128 TMEM columns and issues tcgen05.mma kind::f8f6f4
//              (M=128, N=64, K=32 per instruction) into one of two TMEM
//              accumulators; tcgen05.commit frees the smem stage and hands
//              the accumulator to the epilogue
//   warps 2-5  epilogue: each thread owns one TMEM lane (= one entry), reads
//              its 64 head accumulators with tcgen05.ld and reduces
//              s_k * sum_h (w_h s_q,h) * max(acc_h, 0) -> one fp32 score
// The head reduction never leaves registers; scores are written once,
// coalesced.  The visible tiles of a row are split evenly over the row's
// blocks (about four blocks per SM in one wave).  The FP8 query of each row
// is prepared once (index_prep_kernel, or by the append launch that precedes
// the scan: csa2_append_quant_ex) into the caller's workspace, already in the
// MMA's swizzled layout, and bulk-copied into every block of that row.  All
// waits are bounded: a wait that gives up sets the device
// status bit and an abort flag that stops every role; in-flight copies and
// MMAs are then drained (bounded) and TMEM is freed before the block exits.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kThreads = 192;
constexpr int kStages = 2;   // measured: deeper rings lower the scan's DRAM throughput
constexpr int kTileRows = 128;
constexpr int kHeads = 64;          // N of the MMA (indexer heads, zero padded)
constexpr uint32_t kTmemCols = 128; // two 64-column fp32 accumulators
constexpr uint32_t kWaitLimit = 1u << 22;

template <int DI>
struct IndexSmem {
  alignas(1024) uint8_t tile[kStages][kTileRows * DI];   // A operand ring (K-major, swizzled)
  alignas(1024) uint8_t q8[kHeads * DI];                 // B operand (K-major, swizzled)
  alignas(16) float wq[kHeads];                          // w_h * s_q,h
  uint64_t full[kStages], empty[kStages], tfull[2], tempty[2], drain, qbar, never;
  uint32_t tmem_base;
  int abort;
  int n_issued, n_mma;
};

// Bounded wait that also gives up early once another role raised `abort`.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u && *abort) return false;
  }
  *abort = 1;
  return false;
}

// acc[0..1] += w[0..1] * x[0..1] as one packed f32x2 fused multiply-add (each
// lane rounds exactly as a scalar fmaf).
__device__ __forceinline__ void fma2(float &a0, float &a1, float w0, float w1, float x0, float x1) {
  unsigned long long acc, w, x;
  asm("mov.b64 %0, {%1, %2};" : "=l"(acc) : "f"(a0), "f"(a1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(w) : "f"(w0), "f"(w1));
  asm("mov.b64 %0, {%1, %2};" : "=l"(x) : "f"(x0), "f"(x1));
  asm("fma.rn.f32x2 %0, %1, %2, %0;" : "+l"(acc) : "l"(w), "l"(x));
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a0), "=f"(a1) : "l"(acc));
}

// s4[j] += w_h * max(acc_h, 0) for heads h = j, j+4, ... of one 32-head half
// (wq: the half's 32 weights, 16-byte aligned).
__device__ __forceinline__ void head_reduce32(float *s4, const float *wq, const uint32_t *acc) {
  const float4 *wp = reinterpret_cast<const float4 *>(wq);
#pragma unroll
  for (int h4 = 0; h4 < 8; ++h4) {
    const float4 w = wp[h4];
    const float r0 = fmaxf(__uint_as_float(acc[4 * h4]), 0.f), r1 = fmaxf(__uint_as_float(acc[4 * h4 + 1]), 0.f);
    const float r2 = fmaxf(__uint_as_float(acc[4 * h4 + 2]), 0.f), r3 = fmaxf(__uint_as_float(acc[4 * h4 + 3]), 0.f);
    fma2(s4[0], s4[1], w.x, w.y, r0, r1);
    fma2(s4[2], s4[3], w.z, w.w, r2, r3);
  }
}

// The same reduction for NH consecutive heads (NH a multiple of 4) with the
// weights held in registers.
template <int NH>
__device__ __forceinline__ void head_reduce_reg(float *s4, const float *w, const uint32_t *acc) {
#pragma unroll
  for (int h4 = 0; h4 < NH / 4; ++h4) {
    const float r0 = fmaxf(__uint_as_float(acc[4 * h4]), 0.f), r1 = fmaxf(__uint_as_float(acc[4 * h4 + 1]), 0.f);
    const float r2 = fmaxf(__uint_as_float(acc[4 * h4 + 2]), 0.f), r3 = fmaxf(__uint_as_float(acc[4 * h4 + 3]), 0.f);
    fma2(s4[0], s4[1], w[4 * h4], w[4 * h4 + 1], r0, r1);
    fma2(s4[2], s4[3], w[4 * h4 + 2], w[4 * h4 + 3], r2, r3);
  }
}

}  // namespace

// Indexer query of each row (prep_query_head): grid (rows, 8) x 256 threads,
// one warp per head; the codes are formed while the previous launch runs.
template <int DI>
__global__ void __launch_bounds__(256) index_prep_kernel(const IndexArgs a) {
  pdl_launch_dependents();
  prep_query_head<DI, true>(a, blockIdx.x, blockIdx.y * 8 + (threadIdx.x >> 5), threadIdx.x & 31);
}

template <int DI, bool REINDEX, bool BMAX>
__global__ void __launch_bounds__(kThreads, 4) index_kernel(const __grid_constant__ CUtensorMap ik_map,
                                                            const IndexArgs a) {
  constexpr int KS = DI / 32;   // MMA k-steps (32 bytes of E4M3 each)
  constexpr uint32_t kIdesc = mma_idesc(128, kHeads, 0u /*E4M3*/, 0u /*E4M3*/);
  extern __shared__ uint8_t smem_raw[];
  IndexSmem<DI> &S = *reinterpret_cast<IndexSmem<DI> *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  volatile int *abort = &S.abort;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.y;   // b * T_q + query
  const int b = row / a.T_q;

  // ---- set-up that touches no global memory: barriers (warp 0), TMEM (warp 1)
  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) { mbar_init(&S.full[s], 1); mbar_init(&S.empty[s], 1); }
    for (int x = 0; x < 2; ++x) { mbar_init(&S.tfull[x], 1); mbar_init(&S.tempty[x], 4); }
    mbar_init(&S.drain, 1);
    mbar_init(&S.qbar, 1);
    mbar_init(&S.never, 1);   // nothing arrives on it (diagnostic timeout)
    S.abort = 0;
    S.n_issued = 0;
    S.n_mma = 0;
    fence_barrier_init();
    prefetch_tmap(&ik_map);
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  // the query position is an input no launch writes; with it, the first key
  // tiles and scales are prefetched into L2 while the previous launch (the
  // append that writes the newest entry) finishes
  const int t = a.q_pos[row];
  if (!REINDEX && warp == 2 && lane < kStages && t >= 0) {
    int n_guess = (t + 1) / a.m;
    if (n_guess > a.cap) n_guess = a.cap;
    const int tiles_g = (n_guess + kTileRows - 1) / kTileRows;
    const int tile = (int)(((int64_t)blockIdx.x * tiles_g) / gridDim.x) + lane;
    if (tile < (int)(((int64_t)(blockIdx.x + 1) * tiles_g) / gridDim.x)) {
      tma_prefetch_l2_2d(&ik_map, 0, b * a.cap + tile * kTileRows);
      prefetch_l2(a.ik_scale + (size_t)b * a.cap + (size_t)tile * kTileRows, kTileRows * 4);
    }
  }
  pdl_wait();

  // ---- this block's tiles: the row's visible tiles split evenly over gridDim.x
  int n_vis = (t + 1) / a.m;
  const int ne = a.n_entries[b];
  if (n_vis > ne) n_vis = ne;
  if (n_vis > a.cap) n_vis = a.cap;
  if (n_vis < 0 || t < 0) n_vis = 0;
  const int tiles_row = REINDEX ? a.tiles_per_row : (n_vis + kTileRows - 1) / kTileRows;
  const int tile0 = (int)(((int64_t)blockIdx.x * tiles_row) / gridDim.x);
  const int tile1 = (int)(((int64_t)(blockIdx.x + 1) * tiles_row) / gridDim.x);
  if (!REINDEX && blockIdx.x == 0 && tid == 0 && a.n_valid) a.n_valid[row] = n_vis;
  const int ntiles = tile1 - tile0;
  const int32_t *pool = REINDEX ? a.pool + (size_t)row * a.P : nullptr;

  auto issue = [&](int i) {   // tile tile0+i into stage i % kStages
    const int s = i % kStages;
    const int tile = tile0 + i;
    mbar_arrive_expect_tx(&S.full[s], kTileRows * DI);
    if (REINDEX) {   // 16 boxes of 8 rows at the pool's blocks
#pragma unroll 1
      for (int g = 0; g < 16; ++g) {
        int blk = pool[tile * 16 + g];
        if (blk < 0 || blk >= a.cap / 8) blk = 0;   // masked in the epilogue
        tma_load_2d(&S.tile[s][g * 8 * DI], &ik_map, 0, b * a.cap + blk * 8, &S.full[s]);
      }
    } else {         // one 128-row box
      tma_load_2d(&S.tile[s][0], &ik_map, 0, b * a.cap + tile * kTileRows, &S.full[s]);
    }
  };
  tc_fence_before();
  __syncthreads();   // barriers initialised, TMEM allocated
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  if (ntiles > 0 && tid == 0) {
    // the prepared query (B operand) and head weights of this row, then the first tiles
    mbar_arrive_expect_tx(&S.qbar, kHeads * DI + kHeads * 4);
    bulk_load(S.q8, a.q8 + (size_t)row * kHeads * DI, kHeads * DI, &S.qbar);
    bulk_load(S.wq, a.wq + (size_t)row * kHeads, kHeads * 4, &S.qbar);
    const int first = ntiles < kStages ? ntiles : kStages;
    for (int i = 0; i < first; ++i) issue(i);
    S.n_issued = first;
  }

  if (ntiles <= 0) {
    // nothing to score
  } else   if (warp == 0) {
    // ------------------------------------------------ TMA producer
    if (lane == 0) {
      for (int i = kStages; i < ntiles; ++i) {
        const int s = i % kStages;
        if (!wait_or_abort(&S.empty[s], ((i / kStages) - 1) & 1, abort)) break;
        issue(i);
        S.n_issued = i + 1;
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(S.q8);
      if (a.inject_polls && !mbar_wait_bounded(&S.never, 0, a.inject_polls)) *abort = 1;
      const bool qok = !*abort && wait_or_abort(&S.qbar, 0, abort);
      for (int i = 0; i < ntiles && qok; ++i) {
        const int s = i % kStages, ab = i & 1;
        if (!wait_or_abort(&S.full[s], (i / kStages) & 1, abort)) break;
        if (i >= 2 && !wait_or_abort(&S.tempty[ab], ((i / 2) - 1) & 1, abort)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(S.tile[s]);
#pragma unroll
        for (int kk = 0; kk < KS; ++kk)
          tc_mma_f8(tmem + ab * kHeads, smem_desc_kmajor(a_addr + kk * 32, DI),
                    smem_desc_kmajor(q_addr + kk * 32, DI), kIdesc, kk > 0 ? 1u : 0u);
        tc_commit(&S.empty[s]);    // stage s may be refilled once these MMAs are done
        tc_commit(&S.tfull[ab]);   // accumulator ab is ready for the epilogue
        S.n_mma = i + 1;
      }
    }
  } else {
    // ------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;                    // TMEM lane quarter of this warp
    const int r = 32 * q + lane;               // tile row = TMEM lane
    // entry id, validity and key scale of this lane's row in tile i
    auto row_of = [&](int i, int &e, bool &valid, float &sk) {
      const int tile = tile0 + i;
      if (REINDEX) {
        const int blk = pool[tile * 16 + (r >> 3)];
        e = blk * 8 + (r & 7);
        valid = blk >= 0 && blk < a.cap / 8 && e < n_vis;
      } else {
        e = tile * kTileRows + r;
        valid = e < n_vis;
      }
      sk = valid ? a.ik_scale[(size_t)b * a.cap + e] : 0.f;
    };
    int e_next;
    bool v_next;
    float sk_next;
    row_of(0, e_next, v_next, sk_next);
    int qok = 1;
    if (lane == 0) qok = wait_or_abort(&S.qbar, 0, abort);   // head weights landed in smem
    qok = __shfl_sync(0xffffffffu, qok, 0);
    __syncwarp();
    for (int i = 0; i < ntiles && qok; ++i) {
      const int ab = i & 1;
      const int tile = tile0 + i;
      const int e = e_next;
      const bool valid = v_next;
      const float sk = sk_next;
      if (i + 1 < ntiles) row_of(i + 1, e_next, v_next, sk_next);   // prefetch one tile ahead
      int ok = 1;
      if (lane == 0) ok = wait_or_abort(&S.tfull[ab], (i / 2) & 1, abort);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      // heads in two halves of 32 columns (fewer live registers); chain j
      // takes heads j, j+4, ... in ascending order
      const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + ab * kHeads;
      float s4[4] = {0.f, 0.f, 0.f, 0.f};   // independent chains
#pragma unroll
      for (int hh = 0; hh < 2; ++hh) {
        uint32_t acc[32];
        tmem_ld_x32(taddr + 32 * hh, acc);
        tmem_wait_ld();
        if (hh == 1) {   // the accumulator is free once both halves are in registers
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.tempty[ab]);
        }
        head_reduce32(s4, &S.wq[32 * hh], acc);
      }
      const float sum = (s4[0] + s4[1]) + (s4[2] + s4[3]);
      float *out = a.scores + (size_t)row * a.ld;
      if (REINDEX) out[tile * kTileRows + r] = valid ? sum * sk : -INFINITY;
      else if (valid) out[e] = sum * sk;
      if (BMAX) {   // the maximum of each block of 8 entries (8 consecutive lanes)
        float m = valid ? sum * sk : -INFINITY;
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
        m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
        if ((r & 7) == 0 && e < n_vis) a.bmax[(size_t)row * a.ld_b + (e >> 3)] = m;
      }
    }
  }

  // ---- teardown: on an abort, drain in-flight copies and MMAs (bounded),
  // then free TMEM
  pdl_launch_dependents();
  __syncthreads();
  if (S.abort) {
    if (tid == 0) {
      flag(a.status, CSA2_DEV_TIMEOUT);
      if (ntiles > 0) mbar_wait_bounded(&S.qbar, 0, kWaitLimit);
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

// ---------------------------------------------------------------------------
// Full scan of R consecutive query rows of one sequence per block (T_q >= 2:
// multi-token decode and prefill).  The rows share the sequence's keys, so
// each 128-entry key tile feeds one MMA with N = 64 R (the R rows' prepared
// queries are consecutive 64-row blocks of one K-major operand), and the
// accumulator of a tile is 64 R TMEM columns (two buffers: 128 R columns).
//   warp 0     TMA producer (4-stage ring of key tiles)
//   warp 1     TMEM allocation, tcgen05.mma kind::f8f6f4 M128 N(64R) K32
//   warps 2..  epilogue, 2R warps: warp w reads TMEM lane quarter w%4 of two
//              rows; per (entry, row) the same head reduction as the one-row
//              kernel (chains j: heads j, j+4, ... ascending), so scores do
//              not depend on the grouping
// Each epilogue thread holds its two rows' 64 head weights in registers: read
// from shared memory for every tile instead, the weights alone kept the L1
// data pipe 80% busy (each 16-byte broadcast load takes several wavefronts).
// The MMA issuer keeps a warp of its own: issuing the MMAs from one lane of
// an epilogue warp (which would free registers) made the scan twice as slow.
// With 10 warps the register budget is 168 per thread, hence 16-column TMEM
// reads.
// Entries beyond a row's causal limit are not written.
constexpr int kMultiStages = 4;
constexpr int kMultiChunk = 16;   // TMEM columns per tcgen05.ld + wait in the epilogue (register budget)
constexpr int kMultiRpw = 2;      // query rows per epilogue warp
template <int R>
constexpr int multi_threads() { return 64 + 4 * (R / kMultiRpw) * 32; }

template <int DI, int R>
struct MultiSmem {
  alignas(1024) uint8_t tile[kMultiStages][kTileRows * DI];
  alignas(1024) uint8_t q8[R * kHeads * DI];
  alignas(16) float wq[R][kHeads];
  uint64_t full[kMultiStages], empty[kMultiStages], tfull[2], tempty[2], drain, qbar, never;
  uint32_t tmem_base;
  int abort;
  int n_issued, n_mma;
};

template <int DI, int R, bool BMAX>
__global__ void __launch_bounds__(multi_threads<R>(), 1) index_multi_kernel(const __grid_constant__ CUtensorMap ik_map,
                                                                           const IndexArgs a) {
  constexpr int KS = DI / 32;
  constexpr uint32_t kCols = 2 * R * kHeads;   // 256 (R = 2) or 512 (R = 4)
  constexpr uint32_t kIdesc = mma_idesc(128, R * kHeads, 0u /*E4M3*/, 0u /*E4M3*/);
  extern __shared__ uint8_t smem_raw[];
  MultiSmem<DI, R> &S = *reinterpret_cast<MultiSmem<DI, R> *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  volatile int *abort = &S.abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int groups = a.T_q / R;                // row groups per sequence
  const int b = blockIdx.y / groups;
  const int row0 = b * a.T_q + (blockIdx.y % groups) * R;

  if (tid == 0) {
    for (int s = 0; s < kMultiStages; ++s) { mbar_init(&S.full[s], 1); mbar_init(&S.empty[s], 1); }
    for (int x = 0; x < 2; ++x) { mbar_init(&S.tfull[x], 1); mbar_init(&S.tempty[x], 4 * R / kMultiRpw); }
    mbar_init(&S.drain, 1);
    mbar_init(&S.qbar, 1);
    mbar_init(&S.never, 1);   // nothing arrives on it (diagnostic timeout)
    S.abort = 0;
    S.n_issued = 0;
    S.n_mma = 0;
    fence_barrier_init();
    prefetch_tmap(&ik_map);
  }
  if (warp == 1) {
    tmem_alloc(&S.tmem_base, kCols);
    tmem_relinquish();
  }
  pdl_wait();

  // ---- the group's rows and this block's tiles (the widest row sets the range)
  const int ne = a.n_entries[b];
  const int my_row = warp >= 2 ? (warp - 2) / 4 * kMultiRpw : 0;   // epilogue warps: first row they reduce
  int n_vis_max = 0, nv_mine[kMultiRpw];
#pragma unroll
  for (int i = 0; i < R; ++i) {
    const int t = a.q_pos[row0 + i];
    int n = (t + 1) / a.m;
    if (n > ne) n = ne;
    if (n > a.cap) n = a.cap;
    if (n < 0 || t < 0) n = 0;
    n_vis_max = n > n_vis_max ? n : n_vis_max;
    if (blockIdx.x == 0 && tid == 0 && a.n_valid) a.n_valid[row0 + i] = n;
#pragma unroll
    for (int k = 0; k < kMultiRpw; ++k)
      if (i == my_row + k) nv_mine[k] = n;
  }
  const int tiles_row = (n_vis_max + kTileRows - 1) / kTileRows;
  const int tile0 = (int)(((int64_t)blockIdx.x * tiles_row) / gridDim.x);
  const int tile1 = (int)(((int64_t)(blockIdx.x + 1) * tiles_row) / gridDim.x);
  const int ntiles = tile1 - tile0;

  auto issue = [&](int i) {
    const int s = i % kMultiStages;
    mbar_arrive_expect_tx(&S.full[s], kTileRows * DI);
    tma_load_2d(&S.tile[s][0], &ik_map, 0, b * a.cap + (tile0 + i) * kTileRows, &S.full[s]);
  };
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  if (ntiles > 0 && tid == 0) {
    // the R prepared query rows are consecutive in the workspace
    mbar_arrive_expect_tx(&S.qbar, R * kHeads * DI + R * kHeads * 4);
    bulk_load(S.q8, a.q8 + (size_t)row0 * kHeads * DI, R * kHeads * DI, &S.qbar);
    bulk_load(&S.wq[0][0], a.wq + (size_t)row0 * kHeads, R * kHeads * 4, &S.qbar);
    const int first = ntiles < kMultiStages ? ntiles : kMultiStages;
    for (int i = 0; i < first; ++i) issue(i);
    S.n_issued = first;
  }

  if (ntiles <= 0) {
    // nothing to score
  } else if (warp == 0) {
    if (lane == 0) {
      for (int i = kMultiStages; i < ntiles; ++i) {
        const int s = i % kMultiStages;
        if (!wait_or_abort(&S.empty[s], ((i / kMultiStages) - 1) & 1, abort)) break;
        issue(i);
        S.n_issued = i + 1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t q_addr = smem_u32(S.q8);
      if (a.inject_polls && !mbar_wait_bounded(&S.never, 0, a.inject_polls)) *abort = 1;
      const bool qok = !*abort && wait_or_abort(&S.qbar, 0, abort);
      for (int i = 0; i < ntiles && qok; ++i) {
        const int s = i % kMultiStages, ab = i & 1;
        if (!wait_or_abort(&S.full[s], (i / kMultiStages) & 1, abort)) break;
        if (i >= 2 && !wait_or_abort(&S.tempty[ab], ((i / 2) - 1) & 1, abort)) break;
        tc_fence_after();
        const uint32_t a_addr = smem_u32(S.tile[s]);
#pragma unroll
        for (int kk = 0; kk < KS; ++kk)
          tc_mma_f8(tmem + ab * R * kHeads, smem_desc_kmajor(a_addr + kk * 32, DI),
                    smem_desc_kmajor(q_addr + kk * 32, DI), kIdesc, kk > 0 ? 1u : 0u);
        tc_commit(&S.empty[s]);
        tc_commit(&S.tfull[ab]);
        S.n_mma = i + 1;
      }
    }
  } else {
    const int q = warp & 3;                  // TMEM lane quarter (warp w accesses lanes 32 (w % 4) ..)
    const int r = 32 * q + lane;
    int qok = 1;
    if (lane == 0) qok = wait_or_abort(&S.qbar, 0, abort);   // head weights in smem
    qok = __shfl_sync(0xffffffffu, qok, 0);
    // the rows' head weights stay in registers: re-reading them from shared
    // memory for every tile (64 x 128 B per warp and row) would saturate the
    // L1 pipe
    float wr[kMultiRpw][kHeads];
    if (qok) {
#pragma unroll
      for (int k = 0; k < kMultiRpw; ++k) {
        const float4 *wp = reinterpret_cast<const float4 *>(&S.wq[my_row + k][0]);
#pragma unroll
        for (int h4 = 0; h4 < kHeads / 4; ++h4) {
          const float4 w = wp[h4];
          wr[k][4 * h4] = w.x; wr[k][4 * h4 + 1] = w.y; wr[k][4 * h4 + 2] = w.z; wr[k][4 * h4 + 3] = w.w;
        }
      }
    }
    for (int i = 0; i < ntiles && qok; ++i) {
      const int ab = i & 1;
      const int e = (tile0 + i) * kTileRows + r;
      const float sk = e < n_vis_max ? a.ik_scale[(size_t)b * a.cap + e] : 0.f;
      int ok = 1;
      if (lane == 0) ok = wait_or_abort(&S.tfull[ab], (i / 2) & 1, abort);
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
#pragma unroll
      for (int k = 0; k < kMultiRpw; ++k) {
        const uint32_t taddr = tmem + ((uint32_t)(32 * q) << 16) + ab * R * kHeads + (my_row + k) * kHeads;
        float s4[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int c = 0; c < kHeads / kMultiChunk; ++c) {
          uint32_t acc[kMultiChunk];
          tmem_ld_x16(taddr + c * kMultiChunk, acc);
          tmem_wait_ld();
          if (k == kMultiRpw - 1 && c == kHeads / kMultiChunk - 1) {   // the accumulator is free once read
            tc_fence_before();
            __syncwarp();
            if (lane == 0) mbar_arrive(&S.tempty[ab]);
          }
          head_reduce_reg<kMultiChunk>(s4, &wr[k][c * kMultiChunk], acc);
        }
        const float sc = ((s4[0] + s4[1]) + (s4[2] + s4[3])) * sk;
        if (e < nv_mine[k]) a.scores[(size_t)(row0 + my_row + k) * a.ld + e] = sc;
        if (BMAX) {   // the maximum of each block of 8 entries (8 consecutive lanes)
          float m = e < nv_mine[k] ? sc : -INFINITY;
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 1));
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 2));
          m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, 4));
          if ((r & 7) == 0 && e < nv_mine[k]) a.bmax[(size_t)(row0 + my_row + k) * a.ld_b + (e >> 3)] = m;
        }
      }
    }
  }

  pdl_launch_dependents();
  __syncthreads();
  if (S.abort) {
    if (tid == 0) {
      flag(a.status, CSA2_DEV_TIMEOUT);
      if (ntiles > 0) mbar_wait_bounded(&S.qbar, 0, kWaitLimit);
      for (int j = S.n_mma; j < S.n_issued; ++j)
        mbar_wait_bounded(&S.full[j % kMultiStages], (j / kMultiStages) & 1, kWaitLimit);
    }
    if (tid == 32) {
      tc_commit(&S.drain);
      mbar_wait_bounded(&S.drain, 0, kWaitLimit);
    }
    __syncthreads();
  }
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

int index_rows_per_block(int T_q, bool reindex) {
  if (reindex) return 1;
  if (T_q % 4 == 0) return 4;
  if (T_q % 2 == 0) return 2;
  return 1;
}

size_t index_workspace_bytes(int rows, int dI) {
  const size_t q = ((size_t)rows * kHeads * dI + 15) & ~size_t(15);
  return q + (size_t)rows * kHeads * 4;
}

template <int DI, int R, bool BMAX>
static cudaError_t launch_multi_t(const CUtensorMap &map, const IndexArgs &a, cudaStream_t s) {
  if (!a.prepared) {
    cudaError_t pe = launch_pdl(index_prep_kernel<DI>, dim3(a.B * a.T_q, kHeads / 8), dim3(256), 0, s, dim3(1, 1, 1), a);
    if (pe != cudaSuccess) return pe;
  }
  // R = 4 takes all 512 TMEM columns: ask for enough shared memory that no
  // second block of the kernel shares the SM (it would wait in tcgen05.alloc)
  size_t smem = sizeof(MultiSmem<DI, R>) + 1024;
  if (R == 4 && smem < 120 * 1024) smem = 120 * 1024;
  auto k = index_multi_kernel<DI, R, BMAX>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.ctas_per_row, a.B * (a.T_q / R));
  return launch_pdl(k, grid, dim3(multi_threads<R>()), smem, s, dim3(1, 1, 1), map, a);
}

// The block-maxima output of the fused selection is a separate instantiation:
// its few extra instructions in the epilogue loop slowed the prefill scan by
// 14% when it was a run-time branch.
template <int DI, int R>
static cudaError_t launch_multi(const CUtensorMap &map, const IndexArgs &a, cudaStream_t s) {
  return a.bmax ? launch_multi_t<DI, R, true>(map, a, s) : launch_multi_t<DI, R, false>(map, a, s);
}

template <int DI, bool REINDEX, bool BMAX>
static cudaError_t launch_t(const CUtensorMap &map, const IndexArgs &a, cudaStream_t s) {
  if (!a.prepared) {
    cudaError_t pe = launch_pdl(index_prep_kernel<DI>, dim3(a.B * a.T_q, kHeads / 8), dim3(256), 0, s, dim3(1, 1, 1), a);
    if (pe != cudaSuccess) return pe;
  }
  const size_t smem = sizeof(IndexSmem<DI>) + 1024;
  auto k = index_kernel<DI, REINDEX, BMAX>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid(a.ctas_per_row, a.B * a.T_q);
  return launch_pdl(k, grid, dim3(kThreads), smem, s, dim3(1, 1, 1), map, a);
}

cudaError_t launch_index(const CUtensorMap &map, const IndexArgs &a, bool reindex, int sms, cudaStream_t s) {
  (void)sms;
  const int R = index_rows_per_block(a.T_q, reindex);
  if (R == 4) return a.dI == 128 ? launch_multi<128, 4>(map, a, s) : launch_multi<64, 4>(map, a, s);
  if (R == 2) return a.dI == 128 ? launch_multi<128, 2>(map, a, s) : launch_multi<64, 2>(map, a, s);
  if (reindex) return a.dI == 128 ? launch_t<128, true, false>(map, a, s) : launch_t<64, true, false>(map, a, s);
  if (a.bmax) return a.dI == 128 ? launch_t<128, false, true>(map, a, s) : launch_t<64, false, true>(map, a, s);
  return a.dI == 128 ? launch_t<128, false, false>(map, a, s) : launch_t<64, false, false>(map, a, s);
}

}  // namespace csa2
