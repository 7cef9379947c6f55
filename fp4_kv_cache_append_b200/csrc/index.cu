// Indexer scoring: score_j = sum_h w_h ReLU(s_q,h s_k,j <q8_h, k8_j>) over the
// FP8 indexer keys (Full: every visible entry; Reindex: the 8-entry blocks of
// the candidate pool).
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2": each Full layer
//   scores the whole context with its own indexer; the Hierarchical Sparse
//   Indexer lets later Reindex layers rescore only the <= 2,048 x 8 pool.
// Layout of the work: entries on the M side (128-entry tiles), indexer heads
// on N (<= 64), d_I on K.  Tiles stream from HBM by 2D TMA (boxes of 8 rows x
// d_I bytes, hardware 128B/64B swizzle) through a STAGES-deep mbarrier ring;
// a Reindex tile is 16 boxes at the pool's block rows, a Full tile 16 boxes
// at consecutive rows.  The head reduction happens in the epilogue on the
// accumulator registers, so each entry's score is produced by one quad of
// lanes and written once.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kThreads = 128;      // 4 warps x 32 entries
constexpr int kStages = 4;
constexpr int kTileRows = 128;
constexpr int kMaxHeads = 64;
constexpr uint32_t kWaitLimit = 1u << 22;

template <int DI>
struct IndexSmem {
  alignas(1024) uint8_t tile[kStages][kTileRows * DI];
  uint8_t q8[kMaxHeads][DI + 16];       // padded rows: conflict-free 32-bit reads
  float wq[kMaxHeads];                  // w_h * s_q,h
  uint64_t full[kStages];
};

}  // namespace

template <int DI, bool REINDEX>
__global__ void __launch_bounds__(kThreads) index_kernel(const __grid_constant__ CUtensorMap ik_map,
                                                         const IndexArgs a) {
  constexpr int MASK = DI == 128 ? 7 : 3;
  constexpr int KS = DI / 32;          // k-steps of 32 bytes
  extern __shared__ uint8_t smem_raw[];
  IndexSmem<DI> &S = *reinterpret_cast<IndexSmem<DI> *>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.y;                 // b * T_q + query
  const int b = row / a.T_q;
  const int t = a.q_pos[row];
  int n_vis = (t + 1) / a.m;
  const int ne = a.n_entries[b];
  if (n_vis > ne) n_vis = ne;
  if (n_vis > a.cap) n_vis = a.cap;
  if (n_vis < 0 || t < 0) n_vis = 0;

  const int tile0 = blockIdx.x * a.tiles_per_cta;
  int tiles_row = REINDEX ? a.tiles_per_row : (n_vis + kTileRows - 1) / kTileRows;
  int tile1 = tile0 + a.tiles_per_cta;
  if (tile1 > tiles_row) tile1 = tiles_row;
  if (!REINDEX && blockIdx.x == 0 && tid == 0 && a.n_valid) a.n_valid[row] = n_vis;
  const int ntiles = tile1 - tile0;
  if (ntiles <= 0) return;

  const int32_t *pool = REINDEX ? a.pool + (size_t)row * a.P : nullptr;

  // ---- barriers, then the producer starts streaming immediately
  if (tid == 0) {
    prefetch_tmap(&ik_map);
    for (int s = 0; s < kStages; ++s) mbar_init(&S.full[s], 1);
    fence_barrier_init();
  }
  __syncthreads();

  auto issue = [&](int i) {  // tile0 + i into stage i % kStages (thread 0 only)
    const int s = i % kStages;
    const int tile = tile0 + i;
    mbar_arrive_expect_tx(&S.full[s], kTileRows * DI);
#pragma unroll 1
    for (int g = 0; g < 16; ++g) {
      int r;
      if (REINDEX) {
        int blk = pool[tile * 16 + g];
        if (blk < 0 || blk >= a.cap / 8) blk = 0;
        r = b * a.cap + blk * 8;
      } else {
        r = b * a.cap + tile * kTileRows + g * 8;
      }
      tma_load_2d(&S.tile[s][g * 8 * DI], &ik_map, 0, r, &S.full[s]);
    }
  };
  if (tid == 0) {
    for (int i = 0; i < ntiles && i < kStages; ++i) issue(i);
  }

  // ---- indexer query: per head, FP8 with scale amax/448 (same rule as the keys)
  const uint16_t *qrow = a.q_idx + (size_t)row * a.H_I * DI;
  const float *wrow = a.w + (size_t)row * a.H_I;
  for (int h = warp; h < kMaxHeads; h += kThreads / 32) {
    if (h < a.H_I) {
      float v[DI / 32];
      float amax = 0.f;
#pragma unroll
      for (int i = 0; i < DI / 32; ++i) {
        v[i] = bf16_to_f32(qrow[h * DI + lane + 32 * i]);
        amax = fmaxf(amax, fabsf(v[i]));
      }
      for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
      const float sq = __fdiv_rn(amax, 448.0f);
#pragma unroll
      for (int i = 0; i < DI / 32; ++i)
        S.q8[h][lane + 32 * i] = (uint8_t)(sq == 0.f ? 0u : f32_to_e4m3(__fdiv_rn(v[i], sq)));
      if (lane == 0) S.wq[h] = wrow[h] * sq;
    } else {
#pragma unroll
      for (int i = 0; i < DI / 32; ++i) S.q8[h][lane + 32 * i] = 0;
      if (lane == 0) S.wq[h] = 0.f;
    }
  }
  __syncthreads();

  // B fragments (q8 as the 32x8 col-major operand: column n = head) and the
  // head weights of this lane's accumulator columns.
  const int gid = lane >> 2, tq = lane & 3;
  const int ntn = (a.H_I + 7) / 8;
  uint32_t bf[8][KS][2];
  float wl[8][2];
#pragma unroll
  for (int n = 0; n < 8; ++n) {
#pragma unroll
    for (int k = 0; k < KS; ++k) {
      bf[n][k][0] = *reinterpret_cast<const uint32_t *>(&S.q8[n * 8 + gid][k * 32 + tq * 4]);
      bf[n][k][1] = *reinterpret_cast<const uint32_t *>(&S.q8[n * 8 + gid][k * 32 + 16 + tq * 4]);
    }
    wl[n][0] = S.wq[n * 8 + tq * 2];
    wl[n][1] = S.wq[n * 8 + tq * 2 + 1];
  }

  // ---- main loop over tiles
  for (int i = 0; i < ntiles; ++i) {
    const int s = i % kStages;
    const int tile = tile0 + i;
    const bool ok = mbar_wait_bounded(&S.full[s], (i / kStages) & 1, kWaitLimit);
    if (__syncthreads_or(!ok)) {   // block-uniform decision
      if (tid == 0) {
        flag(a.status, CSA2_DEV_TIMEOUT);
        // copies of tiles i .. i+kStages-1 may still be landing in this
        // CTA's shared memory: wait for them (bounded) before exiting
        const int end = ntiles < i + kStages ? ntiles : i + kStages;
        for (int j = i; j < end; ++j) mbar_wait_bounded(&S.full[j % kStages], (j / kStages) & 1, kWaitLimit);
      }
      __syncthreads();
      return;
    }
    const uint32_t base = smem_u32(S.tile[s]);
#pragma unroll
    for (int ms = 0; ms < 2; ++ms) {
      const int r0 = warp * 32 + ms * 16;
      // entry ids and scales of the two rows this lane finishes
      const int rl = r0 + gid, rh = rl + 8;
      int el, eh;
      bool vl, vh;
      if (REINDEX) {
        const int bl = pool[tile * 16 + (rl >> 3)], bh = pool[tile * 16 + (rh >> 3)];
        el = bl * 8 + (rl & 7);
        eh = bh * 8 + (rh & 7);
        vl = bl >= 0 && bl < a.cap / 8 && el < n_vis;
        vh = bh >= 0 && bh < a.cap / 8 && eh < n_vis;
      } else {
        el = tile * kTileRows + rl;
        eh = tile * kTileRows + rh;
        vl = el < n_vis;
        vh = eh < n_vis;
      }
      const float skl = vl ? a.ik_scale[(size_t)b * a.cap + el] : 0.f;
      const float skh = vh ? a.ik_scale[(size_t)b * a.cap + eh] : 0.f;

      float acc[8][4];
#pragma unroll
      for (int n = 0; n < 8; ++n) acc[n][0] = acc[n][1] = acc[n][2] = acc[n][3] = 0.f;
#pragma unroll
      for (int k = 0; k < KS; ++k) {
        // A 16x32: matrices (rows 0-7 | 8-15) x (bytes 0-15 | 16-31)
        const int r = r0 + (lane & 7) + ((lane >> 3) & 1) * 8;
        const int ch = 2 * k + (lane >> 4);
        uint32_t af[4];
        ldsm_x4(base + swz<MASK>(r * DI + ch * 16), af[0], af[1], af[2], af[3]);
#pragma unroll
        for (int n = 0; n < 8; ++n)
          if (n < ntn) mma_e4m3_16832(acc[n], af, bf[n][k]);
      }
      float sl = 0.f, sh = 0.f;
#pragma unroll
      for (int n = 0; n < 8; ++n) {
        sl += wl[n][0] * fmaxf(acc[n][0], 0.f) + wl[n][1] * fmaxf(acc[n][1], 0.f);
        sh += wl[n][0] * fmaxf(acc[n][2], 0.f) + wl[n][1] * fmaxf(acc[n][3], 0.f);
      }
      sl += __shfl_xor_sync(0xffffffffu, sl, 1);
      sl += __shfl_xor_sync(0xffffffffu, sl, 2);
      sh += __shfl_xor_sync(0xffffffffu, sh, 1);
      sh += __shfl_xor_sync(0xffffffffu, sh, 2);
      if (tq == 0) {
        float *out = a.scores + (size_t)row * a.ld;
        if (REINDEX) {
          out[tile * kTileRows + rl] = vl ? sl * skl : -INFINITY;
          out[tile * kTileRows + rh] = vh ? sh * skh : -INFINITY;
        } else {
          if (vl) out[el] = sl * skl;
          if (vh) out[eh] = sh * skh;
        }
      }
    }
    __syncthreads();  // every warp is done with stage s
    if (tid == 0 && i + kStages < ntiles) {
      fence_proxy_async();
      issue(i + kStages);
    }
  }
}

template <int DI, bool REINDEX>
static cudaError_t launch_t(const CUtensorMap &map, const IndexArgs &a, cudaStream_t s) {
  const size_t smem = sizeof(IndexSmem<DI>) + 1024;
  auto k = index_kernel<DI, REINDEX>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  dim3 grid((a.tiles_per_row + a.tiles_per_cta - 1) / a.tiles_per_cta, a.B * a.T_q);
  k<<<grid, kThreads, smem, s>>>(map, a);
  return cudaGetLastError();
}

cudaError_t launch_index(const CUtensorMap &map, const IndexArgs &a, bool reindex, int sms, cudaStream_t s) {
  (void)sms;
  if (a.dI == 128) return reindex ? launch_t<128, true>(map, a, s) : launch_t<128, false>(map, a, s);
  return reindex ? launch_t<64, true>(map, a, s) : launch_t<64, false>(map, a, s);
}

}  // namespace csa2
