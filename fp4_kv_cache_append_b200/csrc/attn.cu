// Sparse MQA attention over the selected FP4 entries and the FP8 window:
// the pipelined form, for launches of several waves (prefill chunks, large
// decode batches); attn_lat.cu holds the form for launches of one wave, and
// launch_attn below chooses between them.
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2": global sparse
//   retrieval plus the 128-token local window in one attention; section
//   "3) FP4 main KV + SWA Bounded Replay": FP4 (E2M1 + E4M3/16ch) main KV,
//   FP8 window KV.  All query heads share one KV (K = V).
//
// One block per (query row, key split); keys in tiles of 64 (the selected
// entries first, then the window rows), dequantised into one of TWO fp16 K^
// buffers, so that a tile's gather and dequantisation run while the previous
// tile's S, softmax and O^T are in flight.  Warp roles, handing work over
// through mbarriers:
//   warps 0-7   gather + dequantise: thread (key slot r, quarter qq) owns 16
//               channels of every 64-channel chunk of its key (8 code bytes +
//               one E4M3 scale, or 16 E4M3 window bytes); the next tile's
//               loads are issued before this tile is dequantised; values are
//               written exactly as fp16 (hardware E2M1/E4M3 -> f16x2
//               converts; E2M1 x E4M3 is exact in fp16) into the K-major
//               128B-swizzled buffer of the tile, handed over in chunk pairs;
//               a buffer is refilled once the O^T MMAs of its previous tile
//               completed
//   warp 12     tcgen05.mma issuer (converged warp, one elected lane issues):
//               S^T = K^ Q^T into one of two TMEM accumulators (M = 64 keys,
//               N = 64 heads, K = 16, kind::f16) as chunk pairs land; then,
//               once a tile's P is written, O^T += V^T P^T per 128-channel
//               block (V^T is the same K^ buffer read MN-major) and the row
//               sums L += 1 P^T with an all-ones A operand held in TMEM.  The
//               O^T MMAs of tile i-2 are issued before the S MMAs of tile i
//               (their buffer), those of tile i-1 as soon as its P lands
//   warps 8-11  first Q (bf16 -> fp16 B operand), then softmax: warp q reads
//               the S^T lanes of keys 16q .. 16q+15 with the 16x32bx2 TMEM
//               load, thread = (key, 32-head half); the reference max of a
//               head moves only when a tile raises it by more than 2^15 (O^T
//               and L are then rescaled in TMEM, after the previous tile's
//               O^T MMAs completed), so P = 2^(s - m) stays within fp16
//               range; P is written as the MN-major B operand [key][head]
// Window rows keep their raw E4M3 values: the layer's window scale multiplies
// their logits, and O^T (not L) is divided by it when the window tiles start
// and multiplied by it at the end, so their values count scaled and their P
// unscaled.  The splits of one row form a thread-block cluster: each writes
// O / l per head (fp16, [head][channel]) and its (max, sum) per head to the
// workspace, and after one cluster barrier each split merges a slice of the
// channels from all splits (weights 2^(m_s - M) l_s / L) and writes the bf16
// output.  Launch shape (plan_attn): the split count minimises waves x (tiles
// per split + merge cost) with one block per SM; at small batch each split is
// a pair of blocks (grid z) that both compute S and P and each issue the O^T
// MMAs of, write and merge half of the channels.
// Every wait is bounded: one that gives up flags the device status and stops
// every role; issued MMAs are drained and TMEM freed before the block exits.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kDqWarps = 8;                  // gather + dequantise
constexpr int kSmWarp0 = 8;                  // softmax warps 8..11
constexpr int kMmaWarp = 12;
constexpr int kThreads = 13 * 32;
constexpr int kDq = kDqWarps * 32;           // dequantise threads
constexpr int kTile = 64;                    // keys per tile (M of S^T)
constexpr int kPlanTile = 128;               // the split planner's unit (the latency form's tile)
constexpr int kHeads = 64;                   // heads padded to 64 (N)
constexpr float kLog2e = 1.4426950408889634f;
// log2 headroom before a head's reference max moves: P = 2^(s - m_ref) stays
// below 2^15 (fp16 holds up to 65,504; L and O^T accumulate in fp32), and each
// move costs a wait for the previous tile's O^T and a TMEM rescale
constexpr float kLazy = 15.0f;
constexpr uint32_t kWaitLimit = 1u << 22;
constexpr int kSmBar = 1;                    // named barrier of the softmax warps
constexpr int kEpiBar = 2;                   // named barrier of the epilogue (gather) warps
// TMEM columns: S^T of two tiles [0, 128), O^T blocks [128, 128 + 64 MT), L [384, 448), ones [448, 480)
constexpr uint32_t kColS = 0, kColO = 128, kColL = 384, kColOnes = 448, kTmemCols = 512;
// Merge items (head, 8 channels) per thread whose loads are in flight together.
constexpr int kMergeItems = 1;

template <int D>
struct AttnSmem {
  alignas(1024) uint8_t kh[2][(D / 64) * kTile * 128];   // two K^ tiles: D/64 chunks of [64 keys x 128 B]
  alignas(1024) uint8_t q[(D / 64) * kHeads * 128];      // Q: D/64 chunks of [64 heads x 128 B]
  alignas(1024) uint8_t p[2][kTile * 128];               // P of two tiles: [64 keys][64 heads] fp16, MN-major
  float m_ref[kHeads], alpha[kHeads], lsum[kHeads], linv[kHeads];
  float red[4][kHeads];
  float wgt[8][kHeads];                                  // merge weights of the splits
  uint64_t chunk_full[2][D / 128];                       // per buffer, per pair of chunks
  uint64_t kfree[2];                                     // per buffer: its tile's O^T and L MMAs are done
  uint64_t s_full[2], p_full[2], fin, q_ready;
  uint32_t tmem_base;
  int abort;
  int rescale_at;                                        // tile whose softmax moved a reference max
};

// Byte offset of 16-byte piece `pc` (8 fp16 elements) of row `r` in a
// K-major 128B-swizzled operand whose chunks of 64 elements hold `rows` rows.
__device__ __forceinline__ uint32_t sw_off(int r, int pc, int rows) {
  return (uint32_t)((pc >> 3) * rows * 128 + r * 128 + (((pc & 7) ^ (r & 7)) << 4));
}

// Maximum over the 16 lanes of a half-warp of each of 32 columns, by a
// transposing butterfly: afterwards lane l of the half holds in t[0] and t[1]
// the maxima of columns 2(l % 16) and 2(l % 16) + 1 (t is consumed).
__device__ __forceinline__ void reduce_scatter16x32_max(float *t, int lane) {
#pragma unroll
  for (int oc = 16; oc >= 2; oc >>= 1) {
    const int ol = oc >> 1;   // partner lane within the half
    const bool up = (lane & ol) != 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j < oc) {
        const float lo = t[j], hi = t[j + oc];
        const float recv = __shfl_xor_sync(0xffffffffu, up ? lo : hi, ol);
        t[j] = fmaxf(up ? hi : lo, recv);
      }
    }
  }
}

// 2^x by the hardware's approximate exponential (relative error ~2^-22,
// far below the fp16 rounding of P it feeds).
__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// f32 (max, sum) per (row, split, head), after the fp16 partials.
__device__ __forceinline__ float *partial_stats(const AttnArgs &a, size_t nrows) {
  return reinterpret_cast<float *>(reinterpret_cast<uint8_t *>(a.ws) + nrows * a.nsplit * (size_t)a.D * kHeads * 2);
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Bounded wait that also gives up early once another role raised `abort`.
__device__ __forceinline__ bool wait_or_abort(uint64_t *bar, uint32_t parity, volatile int *abort) {
  for (uint32_t i = 0; i < kWaitLimit; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 255u && *abort) return false;
  }
  *abort = 1;
  return false;
}

// Key slot `slot` of tile c: the entry id of a selected entry or the ring slot
// of a window row; -1 = masked.
__device__ __forceinline__ int key_id(const AttnArgs &a, int row, int c, int n_fp4_tiles, int wlo, int nwin,
                                      int slot) {
  if (c < n_fp4_tiles) {
    const int k = c * kTile + slot;
    if (k >= a.K) return -1;
    const int e = a.idx[(size_t)row * a.K + k];
    return (e >= 0 && e < a.cap) ? e : -1;
  }
  const int j = (c - n_fp4_tiles) * kTile + slot;
  return j < nwin ? (wlo + j) % a.W_cap : -1;
}

}  // namespace


template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const AttnArgs a) {
  constexpr int NCH = D / 64;                      // 64-channel chunks of a tile
  constexpr int NPR = NCH / 2;                     // chunk pairs (hand-over unit)
  constexpr int MT = D / 128;                      // O^T TMEM blocks of 128 channels
  constexpr int QP = kHeads * (D / 8);             // 16-byte pieces of Q
  constexpr int QI = QP / 128;                     // ... per softmax thread
  constexpr uint32_t kIdS = mma_idesc(kTile, kHeads, 0u /*f16*/, 0u /*f16*/);
  constexpr uint32_t kIdO = mma_idesc(128, kHeads, 0u, 0u) | (1u << 15) | (1u << 16);   // A (V^T), B (P^T) MN-major
  constexpr uint32_t kIdL = mma_idesc(128, kHeads, 0u, 0u) | (1u << 16);                // A (ones, TMEM), B (P^T) MN-major
  extern __shared__ uint8_t smem_raw[];
  AttnSmem<D> &S = *reinterpret_cast<AttnSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                   ~uintptr_t(1023));
  volatile int *abort = &S.abort;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;   // b * T_q + query
  const int split = blockIdx.y;
  const int b = row / a.T_q;
  const int mt_lo = (int)blockIdx.z * (MT / a.csplit), mt_hi = mt_lo + MT / a.csplit;   // O^T blocks of this block
  pdl_launch_dependents();

  // ---- set-up that touches no global memory overlaps the previous kernel
  if (tid == 0) {
    for (int u = 0; u < 2; ++u) {
      for (int k = 0; k < NPR; ++k) mbar_init(&S.chunk_full[u][k], kDqWarps);
      mbar_init(&S.kfree[u], 1);
      mbar_init(&S.s_full[u], 1);
      mbar_init(&S.p_full[u], 4);
    }
    mbar_init(&S.fin, 1);
    mbar_init(&S.q_ready, 4);
    S.abort = 0;
    S.rescale_at = -1;
    fence_barrier_init();
  }
  if (tid < kHeads) { S.m_ref[tid] = -INFINITY; S.alpha[tid] = 1.f; }
  if (warp == kMmaWarp) {
    tmem_alloc(&S.tmem_base, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  if (warp >= kSmWarp0 && warp < kSmWarp0 + 4) {   // the all-ones A operand of the row-sum MMA
    uint32_t ones[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) ones[j] = 0x3C003C00u;
    tmem_st_x32(tmem + ((uint32_t)(32 * (warp & 3)) << 16) + kColOnes, ones);
    tmem_wait_st();
  }
  pdl_wait();
  const int t = a.q_pos[row];

  // ---- keys of this split: 64-key tiles, the row's tiles divided evenly
  const int n_fp4_tiles = (a.K + kTile - 1) / kTile;
  int wlo = t - a.window + 1;
  if (wlo < 0) wlo = 0;
  const int nwin = (t >= 0 && a.window > 0) ? t - wlo + 1 : 0;
  const int total = n_fp4_tiles + (nwin + kTile - 1) / kTile;
  const int cps = (total + a.nsplit - 1) / a.nsplit;
  const int c_begin = split * cps;
  int c_end = c_begin + cps;
  if (c_end > total) c_end = total;
  const int n_tiles = c_end > c_begin ? c_end - c_begin : 0;
  tc_fence_before();
  __syncthreads();   // the ones are in TMEM before any MMA
  tc_fence_after();

  if (warp < kDqWarps) {
    // ================================================ gather + dequantise
    const int r = tid >> 2, qq = tid & 3;   // key slot, 16-channel quarter of every chunk
    // a tile's loads, all in flight at once: FP4 = 8 code bytes per chunk plus
    // the entry's 32 scale bytes, window = 16 E4M3 bytes per chunk
    // the entry's D/16 scale bytes as D/64 words: word k holds the scales of
    // chunk k, byte qq the one of this thread's 16 channels
    auto load_tile = [&](int c, uint4 *raw, uint32_t *scw) {
      const int id = key_id(a, row, c, n_fp4_tiles, wlo, nwin, r);
      if (c < n_fp4_tiles) {
        const size_t er = (size_t)b * a.cap + (id >= 0 ? id : 0);
        const uint2 *cp = reinterpret_cast<const uint2 *>(a.codes + er * (D / 2)) + qq;
#pragma unroll
        for (int k = 0; k < NCH; ++k) {
          const uint2 v = id >= 0 ? __ldg(cp + 4 * k) : make_uint2(0, 0);
          raw[k] = make_uint4(v.x, v.y, 0, 0);
        }
        if constexpr (NCH >= 4) {   // 16- or 32-byte scale rows: 16-byte loads
          const uint4 *sp = reinterpret_cast<const uint4 *>(a.scales + er * (D / 16));
#pragma unroll
          for (int u = 0; u < NCH / 4; ++u) {
            const uint4 v = id >= 0 ? __ldg(sp + u) : make_uint4(0, 0, 0, 0);
            scw[4 * u] = v.x; scw[4 * u + 1] = v.y; scw[4 * u + 2] = v.z; scw[4 * u + 3] = v.w;
          }
        } else {                    // 8-byte scale rows
          const uint2 v = id >= 0 ? __ldg(reinterpret_cast<const uint2 *>(a.scales + er * (D / 16))) : make_uint2(0, 0);
          scw[0] = v.x; scw[1] = v.y;
        }
      } else {
        const uint4 *wp = reinterpret_cast<const uint4 *>(a.swa_rows + ((size_t)b * a.W_cap + (id >= 0 ? id : 0)) * D) + qq;
#pragma unroll
        for (int k = 0; k < NCH; ++k) raw[k] = id >= 0 ? __ldg(wp + 4 * k) : make_uint4(0, 0, 0, 0);
      }
    };
    uint4 raw[NCH];
    uint32_t scw[NCH];
    if (n_tiles > 0) load_tile(c_begin, raw, scw);
#pragma unroll 1
    for (int it = 0; it < n_tiles; ++it) {
      const int c = c_begin + it;
      const bool is_win = c >= n_fp4_tiles;
      const int buf = it & 1;
      uint8_t *kh = S.kh[buf];
      // the next tile's loads go out before this tile is dequantised
      uint4 rawn[NCH];
      uint32_t scwn[NCH];
      if (it + 1 < n_tiles) load_tile(c + 1, rawn, scwn);
      // the buffer is free once the O^T MMAs of its previous tile completed
      bool ok = true;
      if (it >= 2) {
        int w_ok = 1;
        if (lane == 0) w_ok = wait_or_abort(&S.kfree[buf], ((it >> 1) - 1) & 1, abort);
        ok = __shfl_sync(0xffffffffu, w_ok, 0) != 0;
      }
      if (!ok) break;
#pragma unroll
      for (int k = 0; k < NCH; ++k) {
        uint32_t h[8];
        if (!is_win) {
          const uint32_t sb = (scw[k] >> (8 * qq)) & 0xFFu;   // scale byte 4k + qq
          const uint32_t s2 = e4m3x2_to_f16x2(sb | (sb << 8));
          const __half2 sk = *reinterpret_cast<const __half2 *>(&s2);
          e2m1x8_to_f16x2(raw[k].x, h);
          e2m1x8_to_f16x2(raw[k].y, h + 4);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const __half2 v = __hmul2(*reinterpret_cast<const __half2 *>(&h[e]), sk);
            h[e] = *reinterpret_cast<const uint32_t *>(&v);
          }
        } else {
          e4m3x4_to_f16x2(raw[k].x, h);
          e4m3x4_to_f16x2(raw[k].y, h + 2);
          e4m3x4_to_f16x2(raw[k].z, h + 4);
          e4m3x4_to_f16x2(raw[k].w, h + 6);
        }
#pragma unroll
        for (int j = 0; j < 2; ++j)
          *reinterpret_cast<uint4 *>(kh + sw_off(r, 8 * k + 2 * qq + j, kTile)) =
              make_uint4(h[4 * j], h[4 * j + 1], h[4 * j + 2], h[4 * j + 3]);
        if (k & 1) {   // chunks are handed over in pairs: one proxy fence per two
          fence_proxy_async();   // generic stores -> visible to the tensor core
          __syncwarp();
          if (lane == 0) mbar_arrive(&S.chunk_full[buf][k >> 1]);
        }
      }
#pragma unroll
      for (int k = 0; k < NCH; ++k) raw[k] = rawn[k];
#pragma unroll
      for (int k = 0; k < NCH; ++k) scw[k] = scwn[k];
    }
  } else if (warp < kSmWarp0 + 4) {
    // ================================================ softmax
    const int q = warp & 3;                 // TMEM lane quarter
    const int hh = lane >> 4;               // 32-head half of this thread
    const int r = 16 * q + (lane & 15);     // key slot (S^T row; TMEM lane 32q + r % 16)
    const int st = tid - kSmWarp0 * 32;     // 0..127
    const uint32_t srow = tmem + ((uint32_t)(32 * q) << 16);
    // Q: bf16 -> fp16 into the B-operand layout, while the gather warps load
    // the first tiles (the MMA issuer waits for q_ready)
    if (n_tiles > 0) {
      const uint16_t *qrow = a.q + (size_t)row * a.H * D;
#pragma unroll 1
      for (int u0 = 0; u0 < QI; u0 += 16) {
        uint4 qraw[16];
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          const int i = st + (u0 + u) * 128;
          const int h = i / (D / 8), pc = i % (D / 8);
          qraw[u] = (u0 + u < QI && h < a.H) ? __ldg(reinterpret_cast<const uint4 *>(qrow + (size_t)h * D + pc * 8))
                                             : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 16; ++u) {
          if (u0 + u >= QI) break;
          const int i = st + (u0 + u) * 128;
          const int h = i / (D / 8), pc = i % (D / 8);
          const uint32_t w[4] = {qraw[u].x, qraw[u].y, qraw[u].z, qraw[u].w};
          uint32_t o[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const __half2 hv = __floats2half2_rn(bf16_to_f32(w[k] & 0xFFFFu), bf16_to_f32(w[k] >> 16));
            o[k] = *reinterpret_cast<const uint32_t *>(&hv);
          }
          *reinterpret_cast<uint4 *>(S.q + sw_off(h, pc, kHeads)) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
      fence_proxy_async();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.q_ready);
    }
    auto warp_wait = [&](uint64_t *bar, uint32_t parity) {
      int w_ok = 1;
      if (lane == 0) w_ok = wait_or_abort(bar, parity, abort);
      return __shfl_sync(0xffffffffu, w_ok, 0) != 0;
    };
#pragma unroll 1
    for (int it = 0; it < n_tiles; ++it) {
      const int c = c_begin + it;
      const bool is_win = c >= n_fp4_tiles;
      const int buf = it & 1;
      const int id = key_id(a, row, c, n_fp4_tiles, wlo, nwin, r);
      if (hh == 0 && c < n_fp4_tiles && c * kTile + r < a.K) {   // flag selected entries outside the cache
        const int e = a.idx[(size_t)row * a.K + c * kTile + r];
        if (e >= a.cap) flag(a.status, CSA2_DEV_INDEX_RANGE);
      }
      const bool valid = id >= 0;
      if (!warp_wait(&S.s_full[buf], (it >> 1) & 1)) break;
      tc_fence_after();
      const float lsc = a.scale * (is_win ? a.s_swa : 1.0f) * kLog2e;
      const bool first = it == 0;
      float sv[32];
      auto load_logits = [&]() {   // heads 32 hh .. 32 hh + 31 of key r
        uint32_t rv[32];
        tmem_ld_16x32bx2_x32(srow + kColS + buf * kHeads, rv);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) sv[j] = valid ? __uint_as_float(rv[j]) * lsc : -INFINITY;
      };
      load_logits();
      // after the first tile the reference max usually holds: the per-head
      // maxima are needed only when a logit exceeds it by more than 2^15
      bool over = first;
      if (!first) {
        const float4 *mp = reinterpret_cast<const float4 *>(S.m_ref + 32 * hh);
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 m4 = mp[j4];
          over |= (sv[4 * j4] > m4.x + kLazy) | (sv[4 * j4 + 1] > m4.y + kLazy) | (sv[4 * j4 + 2] > m4.z + kLazy) |
                  (sv[4 * j4 + 3] > m4.w + kLazy);
        }
      }
      const bool need_max = named_bar_or(kSmBar, 128, over);
      if (need_max) {
        reduce_scatter16x32_max(sv, lane);   // heads 32 hh + 2 (lane % 16) + {0, 1} (consumes sv)
        S.red[q][32 * hh + 2 * (lane & 15)] = sv[0];
        S.red[q][32 * hh + 2 * (lane & 15) + 1] = sv[1];
        named_bar(kSmBar, 128);
        if (st < kHeads) {   // new reference max of head st
          const float m_old = S.m_ref[st];
          const float mt = fmaxf(fmaxf(S.red[0][st], S.red[1][st]), fmaxf(S.red[2][st], S.red[3][st]));
          float al = 1.f;
          if (mt != -INFINITY) {
            if (m_old == -INFINITY) {
              S.m_ref[st] = mt;
              al = 0.f;
            } else if (mt > m_old + kLazy) {
              S.m_ref[st] = mt;
              al = exp2f(m_old - mt);
              if (!first) S.rescale_at = it;
            }
          }
          S.alpha[st] = al;
        }
        named_bar(kSmBar, 128);
        load_logits();
      }
      // P of this buffer was read by the O^T MMAs of tile it - 2
      if (it >= 2 && !warp_wait(&S.kfree[buf], ((it >> 1) - 1) & 1)) break;
      // P = 2^(s - m_ref): heads 32 hh .. of row r of the P operand (fp16)
      {
        uint8_t *prow = S.p[buf] + r * 128;
        const float4 *mp = reinterpret_cast<const float4 *>(S.m_ref + 32 * hh);
        uint32_t ph[16];
#pragma unroll
        for (int j4 = 0; j4 < 8; ++j4) {
          const float4 m4 = mp[j4];
          const float mm[4] = {m4.x, m4.y, m4.z, m4.w};
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int j = 4 * j4 + k;
            sv[j] = (sv[j] == -INFINITY || mm[k] == -INFINITY) ? 0.f : ex2_approx(sv[j] - mm[k]);
          }
          const __half2 h0 = __floats2half2_rn(sv[4 * j4], sv[4 * j4 + 1]);
          const __half2 h1 = __floats2half2_rn(sv[4 * j4 + 2], sv[4 * j4 + 3]);
          ph[2 * j4] = *reinterpret_cast<const uint32_t *>(&h0);
          ph[2 * j4 + 1] = *reinterpret_cast<const uint32_t *>(&h1);
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
          *reinterpret_cast<uint4 *>(prow + (((4 * hh + i) ^ (r & 7)) << 4)) =
              make_uint4(ph[4 * i], ph[4 * i + 1], ph[4 * i + 2], ph[4 * i + 3]);
      }
      // rare: a head's reference max moved -> rescale its O^T and L columns;
      // and at the first window tile after FP4 tiles, O^T is divided by the
      // window scale (window rows enter O^T unscaled; the epilogue multiplies
      // the O of a block that saw window tiles by the scale).  The previous
      // tile's O^T and L MMAs must have completed first.
      const bool moved = need_max && S.rescale_at == it;
      const bool to_win = is_win && c == n_fp4_tiles && it > 0;
      if (moved || to_win) {
        if (!warp_wait(&S.kfree[(it - 1) & 1], ((it - 1) >> 1) & 1)) break;
        tc_fence_after();
        const float inv_s = to_win ? 1.0f / a.s_swa : 1.0f;
#pragma unroll 1
        for (int blk = 0; blk <= MT; ++blk) {
          if (blk < MT && (blk < mt_lo || blk >= mt_hi)) continue;
          if (blk == MT && !moved) continue;
          const uint32_t base = srow + (blk < MT ? kColO + 64 * blk : kColL);
          const float f = blk < MT ? inv_s : 1.0f;
#pragma unroll 1
          for (int h2 = 0; h2 < 2; ++h2) {
            uint32_t o[32];
            tmem_ld_x32(base + 32 * h2, o);
            tmem_wait_ld();
#pragma unroll
            for (int j = 0; j < 32; ++j)
              o[j] = __float_as_uint(__uint_as_float(o[j]) * ((moved ? S.alpha[32 * h2 + j] : 1.0f) * f));
            tmem_st_x32(base + 32 * h2, o);
          }
        }
        tmem_wait_st();
      }
      fence_proxy_async();   // P (generic stores) -> visible to the tensor core
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&S.p_full[buf]);
    }
  } else {
    // ================================================ MMA issuer: the whole warp runs
    // the loop converged (every lane polls the barriers), one elected lane
    // issues the MMAs and their commits
    const uint32_t q_base = smem_u32(S.q);
    const uint64_t dq0 = smem_desc_kmajor(q_base, 128);
    auto all_wait = [&](uint64_t *bar, uint32_t parity) {
      return __all_sync(0xffffffffu, wait_or_abort(bar, parity, abort)) != 0;
    };
    // L^T += 1 P^T and O^T += V^T P^T of tile j; the commit frees its buffer
    auto issue_o = [&](int j) {
      const int pb = j & 1;
      const uint64_t dv = smem_desc_mnmajor_sw128(smem_u32(S.kh[pb]), kTile * 128, 1024);
      const uint64_t dp = smem_desc_mnmajor_sw128(smem_u32(S.p[pb]), kTile * 128, 1024);
      const uint32_t acc0 = j > 0 ? 1u : 0u;
      tc_fence_after();
      if (elect_one()) {
#pragma unroll
        for (int ks = 0; ks < kTile / 16; ++ks)
          tc_mma_f16_ta(tmem + kColL, tmem + kColOnes, dp + (((2 * ks) * 1024) >> 4), kIdL, (ks > 0) ? 1u : acc0);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          if (mt >= mt_lo && mt < mt_hi) {
#pragma unroll
            for (int ks = 0; ks < kTile / 16; ++ks)
              tc_mma_f16(tmem + kColO + mt * kHeads, dv + (((2 * mt) * (kTile * 128) + (2 * ks) * 1024) >> 4),
                         dp + (((2 * ks) * 1024) >> 4), kIdO, (ks > 0) ? 1u : acc0);
          }
        }
        tc_commit(&S.kfree[pb]);
      }
      __syncwarp();
    };
    bool ok = n_tiles == 0 || all_wait(&S.q_ready, 0);
    int o_next = 0;   // the next tile whose O^T MMAs are to be issued
#pragma unroll 1
    for (int it = 0; it < n_tiles && ok; ++it) {
      const int buf = it & 1;
      // the O^T MMAs of tile it - 2 read this buffer: issued before its refill is waited for
      while (ok && o_next <= it - 2) {
        ok = all_wait(&S.p_full[o_next & 1], (o_next >> 1) & 1);
        if (ok) issue_o(o_next++);
      }
      if (!ok) break;
      // the bases pass through an opaque copy each tile, so that the unrolled
      // loop below forms each descriptor next to its MMA
      uint64_t dk = smem_desc_kmajor(smem_u32(S.kh[buf]), 128), dq = dq0;
      asm volatile("" : "+l"(dk), "+l"(dq));
      // S^T = K^ Q^T, pair by pair as the chunks land
#pragma unroll
      for (int pr = 0; pr < NPR; ++pr) {
        // the previous tile's O^T as soon as its P landed
        if (o_next == it - 1 && __all_sync(0xffffffffu, mbar_test_wait(&S.p_full[o_next & 1], (o_next >> 1) & 1)))
          issue_o(o_next++);
        if (!all_wait(&S.chunk_full[buf][pr], (it >> 1) & 1)) { ok = false; break; }
        tc_fence_after();
        if (elect_one()) {
#pragma unroll
          for (int k2 = 0; k2 < 2; ++k2) {
            const int k = 2 * pr + k2;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)   // descriptors advance by (byte offset >> 4)
              tc_mma_f16(tmem + kColS + buf * kHeads, dk + ((k * (kTile * 128) + kk * 32) >> 4),
                         dq + ((k * (kHeads * 128) + kk * 32) >> 4), kIdS, (k > 0 || kk > 0) ? 1u : 0u);
          }
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) tc_commit(&S.s_full[buf]);
      __syncwarp();
    }
    while (ok && o_next < n_tiles) {
      ok = all_wait(&S.p_full[o_next & 1], (o_next >> 1) & 1);
      if (ok) issue_o(o_next++);
    }
    if (elect_one()) tc_commit(&S.fin);   // arrives once every MMA issued above is done
    __syncwarp();
  }

  // ---- epilogue: O^T (TMEM lane = channel within a 128-channel block)
  bool ok = *abort == 0;
  if (ok && n_tiles > 0 && tid < kDq) ok = wait_or_abort(&S.fin, 0, abort);
  const bool failed = __syncthreads_or(!ok) || *abort != 0;
  const size_t nrows = (size_t)a.B * a.T_q;
  if (failed) {
    if (tid == 0) flag(a.status, CSA2_DEV_TIMEOUT);
    if (warp == kMmaWarp && lane == 0) mbar_wait_bounded(&S.fin, 0, kWaitLimit);   // every issued MMA done
  } else if (tid < kDq) {
    tc_fence_after();
    const int quarter = warp & 3, half = warp >> 2;   // TMEM lane quarter, 32-head half
    const uint32_t lrow = tmem + ((uint32_t)(32 * quarter) << 16);
    float linv[32];
    {
      uint32_t lv[32];
      if (n_tiles > 0) {
        tmem_ld_x32(lrow + kColL + 32 * half, lv);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) lv[j] = 0u;
      }
      // window rows entered O^T unscaled: a block that saw window tiles scales its O
      const float osc = c_end > n_fp4_tiles && n_tiles > 0 ? a.s_swa : 1.0f;
      // every lane holds every head's sum: the quarter-0 warps take one head
      // per lane, so each head's reciprocal is formed once
      if (quarter == 0) {
        float l = 0.f;
#pragma unroll
        for (int j = 0; j < 32; ++j) l = j == lane ? __uint_as_float(lv[j]) : l;
        S.lsum[32 * half + lane] = l;
        S.linv[32 * half + lane] = l > 0.f ? osc / l : 0.f;
      }
      named_bar(kEpiBar, kDq);
#pragma unroll
      for (int j = 0; j < 32; ++j) linv[j] = S.linv[32 * half + j];
    }
    // O / l per head, staged head-major [64 heads][D] in the K^ tile (free
    // once the last O^T MMA completed) -- bf16 for one split, fp16 partials
    // for several -- then written out in 16-byte pieces.
    uint16_t *ob = reinterpret_cast<uint16_t *>(S.kh);
#pragma unroll 1
    for (int mt = mt_lo; mt < mt_hi; ++mt) {
      const int ch = mt * 128 + 32 * quarter + lane;
      uint32_t o[32];
      if (n_tiles > 0) {
        tmem_ld_x32(lrow + kColO + mt * kHeads + 32 * half, o);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = 0u;
      }
      if (a.nsplit == 1) {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const __nv_bfloat16 bv = __float2bfloat16_rn(__uint_as_float(o[j]) * linv[j]);
          ob[(32 * half + j) * D + ch] = *reinterpret_cast<const uint16_t *>(&bv);
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const __half hv = __float2half_rn(__uint_as_float(o[j]) * linv[j]);
          ob[(32 * half + j) * D + ch] = *reinterpret_cast<const uint16_t *>(&hv);
        }
      }
    }
  }
  __syncthreads();
  if (!failed) {
    if (a.nsplit == 1) {
      const uint4 *src = reinterpret_cast<const uint4 *>(S.kh);
      uint4 *dst = reinterpret_cast<uint4 *>(a.out + (size_t)row * a.H * D);
      const int n16 = a.H * (D / 8);
#pragma unroll 4
      for (int i = tid; i < n16; i += kThreads) dst[i] = src[i];
    } else {
      // this block's channels [z_lo, z_lo + D / csplit) of every head
      const int Dz = D / a.csplit, z_lo = mt_lo * 128;
      const uint4 *src = reinterpret_cast<const uint4 *>(S.kh);
      uint4 *dst = reinterpret_cast<uint4 *>(reinterpret_cast<__half *>(a.ws) +
                                             ((size_t)row * a.nsplit + split) * kHeads * D);
      const int per = Dz / 8, n16 = kHeads * per;
#pragma unroll 4
      for (int i = tid; i < n16; i += kThreads) {
        const int h = i / per, pc = z_lo / 8 + i % per;
        dst[h * (D / 8) + pc] = src[h * (D / 8) + pc];
      }
      if (tid < kHeads) {
        float *pm = partial_stats(a, nrows) + ((size_t)row * a.nsplit + split) * kHeads;
        float *pl = pm + nrows * a.nsplit * kHeads;
        pm[tid] = S.m_ref[tid];
        pl[tid] = S.lsum[tid];
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kTmemCols);
  }

  // ---- merge of the splits (the row's blocks form one cluster)
  if (a.nsplit > 1) {
    cluster_sync_all();   // every split's partials are written
    // this split's channel slice; item = (head, 8 channels): 16 bytes per split in, 16 bytes out
    const int Dz = D / a.csplit, z_lo = (int)blockIdx.z * Dz;   // this block's channel half (or all)
    const int cs = ((Dz / a.nsplit) + 7) / 8 * 8;
    const int c_lo = z_lo + split * cs;
    const int c_hi = c_lo + cs < z_lo + Dz ? c_lo + cs : z_lo + Dz;
    const int ng = c_hi > c_lo ? (c_hi - c_lo) / 8 : 0;
    const int n_items = a.H * ng;
    const __half *base = reinterpret_cast<const __half *>(a.ws) + (size_t)row * a.nsplit * kHeads * D;
    uint4 x[kMergeItems][8];
    auto load_items = [&](int it0) {   // kMergeItems items' loads in flight
#pragma unroll
      for (int v = 0; v < kMergeItems; ++v) {
        const int it = it0 + v * kThreads;
        const int h = it / (ng > 0 ? ng : 1), ch = c_lo + 8 * (it % (ng > 0 ? ng : 1));
#pragma unroll
        for (int s = 0; s < 8; ++s)
          x[v][s] = (it < n_items && s < a.nsplit)
                        ? __ldcg(reinterpret_cast<const uint4 *>(base + ((size_t)s * kHeads + h) * D + ch))
                        : make_uint4(0, 0, 0, 0);
      }
    };
    load_items(tid);   // the first round of partials is in flight with the statistics
    const float *pm = partial_stats(a, nrows) + (size_t)row * a.nsplit * kHeads;
    const float *pl = pm + nrows * a.nsplit * kHeads;
    if (tid < kHeads) {   // all 2 x nsplit loads in flight together
      float ms[8], ls[8];
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        ms[s] = s < a.nsplit ? __ldcg(pm + s * kHeads + tid) : -INFINITY;
        ls[s] = s < a.nsplit ? __ldcg(pl + s * kHeads + tid) : 0.f;
      }
      float M = -INFINITY;
#pragma unroll
      for (int s = 0; s < 8; ++s) M = fmaxf(M, ms[s]);
      float L = 0.f;
#pragma unroll
      for (int s = 0; s < 8; ++s) {
        ms[s] = ms[s] == -INFINITY ? 0.f : exp2f(ms[s] - M) * ls[s];   // the partials are O_s / l_s
        L += ms[s];
      }
      const float inv = L > 0.f ? 1.f / L : 0.f;
#pragma unroll
      for (int s = 0; s < 8; ++s) S.wgt[s][tid] = ms[s] * inv;
    }
    __syncthreads();
#pragma unroll 1
    for (int it0 = tid; it0 < n_items; it0 += kMergeItems * kThreads) {
      if (it0 != tid) load_items(it0);
#pragma unroll
      for (int v = 0; v < kMergeItems; ++v) {
        const int it = it0 + v * kThreads;
        if (it >= n_items) continue;
        const int h = it / ng, ch = c_lo + 8 * (it % ng);
        float acc[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) acc[i] = 0.f;
#pragma unroll
        for (int s = 0; s < 8; ++s) {
          if (s >= a.nsplit) break;
          const float w = S.wgt[s][h];
          const uint32_t w4[4] = {x[v][s].x, x[v][s].y, x[v][s].z, x[v][s].w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float2 f = __half22float2(*reinterpret_cast<const __half2 *>(&w4[i]));
            acc[2 * i] += w * f.x;
            acc[2 * i + 1] += w * f.y;
          }
        }
        uint32_t pk[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const __nv_bfloat162 bv = __floats2bfloat162_rn(acc[2 * i], acc[2 * i + 1]);
          pk[i] = *reinterpret_cast<const uint32_t *>(&bv);
        }
        *reinterpret_cast<uint4 *>(a.out + ((size_t)row * a.H + h) * D + ch) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
      }
    }
  }
}

AttnPlan plan_attn(int B, int T_q, int H, int D, int K, int window, int sms) {
  (void)H;
  AttnPlan p;
  const int rows = B * T_q;
  const int nc = (K + kPlanTile - 1) / kPlanTile + (window + kPlanTile - 1) / kPlanTile;
  // One block per SM at a time (shared memory), so a launch takes
  // ceil(blocks / SMs) waves; a block costs one unit per key tile, plus
  // about 0.8 for writing and merging split partials, plus 0.2 of set-up.
  // Take the split count of least cost (at most 8: the splits of a row form
  // one cluster).
  int nsplit = 1, cps = nc;
  double best = 1e30;
  for (int ns = 1; ns <= 8 && ns <= nc; ++ns) {
    const int c = (nc + ns - 1) / ns;
    const int ne = (nc + c - 1) / c;
    const long long waves = ((long long)rows * ne + sms - 1) / sms;
    const double cost = (double)waves * (c + (ne > 1 ? 0.8 : 0.0) + 0.2);
    if (cost < best - 1e-9) { best = cost; nsplit = ne; cps = c; }
  }
  p.nsplit = nsplit;
  p.chunks_per_split = cps;
  // small batches: two blocks per split, each issuing the O^T MMAs of, and
  // writing and merging, half of the channels (both compute S and P)
  p.csplit = (nsplit > 1 && D % 256 == 0 && (long long)rows * nsplit * 2 <= sms) ? 2 : 1;
  // Measured on B200 (dec_full shapes, 1 to 4,096 rows): the form in which
  // all warps take each phase of a tile in turn is the faster while every
  // block of the launch is resident at once and runs a single 128-key tile
  // (by about 2 us at 8 and 16 rows); once blocks run several tiles, or the
  // launch takes several waves, the pipelined form below (43 vs 45 us at 128
  // rows, 251 vs 295 us at 1,024).
  p.latency_form = ((long long)rows * nsplit * p.csplit <= sms && cps <= 1) ? 1 : 0;
  // fp16 partials [rows][nsplit][64][D] then f32 max and sum [rows][nsplit][64] each
  p.bytes = nsplit > 1 ? (size_t)rows * nsplit * kHeads * ((size_t)D * 2 + 2 * sizeof(float)) : 0;
  return p;
}

template <int D>
static cudaError_t launch_attn_t(const AttnArgs &a, cudaStream_t s) {
  const size_t smem = sizeof(AttnSmem<D>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_kernel<D>, dim3(a.B * a.T_q, a.nsplit, a.csplit), dim3(kThreads), smem, s,
                    dim3(1, (unsigned)a.nsplit, 1), a);
}

cudaError_t launch_attn(const AttnArgs &a, cudaStream_t s) {
  if (a.latency_form) return launch_attn_lat(a, s);
  switch (a.D) {
    case 128: return launch_attn_t<128>(a, s);
    case 256: return launch_attn_t<256>(a, s);
    default: return launch_attn_t<512>(a, s);
  }
}

}  // namespace csa2
