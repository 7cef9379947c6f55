// Sparse MQA attention over the selected FP4 entries and the FP8 window.
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2": global sparse
//   retrieval plus the 128-token local window in one attention; section
//   "3) FP4 main KV + SWA Bounded Replay": FP4 (E2M1 + E4M3/16ch) main KV,
//   FP8 window KV.  All query heads share one KV (K = V).
//
// The latency form of the attention: chosen when the launch fits in one wave
// (every block resident at once, as at decode batch sizes), where each block
// runs one or a few tiles and the time is the chain of one tile's phases.
// All eight warps take every phase in turn, so each phase runs on the whole
// block.  (attn.cu holds the pipelined form for launches of several waves,
// with the split planner and the dispatch between the two.)
//
// One block per (query row, key split); keys in tiles of 128 (the selected
// entries first, then the window rows).  Per tile:
//   1. every thread issues all of its gather loads at once (FP4 codes +
//      scales, or E4M3 rows) and dequantises them exactly into fp16 with the
//      hardware E2M1/E4M3 -> f16x2 converts (E2M1 x E4M3 products and E4M3
//      values are exact in fp16), laid out in shared memory as a K-major
//      128B-swizzled operand;
//   2. S^T = K^ Q^T on tcgen05 (kind::f16, M = 128 keys, N = 64 heads,
//      K = D): TMEM lane = key, column = head;
//   3. all 8 warps (TMEM lane quarter x 32-head half) form the per-head
//      maxima and sums over the 128 keys and write P (fp16) row by row as an
//      MN-major operand [key][head];
//   4. O^T += V^T P^T on tcgen05 (M = 128 channels per TMEM block, N = 64
//      heads, K = 128 keys).  V^T is the same shared-memory tile as K^, read
//      as an MN-major operand, so the tile is dequantised once.
// The softmax reference max of a head moves only when a tile raises it by more
// than 2^8 (then O^T and the running sum are rescaled in place), so P stays
// within fp16 range and rescaling is rare.  Window rows keep their raw E4M3
// values; the layer's window scale multiplies their logits and their P.
// The splits of one row form a thread-block cluster: each writes O / l per
// head (fp16, [head][channel]) and its (max, sum) per head to the workspace, and
// after one cluster barrier each split merges a slice of the channels from all
// splits (weights 2^(m_s - M) l_s / L) and writes the bf16 output.
// Launch shape (plan_attn): the split count minimises waves x (tiles per split
// + merge cost) with one block per SM; at small batch each split is a pair of
// blocks (grid z) that both compute S and P and each issue the O^T MMAs of,
// write and merge half of the channels.  A block that runs several tiles has
// L2 fetch the next tile's rows during the current tile's MMAs and skips the
// per-head max reduction while the reference max holds.
// Each block runs its code about once, from a cold instruction cache, so the
// unrolled size of the straight-line parts (merge, maxima) is kept down:
// fetching code costs as much as executing it here.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kThreads = 256;
constexpr int kMmaWarp = 4;        // issues the MMAs (converged, one elected lane)
constexpr int kTile = 128;         // keys per tile (M of S^T)
constexpr int kHeads = 64;         // heads padded to 64 (N)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.0f;      // log2 headroom before the reference max moves
constexpr uint32_t kWaitLimit = 1u << 22;
// Merge items (head, 8 channels) per thread whose loads are in flight
// together.  Each block runs the merge once, from a cold instruction cache,
// so its unrolled size matters: 2 items keep one round of L2 reads for a
// dec_full split (448 items) at 10 KB less code than 4.
constexpr int kMergeItems = 2;

template <int D>
struct AttnSmem {
  alignas(1024) uint8_t kh[(D / 64) * kTile * 128];   // K^ tile: D/64 chunks of [128 keys x 128 B]
  alignas(1024) uint8_t q[(D / 64) * kHeads * 128];   // Q: D/64 chunks of [64 heads x 128 B]
  alignas(1024) uint8_t p[kTile * 128];               // P: [128 keys][64 heads] fp16, MN-major
  int key_ent[2][kTile];                              // entry id or window slot, -1 = masked
  float red[4][kHeads];
  float m_ref[kHeads], l_run[kHeads], alpha[kHeads], linv[kHeads];
  float wgt[8][kHeads];                               // merge weights of the splits
  uint64_t sbar, obar;
  uint32_t tmem_base;
  int rescale;
};

// Byte offset of 16-byte piece `pc` (8 fp16 elements) of row `r` in a
// K-major 128B-swizzled operand whose chunks of 64 elements hold `rows` rows.
__device__ __forceinline__ uint32_t sw_off(int r, int pc, int rows) {
  return (uint32_t)((pc >> 3) * rows * 128 + r * 128 + (((pc & 7) ^ (r & 7)) << 4));
}

// After the call, lane l holds in t[0] the sum over the warp of column l.
__device__ __forceinline__ void reduce_scatter32(float *t, int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j < o) {
        const float lo = t[j], hi = t[j + o];
        const float recv = __shfl_xor_sync(0xffffffffu, up ? lo : hi, o);
        t[j] = (up ? hi : lo) + recv;
      }
    }
  }
}

// After the call, lane l holds in t[0] the maximum over the warp of column l
// (the same transposing butterfly; t is consumed).
__device__ __forceinline__ void reduce_scatter32_max(float *t, int lane) {
#pragma unroll
  for (int o = 16; o >= 1; o >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (j < o) {
        const float lo = t[j], hi = t[j + o];
        const float recv = __shfl_xor_sync(0xffffffffu, up ? lo : hi, o);
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

__device__ __forceinline__ void prefetch_l2(const void *p) {
  asm volatile("prefetch.global.L2 [%0];" ::"l"(p));
}

// Key ids of tile c (threads 0..127): entry ids of the selected entries, or
// ring slots of the window rows; -1 = masked.  With `warm`, each thread also
// asks L2 for its key's bytes (codes and scales, or the window row), so the
// tile's gather, issued a few thousand cycles later, finds them there.
template <int D>
__device__ __forceinline__ void load_key_ids(const AttnArgs &a, int row, int b, int c, int n_fp4_tiles, int wlo,
                                             int nwin, int *dst, int tid, bool warm) {
  if (tid >= kTile) return;
  int id = -1;
  if (c < n_fp4_tiles) {
    const int k = c * kTile + tid;
    if (k < a.K) {
      const int e = a.idx[(size_t)row * a.K + k];
      if (e >= a.cap) flag(a.status, CSA2_DEV_INDEX_RANGE);
      id = (e >= 0 && e < a.cap) ? e : -1;
    }
    if (warm && id >= 0) {
      const size_t er = (size_t)b * a.cap + id;
#pragma unroll
      for (int o = 0; o < D / 2; o += 128) prefetch_l2(a.codes + er * (D / 2) + o);
      prefetch_l2(a.scales + er * (D / 16));
    }
  } else {
    const int j = (c - n_fp4_tiles) * kTile + tid;
    id = j < nwin ? (wlo + j) % a.W_cap : -1;
    if (warm && id >= 0) {
#pragma unroll
      for (int o = 0; o < D; o += 128) prefetch_l2(a.swa_rows + ((size_t)b * a.W_cap + id) * D + o);
    }
  }
  dst[tid] = id;
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_lat_kernel(const AttnArgs a) {
  constexpr int MT = D / 128;                      // O^T TMEM blocks of 128 channels
  constexpr int QI = kHeads * (D / 8) / kThreads;  // 16-byte pieces of Q per thread
  constexpr int GF = D / 64;                       // FP4 items (32 channels) per thread and tile
  constexpr int GW = D / 32;                       // window items (16 channels) per thread and tile
  constexpr uint32_t kCols = D == 128 ? 128u : (D == 256 ? 256u : 512u);
  constexpr uint32_t kIdS = mma_idesc(128, kHeads, 0u /*f16*/, 0u /*f16*/);
  constexpr uint32_t kIdO = kIdS | (1u << 15) | (1u << 16);   // A (V^T) and B (P^T) MN-major
  extern __shared__ uint8_t smem_raw[];
  AttnSmem<D> &S = *reinterpret_cast<AttnSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                   ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int quarter = warp & 3, half = warp >> 2;   // TMEM lane quarter, 32-head half
  const int row = blockIdx.x;   // b * T_q + query
  const int split = blockIdx.y;
  const int b = row / a.T_q;
  const int mt_lo = (int)blockIdx.z * (MT / a.csplit), mt_hi = mt_lo + MT / a.csplit;   // O^T blocks of this block
  pdl_launch_dependents();

  // ---- set-up that touches no global memory overlaps the previous kernel
  if (tid == 0) {
    mbar_init(&S.sbar, 1);
    mbar_init(&S.obar, 1);
    S.rescale = 0;
    fence_barrier_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(&S.tmem_base, kCols);
    tmem_relinquish();
  }
  // ---- Q: bf16 -> fp16 into the B-operand layout.  The query and its
  // position are inputs of the call that no launch of this library writes, so
  // they are read before the wait for the previous launch (the Top-K that
  // produces the entry ids).
  const int t = a.q_pos[row];
  {
    const uint16_t *qrow = a.q + (size_t)row * a.H * D;
    uint4 qraw[QI];
#pragma unroll
    for (int u = 0; u < QI; ++u) {
      const int i = tid + u * kThreads;
      const int h = i / (D / 8), pc = i % (D / 8);
      qraw[u] = h < a.H ? __ldg(reinterpret_cast<const uint4 *>(qrow + (size_t)h * D + pc * 8)) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < QI; ++u) {
      const int i = tid + u * kThreads;
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
  pdl_wait();

  // ---- keys of this split
  const int n_fp4_tiles = (a.K + kTile - 1) / kTile;
  int wlo = t - a.window + 1;
  if (wlo < 0) wlo = 0;
  const int nwin = (t >= 0 && a.window > 0) ? t - wlo + 1 : 0;
  const int total = n_fp4_tiles + (nwin + kTile - 1) / kTile;
  const int c_begin = split * a.chunks_per_split;
  int c_end = c_begin + a.chunks_per_split;
  if (c_end > total) c_end = total;

  // ---- the first tile's key ids
  if (c_begin < c_end) load_key_ids<D>(a, row, b, c_begin, n_fp4_tiles, wlo, nwin, S.key_ent[c_begin & 1], tid, false);
  if (tid < kHeads) { S.m_ref[tid] = -INFINITY; S.l_run[tid] = 0.f; S.alpha[tid] = 1.f; }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const uint32_t kh_base = smem_u32(S.kh), q_base = smem_u32(S.q), p_base = smem_u32(S.p);

  bool aborted = false;
  int n_done = 0;   // tiles whose O^T MMAs were issued
#pragma unroll 1
  for (int c = c_begin; c < c_end; ++c) {
    const bool is_win = c >= n_fp4_tiles;
    const int *ids = S.key_ent[c & 1];
    // ---- 1a. gather loads, all issued before any is used: FP4 item = 32
    // channels (16 code bytes + 2 scale bytes), window item = 16 E4M3 bytes
    uint4 raw[GW];
    uint32_t sc[GF];
    if (!is_win) {
#pragma unroll
      for (int u = 0; u < GF; ++u) {
        const int i = tid + u * kThreads;
        const int r = i / (D / 32), g = i % (D / 32);
        const int id = ids[r];
        raw[u] = make_uint4(0, 0, 0, 0);
        sc[u] = 0u;
        if (id >= 0) {
          const size_t er = (size_t)b * a.cap + id;
          raw[u] = __ldg(reinterpret_cast<const uint4 *>(a.codes + er * (D / 2)) + g);
          sc[u] = __ldg(reinterpret_cast<const uint16_t *>(a.scales + er * (D / 16)) + g);
        }
      }
    } else {
#pragma unroll
      for (int u = 0; u < GW; ++u) {
        const int i = tid + u * kThreads;
        const int r = i / (D / 16), g = i % (D / 16);
        const int id = ids[r];
        raw[u] = id >= 0 ? __ldg(reinterpret_cast<const uint4 *>(a.swa_rows + ((size_t)b * a.W_cap + id) * D) + g)
                         : make_uint4(0, 0, 0, 0);
      }
    }
    // the previous tile's O^T MMAs read K^ and P: wait before overwriting
    bool ok = true;
    if (n_done > 0) ok = mbar_wait_bounded(&S.obar, (n_done - 1) & 1, kWaitLimit);
    if (__syncthreads_or(!ok)) { aborted = true; break; }

    // ---- 1b. dequantise (hardware converts, exact) into the swizzled K^ tile
    if (!is_win) {
#pragma unroll
      for (int u = 0; u < GF; ++u) {
        const int i = tid + u * kThreads;
        const int r = i / (D / 32), g = i % (D / 32);
        const uint32_t s2 = e4m3x2_to_f16x2(sc[u]);   // scales of channels 32g.. and 32g+16..
        const __half2 slo = __low2half2(*reinterpret_cast<const __half2 *>(&s2));
        const __half2 shi = __high2half2(*reinterpret_cast<const __half2 *>(&s2));
        const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {   // 8 channels -> one 16-byte piece
          uint32_t h[4];
          e2m1x8_to_f16x2(w[k], h);
          const __half2 sk = k < 2 ? slo : shi;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const __half2 v = __hmul2(*reinterpret_cast<const __half2 *>(&h[e]), sk);
            h[e] = *reinterpret_cast<const uint32_t *>(&v);
          }
          *reinterpret_cast<uint4 *>(S.kh + sw_off(r, 4 * g + k, kTile)) = make_uint4(h[0], h[1], h[2], h[3]);
        }
      }
    } else {
#pragma unroll
      for (int u = 0; u < GW; ++u) {
        const int i = tid + u * kThreads;
        const int r = i / (D / 16), g = i % (D / 16);
        uint32_t h[8];
        e4m3x4_to_f16x2(raw[u].x, h);
        e4m3x4_to_f16x2(raw[u].y, h + 2);
        e4m3x4_to_f16x2(raw[u].z, h + 4);
        e4m3x4_to_f16x2(raw[u].w, h + 6);
        *reinterpret_cast<uint4 *>(S.kh + sw_off(r, 2 * g, kTile)) = make_uint4(h[0], h[1], h[2], h[3]);
        *reinterpret_cast<uint4 *>(S.kh + sw_off(r, 2 * g + 1, kTile)) = make_uint4(h[4], h[5], h[6], h[7]);
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- 2. S^T = K^ Q^T (warp 4 converged, one elected lane issues)
    if (warp == kMmaWarp) {
      // descriptors advance by (byte offset >> 4) in their start-address field
      tc_fence_after();
      const uint64_t da = smem_desc_kmajor(kh_base, 128), db = smem_desc_kmajor(q_base, 128);
      if (elect_one()) {
#pragma unroll
        for (int ks = 0; ks < D / 16; ++ks) {
          const uint32_t off = (uint32_t)((ks & 3) * 32);
          tc_mma_f16(tmem, da + (((ks >> 2) * (kTile * 128) + off) >> 4),
                     db + (((ks >> 2) * (kHeads * 128) + off) >> 4), kIdS, ks > 0 ? 1u : 0u);
        }
        tc_commit(&S.sbar);
      }
      __syncwarp();
    }
    // the next tile's key ids (the other buffer) while the MMAs run
    if (c + 1 < c_end) load_key_ids<D>(a, row, b, c + 1, n_fp4_tiles, wlo, nwin, S.key_ent[(c + 1) & 1], tid, true);
    ok = mbar_wait_bounded(&S.sbar, (c - c_begin) & 1, kWaitLimit);
    if (__syncthreads_or(!ok)) { aborted = true; break; }
    tc_fence_after();

    // ---- 3. softmax: warp (quarter, half) holds keys 32*quarter + lane,
    // heads 32*half .. 32*half + 31
    const float lsc = a.scale * (is_win ? a.s_swa : 1.0f) * kLog2e;
    const float psc = is_win ? a.s_swa : 1.0f;
    const bool first = (c == c_begin);
    const int r = 32 * quarter + lane;
    float sv[32];
    const bool valid = ids[r] >= 0;
    auto load_logits = [&]() {
      uint32_t rv[32];
      tmem_ld_x32(tmem + ((uint32_t)(32 * quarter) << 16) + 32 * half, rv);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 32; ++j) sv[j] = valid ? __uint_as_float(rv[j]) * lsc : -INFINITY;
    };
    load_logits();
    // After the first tile the reference max usually holds: the per-head
    // maxima are needed only when some logit exceeds it by more than 2^8.
    bool need_max = first;
    if (!first) {
      const float4 *mp = reinterpret_cast<const float4 *>(&S.m_ref[32 * half]);
      bool over = false;
#pragma unroll
      for (int j4 = 0; j4 < 8; ++j4) {
        const float4 m4 = mp[j4];
        over |= (sv[4 * j4] > m4.x + kLazy) | (sv[4 * j4 + 1] > m4.y + kLazy) | (sv[4 * j4 + 2] > m4.z + kLazy) |
                (sv[4 * j4 + 3] > m4.w + kLazy);
      }
      need_max = __syncthreads_or(over);
    }
    if (need_max) {
      // per-head maxima of this warp's 32 keys (the butterfly consumes sv;
      // the logits are read from TMEM again afterwards)
      reduce_scatter32_max(sv, lane);
      S.red[quarter][32 * half + lane] = sv[0];
      __syncthreads();
      load_logits();
    }
    if (need_max && tid < kHeads) {   // new reference max of head tid
      const float m_old = S.m_ref[tid];
      const float mt = fmaxf(fmaxf(S.red[0][tid], S.red[1][tid]), fmaxf(S.red[2][tid], S.red[3][tid]));
      float al = 1.f;
      if (mt != -INFINITY) {
        if (m_old == -INFINITY) {
          S.m_ref[tid] = mt;
          al = 0.f;
        } else if (mt > m_old + kLazy) {
          S.m_ref[tid] = mt;
          al = exp2f(m_old - mt);
          if (!first) S.rescale = 1;
        }
      }
      S.alpha[tid] = al;
      S.l_run[tid] *= al;
    }
    if (need_max) __syncthreads();
    // P = 2^(s - m_ref): row r of the P operand (fp16, window rows scaled)
    {
      const float4 *mp = reinterpret_cast<const float4 *>(&S.m_ref[32 * half]);
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
        const __half2 h0 = __floats2half2_rn(sv[4 * j4] * psc, sv[4 * j4 + 1] * psc);
        const __half2 h1 = __floats2half2_rn(sv[4 * j4 + 2] * psc, sv[4 * j4 + 3] * psc);
        ph[2 * j4] = *reinterpret_cast<const uint32_t *>(&h0);
        ph[2 * j4 + 1] = *reinterpret_cast<const uint32_t *>(&h1);
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
        *reinterpret_cast<uint4 *>(S.p + r * 128 + (((4 * half + i) ^ (r & 7)) << 4)) =
            make_uint4(ph[4 * i], ph[4 * i + 1], ph[4 * i + 2], ph[4 * i + 3]);
      reduce_scatter32(sv, lane);   // sv[0] = sum over this warp's keys of head 32*half + lane
    }
    S.red[quarter][32 * half + lane] = sv[0];   // the max readers finished before the last barrier
    __syncthreads();
    if (tid < kHeads) S.l_run[tid] += (S.red[0][tid] + S.red[1][tid]) + (S.red[2][tid] + S.red[3][tid]);
    // rare: a head's reference max moved -> rescale its O^T column
    if (S.rescale) {
#pragma unroll 1
      for (int mt = mt_lo; mt < mt_hi; ++mt) {
        const uint32_t taddr = tmem + ((uint32_t)(32 * quarter) << 16) + kHeads + mt * kHeads + 32 * half;
        uint32_t o[32];
        tmem_ld_x32(taddr, o);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 32; ++j) o[j] = __float_as_uint(__uint_as_float(o[j]) * S.alpha[32 * half + j]);
        tmem_st_x32(taddr, o);
      }
      tmem_wait_st();
    }
    fence_proxy_async();   // P (generic stores) -> visible to the tensor core
    tc_fence_before();
    __syncthreads();
    if (tid == 0) S.rescale = 0;

    // ---- 4. O^T += V^T P^T
    if (warp == kMmaWarp) {
      tc_fence_after();
      const uint64_t da = smem_desc_mnmajor_sw128(kh_base, kTile * 128, 1024);
      const uint64_t db = smem_desc_mnmajor_sw128(p_base, kTile * 128, 1024);
      if (elect_one()) {
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
          if (mt < mt_lo || mt >= mt_hi) continue;
#pragma unroll
          for (int ks = 0; ks < kTile / 16; ++ks)
            tc_mma_f16(tmem + kHeads + mt * kHeads, da + (((2 * mt) * (kTile * 128) + (2 * ks) * 1024) >> 4),
                       db + (((2 * ks) * 1024) >> 4), kIdO, (ks > 0 || !first) ? 1u : 0u);
        }
        tc_commit(&S.obar);
      }
      __syncwarp();
    }
    ++n_done;
  }

  // ---- epilogue: O^T (TMEM lane = channel within a 128-channel block)
  bool ok = !aborted;
  if (ok && n_done > 0) ok = mbar_wait_bounded(&S.obar, (n_done - 1) & 1, kWaitLimit);
  const bool failed = __syncthreads_or(!ok);
  if (failed) {
    if (tid == 0) flag(a.status, CSA2_DEV_TIMEOUT);
    if (warp == kMmaWarp && n_done > 0) {   // let every issued MMA finish before TMEM is freed
      if (elect_one()) {                     // the lane that issued them
        mbar_init(&S.sbar, 1);
        fence_barrier_init();
        tc_commit(&S.sbar);
        mbar_wait_bounded(&S.sbar, 0, kWaitLimit);
      }
      __syncwarp();
    }
  } else {
    tc_fence_after();
    const size_t nrows = (size_t)a.B * a.T_q;
    // O / l per head.  One split: bf16, staged head-major [64 heads][D] in
    // the K^ tile (free once the last O^T MMA completed), then written out in
    // 16-byte pieces.  Several splits: fp16 partials straight from registers
    // (a channel per lane; staging measured slower on this latency-bound path).
    // 1 / l per head, once per head (not per thread)
    if (tid < kHeads) {
      const float l = S.l_run[tid];
      S.linv[tid] = l > 0.f ? 1.f / l : 0.f;
    }
    __syncthreads();
    float linv[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) linv[j] = S.linv[32 * half + j];
    uint16_t *ob = reinterpret_cast<uint16_t *>(S.kh);
#pragma unroll 1
    for (int mt = mt_lo; mt < mt_hi; ++mt) {
      const int ch = mt * 128 + 32 * quarter + lane;
      uint32_t o[32];
      if (n_done > 0) {
        tmem_ld_x32(tmem + ((uint32_t)(32 * quarter) << 16) + kHeads + mt * kHeads + 32 * half, o);
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
        __half *po = reinterpret_cast<__half *>(a.ws) + ((size_t)row * a.nsplit + split) * kHeads * D + ch;
#pragma unroll
        for (int j = 0; j < 32; ++j) po[(size_t)(32 * half + j) * D] = __float2half_rn(__uint_as_float(o[j]) * linv[j]);
      }
    }
    if (a.nsplit == 1) {
      __syncthreads();
      const uint4 *src = reinterpret_cast<const uint4 *>(ob);
      uint4 *dst = reinterpret_cast<uint4 *>(a.out + (size_t)row * a.H * D);
      const int n16 = a.H * (D / 8);
#pragma unroll 4
      for (int i = tid; i < n16; i += kThreads) dst[i] = src[i];
    }
    if (a.nsplit > 1 && tid < kHeads) {
      float *pm = partial_stats(a, nrows) + ((size_t)row * a.nsplit + split) * kHeads;
      float *pl = pm + nrows * a.nsplit * kHeads;
      pm[tid] = S.m_ref[tid];
      pl[tid] = S.l_run[tid];
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }

  // ---- merge of the splits (the row's blocks form one cluster)
  if (a.nsplit > 1) {
    cluster_sync_all();   // every split's partials are written
    const size_t nrows = (size_t)a.B * a.T_q;
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
    // this split's channel slice; item = (head, 8 channels): 16 bytes per split in, 16 bytes out
    const int Dz = D / a.csplit, z_lo = (int)blockIdx.z * Dz;   // this block's channel half (or all)
    const int cs = ((Dz / a.nsplit) + 7) / 8 * 8;
    const int c_lo = z_lo + split * cs;
    const int c_hi = c_lo + cs < z_lo + Dz ? c_lo + cs : z_lo + Dz;
    const int ng = c_hi > c_lo ? (c_hi - c_lo) / 8 : 0;
    const int n_items = a.H * ng;
    const __half *base = reinterpret_cast<const __half *>(a.ws) + (size_t)row * a.nsplit * kHeads * D;
#pragma unroll 1
    for (int it0 = tid; it0 < n_items; it0 += kMergeItems * kThreads) {   // kMergeItems items' loads in flight
      uint4 x[kMergeItems][8];
#pragma unroll
      for (int v = 0; v < kMergeItems; ++v) {
        const int it = it0 + v * kThreads;
        const int h = it / ng, ch = c_lo + 8 * (it % ng);
#pragma unroll
        for (int s = 0; s < 8; ++s)
          x[v][s] = (it < n_items && s < a.nsplit)
                        ? __ldcg(reinterpret_cast<const uint4 *>(base + ((size_t)s * kHeads + h) * D + ch))
                        : make_uint4(0, 0, 0, 0);
      }
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

template <int D>
static cudaError_t launch_attn_lat_t(const AttnArgs &a, cudaStream_t s) {
  const size_t smem = sizeof(AttnSmem<D>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_lat_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(attn_lat_kernel<D>, dim3(a.B * a.T_q, a.nsplit, a.csplit), dim3(kThreads), smem, s,
                    dim3(1, (unsigned)a.nsplit, 1),
                    a);
}

cudaError_t launch_attn_lat(const AttnArgs &a, cudaStream_t s) {
  switch (a.D) {
    case 128: return launch_attn_lat_t<128>(a, s);
    case 256: return launch_attn_lat_t<256>(a, s);
    default: return launch_attn_lat_t<512>(a, s);
  }
}

}  // namespace csa2
