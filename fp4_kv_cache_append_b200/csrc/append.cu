// Append kernel: pool m tokens into a compressed entry, quantise it to FP4
// (E2M1 + one E4M3 scale per 16 channels), project and FP8-quantise its
// indexer key, and write FP8 window rows.
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2": m tokens -> one
//   entry with no overlap and no absolute-position term; the indexer key is
//   projected from the main KV.  Section "3) FP4 main KV + SWA Bounded
//   Replay": FP4 main KV, FP8 window KV.
// One 512-thread block per group of up to 8 new entries (thread t < D/2 owns
// channels 2t, 2t+1 and writes code byte t; all threads share the projection:
// one fused multiply-add chain per (entry, key output), channels ascending)
// and one block per window row.  The quantised bytes are
// decided in binary32 with IEEE division, no contraction (explicit _rn
// intrinsics), so they are reproducible bit for bit.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace csa2 {

// e^x for x in [-80, 0], binary32: Cody-Waite reduction x = n ln2 + r with
// ln2 split into a 17-bit head (exact n*head for |n| < 128) and the rounded
// tail, then the degree-7 Taylor polynomial of e^r by Horner's rule with
// fused multiply-adds, scaled by 2^n built from its exponent field.  Below
// -80 the result is 0.  The gate weights of an m = 2 entry depend on this
// exact operation sequence.
__device__ __forceinline__ float gate_exp(float x) {
  if (!(x >= -80.0f)) return 0.0f;
  if (x > 0.0f) x = 0.0f;
  const float n = rintf(__fmul_rn(x, 0x1.715476p+0f));
  float r = __fmaf_rn(-n, 0x1.62e4p-1f, x);
  r = __fmaf_rn(-n, 0x1.7f7d1cp-20f, r);
  float p = 0x1.a01a02p-13f;
  p = __fmaf_rn(p, r, 0x1.6c16c2p-10f);
  p = __fmaf_rn(p, r, 0x1.111112p-7f);
  p = __fmaf_rn(p, r, 0x1.555556p-5f);
  p = __fmaf_rn(p, r, 0x1.555556p-3f);
  p = __fmaf_rn(p, r, 0.5f);
  p = __fmaf_rn(p, r, 1.0f);
  p = __fmaf_rn(p, r, 1.0f);
  return __fmul_rn(p, __uint_as_float((uint32_t)((int)n + 127) << 23));
}

// Softmax-gated pair (per channel): the larger logit gets 1/(1+e), the other
// e/(1+e), e = exp(-|z_a - z_b|); pooled = fl(w_a kv_a) + fl(w_b kv_b).
__device__ __forceinline__ float pool_pair(float ka, float kb, float za, float zb) {
  const float e = gate_exp(-fabsf(__fsub_rn(za, zb)));
  const float s = __fadd_rn(1.0f, e);
  const float w_big = __fdiv_rn(1.0f, s), w_small = __fdiv_rn(e, s);
  const float wa = (za >= zb) ? w_big : w_small;
  const float wb = (za >= zb) ? w_small : w_big;
  return __fadd_rn(__fmul_rn(wa, ka), __fmul_rn(wb, kb));
}

// Indexer keys of entries e0 .. e0+count-1 (count <= 32) of
// sequence b from their dequantised values xh [count][D] (shared memory),
// with W_ik staged in shared memory as ws [D][dI]: k_i = sum_c x^_c W[c][i]
// as ONE fused multiply-add chain per output, channels in ascending order
// from +0; then per entry s_k = amax/448 and E4M3 codes of k/s_k.  Thread t
// owns output i = t % dI of entries t / dI + k * slots (slots = blockDim /
// dI, k < kChains): its chains run side by side, share every W_ik element it
// reads and take 4 channels of an entry per 16-byte load.  Every thread of
// the block must call it.
template <int D, int DI>
__device__ __forceinline__ void entry_chains(int count, const float *xh, float *kbuf, const uint16_t *ws) {
  constexpr int kChains = 8;   // 32 entries over 4 (d_I = 128) slots of 512 threads; d_I = 64 uses 4 of them
  constexpr int kSlots = 512 / DI;
  const int t = threadIdx.x;
  const int i = t % DI, s0 = t / DI;
  if (s0 >= count) return;
  // which of this thread's chains exist, decided once (warp-uniform)
  bool act[kChains];
#pragma unroll
  for (int k = 0; k < kChains; ++k) act[k] = s0 + k * kSlots < count;
  float acc[kChains];
#pragma unroll
  for (int k = 0; k < kChains; ++k) acc[k] = 0.0f;
  const uint16_t *wcol = ws + i;
  const float *xr = xh + s0 * D;   // chain k reads row s0 + k * kSlots: a constant offset
#pragma unroll 2
  for (int c = 0; c < D; c += 4) {
    const float w0 = bf16_to_f32(wcol[c * DI]), w1 = bf16_to_f32(wcol[(c + 1) * DI]);
    const float w2 = bf16_to_f32(wcol[(c + 2) * DI]), w3 = bf16_to_f32(wcol[(c + 3) * DI]);
#pragma unroll
    for (int k = 0; k < kChains; ++k) {
      if (act[k]) {
        const float4 x = *reinterpret_cast<const float4 *>(xr + k * kSlots * D + c);
        float v = acc[k];
        v = __fmaf_rn(x.x, w0, v);
        v = __fmaf_rn(x.y, w1, v);
        v = __fmaf_rn(x.z, w2, v);
        acc[k] = __fmaf_rn(x.w, w3, v);
      }
    }
  }
#pragma unroll
  for (int k = 0; k < kChains; ++k)
    if (act[k]) kbuf[(s0 + k * kSlots) * DI + i] = acc[k];
}

__device__ void entry_keys(const AppendArgs &a, int b, int e0, int count, const float *xh, float *kbuf,
                           const uint16_t *ws) {
  const int t = threadIdx.x, dI = a.dI;
  switch (a.D * 1000 + dI) {   // the chains with compile-time strides
    case 512128: entry_chains<512, 128>(count, xh, kbuf, ws); break;
    case 512064: entry_chains<512, 64>(count, xh, kbuf, ws); break;
    case 256128: entry_chains<256, 128>(count, xh, kbuf, ws); break;
    case 256064: entry_chains<256, 64>(count, xh, kbuf, ws); break;
    case 128128: entry_chains<128, 128>(count, xh, kbuf, ws); break;
    default: entry_chains<128, 64>(count, xh, kbuf, ws); break;
  }
  __syncthreads();
  // ---- FP8 key per entry: warp w takes entries w, w + warps, ...
  const int warp = t >> 5, lane = t & 31, nw = (int)blockDim.x >> 5;
  for (int jj = warp; jj < count; jj += nw) {
    const int e = e0 + jj;
    float kmax = 0.0f;
    for (int i = lane; i < dI; i += 32) kmax = fmaxf(kmax, fabsf(kbuf[jj * dI + i]));
    for (int o = 16; o > 0; o >>= 1) kmax = fmaxf(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
    const float sk = __fdiv_rn(kmax, 448.0f);
    if (e < a.cap) {
      const size_t row = (size_t)b * a.cap + e;
      for (int i = lane; i < dI; i += 32)
        a.ik[row * dI + i] = (uint8_t)(sk == 0.0f ? 0u : f32_to_e4m3(__fdiv_rn(kbuf[jj * dI + i], sk)));
      if (lane == 0) a.ik_scale[row] = sk;
    }
  }
}

// Entries j0 .. j0+count-1 (count <= entries_per_block <= 32) of sequence b.  The
// projection reads each W_ik element once for all of the block's entries.
__device__ void append_entries(const AppendArgs &a, int b, int j0, float *sm) {
  const int t = threadIdx.x;
  const int D = a.D, dI = a.dI, m = a.m;
  const int p0 = a.pos0[b];
  if (p0 < 0) {
    if (t == 0 && j0 == 0) flag(a.status, CSA2_DEV_BAD_POSITION);
    return;
  }
  if (j0 == 0 && t == 0) a.n_entries[b] = (p0 + a.T) / m;
  const int n_new = (p0 + a.T) / m - p0 / m;
  int count = n_new - j0;
  if (count > a.entries_per_block) count = a.entries_per_block;

  float *xh = sm;                                   // [E][D]
  float *kbuf = xh + a.entries_per_block * D;       // [E][dI] binary32 keys
  uint16_t *ws = reinterpret_cast<uint16_t *>(kbuf + a.entries_per_block * dI + 32);  // W_ik [D][dI] bf16, 16-byte aligned
  // stage W_ik in shared memory with 16-byte loads (issued before the
  // quantisation so their latency overlaps it)
  if (count > 0) {
    const uint4 *src = reinterpret_cast<const uint4 *>(a.w_ik);
    uint4 *dst = reinterpret_cast<uint4 *>(ws);
    for (int i = t; i < D * dI / 8; i += blockDim.x) dst[i] = src[i];
  }

  // ---- pool + FP4 per entry: thread t owns channels 2p, 2p+1 (p = t % (D/2),
  // 8 threads per 16-channel group) of entries t / (D/2) + k * (blockDim /
  // (D/2)); each round's loads (8 entries) are issued before any is used
  {
    const int P2 = D / 2, G2 = (int)blockDim.x / P2, p = t % P2;
    for (int base = t / P2; base < count; base += 8 * G2) {
      uint32_t ka[8], kb[8], ga[8], gb[8];
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int jj = base + r * G2;
        if (jj >= count) break;
        const int e = p0 / m + j0 + jj;
        if (m == 1) {
          ka[r] = reinterpret_cast<const uint32_t *>(a.kv + ((size_t)b * a.T + (e - p0)) * D)[p];
        } else {
          const int ta = 2 * e - p0;  // -1 only for the block's first entry with p0 odd: the pending token
          const uint16_t *kva = ta < 0 ? a.pending_kv + (size_t)b * D : a.kv + ((size_t)b * a.T + ta) * D;
          const uint16_t *za = ta < 0 ? a.pending_gate + (size_t)b * D : a.gate + ((size_t)b * a.T + ta) * D;
          ka[r] = reinterpret_cast<const uint32_t *>(kva)[p];
          kb[r] = reinterpret_cast<const uint32_t *>(a.kv + ((size_t)b * a.T + ta + 1) * D)[p];
          ga[r] = reinterpret_cast<const uint32_t *>(za)[p];
          gb[r] = reinterpret_cast<const uint32_t *>(a.gate + ((size_t)b * a.T + ta + 1) * D)[p];
        }
      }
#pragma unroll
      for (int r = 0; r < 8; ++r) {
        const int jj = base + r * G2;
        if (jj >= count) break;
        const int e = p0 / m + j0 + jj;
        float x0, x1;
        if (m == 1) {
          x0 = bf16_to_f32((uint16_t)(ka[r] & 0xFFFFu));
          x1 = bf16_to_f32((uint16_t)(ka[r] >> 16));
        } else {
          x0 = pool_pair(bf16_to_f32(ka[r] & 0xFFFFu), bf16_to_f32(kb[r] & 0xFFFFu), bf16_to_f32(ga[r] & 0xFFFFu),
                         bf16_to_f32(gb[r] & 0xFFFFu));
          x1 = pool_pair(bf16_to_f32(ka[r] >> 16), bf16_to_f32(kb[r] >> 16), bf16_to_f32(ga[r] >> 16),
                         bf16_to_f32(gb[r] >> 16));
        }
        float amax = fmaxf(fabsf(x0), fabsf(x1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
        uint32_t sb = amax == 0.0f ? 0u : f32_to_e4m3(__fdiv_rn(amax, 6.0f));
        const float sc = e4m3_to_f32(sb);
        uint32_t c0 = 0, c1 = 0;
        if (sc != 0.0f) {
          c0 = f32_to_e2m1(__fdiv_rn(x0, sc));
          c1 = f32_to_e2m1(__fdiv_rn(x1, sc));
        } else {
          sb = 0;
        }
        if (e < a.cap) {
          const size_t row = (size_t)b * a.cap + e;
          a.codes[row * (D / 2) + p] = (uint8_t)(c0 | (c1 << 4));
          if ((p & 7) == 0) a.scales[row * (D / 16) + (p >> 3)] = (uint8_t)sb;
        } else if (p == 0) {
          flag(a.status, CSA2_DEV_APPEND_RANGE);
        }
        xh[jj * D + 2 * p] = __fmul_rn(e2m1_to_f32(c0), sc);
        xh[jj * D + 2 * p + 1] = __fmul_rn(e2m1_to_f32(c1), sc);
      }
    }
  }
  // m = 2: the chunk's last token opens a pair -> it waits in the pending
  // buffer.  Block j0 == 0 is the only one that reads or writes it; it reads
  // first (above) and writes after the barrier.
  __syncthreads();
  if (m == 2 && j0 == 0 && ((p0 + a.T) & 1) && t < D / 2) {
    const size_t src = ((size_t)b * a.T + (a.T - 1)) * D;
    reinterpret_cast<uint32_t *>(a.pending_kv + (size_t)b * D)[t] = reinterpret_cast<const uint32_t *>(a.kv + src)[t];
    reinterpret_cast<uint32_t *>(a.pending_gate + (size_t)b * D)[t] = reinterpret_cast<const uint32_t *>(a.gate + src)[t];
  }
  if (count <= 0) return;

  entry_keys(a, b, p0 / m + j0, count, xh, kbuf, ws);
}

__device__ void append_window_row(const AppendArgs &a, int b, int r) {
  const int t = threadIdx.x;
  if (t >= a.D / 2) return;
  const int p0 = a.pos0[b];
  const int cnt = a.T < a.W_cap ? a.T : a.W_cap;
  const int tau = a.T - cnt + r;
  const int p = p0 + tau;
  if (p < 0) {
    if (t == 0) flag(a.status, CSA2_DEV_BAD_POSITION);
    return;
  }
  const uint32_t v = reinterpret_cast<const uint32_t *>(a.kv_swa + ((size_t)b * a.T + tau) * a.D)[t];
  const uint32_t lo = f32_to_e4m3(__fdiv_rn(bf16_to_f32((uint16_t)(v & 0xFFFFu)), a.s_swa));
  const uint32_t hi = f32_to_e4m3(__fdiv_rn(bf16_to_f32((uint16_t)(v >> 16)), a.s_swa));
  uint8_t *dst = a.swa_rows + ((size_t)b * a.W_cap + (p % a.W_cap)) * a.D;
  reinterpret_cast<uint16_t *>(dst)[t] = (uint16_t)(lo | (hi << 8));
}

// Blocks beyond the cache work prepare the following scan's indexer query:
// 8 blocks per query row, warp w of block j handles head 8j + w.  WAIT: the
// codes are formed before the wait for the previous launch, stored after it.
template <bool WAIT>
__device__ __forceinline__ void prep_block(const AppendArgs &a, int i) {
  const int row = i / 8, h = (i % 8) * 8 + (int)(threadIdx.x >> 5);
  if (row >= a.prep.rows || threadIdx.x >= 256) return;
  if (a.prep.dI == 128) prep_query_head<128, WAIT>(a.prep, row, h, threadIdx.x & 31);
  else prep_query_head<64, WAIT>(a.prep, row, h, threadIdx.x & 31);
}

__global__ void append_kernel(const AppendArgs a) {
  extern __shared__ float sm[];
  pdl_launch_dependents();
  pdl_wait();
  const int nm = a.B * a.main_blocks_per_seq;
  const int nw = a.B * a.swa_blocks_per_seq;
  if ((int)blockIdx.x >= nm + nw) {
    prep_block<false>(a, (int)blockIdx.x - nm - nw);
    return;
  }
  if ((int)blockIdx.x < nm) {
    append_entries(a, blockIdx.x / a.main_blocks_per_seq,
                   (blockIdx.x % a.main_blocks_per_seq) * a.entries_per_block, sm);
  } else {
    const int i = blockIdx.x - nm;
    append_window_row(a, i / a.swa_blocks_per_seq, i % a.swa_blocks_per_seq);
  }
}

// Operands of channels c0 .. c0+31 of one indexer-key output: x^ (binary32)
// and the output's row of the transposed W_ik slice (bf16, channels contiguous).
__device__ __forceinline__ void dec_key_load(const float *xh, const uint16_t *wrow, int c0, float4 (&x)[8],
                                             uint4 (&w)[4]) {
#pragma unroll
  for (int j = 0; j < 8; ++j) x[j] = reinterpret_cast<const float4 *>(xh + c0)[j];
#pragma unroll
  for (int j = 0; j < 4; ++j) w[j] = reinterpret_cast<const uint4 *>(wrow + c0)[j];
}
// 32 multiply-adds in ascending channel order; a 32-bit word holds the bf16 of
// an even channel in its low half and of the next channel in its high half.
__device__ __forceinline__ float dec_key_chunk(float acc, const float4 (&x)[8], const uint4 (&w)[4]) {
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const uint32_t u[4] = {w[j].x, w[j].y, w[j].z, w[j].w};
    const float v[8] = {x[2 * j].x, x[2 * j].y, x[2 * j].z, x[2 * j].w,
                        x[2 * j + 1].x, x[2 * j + 1].y, x[2 * j + 1].z, x[2 * j + 1].w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      acc = __fmaf_rn(v[2 * k], __uint_as_float(u[k] << 16), acc);
      acc = __fmaf_rn(v[2 * k + 1], __uint_as_float(u[k] & 0xFFFF0000u), acc);
    }
  }
  return acc;
}
// One indexer-key output as one fused multiply-add chain over the channels in
// ascending order from +0.  The next 32 channels' operands are loaded while
// the current 32 multiply-adds run, so the chain runs at the multiply-add
// latency (D is a multiple of 64).
__device__ __forceinline__ float dec_key_chain(const float *xh, const uint16_t *wrow, int D) {
  float acc = 0.0f;
  float4 xa[8], xb[8];
  uint4 wa[4], wb[4];
  dec_key_load(xh, wrow, 0, xa, wa);
#pragma unroll 1
  for (int c0 = 0; c0 < D; c0 += 64) {
    dec_key_load(xh, wrow, c0 + 32, xb, wb);
    acc = dec_key_chunk(acc, xa, wa);
    if (c0 + 64 < D) dec_key_load(xh, wrow, c0 + 64, xa, wa);
    acc = dec_key_chunk(acc, xb, wb);
  }
  return acc;
}

// Decode (one new token per sequence, m = 1): a cluster of 8 blocks per
// sequence.  Every block quantises the new entry (the same binary32 steps as
// append_entries, so all blocks hold the same x^); block c projects indexer
// outputs [c*dI/8, (c+1)*dI/8) from its slice of W_ik and writes 1/8 of the
// window row; the FP8 key scale needs the maximum over all outputs, which the
// blocks push into each other's shared memory before one cluster barrier.
// Block 0 writes the FP4 codes, the scales, the key scale and n_entries.
// The kernel reads only inputs that no launch of the library writes (the
// token, its window copy, W_ik, the positions, the indexer query), so all of
// its arithmetic runs while the previous launch (the previous step's
// attention, which reads the cache and the window ring) is still running; it
// waits for that launch only before its first store.
constexpr int kDecCl = 8;
constexpr int kWT = 512 + 8;   // row stride (bf16) of the transposed W_ik slice: rows on distinct banks

__global__ void __cluster_dims__(kDecCl, 1, 1) __launch_bounds__(256) append_decode_kernel(const AppendArgs a) {
  __shared__ alignas(16) float xh[512];
  __shared__ alignas(16) uint16_t wsl[16 * kWT];   // W_ik[:, c*OPB .. c*OPB+OPB) transposed: [OPB][D (+8)]
  __shared__ float kmx[kDecCl];                    // the blocks' local key maxima
  cg::cluster_group cl = cg::this_cluster();
  const int c = (int)cl.block_rank();
  const int b = blockIdx.y, t = threadIdx.x;
  const int D = a.D, dI = a.dI, OPB = dI / kDecCl;
  pdl_launch_dependents();
  if (b >= a.B) {   // a cluster of query-preparation blocks (no cluster barrier)
    prep_block<true>(a, (b - a.B) * kDecCl + c);
    return;
  }
  const int p0 = a.pos0[b];
  if (p0 < 0) {   // the same in every block of the cluster: none of them waits at the cluster barrier
    if (t == 0 && c == 0) {
      pdl_wait();
      flag(a.status, CSA2_DEV_BAD_POSITION);
    }
    return;
  }
  const int e = p0;   // m = 1: token p0 completes entry p0
  // ---- loads, all issued before any is used: the entry's kv pair, its window
  // pair, and this block's W_ik slice (16-byte pieces, at most 4 per thread)
  uint32_t kvp = 0u, swp = 0u;
  if (t < D / 2) kvp = reinterpret_cast<const uint32_t *>(a.kv + (size_t)b * D)[t];
  const int wch = D / (2 * kDecCl);   // window channel pairs per block
  if (a.swa_rows && t < wch) swp = reinterpret_cast<const uint32_t *>(a.kv_swa + (size_t)b * D)[c * wch + t];
  {
    const int ppr = OPB * 2 / 16;   // 16-byte pieces per W row of the slice
    const uint4 *src = reinterpret_cast<const uint4 *>(a.w_ik);
    uint4 wv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = t + u * 256;
      if (i < D * ppr) wv[u] = __ldg(src + ((size_t)(i / ppr) * dI + c * OPB) * 2 / 16 + i % ppr);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {   // piece = channel i / ppr, outputs 8 (i % ppr) .. + 7
      const int i = t + u * 256;
      if (i < D * ppr) {
        const int ch = i / ppr, o0 = 8 * (i % ppr);
        const uint32_t w[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          wsl[(o0 + 2 * k) * kWT + ch] = (uint16_t)(w[k] & 0xFFFFu);
          wsl[(o0 + 2 * k + 1) * kWT + ch] = (uint16_t)(w[k] >> 16);
        }
      }
    }
  }

  // ---- FP4: thread t < D/2 owns channels 2t, 2t+1 (8 threads per 16-channel group)
  uint32_t code_pair = 0u, scale_byte = 0u;
  if (t < D / 2) {
    const float x0 = bf16_to_f32((uint16_t)(kvp & 0xFFFFu)), x1 = bf16_to_f32((uint16_t)(kvp >> 16));
    float amax = fmaxf(fabsf(x0), fabsf(x1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 4));
    uint32_t sb = amax == 0.0f ? 0u : f32_to_e4m3(__fdiv_rn(amax, 6.0f));
    const float sc = e4m3_to_f32(sb);
    uint32_t c0 = 0, c1 = 0;
    if (sc != 0.0f) {
      c0 = f32_to_e2m1(__fdiv_rn(x0, sc));
      c1 = f32_to_e2m1(__fdiv_rn(x1, sc));
    } else {
      sb = 0;
    }
    code_pair = c0 | (c1 << 4);
    scale_byte = sb;
    xh[2 * t] = __fmul_rn(e2m1_to_f32(c0), sc);
    xh[2 * t + 1] = __fmul_rn(e2m1_to_f32(c1), sc);
  }
  // ---- window: channels [2*wch*c, 2*wch*(c+1)) of the ring slot p0 mod W_cap
  uint32_t win_pair = 0u;
  if (a.swa_rows && t < wch) {
    const uint32_t lo = f32_to_e4m3(__fdiv_rn(bf16_to_f32((uint16_t)(swp & 0xFFFFu)), a.s_swa));
    const uint32_t hi = f32_to_e4m3(__fdiv_rn(bf16_to_f32((uint16_t)(swp >> 16)), a.s_swa));
    win_pair = lo | (hi << 8);
  }
  __syncthreads();
  // ---- indexer key: thread o < OPB forms output c*OPB + o as one fused
  // multiply-add chain over the channels in ascending order from +0, as
  // append_entries does
  float k = 0.0f;
  if (t < 32) {
    if (t < OPB) {
      k = dec_key_chain(xh, wsl + t * kWT, D);
    }
    float m = t < OPB ? fabsf(k) : 0.0f;
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xffffffffu, m, o));
    if (t < kDecCl) *cl.map_shared_rank(&kmx[c], t) = m;   // push into every block
  }
  cl.sync();
  float sk = 0.0f;
  uint32_t kcode = 0u;
  if (t < OPB) {
    float kmax = kmx[0];
#pragma unroll
    for (int r = 1; r < kDecCl; ++r) kmax = fmaxf(kmax, kmx[r]);
    sk = __fdiv_rn(kmax, 448.0f);
    kcode = sk == 0.0f ? 0u : f32_to_e4m3(__fdiv_rn(k, sk));
  }

  // ---- stores, once the previous launch has finished with the cache
  pdl_wait();
  if (c == 0 && t < D / 2) {
    if (e < a.cap) {
      const size_t row = (size_t)b * a.cap + e;
      a.codes[row * (D / 2) + t] = (uint8_t)code_pair;
      if ((t & 7) == 0) a.scales[row * (D / 16) + (t >> 3)] = (uint8_t)scale_byte;
    } else if (t == 0) {
      flag(a.status, CSA2_DEV_APPEND_RANGE);
    }
  }
  if (a.swa_rows && t < wch) {
    uint8_t *dst = a.swa_rows + ((size_t)b * a.W_cap + (p0 % a.W_cap)) * D;
    reinterpret_cast<uint16_t *>(dst)[c * wch + t] = (uint16_t)win_pair;
  }
  if (t < OPB && e < a.cap) {
    const size_t row = (size_t)b * a.cap + e;
    a.ik[row * dI + c * OPB + t] = (uint8_t)kcode;
    if (c == 0 && t == 0) a.ik_scale[row] = sk;
  }
  if (c == 0 && t == 0) a.n_entries[b] = p0 + 1;
}

// Indexer keys of entries already stored as FP4 (the projected append writes
// codes and scales first): one 512-thread block per group of up to 8 new
// entries of a sequence; the entries are dequantised exactly (E2M1 x E4M3)
// and projected by entry_keys, the same arithmetic as a token append.
__global__ void __launch_bounds__(512) append_keys_kernel(const AppendArgs a) {
  extern __shared__ float sm[];
  pdl_launch_dependents();
  pdl_wait();
  const int t = threadIdx.x, D = a.D, dI = a.dI;
  const int b = blockIdx.x / a.main_blocks_per_seq;
  const int j0 = (blockIdx.x % a.main_blocks_per_seq) * a.entries_per_block;
  const int p0 = a.pos0[b];
  if (p0 < 0) return;   // flagged by the projection kernel
  int count = a.T - j0;
  if (count > a.entries_per_block) count = a.entries_per_block;
  if (count <= 0) return;
  float *xh = sm;
  float *kbuf = xh + a.entries_per_block * D;
  uint16_t *ws = reinterpret_cast<uint16_t *>(kbuf + a.entries_per_block * dI + 32);
  {
    const uint4 *src = reinterpret_cast<const uint4 *>(a.w_ik);
    uint4 *dst = reinterpret_cast<uint4 *>(ws);
    for (int i = t; i < D * dI / 8; i += blockDim.x) dst[i] = src[i];
  }
  for (int i = t; i < count * D; i += blockDim.x) {
    const int jj = i / D, c = i % D, e = p0 + j0 + jj;
    float v = 0.0f;
    if (e < a.cap) {
      const size_t row = (size_t)b * a.cap + e;
      const uint32_t code = (a.codes[row * (D / 2) + c / 2] >> ((c & 1) * 4)) & 0xFu;
      v = __fmul_rn(e2m1_to_f32(code), e4m3_to_f32(a.scales[row * (D / 16) + c / 16]));
    }
    xh[jj * D + c] = v;
  }
  __syncthreads();
  entry_keys(a, b, p0 + j0, count, xh, kbuf, ws);
}

cudaError_t launch_append_keys(const AppendArgs &a, cudaStream_t s) {
  const int blocks = a.B * a.main_blocks_per_seq;
  if (blocks == 0) return cudaSuccess;
  const size_t smem = sizeof(float) * ((size_t)a.entries_per_block * (a.D + a.dI) + 32) +
                      sizeof(uint16_t) * (size_t)a.D * a.dI;
  cudaError_t e = cudaFuncSetAttribute(append_keys_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(append_keys_kernel, dim3(blocks), dim3(512), smem, s, dim3(1, 1, 1), a);
}

cudaError_t launch_append(const AppendArgs &a, cudaStream_t s) {
  if (a.codes && a.m == 1 && a.T == 1 && a.D <= 512 && a.dI % (8 * kDecCl) == 0 && a.dI / kDecCl <= 16 &&
      (!a.swa_rows || a.W_cap >= 1))
    return launch_pdl(append_decode_kernel, dim3(kDecCl, a.B + a.prep.rows), dim3(256), 0, s, dim3(1, 1, 1), a);
  const int blocks = a.B * (a.main_blocks_per_seq + a.swa_blocks_per_seq) + 8 * a.prep.rows;
  if (blocks == 0) return cudaSuccess;
  const int threads = 512;   // quantisation uses the first D/2, the projection all of them
  // [E][D] + [E][dI] floats, 32 floats, then W_ik [D][dI] bf16
  const size_t smem = a.codes ? sizeof(float) * ((size_t)a.entries_per_block * (a.D + a.dI) + 32) +
                                    sizeof(uint16_t) * (size_t)a.D * a.dI
                              : 0;
  cudaError_t e = cudaFuncSetAttribute(append_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(append_kernel, dim3(blocks), dim3(threads), smem, s, dim3(1, 1, 1), a);
}

}  // namespace csa2
