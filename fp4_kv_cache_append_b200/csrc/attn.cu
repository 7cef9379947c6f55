// Sparse MQA attention over the selected FP4 entries and the FP8 window.
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2": global sparse
//   retrieval plus the 128-token local window in one attention; section
//   "3) FP4 main KV + SWA Bounded Replay": FP4 (E2M1 + E4M3/16ch) main KV,
//   FP8 window KV.  All query heads share one KV (K = V).
//
// One block per (query row, key split); keys in tiles of 128 (the selected
// entries first, then the window rows).  Per tile:
//   1. all 8 warps gather the tile's rows (FP4 codes + scales, or E4M3 rows)
//      and dequantise them exactly into fp16 in shared memory, laid out as a
//      K-major 128B-swizzled operand (E2M1 x E4M3 and E4M3 are exact in fp16);
//   2. S^T = K^ Q^T on tcgen05 (kind::f16, M = 128 keys, N = 64 heads,
//      K = D): TMEM lane = key, column = head;
//   3. warps 0-3 (one TMEM lane quarter each) read S^T, reduce the per-head
//      maximum and sum across the 128 lanes with a reduce-scatter butterfly,
//      exponentiate (base 2) and write P^T (fp16) as the next B operand;
//   4. O^T += V^T P^T on tcgen05 (M = 128 channels per TMEM block, N = 64
//      heads, K = 128 keys).  V^T is the same shared-memory tile as K^, read
//      as an MN-major operand, so the tile is dequantised once.
// The softmax reference max of a head moves only when a tile raises it by more
// than 2^8 (then O^T and the running sum are rescaled in place), so P stays
// within fp16 range and rescaling is rare.  Window rows keep their raw E4M3
// values; the layer's window scale multiplies their logits and their P.
// With several splits per row each writes (m, l, O) partials that
// attn_combine_kernel merges.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kThreads = 256;
constexpr int kTile = 128;         // keys per tile (M of S^T)
constexpr int kHeads = 64;         // heads padded to 64 (N)
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLazy = 8.0f;      // log2 headroom before the reference max moves
constexpr uint32_t kWaitLimit = 1u << 22;

// fp16 bits of the 16 E2M1 codes (0, .5, 1, 1.5, 2, 3, 4, 6 and negatives).
__constant__ uint16_t kE2m1Half[16] = {0x0000, 0x3800, 0x3C00, 0x3E00, 0x4000, 0x4200, 0x4400, 0x4600,
                                       0x8000, 0xB800, 0xBC00, 0xBE00, 0xC000, 0xC200, 0xC400, 0xC600};

// E4M3 byte -> fp16 bits (exact): normal e>0 maps to fp16 exponent e+8,
// subnormal m*2^-9 is an fp16 normal.
__device__ __forceinline__ uint32_t e4m3_to_half_bits(uint32_t b) {
  const uint32_t s = (b & 0x80u) << 8, e = (b >> 3) & 15u, m = b & 7u;
  if (e) return s | ((e + 8u) << 10) | (m << 7);
  if (m == 0) return s;
  const uint32_t p = 31u - __clz(m);   // m * 2^-9 = 2^(p-9) * (m / 2^p)
  return s | ((p - 9u + 15u) << 10) | (((m << (3u - p)) & 7u) << 7);
}

template <int D>
struct AttnSmem {
  alignas(1024) uint8_t kh[(D / 64) * kTile * 128];   // K^ tile: D/64 chunks of [128 keys x 128 B]
  alignas(1024) uint8_t q[(D / 64) * kHeads * 128];   // Q: D/64 chunks of [64 heads x 128 B]
  alignas(1024) uint8_t p[2 * kHeads * 128];          // P^T: 2 chunks of [64 heads x 128 B]
  uint32_t lut[256];                                  // code byte -> fp16 pair (low nibble first)
  int key_ent[kTile];                                 // entry id or window slot, -1 = masked
  float red[4][kHeads];
  float m_ref[kHeads], l_run[kHeads], alpha[kHeads];
  uint64_t sbar, obar;
  uint32_t tmem_base;
  int rescale;
};

// Byte offset of 16-byte piece `pc` (8 fp16 elements) of row `r` in a
// K-major 128B-swizzled operand whose chunks of 64 elements hold `rows` rows.
__device__ __forceinline__ uint32_t sw_off(int r, int pc, int rows) {
  return (uint32_t)((pc >> 3) * rows * 128 + r * 128 + (((pc & 7) ^ (r & 7)) << 4));
}

// Reduce-scatter of 64 values across the 32 lanes of a warp: afterwards
// t[0], t[1] hold the reduction over the warp of columns c, c+1 with
// c = the lane's column base (returned).
template <bool MAX>
__device__ __forceinline__ int reduce_scatter64(float *t, int lane) {
  int base = 0;
#pragma unroll
  for (int o = 16, n = 32; o >= 1; o >>= 1, n >>= 1) {
    const bool up = (lane & o) != 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      if (j < n) {
        const float lo = t[j], hi = t[j + n];
        const float send = up ? lo : hi, keep = up ? hi : lo;
        const float recv = __shfl_xor_sync(0xffffffffu, send, o);
        t[j] = MAX ? fmaxf(keep, recv) : keep + recv;
      }
    }
    if (up) base += n;
  }
  return base;
}

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const AttnArgs a) {
  constexpr int NCH = D / 64;                      // 64-channel chunks
  constexpr int MT = D / 128;                      // O^T TMEM blocks of 128 channels
  constexpr uint32_t kCols = D == 128 ? 128u : (D == 256 ? 256u : 512u);
  constexpr uint32_t kIdS = mma_idesc(128, kHeads, 0u /*f16*/, 0u /*f16*/);
  constexpr uint32_t kIdO = kIdS | (1u << 15);     // A (V^T) MN-major
  extern __shared__ uint8_t smem_raw[];
  AttnSmem<D> &S = *reinterpret_cast<AttnSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                                   ~uintptr_t(1023));
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int row = blockIdx.x;   // b * T_q + query
  const int split = blockIdx.y;
  const int b = row / a.T_q;
  const int t = a.q_pos[row];

  // ---- keys of this split
  const int n_fp4_tiles = (a.K + kTile - 1) / kTile;
  int wlo = t - a.window + 1;
  if (wlo < 0) wlo = 0;
  const int nwin = (t >= 0 && a.window > 0) ? t - wlo + 1 : 0;
  const int total = n_fp4_tiles + (nwin + kTile - 1) / kTile;
  const int c_begin = split * a.chunks_per_split;
  int c_end = c_begin + a.chunks_per_split;
  if (c_end > total) c_end = total;

  // ---- set-up
  if (tid == 0) {
    mbar_init(&S.sbar, 1);
    mbar_init(&S.obar, 1);
    S.rescale = 0;
    fence_barrier_init();
  }
  if (warp == 4) {
    tmem_alloc(&S.tmem_base, kCols);
    tmem_relinquish();
  }
  for (int i = tid; i < 256; i += kThreads)
    S.lut[i] = (uint32_t)kE2m1Half[i & 15] | ((uint32_t)kE2m1Half[i >> 4] << 16);
  if (tid < kHeads) { S.m_ref[tid] = -INFINITY; S.l_run[tid] = 0.f; S.alpha[tid] = 1.f; }
  // Q: bf16 -> fp16 into the B-operand layout (heads >= H are zero), in
  // batches of 4 items whose loads are all issued before they are used
  {
    constexpr int QI = kHeads * (D / 8) / kThreads;   // 16-byte items per thread
    const uint16_t *qrow = a.q + (size_t)row * a.H * D;
#pragma unroll 1
    for (int j0 = 0; j0 < QI; j0 += 4) {
      uint4 raw[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = tid + (j0 + u) * kThreads;
        const int h = i / (D / 8), pc = i % (D / 8);
        raw[u] = h < a.H ? *reinterpret_cast<const uint4 *>(qrow + (size_t)h * D + pc * 8) : make_uint4(0, 0, 0, 0);
      }
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int i = tid + (j0 + u) * kThreads;
        const int h = i / (D / 8), pc = i % (D / 8);
        const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
        uint32_t o[4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const __half2 hv = __floats2half2_rn(bf16_to_f32(w[k] & 0xFFFFu), bf16_to_f32(w[k] >> 16));
          o[k] = *reinterpret_cast<const uint32_t *>(&hv);
        }
        *reinterpret_cast<uint4 *>(S.q + sw_off(h, pc, kHeads)) = make_uint4(o[0], o[1], o[2], o[3]);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = S.tmem_base;
  const uint32_t kh_base = smem_u32(S.kh), q_base = smem_u32(S.q), p_base = smem_u32(S.p);

  bool aborted = false;
  int n_done = 0;   // tiles whose O^T MMAs were issued
  for (int c = c_begin; c < c_end && !aborted; ++c) {
    const bool is_win = c >= n_fp4_tiles;
    // ---- key ids
    if (tid < kTile) {
      int id = -1;
      if (!is_win) {
        const int k = c * kTile + tid;
        if (k < a.K) {
          const int e = a.idx[(size_t)row * a.K + k];
          if (e >= a.cap) flag(a.status, CSA2_DEV_INDEX_RANGE);
          id = (e >= 0 && e < a.cap) ? e : -1;
        }
      } else {
        const int j = (c - n_fp4_tiles) * kTile + tid;
        id = j < nwin ? (wlo + j) % a.W_cap : -1;
      }
      S.key_ent[tid] = id;
    }
    // the previous tile's O^T MMAs read K^ and P^T: wait before overwriting
    bool ok = true;
    if (n_done > 0) ok = mbar_wait_bounded(&S.obar, (n_done - 1) & 1, kWaitLimit);
    if (__syncthreads_or(!ok)) { aborted = true; break; }

    // ---- 1. gather + dequantise: item = 16 channels of one row -> 2 pieces,
    // in batches of 4 items whose loads are issued before they are decoded
    {
      constexpr int GI = kTile * (D / 16) / kThreads;   // items per thread
#pragma unroll 1
      for (int j0 = 0; j0 < GI; j0 += 4) {
        uint4 raw[4];   // FP4: codes in .x/.y, scale byte in .z; window: 16 E4M3 bytes
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = tid + (j0 + u) * kThreads;
          const int r = i / (D / 16), g = i % (D / 16);
          const int id = S.key_ent[r];
          raw[u] = make_uint4(0, 0, 0, 0);
          if (id >= 0) {
            if (!is_win) {
              const size_t er = (size_t)b * a.cap + id;
              const uint2 cb = *reinterpret_cast<const uint2 *>(a.codes + er * (D / 2) + g * 8);
              raw[u] = make_uint4(cb.x, cb.y, a.scales[er * (D / 16) + g], 0);
            } else {
              raw[u] = *reinterpret_cast<const uint4 *>(a.swa_rows + ((size_t)b * a.W_cap + id) * D + g * 16);
            }
          }
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = tid + (j0 + u) * kThreads;
          const int r = i / (D / 16), g = i % (D / 16);
          uint32_t out[8];
          if (!is_win) {
            const uint32_t sh = e4m3_to_half_bits(raw[u].z);
            const __half2 s2 = __halves2half2(__ushort_as_half((unsigned short)sh), __ushort_as_half((unsigned short)sh));
            const uint32_t bytes[2] = {raw[u].x, raw[u].y};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t pr = S.lut[(bytes[k >> 2] >> (8 * (k & 3))) & 0xFFu];
              const __half2 v = __hmul2(*reinterpret_cast<const __half2 *>(&pr), s2);
              out[k] = *reinterpret_cast<const uint32_t *>(&v);
            }
          } else {
            const uint32_t w[4] = {raw[u].x, raw[u].y, raw[u].z, raw[u].w};
#pragma unroll
            for (int k = 0; k < 8; ++k) {
              const uint32_t b0 = (w[k >> 1] >> (16 * (k & 1))) & 0xFFu;
              const uint32_t b1 = (w[k >> 1] >> (16 * (k & 1) + 8)) & 0xFFu;
              out[k] = e4m3_to_half_bits(b0) | (e4m3_to_half_bits(b1) << 16);
            }
          }
          *reinterpret_cast<uint4 *>(S.kh + sw_off(r, 2 * g, kTile)) = make_uint4(out[0], out[1], out[2], out[3]);
          *reinterpret_cast<uint4 *>(S.kh + sw_off(r, 2 * g + 1, kTile)) = make_uint4(out[4], out[5], out[6], out[7]);
        }
      }
    }
    fence_proxy_async();
    tc_fence_before();
    __syncthreads();

    // ---- 2. S^T = K^ Q^T
    if (tid == 128) {
      tc_fence_after();
#pragma unroll 1
      for (int ks = 0; ks < D / 16; ++ks) {
        const uint32_t off = (uint32_t)((ks >> 2) * 0 + (ks & 3) * 32);
        const uint32_t a_addr = kh_base + (ks >> 2) * (kTile * 128) + off;
        const uint32_t b_addr = q_base + (ks >> 2) * (kHeads * 128) + off;
        tc_mma_f16(tmem, smem_desc_kmajor(a_addr, 128), smem_desc_kmajor(b_addr, 128), kIdS, ks > 0 ? 1u : 0u);
      }
      tc_commit(&S.sbar);
    }
    ok = mbar_wait_bounded(&S.sbar, (c - c_begin) & 1, kWaitLimit);
    if (__syncthreads_or(!ok)) { aborted = true; break; }
    tc_fence_after();

    // ---- 3. softmax (warps 0-3: TMEM lane = key)
    const float lsc = a.scale * (is_win ? a.s_swa : 1.0f) * kLog2e;
    const float psc = is_win ? a.s_swa : 1.0f;
    const bool first = (c == c_begin);
    if (warp < 4) {
      const int r = 32 * warp + lane;
      float sv[kHeads], tt[kHeads];
      {
        uint32_t raw[kHeads];
        tmem_ld_x32(tmem + ((uint32_t)(32 * warp) << 16), raw);
        tmem_ld_x32(tmem + ((uint32_t)(32 * warp) << 16) + 32, raw + 32);
        tmem_wait_ld();
        const bool valid = S.key_ent[r] >= 0;
#pragma unroll
        for (int h = 0; h < kHeads; ++h) {
          sv[h] = valid ? __uint_as_float(raw[h]) * lsc : -INFINITY;
          tt[h] = sv[h];
        }
      }
      // per-head max over the warp's 32 keys: integer max of order-preserving bits
#pragma unroll
      for (int h = 0; h < kHeads; ++h) {
        const int bits = __float_as_int(tt[h]);
        const int key = bits >= 0 ? bits : (bits ^ 0x7FFFFFFF);
        const int mk = __reduce_max_sync(0xffffffffu, key);
        if (lane == (h & 31)) S.red[warp][h] = __int_as_float(mk >= 0 ? mk : (mk ^ 0x7FFFFFFF));
      }
      named_bar(1, 128);
      int cb;
      if (tid < kHeads) {   // new reference max of head tid
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
      named_bar(1, 128);
      // P = 2^(s - m_ref), written as P^T[head][key] (fp16, window rows scaled)
#pragma unroll
      for (int h = 0; h < kHeads; ++h) {
        const float m = S.m_ref[h];
        const float pv = (sv[h] == -INFINITY || m == -INFINITY) ? 0.f : exp2f(sv[h] - m);
        tt[h] = pv;
        const __half hp = __float2half_rn(pv * psc);
        *reinterpret_cast<__half *>(S.p + sw_off(h, r >> 3, kHeads) + (r & 7) * 2) = hp;
      }
      cb = reduce_scatter64<false>(tt, lane);
      S.red[warp][cb] = tt[0];
      S.red[warp][cb + 1] = tt[1];
      named_bar(1, 128);
      if (tid < kHeads) S.l_run[tid] += (S.red[0][tid] + S.red[1][tid]) + (S.red[2][tid] + S.red[3][tid]);
      named_bar(1, 128);
      // rare: a head's reference max moved -> rescale its O^T column
      if (S.rescale) {
#pragma unroll 1
        for (int mt = 0; mt < MT; ++mt) {
          const uint32_t taddr = tmem + ((uint32_t)(32 * warp) << 16) + kHeads + mt * kHeads;
          uint32_t o[kHeads];
          tmem_ld_x32(taddr, o);
          tmem_ld_x32(taddr + 32, o + 32);
          tmem_wait_ld();
#pragma unroll
          for (int h = 0; h < kHeads; ++h) o[h] = __float_as_uint(__uint_as_float(o[h]) * S.alpha[h]);
          tmem_st_x32(taddr, o);
          tmem_st_x32(taddr + 32, o + 32);
        }
        tmem_wait_st();
        named_bar(1, 128);
        if (tid == 0) S.rescale = 0;
      }
    }
    fence_proxy_async();   // P^T (generic stores) -> visible to the tensor core
    tc_fence_before();
    __syncthreads();

    // ---- 4. O^T += V^T P^T
    if (tid == 128) {
      tc_fence_after();
#pragma unroll 1
      for (int mt = 0; mt < MT; ++mt) {
#pragma unroll 1
        for (int ks = 0; ks < kTile / 16; ++ks) {
          const uint32_t a_addr = kh_base + (2 * mt) * (kTile * 128) + (2 * ks) * 1024;
          const uint32_t b_addr = p_base + (ks >> 2) * (kHeads * 128) + (ks & 3) * 32;
          tc_mma_f16(tmem + kHeads + mt * kHeads, smem_desc_mnmajor_sw128(a_addr, kTile * 128, 1024),
                     smem_desc_kmajor(b_addr, 128), kIdO, (ks > 0 || !first) ? 1u : 0u);
        }
      }
      tc_commit(&S.obar);
    }
    ++n_done;
  }

  // ---- epilogue: O^T (TMEM lane = channel within a 128-channel block)
  bool ok = !aborted;
  if (ok && n_done > 0) ok = mbar_wait_bounded(&S.obar, (n_done - 1) & 1, kWaitLimit);
  if (__syncthreads_or(!ok)) {
    if (tid == 0) flag(a.status, CSA2_DEV_TIMEOUT);
    if (tid == 128 && n_done > 0) {   // let every issued MMA finish before TMEM is freed
      mbar_init(&S.sbar, 1);
      fence_barrier_init();
      tc_commit(&S.sbar);
      mbar_wait_bounded(&S.sbar, 0, kWaitLimit);
    }
    __syncthreads();
  } else {
    tc_fence_after();
    if (warp < 4) {
      const size_t nrows = (size_t)a.B * a.T_q;
#pragma unroll 1
      for (int mt = 0; mt < MT; ++mt) {
        const int ch = mt * 128 + 32 * warp + lane;
        uint32_t o[kHeads];
        if (n_done > 0) {
          const uint32_t taddr = tmem + ((uint32_t)(32 * warp) << 16) + kHeads + mt * kHeads;
          tmem_ld_x32(taddr, o);
          tmem_ld_x32(taddr + 32, o + 32);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int h = 0; h < kHeads; ++h) o[h] = 0u;
        }
        if (a.nsplit == 1) {
          uint16_t *orow = a.out + (size_t)row * a.H * D;
#pragma unroll
          for (int h = 0; h < kHeads; ++h) {
            if (h < a.H) {
              const float l = S.l_run[h];
              const float v = l > 0.f ? __uint_as_float(o[h]) / l : 0.f;
              const __nv_bfloat16 bv = __float2bfloat16_rn(v);
              orow[(size_t)h * D + ch] = *reinterpret_cast<const uint16_t *>(&bv);
            }
          }
        } else {
          float *po = a.ws + ((size_t)row * a.nsplit + split) * kHeads * D;
#pragma unroll
          for (int h = 0; h < kHeads; ++h) po[(size_t)h * D + ch] = __uint_as_float(o[h]);
        }
      }
      if (a.nsplit > 1 && tid < kHeads) {
        float *pm = a.ws + nrows * a.nsplit * kHeads * D + ((size_t)row * a.nsplit + split) * kHeads;
        float *pl = pm + nrows * a.nsplit * kHeads;
        pm[tid] = S.m_ref[tid];
        pl[tid] = S.l_run[tid];
      }
    }
    tc_fence_before();
    __syncthreads();
  }
  if (warp == 4) {
    tc_fence_after();
    tmem_dealloc(tmem, kCols);
  }
}

// out = sum_s 2^(m_s - M) O_s / sum_s 2^(m_s - M) l_s, per (row, head).
template <int D>
__global__ void attn_combine_kernel(const AttnArgs a) {
  const int row = blockIdx.x, h = blockIdx.y;
  const size_t nrows = (size_t)a.B * a.T_q;
  const float *pm = a.ws + nrows * a.nsplit * kHeads * D + (size_t)row * a.nsplit * kHeads;
  const float *pl = pm + nrows * a.nsplit * kHeads;
  float M = -INFINITY;
  for (int s = 0; s < a.nsplit; ++s) M = fmaxf(M, pm[s * kHeads + h]);
  float L = 0.f;
  for (int s = 0; s < a.nsplit; ++s) {
    const float ms = pm[s * kHeads + h];
    if (ms != -INFINITY) L += exp2f(ms - M) * pl[s * kHeads + h];
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  for (int c = threadIdx.x * 4; c < D; c += blockDim.x * 4) {
    float4 acc = make_float4(0, 0, 0, 0);
    for (int s = 0; s < a.nsplit; ++s) {
      const float ms = pm[s * kHeads + h];
      if (ms == -INFINITY) continue;
      const float w = exp2f(ms - M);
      const float4 v = *reinterpret_cast<const float4 *>(a.ws + (((size_t)row * a.nsplit + s) * kHeads + h) * D + c);
      acc.x += w * v.x; acc.y += w * v.y; acc.z += w * v.z; acc.w += w * v.w;
    }
    uint16_t *dst = a.out + ((size_t)row * a.H + h) * D + c;
    const __nv_bfloat162 v0 = __floats2bfloat162_rn(acc.x * inv, acc.y * inv);
    const __nv_bfloat162 v1 = __floats2bfloat162_rn(acc.z * inv, acc.w * inv);
    uint2 pk;
    pk.x = *reinterpret_cast<const uint32_t *>(&v0);
    pk.y = *reinterpret_cast<const uint32_t *>(&v1);
    *reinterpret_cast<uint2 *>(dst) = pk;
  }
}

AttnPlan plan_attn(int B, int T_q, int H, int D, int K, int window, int sms) {
  (void)H;
  AttnPlan p;
  const int rows = B * T_q;
  const int nc = (K + kTile - 1) / kTile + (window + kTile - 1) / kTile;
  int nsplit = 1;
  if (rows < sms) {
    nsplit = (2 * sms + rows - 1) / rows;
    if (nsplit > nc) nsplit = nc;
  }
  const int cps = (nc + nsplit - 1) / nsplit;
  nsplit = (nc + cps - 1) / cps;
  p.nsplit = nsplit;
  p.chunks_per_split = cps;
  p.bytes = nsplit > 1 ? (size_t)rows * nsplit * kHeads * ((size_t)D + 2) * sizeof(float) : 0;
  return p;
}

template <int D>
static cudaError_t launch_attn_t(const AttnArgs &a, cudaStream_t s) {
  const size_t smem = sizeof(AttnSmem<D>) + 1024;
  cudaError_t e = cudaFuncSetAttribute(attn_kernel<D>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  attn_kernel<D><<<dim3(a.B * a.T_q, a.nsplit), kThreads, smem, s>>>(a);
  e = cudaGetLastError();
  if (e != cudaSuccess || a.nsplit == 1) return e;
  attn_combine_kernel<D><<<dim3(a.B * a.T_q, a.H), D / 4 < 128 ? D / 4 : 128, 0, s>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_attn(const AttnArgs &a, cudaStream_t s) {
  switch (a.D) {
    case 128: return launch_attn_t<128>(a, s);
    case 256: return launch_attn_t<256>(a, s);
    default: return launch_attn_t<512>(a, s);
  }
}

}  // namespace csa2
