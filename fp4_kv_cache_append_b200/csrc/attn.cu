// Sparse MQA attention over the selected FP4 entries and the FP8 window.
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2": global sparse
//   retrieval plus the 128-token local window in one attention; section
//   "3) FP4 main KV + SWA Bounded Replay": FP4 (E2M1 + E4M3/16ch) main KV,
//   FP8 window KV.  All query heads share one KV (K = V).
// One block per (query row, key split), 16 warps.  Keys are processed in
// chunks of 64: the chunk's rows are gathered (FP4 codes + scales, or E4M3
// window rows) and dequantised exactly into fp16 in shared memory, then
//   S = Q K^T   (warp: 16 heads x 16 keys, k = D)   and
//   O += P V    (warp: 16 heads x D/4 channels, k = 64 keys)
// run on fp16 tensor-core MMAs with fp32 accumulation; the softmax is online
// (running max / sum per head, base-2 exponent).  E2M1 x E4M3 and E4M3 are
// exact in fp16, so the only roundings before accumulation are q -> fp16 and
// P -> fp16.  Window rows keep their raw E4M3 values; the layer's window scale
// multiplies their logits and their P entries instead.
// With several splits per row, each split writes (m, l, O) partials and
// attn_combine_kernel merges them.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kThreads = 512;
constexpr int kChunk = 64;
constexpr int kHeads = 64;        // heads padded to 64 (4 warp rows of 16)
constexpr float kLog2e = 1.4426950408889634f;

// fp16 bits of the 16 E2M1 codes (0, .5, 1, 1.5, 2, 3, 4, 6 and negatives).
__constant__ uint16_t kE2m1Half[16] = {0x0000, 0x3800, 0x3C00, 0x3E00, 0x4000, 0x4200, 0x4400, 0x4600,
                                       0x8000, 0xB800, 0xBC00, 0xBE00, 0xC000, 0xC200, 0xC400, 0xC600};

// E4M3 byte -> fp16 bits (exact): normal e>0 maps to fp16 exponent e+8,
// subnormal m*2^-9 is an fp16 normal.
__device__ __forceinline__ uint32_t e4m3_to_half_bits(uint32_t b) {
  const uint32_t s = (b & 0x80u) << 8, e = (b >> 3) & 15u, m = b & 7u;
  if (e) return s | ((e + 8u) << 10) | (m << 7);
  if (m == 0) return s;
  // m * 2^-9 = 2^(p-9) * (m / 2^p) with p = floor(log2 m)
  const uint32_t p = 31u - __clz(m);
  return s | ((p - 9u + 15u) << 10) | (((m << (3u - p)) & 7u) << 7);
}

// Byte offset of (row, 16-byte chunk c) in a row-major fp16 tile whose rows
// are `row_bytes` long, with the chunk index XOR-swizzled by row (ldmatrix is
// then free of bank conflicts).
__device__ __forceinline__ uint32_t tile_off(int row, int c, int row_bytes) {
  return row * row_bytes + ((c ^ (row & 7)) << 4);
}

template <int D>
struct AttnSmem {
  alignas(128) uint16_t q[kHeads * D];
  alignas(128) uint16_t k[kChunk * D];
  alignas(128) uint16_t p[kHeads * kChunk];
  uint32_t lut[256];          // code byte -> packed fp16 pair (low nibble first)
  int key_ent[kChunk];        // entry id or window slot, -1 = masked
  float red_max[4][kHeads];
  float red_sum[4][kHeads];
  float m_run[kHeads], l_run[kHeads], alpha[kHeads];
};

}  // namespace

template <int D>
__global__ void __launch_bounds__(kThreads, 1) attn_kernel(const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  AttnSmem<D> &S = *reinterpret_cast<AttnSmem<D> *>((reinterpret_cast<uintptr_t>(smem_raw) + 127) & ~uintptr_t(127));
  constexpr int RB = D * 2;          // row bytes of an fp16 tile
  constexpr int NCH = D / 8;         // 16-byte chunks per row
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int gid = lane >> 2, tq = lane & 3;
  const int row = blockIdx.x;        // b * T_q + query
  const int split = blockIdx.y;
  const int b = row / a.T_q;
  const int t = a.q_pos[row];

  // ---- per-row key bookkeeping
  const int n_fp4_chunks = (a.K + kChunk - 1) / kChunk;
  int wlo = t - a.window + 1;
  if (wlo < 0) wlo = 0;
  const int nwin = (t >= 0 && a.window > 0) ? t - wlo + 1 : 0;
  const int n_win_chunks = (nwin + kChunk - 1) / kChunk;
  const int total_chunks = n_fp4_chunks + n_win_chunks;
  const int c_begin = split * a.chunks_per_split;
  int c_end = c_begin + a.chunks_per_split;
  if (c_end > total_chunks) c_end = total_chunks;

  // ---- setup: LUT, Q (bf16 -> fp16), running stats
  for (int i = tid; i < 256; i += kThreads)
    S.lut[i] = (uint32_t)kE2m1Half[i & 15] | ((uint32_t)kE2m1Half[i >> 4] << 16);
  if (tid < kHeads) { S.m_run[tid] = -INFINITY; S.l_run[tid] = 0.f; }
  const uint16_t *qrow = a.q + (size_t)row * a.H * D;
  for (int i = tid; i < kHeads * NCH; i += kThreads) {
    const int h = i / NCH, c = i % NCH;
    uint4 v = make_uint4(0, 0, 0, 0);
    if (h < a.H) {
      const uint4 raw = *reinterpret_cast<const uint4 *>(qrow + (size_t)h * D + c * 8);
      const uint32_t w[4] = {raw.x, raw.y, raw.z, raw.w};
      uint32_t o[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const __half2 hv = __floats2half2_rn(bf16_to_f32(w[j] & 0xFFFFu), bf16_to_f32(w[j] >> 16));
        o[j] = *reinterpret_cast<const uint32_t *>(&hv);
      }
      v = make_uint4(o[0], o[1], o[2], o[3]);
    }
    *reinterpret_cast<uint4 *>(reinterpret_cast<uint8_t *>(S.q) + tile_off(h, c, RB)) = v;
  }

  // MMA roles
  const int hg = warp & 3;            // head group: heads 16hg..16hg+15
  const int kg = warp >> 2;           // S: keys 16kg..16kg+15 of the chunk
  const int cg = warp >> 2;           // O: channels cg*D/4 ..
  constexpr int ONT = D / 4 / 8;      // O n-tiles per warp
  float o[ONT][4];
#pragma unroll
  for (int n = 0; n < ONT; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.f;

  const uint32_t q_base = smem_u32(S.q), k_base = smem_u32(S.k), p_base = smem_u32(S.p);

  for (int c = c_begin; c < c_end; ++c) {
    const bool is_win = c >= n_fp4_chunks;
    __syncthreads();   // previous chunk fully consumed (and setup visible)
    // ---- key ids of this chunk
    if (tid < kChunk) {
      int id = -1;
      if (!is_win) {
        const int k = c * kChunk + tid;
        if (k < a.K) {
          const int e = a.idx[(size_t)row * a.K + k];
          if (e >= a.cap) flag(a.status, CSA2_DEV_INDEX_RANGE);
          id = (e >= 0 && e < a.cap) ? e : -1;
        }
      } else {
        const int j = (c - n_fp4_chunks) * kChunk + tid;
        id = j < nwin ? (wlo + j) % a.W_cap : -1;
      }
      S.key_ent[tid] = id;
    }
    __syncthreads();
    // ---- gather + dequantise 64 rows into S.k (fp16, swizzled)
    // piece = 16 channels of one row (FP4: 8 code bytes + 1 scale; FP8: 16 bytes)
    for (int i = tid; i < kChunk * (D / 16); i += kThreads) {
      const int r = i / (D / 16), pc = i % (D / 16);
      const int id = S.key_ent[r];
      uint32_t out[8] = {0, 0, 0, 0, 0, 0, 0, 0};
      if (id >= 0) {
        if (!is_win) {
          const size_t er = (size_t)b * a.cap + id;
          const uint2 cb = *reinterpret_cast<const uint2 *>(a.codes + er * (D / 2) + pc * 8);
          const uint32_t sb = a.scales[er * (D / 16) + pc];
          const uint32_t sh = e4m3_to_half_bits(sb);
          const __half2 s2 = __halves2half2(__ushort_as_half((unsigned short)sh), __ushort_as_half((unsigned short)sh));
          const uint32_t bytes[2] = {cb.x, cb.y};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t byte = (bytes[j >> 2] >> (8 * (j & 3))) & 0xFFu;
            const uint32_t pr = S.lut[byte];
            const __half2 v = __hmul2(*reinterpret_cast<const __half2 *>(&pr), s2);
            out[j] = *reinterpret_cast<const uint32_t *>(&v);
          }
        } else {
          const uint4 rb = *reinterpret_cast<const uint4 *>(a.swa_rows + ((size_t)b * a.W_cap + id) * D + pc * 16);
          const uint32_t w[4] = {rb.x, rb.y, rb.z, rb.w};
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            const uint32_t b0 = (w[j >> 1] >> (16 * (j & 1))) & 0xFFu;
            const uint32_t b1 = (w[j >> 1] >> (16 * (j & 1) + 8)) & 0xFFu;
            out[j] = e4m3_to_half_bits(b0) | (e4m3_to_half_bits(b1) << 16);
          }
        }
      }
      uint8_t *dst = reinterpret_cast<uint8_t *>(S.k);
      *reinterpret_cast<uint4 *>(dst + tile_off(r, 2 * pc, RB)) = make_uint4(out[0], out[1], out[2], out[3]);
      *reinterpret_cast<uint4 *>(dst + tile_off(r, 2 * pc + 1, RB)) = make_uint4(out[4], out[5], out[6], out[7]);
    }
    __syncthreads();

    // ---- S = Q K^T: warp -> heads 16hg.., keys 16kg..
    float s[2][4] = {{0, 0, 0, 0}, {0, 0, 0, 0}};
#pragma unroll 4
    for (int ks = 0; ks < D / 16; ++ks) {
      uint32_t af[4], bfr[4];
      {
        const int r = 16 * hg + (lane & 15);
        const int ch = 2 * ks + (lane >> 4);
        ldsm_x4(q_base + tile_off(r, ch, RB), af[0], af[1], af[2], af[3]);
      }
      {
        const int r = 16 * kg + (lane & 7) + ((lane >> 4) << 3);
        const int ch = 2 * ks + ((lane >> 3) & 1);
        ldsm_x4(k_base + tile_off(r, ch, RB), bfr[0], bfr[1], bfr[2], bfr[3]);
      }
      mma_f16_16816(s[0], af, bfr);
      mma_f16_16816(s[1], af, bfr + 2);
    }
    // ---- online softmax (base 2)
    const float lsc = a.scale * (is_win ? a.s_swa : 1.0f) * kLog2e;
    const float psc = is_win ? a.s_swa : 1.0f;
    const int hl = 16 * hg + gid, hh = hl + 8;
    float mx_l = -INFINITY, mx_h = -INFINITY;
#pragma unroll
    for (int n = 0; n < 2; ++n) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const int key = 16 * kg + 8 * n + 2 * tq + j;
        const bool valid = S.key_ent[key] >= 0;
        s[n][j] = valid ? s[n][j] * lsc : -INFINITY;
        s[n][2 + j] = valid ? s[n][2 + j] * lsc : -INFINITY;
        mx_l = fmaxf(mx_l, s[n][j]);
        mx_h = fmaxf(mx_h, s[n][2 + j]);
      }
    }
    mx_l = fmaxf(mx_l, __shfl_xor_sync(0xffffffffu, mx_l, 1));
    mx_l = fmaxf(mx_l, __shfl_xor_sync(0xffffffffu, mx_l, 2));
    mx_h = fmaxf(mx_h, __shfl_xor_sync(0xffffffffu, mx_h, 1));
    mx_h = fmaxf(mx_h, __shfl_xor_sync(0xffffffffu, mx_h, 2));
    if (tq == 0) { S.red_max[kg][hl] = mx_l; S.red_max[kg][hh] = mx_h; }
    __syncthreads();
    float m_new_l = S.m_run[hl], m_new_h = S.m_run[hh];
#pragma unroll
    for (int g = 0; g < 4; ++g) { m_new_l = fmaxf(m_new_l, S.red_max[g][hl]); m_new_h = fmaxf(m_new_h, S.red_max[g][hh]); }
    float sum_l = 0.f, sum_h = 0.f;
#pragma unroll
    for (int n = 0; n < 2; ++n) {
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float pl = m_new_l == -INFINITY ? 0.f : exp2f(s[n][j] - m_new_l);
        const float ph = m_new_h == -INFINITY ? 0.f : exp2f(s[n][2 + j] - m_new_h);
        s[n][j] = pl;
        s[n][2 + j] = ph;
        sum_l += pl;
        sum_h += ph;
      }
      // P (fp16, scaled for window rows) -> smem [head][key]
      const int key = 16 * kg + 8 * n + 2 * tq;
      const __half2 vl = __floats2half2_rn(s[n][0] * psc, s[n][1] * psc);
      const __half2 vh = __floats2half2_rn(s[n][2] * psc, s[n][3] * psc);
      uint8_t *pb = reinterpret_cast<uint8_t *>(S.p);
      *reinterpret_cast<__half2 *>(pb + tile_off(hl, key >> 3, kChunk * 2) + (key & 7) * 2) = vl;
      *reinterpret_cast<__half2 *>(pb + tile_off(hh, key >> 3, kChunk * 2) + (key & 7) * 2) = vh;
    }
    sum_l += __shfl_xor_sync(0xffffffffu, sum_l, 1);
    sum_l += __shfl_xor_sync(0xffffffffu, sum_l, 2);
    sum_h += __shfl_xor_sync(0xffffffffu, sum_h, 1);
    sum_h += __shfl_xor_sync(0xffffffffu, sum_h, 2);
    if (tq == 0) { S.red_sum[kg][hl] = sum_l; S.red_sum[kg][hh] = sum_h; }
    __syncthreads();
    if (tid < kHeads) {
      const float m_old = S.m_run[tid];
      float m_new = m_old;
#pragma unroll
      for (int g = 0; g < 4; ++g) m_new = fmaxf(m_new, S.red_max[g][tid]);
      const float al = (m_new == -INFINITY) ? 1.f : exp2f(m_old - m_new);
      float l = S.l_run[tid] * al;
#pragma unroll
      for (int g = 0; g < 4; ++g) l += S.red_sum[g][tid];
      S.alpha[tid] = al;
      S.m_run[tid] = m_new;
      S.l_run[tid] = l;
    }
    __syncthreads();
    // ---- O = alpha O + P V: warp -> heads 16hg.., channels cg*D/4..
    {
      const float al = S.alpha[16 * hg + gid], ah = S.alpha[16 * hg + gid + 8];
#pragma unroll
      for (int n = 0; n < ONT; ++n) { o[n][0] *= al; o[n][1] *= al; o[n][2] *= ah; o[n][3] *= ah; }
#pragma unroll
      for (int ks = 0; ks < kChunk / 16; ++ks) {
        uint32_t af[4];
        {
          const int r = 16 * hg + (lane & 15);
          const int ch = 2 * ks + (lane >> 4);
          ldsm_x4(p_base + tile_off(r, ch, kChunk * 2), af[0], af[1], af[2], af[3]);
        }
#pragma unroll
        for (int n = 0; n < ONT; n += 2) {
          uint32_t bfr[4];
          const int r = 16 * ks + (lane & 7) + (((lane >> 3) & 1) << 3);
          const int ch = (cg * (D / 4)) / 8 + n + (lane >> 4);
          ldsm_x4_t(k_base + tile_off(r, ch, RB), bfr[0], bfr[1], bfr[2], bfr[3]);
          mma_f16_16816(o[n], af, bfr);
          mma_f16_16816(o[n + 1], af, bfr + 2);
        }
      }
    }
  }
  __syncthreads();

  // ---- epilogue
  const int hl = 16 * hg + gid, hh = hl + 8;
  if (a.nsplit == 1) {
    const float ll = S.l_run[hl], lh = S.l_run[hh];
    const float il = ll > 0.f ? 1.f / ll : 0.f, ih = lh > 0.f ? 1.f / lh : 0.f;
    uint16_t *orow = a.out + (size_t)row * a.H * D;
#pragma unroll
    for (int n = 0; n < ONT; ++n) {
      const int ch = cg * (D / 4) + n * 8 + 2 * tq;
      if (hl < a.H) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(o[n][0] * il, o[n][1] * il);
        *reinterpret_cast<__nv_bfloat162 *>(orow + (size_t)hl * D + ch) = v;
      }
      if (hh < a.H) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(o[n][2] * ih, o[n][3] * ih);
        *reinterpret_cast<__nv_bfloat162 *>(orow + (size_t)hh * D + ch) = v;
      }
    }
  } else {
    // partials: O [rows][nsplit][64][D], then m, l [rows][nsplit][64]
    const size_t nrows = (size_t)a.B * a.T_q;
    float *po = a.ws + ((size_t)row * a.nsplit + split) * kHeads * D;
    float *pm = a.ws + nrows * a.nsplit * kHeads * D + ((size_t)row * a.nsplit + split) * kHeads;
    float *pl = pm + nrows * a.nsplit * kHeads;
#pragma unroll
    for (int n = 0; n < ONT; ++n) {
      const int ch = cg * (D / 4) + n * 8 + 2 * tq;
      *reinterpret_cast<float2 *>(po + (size_t)hl * D + ch) = make_float2(o[n][0], o[n][1]);
      *reinterpret_cast<float2 *>(po + (size_t)hh * D + ch) = make_float2(o[n][2], o[n][3]);
    }
    if (tid < kHeads) { pm[tid] = S.m_run[tid]; pl[tid] = S.l_run[tid]; }
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
  const int nc = (K + kChunk - 1) / kChunk + (window + kChunk - 1) / kChunk;
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
  const size_t smem = sizeof(AttnSmem<D>) + 128;
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
