// Top-K selection and the hierarchical candidate pool.
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2": each Full or
//   Reindex layer keeps the Top-512 entries; the first Full layer of the
//   decoder also builds the pool of <= 2,048 blocks x 8 positions that the
//   Reindex layers rescore (paper sec. 2.3.2, 4.2.1, Fig. 5).
// Order: score descending, ties -> smaller column; absent = non-finite.  The
// result lists the chosen columns in ascending order, -1 padded.
//
// Two launches, no cross-block waiting:
//  1. topk_chunk_kernel: one block per (row, chunk of columns) keeps the
//     chunk's best k1 columns (and best p1 blocks of 8) with a 4-pass 8-bit
//     radix select over order-preserving 32-bit keys held in shared memory,
//     then an order-preserving compaction (ballots) into the workspace.
//  2. topk_merge_kernel: one block per row repeats the select over the
//     concatenated candidates (already in column order) and writes the
//     result, mapping columns through the pool for Reindex rows.
// The global Top-K is inside the union of the chunks' Top-Ks because the
// (key, -column) order is total.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kT1 = 512;
constexpr int kT2 = 1024;
constexpr int kMergeSmemCands = 16384;

// Order-preserving key of a score: larger score -> larger key; -0 == +0;
// non-finite -> 0 (absent).
__device__ __forceinline__ uint32_t score_key(float f) {
  if (!isfinite(f)) return 0u;
  if (f == 0.0f) f = 0.0f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct SelState {
  uint32_t thr;     // keys > thr are taken; keys == thr are taken ...
  int take_eq;      // ... for the first take_eq of them in column order
  uint32_t prefix, mask;
  int krem;
  int nvalid;
  int found_bin;
  int warp_gt[32], warp_eq[32];
};

template <int NT>
__device__ int block_sum(int v, int *red) {
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  int s = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) s += red[w];
  return s;
}

// Threshold of the K largest keys among keys[0..n) (0 = absent).  Leaves the
// result in st->thr / st->take_eq.  All threads of the block must call.
// 8-bit digits starting at the highest bit where the present keys differ
// (the bits above are common to all of them), so no pass is spent on a
// digit every key shares.  Histogram updates take one atomic per warp when
// the warp's active keys share a digit (the common case in the first pass).
template <int NT>
__device__ void radix_select(const uint32_t *keys, int n, int K, uint32_t *hist, SelState *st, int *red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int cnt = 0;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for (int i = tid; i < n; i += NT) {
    const uint32_t k = keys[i];
    if (k) { ++cnt; kmin = min(kmin, k); kmax = max(kmax, k); }
  }
  cnt = __reduce_add_sync(0xffffffffu, (unsigned)cnt);
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  __syncthreads();
  if (lane == 0) { red[warp] = cnt; hist[warp] = kmin; hist[32 + warp] = kmax; }
  __syncthreads();
  int nvalid = 0;
  kmin = 0xFFFFFFFFu;
  kmax = 0u;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) { nvalid += red[w]; kmin = min(kmin, hist[w]); kmax = max(kmax, hist[32 + w]); }
  __syncthreads();
  if (nvalid <= K) {   // take every present key
    if (tid == 0) { st->thr = 1u; st->take_eq = 0x7fffffff; st->nvalid = nvalid; }
    __syncthreads();
    return;
  }
  // bits above `top` are the same in every present key
  const int top = 31 - __clz(kmin ^ kmax | 1u);   // highest differing bit (>= 0)
  int shift = top - 7;
  const uint32_t common = top >= 31 ? 0u : (kmin >> (top + 1)) << (top + 1);
  if (tid == 0) {
    st->prefix = common;
    st->mask = top >= 31 ? 0u : ~((1u << (top + 1)) - 1u);
    st->krem = K;
    st->nvalid = nvalid;
  }
  const int iters = (n + NT - 1) / NT;
#pragma unroll 1
  while (true) {
    const int sh = shift < 0 ? 0 : shift;            // last digit may be narrower
    const uint32_t dmask = shift < 0 ? (0xFFu >> (-shift)) : 0xFFu;
    for (int i = tid; i < 256; i += NT) hist[i] = 0u;
    __syncthreads();
    const uint32_t prefix = st->prefix, mask = st->mask;
    for (int j = 0; j < iters; ++j) {
      const int i = j * NT + tid;
      const uint32_t k = i < n ? keys[i] : 0u;
      const bool act = k != 0u && (k & mask) == prefix;
      const uint32_t bin = (k >> sh) & dmask;
      const unsigned am = __ballot_sync(0xffffffffu, act);
      if (am) {
        const int leader = __ffs(am) - 1;
        const uint32_t b0 = __shfl_sync(0xffffffffu, bin, leader);
        if (__all_sync(0xffffffffu, !act || bin == b0)) {
          if (lane == leader) atomicAdd(&hist[b0], (uint32_t)__popc(am));
        } else if (act) {
          atomicAdd(&hist[bin], 1u);
        }
      }
    }
    __syncthreads();
    if (tid < 32) {   // warp 0: lane l owns bins 8l..8l+7; find the bin holding the krem-th largest
      const int krem = st->krem;
      uint32_t own = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) own += hist[8 * lane + q];
      uint32_t suf = own;   // inclusive suffix over lanes >= lane
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += v;
      }
      const uint32_t above_lane = suf - own;   // keys in bins of higher lanes
      const bool here = suf >= (uint32_t)krem && above_lane < (uint32_t)krem;
      if (here) {
        uint32_t above = above_lane;
        int bin = 8 * lane;
        for (int q = 7; q >= 0; --q) {
          const uint32_t h = hist[8 * lane + q];
          if (above + h >= (uint32_t)krem) { bin = 8 * lane + q; break; }
          above += h;
        }
        st->krem = krem - (int)above;
        st->prefix = prefix | ((uint32_t)bin << sh);
        st->mask = mask | (dmask << sh);
      }
    }
    __syncthreads();
    if (sh == 0) break;
    shift -= 8;
  }
  if (tid == 0) { st->thr = st->prefix; st->take_eq = st->krem; }
  __syncthreads();
}

// Column-ordered compaction of the selected keys: emit(pos, i, key) for each
// taken i in increasing i.  Returns the number taken.  All threads call.
template <int NT, class Emit>
__device__ int ordered_emit(const uint32_t *keys, int n, SelState *st, Emit emit) {
  constexpr int NW = NT / 32;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t thr = st->thr;
  const int take_eq = st->take_eq;
  const int per = ((n + NW - 1) / NW + 31) & ~31;
  const int lo = warp * per;
  const int hi = lo + per < n ? lo + per : n;
  int gt = 0, eq = 0;
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const uint32_t k = i < hi ? keys[i] : 0u;
    gt += __popc(__ballot_sync(0xffffffffu, k > thr));
    eq += __popc(__ballot_sync(0xffffffffu, k == thr));
  }
  __syncthreads();
  if (lane == 0) { st->warp_gt[warp] = gt; st->warp_eq[warp] = eq; }
  __syncthreads();
  int gt_before = 0, eq_before = 0, gt_all = 0, eq_all = 0;
  for (int w = 0; w < NW; ++w) {
    if (w < warp) { gt_before += st->warp_gt[w]; eq_before += st->warp_eq[w]; }
    gt_all += st->warp_gt[w];
    eq_all += st->warp_eq[w];
  }
  int out = gt_before + (eq_before < take_eq ? eq_before : take_eq);
  const unsigned lt = (1u << lane) - 1u;
  for (int base = lo; base < hi; base += 32) {
    const int i = base + lane;
    const uint32_t k = i < hi ? keys[i] : 0u;
    const unsigned eqb = __ballot_sync(0xffffffffu, k == thr);
    const int rank = eq_before + __popc(eqb & lt);
    const bool take = k > thr || (k == thr && rank < take_eq);
    const unsigned tb = __ballot_sync(0xffffffffu, take);
    if (take) emit(out + __popc(tb & lt), i, k);
    out += __popc(tb);
    eq_before += __popc(eqb);
  }
  return gt_all + (eq_all < take_eq ? eq_all : take_eq);
}

struct WsView {
  uint32_t *ckey;   // [rows][nchunks][k1]
  int32_t *ccol;
  uint32_t *pkey;   // [rows][nchunks][p1]
  int32_t *pblk;
};

__host__ __device__ inline WsView ws_view(void *ws, int rows, const TopkPlan &p) {
  WsView v;
  const size_t nk = (size_t)rows * p.nchunks * p.k1, np = (size_t)rows * p.nchunks * p.p1;
  uint8_t *q = reinterpret_cast<uint8_t *>(ws);
  v.ckey = reinterpret_cast<uint32_t *>(q);
  q += nk * 4;
  v.ccol = reinterpret_cast<int32_t *>(q);
  q += nk * 4;
  v.pkey = reinterpret_cast<uint32_t *>(q);
  q += np * 4;
  v.pblk = reinterpret_cast<int32_t *>(q);
  return v;
}

__global__ void __launch_bounds__(kT1) topk_chunk_kernel(const TopkArgs a, const TopkPlan p) {
  extern __shared__ uint32_t sm1[];
  __shared__ uint32_t hist[256];
  __shared__ SelState st;
  __shared__ int red[32];
  uint32_t *keys = sm1;                 // [chunk]
  uint32_t *bkeys = sm1 + p.chunk;      // [chunk/8]
  const int row = blockIdx.y, chunk = blockIdx.x, tid = threadIdx.x;
  const int c0 = chunk * p.chunk;
  int ncol = a.n_cols;
  if (a.n_valid) {
    const int nv = a.n_valid[row];
    if (nv < ncol) ncol = nv < 0 ? 0 : nv;
  }
  int cnt = ncol - c0;
  cnt = cnt < 0 ? 0 : (cnt > p.chunk ? p.chunk : cnt);
  const float *srow = a.scores + (size_t)row * a.ld + c0;
  for (int i = tid; i < p.chunk; i += kT1) keys[i] = i < cnt ? score_key(srow[i]) : 0u;
  __syncthreads();

  WsView v = ws_view(a.ws, a.rows, p);
  const size_t base = ((size_t)row * p.nchunks + chunk) * p.k1;
  radix_select<kT1>(keys, p.chunk, p.k1, hist, &st, red);
  const int taken = ordered_emit<kT1>(keys, p.chunk, &st, [&](int pos, int i, uint32_t k) {
    v.ckey[base + pos] = k;
    v.ccol[base + pos] = c0 + i;
  });
  for (int i = taken + tid; i < p.k1; i += kT1) { v.ckey[base + i] = 0u; v.ccol[base + i] = -1; }

  if (a.P_out > 0) {
    const int nb = p.chunk / 8;
    for (int j = tid; j < nb; j += kT1) {
      uint32_t m = 0u;
#pragma unroll
      for (int q = 0; q < 8; ++q) m = max(m, keys[8 * j + q]);
      bkeys[j] = m;
    }
    __syncthreads();
    const size_t pb = ((size_t)row * p.nchunks + chunk) * p.p1;
    radix_select<kT1>(bkeys, nb, p.p1, hist, &st, red);
    const int pt = ordered_emit<kT1>(bkeys, nb, &st, [&](int pos, int j, uint32_t k) {
      v.pkey[pb + pos] = k;
      v.pblk[pb + pos] = c0 / 8 + j;
    });
    for (int i = pt + tid; i < p.p1; i += kT1) { v.pkey[pb + i] = 0u; v.pblk[pb + i] = -1; }
  }
}

__global__ void __launch_bounds__(kT2) topk_merge_kernel(const TopkArgs a, const TopkPlan p) {
  extern __shared__ uint32_t sm2[];
  __shared__ uint32_t hist[256];
  __shared__ SelState st;
  __shared__ int red[32];
  const int row = blockIdx.x, tid = threadIdx.x;
  WsView v = ws_view(a.ws, a.rows, p);

  // ---- entries
  {
    const int n = p.nchunks * p.k1;
    const size_t base = (size_t)row * n;
    const uint32_t *keys = v.ckey + base;
    const int32_t *cols = v.ccol + base;
    if (n <= kMergeSmemCands) {
      uint32_t *k_s = sm2;
      int32_t *c_s = reinterpret_cast<int32_t *>(sm2 + n);
      for (int i = tid; i < n; i += kT2) { k_s[i] = keys[i]; c_s[i] = cols[i]; }
      __syncthreads();
      keys = k_s;
      cols = c_s;
    }
    radix_select<kT2>(keys, n, a.K, hist, &st, red);
    int32_t *out = a.out_idx + (size_t)row * a.K;
    const int32_t *pb = a.pool_blocks ? a.pool_blocks + (size_t)row * (a.n_cols / 8) : nullptr;
    const int taken = ordered_emit<kT2>(keys, n, &st, [&](int pos, int i, uint32_t) {
      const int c = cols[i];
      out[pos] = pb ? pb[c >> 3] * 8 + (c & 7) : c;
    });
    for (int i = taken + tid; i < a.K; i += kT2) out[i] = -1;
    __syncthreads();
  }
  // ---- pool
  if (a.P_out > 0) {
    const int n = p.nchunks * p.p1;
    const size_t base = (size_t)row * n;
    const uint32_t *keys = v.pkey + base;
    const int32_t *blks = v.pblk + base;
    if (n <= kMergeSmemCands) {
      uint32_t *k_s = sm2;
      int32_t *b_s = reinterpret_cast<int32_t *>(sm2 + n);
      for (int i = tid; i < n; i += kT2) { k_s[i] = keys[i]; b_s[i] = blks[i]; }
      __syncthreads();
      keys = k_s;
      blks = b_s;
    }
    radix_select<kT2>(keys, n, a.P_out, hist, &st, red);
    int32_t *out = a.out_pool + (size_t)row * a.P_out;
    const int taken = ordered_emit<kT2>(keys, n, &st, [&](int pos, int i, uint32_t) { out[pos] = blks[i]; });
    for (int i = taken + tid; i < a.P_out; i += kT2) out[i] = -1;
  }
}

}  // namespace

TopkPlan plan_topk(int rows, int n_cols, int K, int P_out) {
  TopkPlan p;
  int chunk = 4096;
  auto kk = [&](int c) { return K < c ? K : c; };
  while (chunk < 32768 && (size_t)((n_cols + chunk - 1) / chunk) * kk(chunk) > 8192) chunk *= 2;
  p.chunk = chunk;
  p.nchunks = n_cols > 0 ? (n_cols + chunk - 1) / chunk : 1;
  p.k1 = kk(chunk);
  p.p1 = P_out > 0 ? (P_out < chunk / 8 ? P_out : chunk / 8) : 0;
  p.bytes = (size_t)rows * p.nchunks * ((size_t)p.k1 + p.p1) * 8;
  return p;
}

cudaError_t launch_topk(const TopkArgs &a, const TopkPlan &p, cudaStream_t s) {
  const size_t sm1 = sizeof(uint32_t) * ((size_t)p.chunk + p.chunk / 8);
  cudaError_t e = cudaFuncSetAttribute(topk_chunk_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm1);
  if (e != cudaSuccess) return e;
  topk_chunk_kernel<<<dim3(p.nchunks, a.rows), kT1, sm1, s>>>(a, p);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  // shared memory holds whichever candidate list fits (the other is read from
  // the workspace directly)
  const int nk = p.nchunks * p.k1, np = p.nchunks * p.p1;
  const int sk = nk <= kMergeSmemCands ? nk : 0, sp = np <= kMergeSmemCands ? np : 0;
  const size_t sm2 = (size_t)(sk > sp ? sk : sp) * 8;
  e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm2);
  if (e != cudaSuccess) return e;
  topk_merge_kernel<<<a.rows, kT2, sm2, s>>>(a, p);
  return cudaGetLastError();
}

}  // namespace csa2
