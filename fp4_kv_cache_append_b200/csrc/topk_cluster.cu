// Top-K selection and hierarchical pool for rows of up to 65,536 columns in
// one launch: a thread-block cluster of 8 blocks per row.
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2": Top-512 per
//   Full/Reindex layer; the first Full decoder layer's pool of 2,048 blocks
//   x 8 positions (paper sec. 2.3.2, 4.2.1, Fig. 5).
// Same contract as the multi-kernel path in topk.cu (score descending, ties
// -> smaller column, non-finite = absent, ascending output, -1 padding,
// block score = max of its present columns), without a workspace:
//   * block r of the cluster owns columns [r*S, (r+1)*S); each thread keeps
//     32 consecutive columns' order-preserving keys (and their 4 block
//     maxima) in registers;
//   * the cluster-wide key range comes from every block's min/max read
//     through distributed shared memory;
//   * rounds of a 2048-bin histogram over the remaining key range, summed
//     across the cluster (block r reduces bins [256r, 256r+256)), narrow
//     the range to the bin holding the K-th key until that bin is either
//     taken whole or is a single key value (at most 3 rounds for 32-bit keys);
//   * ties at that value are shared out in column order from per-block
//     counts, and every block writes its chosen columns, in order, at the
//     offset given by the counts of the blocks before it.
// Entries (K) and blocks (P_out) are selected together in the same rounds.
// Only cluster barriers are used; no block waits on a flag.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace csa2 {

namespace {

constexpr int kCl = 8;        // blocks per row
constexpr int kT = 256;       // threads per block
constexpr int kN = 32;        // columns per thread
constexpr int kNB = kN / 8;   // blocks of 8 columns per thread
constexpr int kBins = 2048;

__device__ __forceinline__ uint32_t ckey(float f) {
  if (!isfinite(f)) return 0u;
  if (f == 0.0f) f = 0.0f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive scan of one int per thread over the block; returns the total.
__device__ __forceinline__ int block_excl_scan(int v, int &excl, int *red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  __syncthreads();
  if (lane == 31) red[warp] = incl;
  __syncthreads();
  int before = 0, total = 0;
#pragma unroll
  for (int w = 0; w < kT / 32; ++w) {
    if (w < warp) before += red[w];
    total += red[w];
  }
  excl = before + incl - v;
  return total;
}

struct Sel {          // state of one selection (entries or blocks), identical in every block
  uint32_t lo, hi;    // key range still undecided
  int need;           // keys still to take inside [lo, hi]
  int shift;
  bool done;
  uint32_t thr_gt;    // final: keys > thr_gt are taken ...
  uint32_t thr_eq;    // ... and `take_eq` of the keys == thr_eq (in column order)
  int take_eq;
};

struct Shared {
  uint32_t hist[2][kBins];
  uint32_t hsum[2][kBins / kCl];
  uint32_t stat[2][3];       // this block: min, max, count of present keys
  int cnt[2][2];             // this block: ties, chosen
  int red[kT / 32];
  uint32_t g[2][3];          // cluster: min, max, count
  int th[2][3];              // threshold bin, keys above it in the range, keys in it
};

}  // namespace

__global__ void __cluster_dims__(kCl, 1, 1) __launch_bounds__(kT) topk_cluster_kernel(const TopkArgs a, int S) {
  __shared__ Shared sh;
  cg::cluster_group cl = cg::this_cluster();
  const int r = (int)cl.block_rank();
  const int row = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int ncol = a.n_cols;
  if (a.n_valid) {
    const int v = a.n_valid[row];
    if (v < ncol) ncol = v < 0 ? 0 : v;
  }
  const int npt = S / kT;                   // columns per thread (a multiple of 8, <= kN)
  const int c0 = r * S + tid * npt;         // this thread's first column
  const float *srow = a.scores + (size_t)row * a.ld;
  const int nsel = a.P_out > 0 ? 2 : 1;
  const int Kt[2] = {a.K, a.P_out};

  // ---- keys in registers (column order within the thread)
  uint32_t key[kN], bkey[kNB];
  // c0 is a multiple of 8, so 16-byte loads are aligned when the row is
  const bool vec = (a.ld & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15u) == 0;
#pragma unroll
  for (int k = 0; k < kN; k += 4) {
    const int col = c0 + k;
    if (vec && k < npt && col + 4 <= ncol) {
      const float4 v = __ldcs(reinterpret_cast<const float4 *>(srow + col));
      key[k] = ckey(v.x);
      key[k + 1] = ckey(v.y);
      key[k + 2] = ckey(v.z);
      key[k + 3] = ckey(v.w);
    } else {
#pragma unroll
      for (int j = 0; j < 4; ++j) key[k + j] = (k + j < npt && col + j < ncol) ? ckey(srow[col + j]) : 0u;
    }
  }
#pragma unroll
  for (int g = 0; g < kNB; ++g) {
    uint32_t m = 0u;
#pragma unroll
    for (int k = 0; k < 8; ++k) m = max(m, key[8 * g + k]);
    bkey[g] = m;
  }

  // ---- local and cluster-wide key range and count
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    if (s >= nsel) break;
    uint32_t mn = 0xFFFFFFFFu, mx = 0u, c = 0u;
    if (s == 0) {
#pragma unroll
      for (int k = 0; k < kN; ++k) if (key[k]) { mn = min(mn, key[k]); mx = max(mx, key[k]); ++c; }
    } else {
#pragma unroll
      for (int g = 0; g < kNB; ++g) if (bkey[g]) { mn = min(mn, bkey[g]); mx = max(mx, bkey[g]); ++c; }
    }
    mn = __reduce_min_sync(0xffffffffu, mn);
    mx = __reduce_max_sync(0xffffffffu, mx);
    c = __reduce_add_sync(0xffffffffu, c);
    if (lane == 0) { sh.hsum[s][warp] = mn; sh.hsum[s][8 + warp] = mx; sh.hsum[s][16 + warp] = c; }
  }
  __syncthreads();
  if (tid < nsel) {
    uint32_t mn = 0xFFFFFFFFu, mx = 0u, c = 0u;
    for (int w = 0; w < kT / 32; ++w) {
      mn = min(mn, sh.hsum[tid][w]);
      mx = max(mx, sh.hsum[tid][8 + w]);
      c += sh.hsum[tid][16 + w];
    }
    sh.stat[tid][0] = mn;
    sh.stat[tid][1] = mx;
    sh.stat[tid][2] = c;
  }
  cl.sync();
  if (warp == 0) {
    for (int s = 0; s < nsel; ++s) {
      uint32_t mn = 0xFFFFFFFFu, mx = 0u, c = 0u;
      if (lane < kCl) {
        const uint32_t *rs = cl.map_shared_rank(&sh.stat[s][0], lane);
        mn = rs[0];
        mx = rs[1];
        c = rs[2];
      }
      mn = __reduce_min_sync(0xffffffffu, mn);
      mx = __reduce_max_sync(0xffffffffu, mx);
      c = __reduce_add_sync(0xffffffffu, c);
      if (lane == 0) { sh.g[s][0] = mn; sh.g[s][1] = mx; sh.g[s][2] = c; }
    }
  }
  __syncthreads();

  Sel sel[2];
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    sel[s].lo = sh.g[s][0];
    sel[s].hi = sh.g[s][1];
    sel[s].need = Kt[s];
    sel[s].shift = 0;
    sel[s].take_eq = 0;
    sel[s].thr_eq = 0u;
    sel[s].thr_gt = 0u;
    // every present key fits: take them all
    sel[s].done = s >= nsel || (int)sh.g[s][2] <= Kt[s];
  }

  // ---- rounds: histogram of the undecided range, cluster-reduced
#pragma unroll 1
  while (!(sel[0].done && sel[1].done)) {
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      const uint32_t span = sel[s].hi - sel[s].lo;
      sel[s].shift = span >= (uint32_t)kBins ? (32 - __clz(span)) - 11 : 0;
      for (int i = tid; i < kBins; i += kT) sh.hist[s][i] = 0u;
    }
    __syncthreads();
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (sel[s].done) continue;
      const uint32_t lo = sel[s].lo, hi = sel[s].hi;
      const int shf = sel[s].shift;
      if (s == 0) {
#pragma unroll
        for (int k = 0; k < kN; ++k)
          if (key[k] && key[k] >= lo && key[k] <= hi) atomicAdd(&sh.hist[0][(key[k] - lo) >> shf], 1u);
      } else {
#pragma unroll
        for (int g = 0; g < kNB; ++g)
          if (bkey[g] && bkey[g] >= lo && bkey[g] <= hi) atomicAdd(&sh.hist[1][(bkey[g] - lo) >> shf], 1u);
      }
    }
    cl.sync();   // every block's histogram is complete
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (sel[s].done) continue;
      const int bin = r * (kBins / kCl) + tid;   // this block reduces 256 bins
      uint32_t v = 0u;
#pragma unroll
      for (int c = 0; c < kCl; ++c) v += cl.map_shared_rank(&sh.hist[s][0], c)[bin];
      sh.hsum[s][tid] = v;
    }
    cl.sync();   // every segment is reduced
#pragma unroll
    for (int s = 0; s < 2; ++s) {
      if (sel[s].done) continue;   // cluster-uniform
      // thread t reads bins [8t, 8t+8) of the reduced histogram
      uint32_t h[8], local = 0u;
      const uint32_t *seg = cl.map_shared_rank(&sh.hsum[s][0], (8 * tid) / (kBins / kCl));
#pragma unroll
      for (int i = 0; i < 8; ++i) { h[i] = seg[(8 * tid) % (kBins / kCl) + i]; local += h[i]; }
      int lower;   // keys in the bins of lower threads
      const int total = block_excl_scan((int)local, lower, sh.red);
      const int above_me = total - lower - (int)local;   // keys in the bins of higher threads
      const int need = sel[s].need;
      if (above_me < need && above_me + (int)local >= need) {   // exactly one thread
        int ab = above_me, t_bin = 8 * tid, cnt_t = (int)h[0];
        for (int i = 7; i >= 0; --i) {
          if (ab + (int)h[i] >= need) { t_bin = 8 * tid + i; cnt_t = (int)h[i]; break; }
          ab += (int)h[i];
        }
        sh.th[s][0] = t_bin;
        sh.th[s][1] = ab;
        sh.th[s][2] = cnt_t;
      }
      __syncthreads();
      const int T = sh.th[s][0], above = sh.th[s][1], cntT = sh.th[s][2];
      const uint32_t lo_T = sel[s].lo + ((uint32_t)T << sel[s].shift);
      const uint32_t w1 = (1u << sel[s].shift) - 1u;
      const uint32_t hi_T = (sel[s].hi - lo_T > w1) ? lo_T + w1 : sel[s].hi;
      const int need2 = need - above;
      if (cntT == need2) {            // bin T is taken whole: every key >= lo_T
        sel[s].thr_gt = lo_T - 1u;
        sel[s].take_eq = 0;
        sel[s].done = true;
      } else if (sel[s].shift == 0) { // bin T is one key value: need2 of its ties
        sel[s].thr_gt = lo_T;
        sel[s].thr_eq = lo_T;
        sel[s].take_eq = need2;
        sel[s].done = true;
      } else {                        // refine inside bin T
        sel[s].lo = lo_T;
        sel[s].hi = hi_T;
        sel[s].need = need2;
      }
    }
    cl.sync();   // reduced segments are no longer read; the next round may overwrite them
  }

  // ---- ties (column order across the cluster) and output offsets
  int my_ties[2] = {0, 0}, my_chosen[2] = {0, 0}, tie_base[2] = {0, 0};
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    int t = 0;
    if (s < nsel && sel[s].take_eq > 0) {
      if (s == 0) {
#pragma unroll
        for (int k = 0; k < kN; ++k) t += key[k] && key[k] == sel[s].thr_eq;
      } else {
#pragma unroll
        for (int g = 0; g < kNB; ++g) t += bkey[g] && bkey[g] == sel[s].thr_eq;
      }
    }
    my_ties[s] = t;
    const int tot = block_excl_scan(t, tie_base[s], sh.red);
    if (tid == 0) sh.cnt[s][0] = tot;
  }
  cl.sync();
  int ties_before[2] = {0, 0}, allow[2] = {0, 0};
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    for (int c = 0; c < r; ++c) ties_before[s] += cl.map_shared_rank(&sh.cnt[s][0], c)[0];
    allow[s] = sel[s].take_eq - ties_before[s];   // ties this block may still take
  }
  // chosen per thread (ties in column order: block prefix + thread prefix)
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    int c = 0, tr = tie_base[s];
    if (s < nsel) {
      if (s == 0) {
#pragma unroll
        for (int k = 0; k < kN; ++k) {
          const uint32_t kk = key[k];
          const bool tie = kk && kk == sel[s].thr_eq && sel[s].take_eq > 0;
          c += (kk && kk > sel[s].thr_gt) || (tie && tr < allow[s]);
          tr += tie;
        }
      } else {
#pragma unroll
        for (int g = 0; g < kNB; ++g) {
          const uint32_t kk = bkey[g];
          const bool tie = kk && kk == sel[s].thr_eq && sel[s].take_eq > 0;
          c += (kk && kk > sel[s].thr_gt) || (tie && tr < allow[s]);
          tr += tie;
        }
      }
    }
    my_chosen[s] = c;
  }
  int pos[2];
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    const int tot = block_excl_scan(my_chosen[s], pos[s], sh.red);
    if (tid == 0) sh.cnt[s][1] = tot;
  }
  cl.sync();
  int base[2] = {0, 0}, total[2] = {0, 0};
#pragma unroll
  for (int s = 0; s < 2; ++s) {
    for (int c = 0; c < kCl; ++c) {
      const int v = cl.map_shared_rank(&sh.cnt[s][1], c)[0];
      if (c < r) base[s] += v;
      total[s] += v;
    }
  }
  // ---- write the chosen columns in order
  {
    int o = base[0] + pos[0], tr = tie_base[0];
    int32_t *out = a.out_idx + (size_t)row * a.K;
    const int32_t *pb = a.pool_blocks ? a.pool_blocks + (size_t)row * (a.n_cols / 8) : nullptr;
#pragma unroll
    for (int k = 0; k < kN; ++k) {
      const uint32_t kk = key[k];
      const bool tie = kk && kk == sel[0].thr_eq && sel[0].take_eq > 0;
      const bool take = (kk && kk > sel[0].thr_gt) || (tie && tr < allow[0]);
      tr += tie;
      if (take) {
        const int col = c0 + k;
        if (o < a.K) out[o] = pb ? pb[col >> 3] * 8 + (col & 7) : col;
        ++o;
      }
    }
    if (r == kCl - 1)
      for (int i = total[0] + tid; i < a.K; i += kT) out[i] = -1;
  }
  if (nsel == 2) {
    int o = base[1] + pos[1], tr = tie_base[1];
    int32_t *out = a.out_pool + (size_t)row * a.P_out;
#pragma unroll
    for (int g = 0; g < kNB; ++g) {
      const uint32_t kk = bkey[g];
      const bool tie = kk && kk == sel[1].thr_eq && sel[1].take_eq > 0;
      const bool take = (kk && kk > sel[1].thr_gt) || (tie && tr < allow[1]);
      tr += tie;
      if (take) {
        if (o < a.P_out) out[o] = (c0 >> 3) + g;
        ++o;
      }
    }
    if (r == kCl - 1)
      for (int i = total[1] + tid; i < a.P_out; i += kT) out[i] = -1;
  }
  cl.sync();   // no block leaves while another may still read its shared memory
}

// Rows of up to kCl * kT * kN columns go through the cluster kernel.
bool topk_cluster_fits(int n_cols) { return n_cols <= kCl * kT * kN; }

cudaError_t launch_topk_cluster(const TopkArgs &a, cudaStream_t s) {
  // slice per block: a multiple of 8 columns per thread
  int npt = (a.n_cols + kCl * kT - 1) / (kCl * kT);
  npt = (npt + 7) / 8 * 8;
  if (npt < 8) npt = 8;
  topk_cluster_kernel<<<dim3(kCl, a.rows), kT, 0, s>>>(a, npt * kT);
  return cudaGetLastError();
}

}  // namespace csa2
