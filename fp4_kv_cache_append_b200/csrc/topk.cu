// Top-K selection and the hierarchical candidate pool for rows of more than
// 65,536 columns (shorter rows use the single-launch cluster kernel of
// topk_cluster.cu): 128 or more rows of at most 131,072 columns without a
// pool take topk_rows_kernel (one block per row, below); the other shapes the
// four-kernel path described here.
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2": each Full or
//   Reindex layer keeps the Top-512 entries; the first Full layer of the
//   decoder also builds the pool of <= 2,048 blocks x 8 positions that the
//   Reindex layers rescore (paper sec. 2.3.2, 4.2.1, Fig. 5).
// Order: score descending, ties -> smaller column; absent = non-finite.  The
// result lists the chosen columns in ascending order, -1 padded.  A block's
// score is the maximum of its present columns.
//
// Scores become order-preserving 32-bit keys (0 = absent).  Four kernels
// after a memset of the per-row counters, none of them waiting on another
// block:
//  0. topk_range_kernel  (rows x column chunks): the row's smallest and
//     largest present key (atomic max of key and of ~key).
//  1. topk_hist_kernel   (same grid): 2048-bin histogram of the digit
//     (key - min) >> shift, the shift chosen so the bins span the row's key
//     range, for entries and for block maxima.
//  2. topk_filter_kernel (same grid): every block derives the threshold bin
//     T (the bin holding the K-th key) from the histogram, and appends the
//     columns above T to the row's "selected" list and the columns in T to
//     its "candidates" list (one atomic per warp and list).
//  3. topk_select_kernel (one block per row): exact radix select among the
//     candidates (a second select on the column among keys equal to the
//     threshold, so ties go to smaller columns); the chosen columns are
//     marked in a bitmap and written in ascending order by a prefix popcount
//     (mapped through the pool for Reindex rows).
// Binning over the actual range keeps the threshold bin small even when a
// row's scores sit within a few percent of each other.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kBins = 2048;          // digit = (key - kmin) >> shift, 11 bits
constexpr int kColsPerBlock = 4096;  // columns per hist/filter block
constexpr int kTF = 256;             // hist/filter threads: 16 columns each
constexpr int kTS = 1024;            // select threads
constexpr int kSmemCands = 12288;    // candidates staged in shared memory by the select kernel

// Order-preserving key of a score: larger score -> larger key; -0 == +0;
// non-finite -> 0 (absent).
__device__ __forceinline__ uint32_t score_key(float f) {
  if (!isfinite(f)) return 0u;
  if (f == 0.0f) f = 0.0f;
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

struct Ws {
  uint32_t *hist, *histb;   // [rows][kBins]
  uint32_t *cnt;            // [rows][4]: selected, candidates, selected blocks, candidate blocks
  uint32_t *range;          // [rows][2]: max key, max of ~key (both start at 0)
  int32_t *sel, *cand, *selb, *candb;
};

// Digit of a present key within the row's key range [kmin, kmax].
struct Binning {
  uint32_t kmin;
  int shift;
  __device__ __forceinline__ int digit(uint32_t key) const { return (int)((key - kmin) >> shift); }
};

__device__ __forceinline__ Ws ws_view(const TopkArgs &a, const TopkPlan &p) {
  uint8_t *q = reinterpret_cast<uint8_t *>(a.ws);
  Ws w;
  w.hist = reinterpret_cast<uint32_t *>(q + p.off_hist);
  w.histb = reinterpret_cast<uint32_t *>(q + p.off_histb);
  w.cnt = reinterpret_cast<uint32_t *>(q + p.off_cnt);
  w.range = reinterpret_cast<uint32_t *>(q + p.off_range);
  w.sel = reinterpret_cast<int32_t *>(q + p.off_sel);
  w.cand = reinterpret_cast<int32_t *>(q + p.off_cand);
  w.selb = reinterpret_cast<int32_t *>(q + p.off_selb);
  w.candb = reinterpret_cast<int32_t *>(q + p.off_candb);
  return w;
}

__device__ __forceinline__ int row_cols(const TopkArgs &a, int row) {
  int n = a.n_cols;
  if (a.n_valid) {
    const int v = a.n_valid[row];
    if (v < n) n = v < 0 ? 0 : v;
  }
  return n;
}

__device__ __forceinline__ Binning row_binning(const Ws &w, int row) {
  const uint32_t kmax = w.range[2 * row], kmin = ~w.range[2 * row + 1];
  Binning b;
  b.kmin = kmin;
  const uint32_t span = kmax > kmin ? kmax - kmin : 0u;
  b.shift = span >= (uint32_t)kBins ? (32 - __clz(span)) - 11 : 0;
  return b;
}

// Histogram update, one atomic per warp when the warp's present keys share a bin.
__device__ __forceinline__ void hist_add(uint32_t *h, uint32_t key, const Binning &bn, int lane) {
  const bool act = key != 0u;
  const uint32_t bin = act ? (uint32_t)bn.digit(key) : 0u;
  const unsigned am = __ballot_sync(0xffffffffu, act);
  if (!am) return;
  const int leader = __ffs(am) - 1;
  const uint32_t b0 = __shfl_sync(0xffffffffu, bin, leader);
  if (__all_sync(0xffffffffu, !act || bin == b0)) {
    if (lane == leader) atomicAdd(&h[b0], (uint32_t)__popc(am));
  } else if (act) {
    atomicAdd(&h[bin], 1u);
  }
}

// Append `val` to list[] for the lanes with flag set; one atomic per warp.
__device__ __forceinline__ void warp_append(bool flag, int32_t val, uint32_t *counter, int32_t *list, int lane) {
  const unsigned m = __ballot_sync(0xffffffffu, flag);
  if (!m) return;
  const int leader = __ffs(m) - 1;
  uint32_t base = 0;
  if (lane == leader) base = atomicAdd(counter, (uint32_t)__popc(m));
  base = __shfl_sync(0xffffffffu, base, leader);
  if (flag) list[base + __popc(m & ((1u << lane) - 1u))] = val;
}

// Threshold bin of the K-th largest key from a row histogram: the bin T whose
// keys, with all keys of higher bins (`above` of them), reach K.  Fewer than
// K present keys: T = -1 and above = their number.  All threads call; every
// thread gets the result.
template <int NT>
__device__ void find_threshold(const uint32_t *hist, int K, int &T, int &above, int *sm_ws) {
  constexpr int BPT = kBins / NT;   // bins per thread
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  uint32_t h[BPT];
  uint32_t local = 0;
#pragma unroll
  for (int i = 0; i < BPT; ++i) { h[i] = hist[tid * BPT + i]; local += h[i]; }
  uint32_t v = local;   // inclusive suffix over lanes >= lane
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_down_sync(0xffffffffu, v, o);
    if (lane + o < 32) v += y;
  }
  __syncthreads();
  if (lane == 0) sm_ws[warp] = (int)v;
  __syncthreads();
  uint32_t higher = 0, total = 0;
#pragma unroll
  for (int w = 0; w < NT / 32; ++w) {
    const uint32_t s = (uint32_t)sm_ws[w];
    total += s;
    if (w > warp) higher += s;
  }
  const uint32_t excl = v - local + higher;   // keys in bins above this thread's
  if (total <= (uint32_t)K) {
    if (tid == 0) { sm_ws[32] = -1; sm_ws[33] = (int)total; }
  } else if (excl < (uint32_t)K && excl + local >= (uint32_t)K) {
    uint32_t ab = excl;
    int t_bin = tid * BPT;
    for (int i = BPT - 1; i >= 0; --i) {
      if (ab + h[i] >= (uint32_t)K) { t_bin = tid * BPT + i; break; }
      ab += h[i];
    }
    sm_ws[32] = t_bin;
    sm_ws[33] = (int)ab;
  }
  __syncthreads();
  T = sm_ws[32];
  above = sm_ws[33];
  __syncthreads();
}

// Threshold of the K largest keys key(0..n-1) (0 = absent): keys > thr are
// taken, and take_eq of the keys == thr.  8-bit digits from the highest bit
// where present keys differ.
struct SelState {
  uint32_t thr, prefix, mask;
  int take_eq, krem;
};

template <int NT, class KeyF>
__device__ void radix_select(KeyF key, int n, int K, uint32_t *hist, SelState *st, int *red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  int cnt = 0;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  for (int i = tid; i < n; i += NT) {
    const uint32_t k = key(i);
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
  if (nvalid <= K) {
    if (tid == 0) { st->thr = 1u; st->take_eq = 0x7fffffff; }
    __syncthreads();
    return;
  }
  const int top = 31 - __clz((kmin ^ kmax) | 1u);   // highest differing bit
  int shift = top - 7;
  if (tid == 0) {
    st->prefix = top >= 31 ? 0u : (kmin >> (top + 1)) << (top + 1);
    st->mask = top >= 31 ? 0u : ~((1u << (top + 1)) - 1u);
    st->krem = K;
  }
  const int iters = (n + NT - 1) / NT;
#pragma unroll 1
  while (true) {
    const int sh = shift < 0 ? 0 : shift;
    const uint32_t dmask = shift < 0 ? (0xFFu >> (-shift)) : 0xFFu;
    for (int i = tid; i < 256; i += NT) hist[i] = 0u;
    __syncthreads();
    const uint32_t prefix = st->prefix, mask = st->mask;
    for (int j = 0; j < iters; ++j) {
      const int i = j * NT + tid;
      const uint32_t k = i < n ? key(i) : 0u;
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
    if (tid < 32) {   // lane l owns bins 8l..8l+7: find the bin holding the krem-th largest
      const int krem = st->krem;
      uint32_t own = 0;
#pragma unroll
      for (int q = 0; q < 8; ++q) own += hist[8 * lane + q];
      uint32_t suf = own;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_down_sync(0xffffffffu, suf, o);
        if (lane + o < 32) suf += v;
      }
      const uint32_t above_lane = suf - own;
      if (suf >= (uint32_t)krem && above_lane < (uint32_t)krem) {
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

__global__ void __launch_bounds__(kTF) topk_range_kernel(const TopkArgs a, const TopkPlan p) {
  __shared__ uint32_t wmax[kTF / 32], wnmin[kTF / 32];
  const int row = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c0 = blockIdx.x * kColsPerBlock;
  const int ncol = row_cols(a, row);
  const float *srow = a.scores + (size_t)row * a.ld;
  uint32_t kmax = 0u, nmin = 0u;   // max key, max of ~key over present keys
#pragma unroll
  for (int j = 0; j < kColsPerBlock / kTF; ++j) {
    const int col = c0 + j * kTF + tid;
    const uint32_t key = col < ncol ? score_key(srow[col]) : 0u;
    if (key) { kmax = max(kmax, key); nmin = max(nmin, ~key); }
  }
  kmax = __reduce_max_sync(0xffffffffu, kmax);
  nmin = __reduce_max_sync(0xffffffffu, nmin);
  if (lane == 0) { wmax[warp] = kmax; wnmin[warp] = nmin; }
  __syncthreads();
  if (tid == 0) {
    for (int w = 1; w < kTF / 32; ++w) { kmax = max(kmax, wmax[w]); nmin = max(nmin, wnmin[w]); }
    if (kmax) {
      const Ws w = ws_view(a, p);
      atomicMax(&w.range[2 * row], kmax);
      atomicMax(&w.range[2 * row + 1], nmin);
    }
  }
}

__global__ void __launch_bounds__(kTF) topk_hist_kernel(const TopkArgs a, const TopkPlan p) {
  __shared__ uint32_t h[kBins], hb[kBins];
  const int row = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const int c0 = blockIdx.x * kColsPerBlock;
  const int ncol = row_cols(a, row);
  for (int i = tid; i < kBins; i += kTF) { h[i] = 0u; hb[i] = 0u; }
  __syncthreads();
  const float *srow = a.scores + (size_t)row * a.ld;
  const Ws w = ws_view(a, p);
  const Binning bn = row_binning(w, row);
  float v[kColsPerBlock / kTF];
#pragma unroll
  for (int j = 0; j < kColsPerBlock / kTF; ++j) {
    const int col = c0 + j * kTF + tid;
    v[j] = col < ncol ? srow[col] : -INFINITY;
  }
#pragma unroll
  for (int j = 0; j < kColsPerBlock / kTF; ++j) {
    const uint32_t key = score_key(v[j]);
    hist_add(h, key, bn, lane);
    if (a.P_out > 0) {   // block of 8 consecutive columns = 8 consecutive lanes
      uint32_t bk = key;
      bk = max(bk, __shfl_xor_sync(0xffffffffu, bk, 1));
      bk = max(bk, __shfl_xor_sync(0xffffffffu, bk, 2));
      bk = max(bk, __shfl_xor_sync(0xffffffffu, bk, 4));
      hist_add(hb, (lane & 7) == 0 ? bk : 0u, bn, lane);
    }
  }
  __syncthreads();
  for (int i = tid; i < kBins; i += kTF) {
    if (h[i]) atomicAdd(&w.hist[(size_t)row * kBins + i], h[i]);
    if (a.P_out > 0 && hb[i]) atomicAdd(&w.histb[(size_t)row * kBins + i], hb[i]);
  }
}

__global__ void __launch_bounds__(kTF) topk_filter_kernel(const TopkArgs a, const TopkPlan p) {
  __shared__ int sm_ws[40];
  const int row = blockIdx.y, tid = threadIdx.x, lane = tid & 31;
  const int c0 = blockIdx.x * kColsPerBlock;
  const int ncol = row_cols(a, row);
  const Ws w = ws_view(a, p);
  const Binning bn = row_binning(w, row);
  int T, above, Tb = -1, aboveb = 0;
  find_threshold<kTF>(w.hist + (size_t)row * kBins, a.K, T, above, sm_ws);
  if (a.P_out > 0) find_threshold<kTF>(w.histb + (size_t)row * kBins, a.P_out, Tb, aboveb, sm_ws);
  (void)above;
  (void)aboveb;
  const float *srow = a.scores + (size_t)row * a.ld;
  uint32_t *cnt = w.cnt + (size_t)row * 4;
  float v[kColsPerBlock / kTF];
#pragma unroll
  for (int j = 0; j < kColsPerBlock / kTF; ++j) {
    const int col = c0 + j * kTF + tid;
    v[j] = col < ncol ? srow[col] : -INFINITY;
  }
#pragma unroll
  for (int j = 0; j < kColsPerBlock / kTF; ++j) {
    const int col = c0 + j * kTF + tid;
    const uint32_t key = score_key(v[j]);
    const int bin = key ? bn.digit(key) : -2;
    warp_append(key && bin > T, col, &cnt[0], w.sel + (size_t)row * a.K, lane);
    warp_append(key && bin == T, col, &cnt[1], w.cand + (size_t)row * a.n_cols, lane);
    if (a.P_out > 0) {
      uint32_t bk = key;
      bk = max(bk, __shfl_xor_sync(0xffffffffu, bk, 1));
      bk = max(bk, __shfl_xor_sync(0xffffffffu, bk, 2));
      bk = max(bk, __shfl_xor_sync(0xffffffffu, bk, 4));
      const bool lead = (lane & 7) == 0 && bk != 0u;
      const int bbin = bk ? bn.digit(bk) : -2;
      warp_append(lead && bbin > Tb, col >> 3, &cnt[2], w.selb + (size_t)row * a.P_out, lane);
      warp_append(lead && bbin == Tb, col >> 3, &cnt[3], w.candb + (size_t)row * p.nb, lane);
    }
  }
}

// One part (entries or blocks) of the select kernel: out[0..K) = the K best
// columns in ascending order (-1 padded), from the selected list, the
// candidate list and the key of each candidate column.  The chosen columns
// are marked in a bitmap of the row's columns; a prefix popcount over the
// bitmap gives each one its output position (no sort).
template <class KeyOfCol>
__device__ void select_part(const uint32_t *hist, const int32_t *sel, const int32_t *cand, uint32_t n_cand,
                            int K, int n_cols, KeyOfCol key_of, const int32_t *pool_blocks, int32_t *out,
                            uint32_t *cand_key, int32_t *cand_col, uint32_t *bitmap, uint32_t *hist256,
                            SelState *st, int *red) {
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int nwords = (n_cols + 31) >> 5;
  for (int i = tid; i < nwords; i += kTS) bitmap[i] = 0u;
  int T, above;
  find_threshold<kTS>(hist, K, T, above, red);   // (synchronises: bitmap cleared)
  for (int i = tid; i < above; i += kTS) {
    const int32_t c = sel[i];
    atomicOr(&bitmap[c >> 5], 1u << (c & 31));
  }
  const int need = T < 0 ? 0 : K - above;
  if (need > 0) {
    const int n = (int)n_cand;
    const bool staged = n <= kSmemCands;
    if (staged) {
      for (int i = tid; i < n; i += kTS) {
        const int32_t c = cand[i];
        cand_col[i] = c;
        cand_key[i] = key_of(c);
      }
      __syncthreads();
    }
    auto kf = [&](int i) -> uint32_t { return staged ? cand_key[i] : key_of(cand[i]); };
    auto cf = [&](int i) -> int32_t { return staged ? cand_col[i] : cand[i]; };
    radix_select<kTS>(kf, n, need, hist256, st, red);
    const uint32_t thr = st->thr;
    const int take_eq = st->take_eq;
    // ties at thr: the take_eq smallest columns (skipped when all ties fit)
    int n_eq = 0;
    for (int i = tid; i < n; i += kTS) n_eq += kf(i) == thr;
    n_eq = __reduce_add_sync(0xffffffffu, (unsigned)n_eq);
    if (lane == 0) red[warp] = n_eq;
    __syncthreads();
    n_eq = 0;
#pragma unroll
    for (int w = 0; w < kTS / 32; ++w) n_eq += red[w];
    __syncthreads();
    uint32_t thr2 = 0u;
    auto tf = [&](int i) -> uint32_t { return kf(i) == thr ? 0xFFFFFFFFu - (uint32_t)cf(i) : 0u; };
    if (n_eq > take_eq) {
      radix_select<kTS>(tf, n, take_eq, hist256, st, red);
      thr2 = st->thr;
    }
    for (int i = tid; i < n; i += kTS) {
      const uint32_t k = kf(i);
      if (k > thr || (k == thr && tf(i) >= thr2)) {
        const int32_t c = cf(i);
        atomicOr(&bitmap[c >> 5], 1u << (c & 31));
      }
    }
  }
  __syncthreads();
  // exclusive prefix popcount over the bitmap words (each thread a run of words)
  const int per = (nwords + kTS - 1) / kTS;
  const int w0 = tid * per, w1 = min(w0 + per, nwords);
  int mine = 0;
  for (int wi = w0; wi < w1; ++wi) mine += __popc(bitmap[wi]);
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) red[warp] = incl;
  __syncthreads();
  int before = incl - mine, total = 0;
#pragma unroll
  for (int w = 0; w < kTS / 32; ++w) {
    const int v = red[w];
    if (w < warp) before += v;
    total += v;
  }
  for (int wi = w0; wi < w1; ++wi) {
    uint32_t bits = bitmap[wi];
    while (bits) {
      const int bpos = __ffs(bits) - 1;
      bits &= bits - 1;
      const int c = wi * 32 + bpos;
      if (before < K) out[before] = pool_blocks ? pool_blocks[c >> 3] * 8 + (c & 7) : c;
      ++before;
    }
  }
  for (int i = total + tid; i < K; i += kTS) out[i] = -1;
  __syncthreads();
}

__global__ void __launch_bounds__(kTS) topk_select_kernel(const TopkArgs a, const TopkPlan p) {
  extern __shared__ uint32_t sm3[];
  __shared__ uint32_t hist256[256];
  __shared__ SelState st;
  __shared__ int red[40];
  uint32_t *cand_key = sm3;                                           // [kSmemCands]
  int32_t *cand_col = reinterpret_cast<int32_t *>(sm3 + kSmemCands);  // [kSmemCands]
  uint32_t *bitmap = sm3 + 2 * kSmemCands;                            // [n_cols / 32]
  const int row = blockIdx.x;
  const Ws w = ws_view(a, p);
  const float *srow = a.scores + (size_t)row * a.ld;
  const int ncol = row_cols(a, row);
  const uint32_t *cnt = w.cnt + (size_t)row * 4;
  const int32_t *pb = a.pool_blocks ? a.pool_blocks + (size_t)row * (a.n_cols / 8) : nullptr;

  auto entry_key = [&](int32_t c) -> uint32_t { return c < ncol ? score_key(srow[c]) : 0u; };
  select_part(w.hist + (size_t)row * kBins, w.sel + (size_t)row * a.K, w.cand + (size_t)row * a.n_cols, cnt[1],
              a.K, a.n_cols, entry_key, pb, a.out_idx + (size_t)row * a.K, cand_key, cand_col, bitmap, hist256,
              &st, red);
  if (a.P_out > 0) {
    auto block_key = [&](int32_t blk) -> uint32_t {
      uint32_t m = 0u;
      for (int q = 0; q < 8; ++q) {
        const int c = blk * 8 + q;
        if (c < ncol) m = max(m, score_key(srow[c]));
      }
      return m;
    };
    select_part(w.histb + (size_t)row * kBins, w.selb + (size_t)row * a.P_out, w.candb + (size_t)row * p.nb,
                cnt[3], a.P_out, p.nb, block_key, nullptr, a.out_pool + (size_t)row * a.P_out, cand_key, cand_col,
                bitmap, hist256, &st, red);
  }
}

size_t align16(size_t x) { return (x + 15) & ~size_t(15); }

// ---------------------------------------------------------------------------
// Many long rows (prefill chunks): one block of kRT threads per row and no
// workspace.  The row is read once from HBM and then from L2 (the blocks
// resident at a time hold about 2 x 148 rows, well inside L2).  A radix
// select over the 32-bit keys in digit levels of 11, 11 and 10 bits: a
// level's histogram counts only the keys whose higher digits equal the ones
// fixed so far, and the selection stops as soon as the bin of the K-th key
// is taken whole (after one or two levels for all but heavily tied rows).
// One marking pass then sets a bitmap of the chosen columns (exact ties at
// the last level go to the smaller columns), and a prefix popcount writes
// them in ascending order.
constexpr int kRT = 512;               // threads of the row kernel
constexpr int kRowsMin = 128;          // rows from which the row kernel is used
constexpr int kRowColsMax = 131072;    // a row's bitmaps fit in shared memory

struct RowSel {
  uint32_t prefix, mask;   // key bits fixed so far (mask: the top bits)
  int need;                // keys still to take among those matching prefix
  int done;                // all keys matching prefix are taken
};

// One atomic per distinct bin of the warp's active lanes.
__device__ __forceinline__ void hist_add_match(uint32_t *h, bool act, uint32_t bin, int lane) {
  const unsigned am = __ballot_sync(0xffffffffu, act);
  if (!am) return;
  const unsigned peers = __match_any_sync(0xffffffffu, act ? bin : 0xFFFFFFFFu);
  if (act && (__ffs(peers) - 1) == lane) atomicAdd(&h[bin], (uint32_t)__popc(peers));
}

// Calls f(column, key) for every column of the row, four columns per thread
// and step where the row is 16-byte aligned.  Every thread of the block makes
// the same number of calls (f may use warp collectives): columns past the
// row's end come with key 0 (absent).
template <class F>
__device__ __forceinline__ void for_row(const float *srow, int n, bool vec, F f) {
  const int tid = threadIdx.x;
  if (vec) {
    const int n4 = n >> 2;
    const float4 *r4 = reinterpret_cast<const float4 *>(srow);
    for (int base = 0; base < n4; base += kRT) {
      const int i = base + tid;
      const float4 v = i < n4 ? r4[i] : make_float4(NAN, NAN, NAN, NAN);
      f(4 * i, score_key(v.x));
      f(4 * i + 1, score_key(v.y));
      f(4 * i + 2, score_key(v.z));
      f(4 * i + 3, score_key(v.w));
    }
    const int c = 4 * n4 + tid;   // the last n % 4 columns
    f(c, c < n ? score_key(srow[c]) : 0u);
  } else {
    for (int base = 0; base < n; base += kRT) {
      const int c = base + tid;
      f(c, c < n ? score_key(srow[c]) : 0u);
    }
  }
}

__global__ void __launch_bounds__(kRT, 2) topk_rows_kernel(const TopkArgs a) {
  extern __shared__ uint32_t smr[];
  const int nwords = (a.n_cols + 31) >> 5;
  uint32_t *hist = smr;                       // [kBins]
  uint32_t *bitmap = smr + kBins;             // [nwords] chosen columns
  uint32_t *tiemap = bitmap + nwords;         // [nwords] exact ties at the last level
  __shared__ RowSel st;
  __shared__ int red[40];
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float *srow = a.scores + (size_t)row * a.ld;
  const int n = row_cols(a, row);
  const bool vec = (a.ld & 3) == 0;
  for (int i = tid; i < nwords; i += kRT) { bitmap[i] = 0u; tiemap[i] = 0u; }
  if (tid == 0) { st.prefix = 0u; st.mask = 0u; st.need = a.K; st.done = 0; }
  __syncthreads();
#pragma unroll 1
  for (int lv = 0; lv < 3; ++lv) {
    const int sh = lv == 0 ? 21 : (lv == 1 ? 10 : 0);
    const uint32_t dm = lv == 2 ? 0x3FFu : 0x7FFu;
    for (int i = tid; i < kBins; i += kRT) hist[i] = 0u;
    __syncthreads();
    const uint32_t prefix = st.prefix, mask = st.mask;
    for_row(srow, n, vec, [&](int, uint32_t key) {
      const bool act = key != 0u && (key & mask) == prefix;
      hist_add_match(hist, act, (key >> sh) & dm, lane);
    });
    __syncthreads();
    int T, above;
    find_threshold<kRT>(hist, st.need, T, above, red);
    if (tid == 0) {
      if (T < 0) {
        st.done = 1;   // the matching keys are fewer than need: all taken
      } else {
        st.need -= above;
        st.prefix |= (uint32_t)T << sh;
        st.mask |= dm << sh;
        if (hist[T] == (uint32_t)st.need) st.done = 1;
      }
    }
    __syncthreads();
    if (st.done) break;
  }
  // marking pass: keys above the fixed digits, and the matching ones (all of
  // them when done, else exact ties: the need smallest columns)
  {
    const uint32_t prefix = st.prefix, mask = st.mask;
    const bool done = st.done != 0;
    for_row(srow, n, vec, [&](int c, uint32_t key) {
      if (key == 0u) return;
      const uint32_t top = key & mask;
      if (top > prefix || (done && top == prefix)) atomicOr(&bitmap[c >> 5], 1u << (c & 31));
      else if (top == prefix) atomicOr(&tiemap[c >> 5], 1u << (c & 31));
    });
  }
  __syncthreads();
  const int per = (nwords + kRT - 1) / kRT;
  const int w0 = tid * per, w1 = min(w0 + per, nwords);
  if (!st.done) {   // the first need tie columns join the chosen ones
    int mine = 0;
    for (int wi = w0; wi < w1; ++wi) mine += __popc(tiemap[wi]);
    int incl = mine;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += y;
    }
    if (lane == 31) red[warp] = incl;
    __syncthreads();
    int before = incl - mine;
#pragma unroll
    for (int w = 0; w < kRT / 32; ++w)
      if (w < warp) before += red[w];
    const int need = st.need;
    for (int wi = w0; wi < w1 && before < need; ++wi) {
      uint32_t bits = tiemap[wi], take = 0u;
      while (bits && before < need) {
        const uint32_t b = bits & (0u - bits);
        take |= b;
        bits ^= b;
        ++before;
      }
      bitmap[wi] |= take;
    }
    __syncthreads();
  }
  // ascending output by prefix popcount over the chosen columns
  int mine = 0;
  for (int wi = w0; wi < w1; ++wi) mine += __popc(bitmap[wi]);
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += y;
  }
  if (lane == 31) red[warp] = incl;
  __syncthreads();
  int before = incl - mine, total = 0;
#pragma unroll
  for (int w = 0; w < kRT / 32; ++w) {
    const int v = red[w];
    if (w < warp) before += v;
    total += v;
  }
  int32_t *out = a.out_idx + (size_t)row * a.K;
  const int32_t *pb = a.pool_blocks ? a.pool_blocks + (size_t)row * (a.n_cols / 8) : nullptr;
  for (int wi = w0; wi < w1; ++wi) {
    uint32_t bits = bitmap[wi];
    while (bits) {
      const int bpos = __ffs(bits) - 1;
      bits &= bits - 1;
      const int c = wi * 32 + bpos;
      if (before < a.K) out[before] = pb ? pb[c >> 3] * 8 + (c & 7) : c;
      ++before;
    }
  }
  for (int i = total + tid; i < a.K; i += kRT) out[i] = -1;
}

bool topk_rows_path(int rows, int n_cols, int P_out) {
  return rows >= kRowsMin && !topk_cluster_fits(n_cols) && n_cols <= kRowColsMax && P_out == 0;
}

}  // namespace

TopkPlan plan_topk(int rows, int n_cols, int K, int P_out) {
  TopkPlan p{};
  if (topk_cluster_fits(n_cols) || topk_rows_path(rows, n_cols, P_out)) return p;   // no workspace
  p.nchunks = n_cols > 0 ? (n_cols + kColsPerBlock - 1) / kColsPerBlock : 1;
  p.nb = (n_cols + 7) / 8;
  const size_t R = (size_t)(rows > 0 ? rows : 0);
  size_t o = 0;
  p.off_hist = o;
  o += R * kBins * 4;
  p.off_histb = o;
  if (P_out > 0) o += R * kBins * 4;
  p.off_cnt = o;
  o += R * 4 * 4;
  p.off_range = o;
  o += R * 2 * 4;
  p.zero_bytes = o;
  o = align16(o);
  p.off_sel = o;
  o = align16(o + R * K * 4);
  p.off_cand = o;
  o = align16(o + R * (size_t)n_cols * 4);
  p.off_selb = o;
  if (P_out > 0) o = align16(o + R * P_out * 4);
  p.off_candb = o;
  if (P_out > 0) o = align16(o + R * (size_t)p.nb * 4);
  p.bytes = o;
  return p;
}

cudaError_t launch_topk(const TopkArgs &a, const TopkPlan &p, cudaStream_t s) {
  if (topk_cluster_fits(a.n_cols)) return launch_topk_cluster(a, s);
  if (topk_rows_path(a.rows, a.n_cols, a.P_out)) {
    const size_t sm = sizeof(uint32_t) * (kBins + 2 * (((size_t)a.n_cols + 31) / 32));
    cudaError_t e = cudaFuncSetAttribute(topk_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
    if (e != cudaSuccess) return e;
    topk_rows_kernel<<<a.rows, kRT, sm, s>>>(a);
    return cudaGetLastError();
  }
  cudaError_t e = cudaMemsetAsync(a.ws, 0, p.zero_bytes, s);
  if (e != cudaSuccess) return e;
  if (a.n_cols > 0) {
    const dim3 grid(p.nchunks, a.rows);
    topk_range_kernel<<<grid, kTF, 0, s>>>(a, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    topk_hist_kernel<<<grid, kTF, 0, s>>>(a, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    topk_filter_kernel<<<grid, kTF, 0, s>>>(a, p);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
  }
  // candidates staged + a bitmap of the row's columns (bits)
  const size_t sm = sizeof(uint32_t) * (2 * (size_t)kSmemCands + ((size_t)a.n_cols + 31) / 32 + 1);
  if (sm > 227 * 1024) return cudaErrorInvalidValue;
  e = cudaFuncSetAttribute(topk_select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
  if (e != cudaSuccess) return e;
  topk_select_kernel<<<a.rows, kTS, sm, s>>>(a, p);
  return cudaGetLastError();
}

}  // namespace csa2
