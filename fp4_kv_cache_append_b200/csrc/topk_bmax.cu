// Top-K selection and the hierarchical pool from the Full scan's block
// maxima: the first selection level runs in the scan's epilogue, which writes,
// next to each score, the maximum of every block of 8 entries.
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2": Top-512 per
//   Full layer; the first Full decoder layer's pool of 2,048 blocks x 8
//   positions (paper sec. 2.3.2, 4.2.1, Fig. 5).
// Same contract as csa2_topk (score descending, ties -> smaller column,
// non-finite = absent, ascending output, -1 padding; block score = max of
// its present columns).
//
// One 512-thread block per row.  Thread t holds the keys of blocks
// 32t .. 32t+31 (order-preserving 32-bit keys of the block maxima, 0 =
// absent).  Two selections run side by side over them:
//   * the pool: the P_out blocks with the largest maxima;
//   * tau: the K-th largest block maximum.
// A selection bins the keys by VALUE, linearly between the smallest and the
// largest present value (256 bins, shared-memory atomics: values spread over
// the bins, so few atomics collide), finds the bin holding the k-th largest
// key, and ranks that bin's keys exactly (key desc, column asc) -- scores of
// a row sit in a few binades, so binning by key bits would put nearly all of
// them in one bin.  A bin of more than kColl keys (heavy ties, or one huge
// outlier squeezing the rest into one bin) is resolved by a radix selection on
// the key bits instead.
// There are at least K distinct entries scoring >= tau (one per block whose
// maximum is >= tau), so the K-th largest score s_K >= tau, and every entry
// of the Top-K lies in a block whose maximum is >= s_K >= tau.  The entries
// of those blocks that score >= tau are the candidates (usually a little over
// K); they are gathered in column order into shared memory and selected
// exactly.  Rows whose candidate blocks hold more than kCap entries (heavy
// ties at tau) select over the whole row instead, reading it from global
// memory once per round.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

namespace {

constexpr int kT = 512;
constexpr int kW = kT / 32;
constexpr int kBpt = 32;           // block maxima per thread: rows of up to 16,384 blocks
constexpr int kCap = 8192;         // candidate entries in shared memory
constexpr int kCpt = kCap / kT;    // candidates per thread

__device__ __forceinline__ uint32_t skey(float f) {
  if (!isfinite(f)) return 0u;   // absent
  if (f == 0.0f) f = 0.0f;       // -0 == +0
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ float kval(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

constexpr int kColl = 2048;        // largest value bin ranked exactly

// Final rule of a selection: take key if key > kthr, or key == kthr and
// (cmode: its column <= cthr; else: its rank among the keys equal to kthr, in
// column order, is below take_eq).
struct SelRule {
  uint32_t kthr;
  int cthr;
  int take_eq;
  int cmode;
};

struct SelSmem {
  uint32_t hist[2][256];             // radix rounds
  uint32_t vhist[256][8];            // value bins, 8 copies per bin (fewer colliding atomics)
  uint32_t prefix[2], mask[2];
  int need[2], done[2];
  SelRule rule[2];
  unsigned long long red[kW];
  int n_present;
  uint32_t kmin, kmax;               // smallest / largest present key
  int vbin_ok;                       // the value range gives usable bins
  int T[2], cnt[2], n_coll[2], fallback[2];
  uint2 coll[2][kColl];              // (key, column) of the threshold bin
};

struct MergeSmem {
  SelSmem sel;
  uint32_t key[kBpt * kT];
};

struct Smem {
  SelSmem sel;
  uint32_t bkey[kBpt * kT];          // block-maximum keys (SmemKeys layout)
  uint32_t cand_key[kCap];           // candidate keys (SmemKeys layout)
  int32_t cand_blk[kCap / 8];        // candidate blocks, ascending
};

// Exclusive block scan of v; afterwards red[kW-1] holds the block total.
__device__ __forceinline__ unsigned long long block_scan(unsigned long long v, unsigned long long *red, int lane,
                                                         int warp) {
  unsigned long long x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  __syncthreads();   // the previous scan's readers of red are done
  if (lane == 31) red[warp] = x;
  __syncthreads();
  if (warp == 0) {
    unsigned long long w = red[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const unsigned long long y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    red[lane] = w;
  }
  __syncthreads();
  return (warp ? red[warp - 1] : 0ull) + x - v;
}

// Keys in shared memory: thread t's element i is column t * npt + i and
// lives at k[i * kT + t] (consecutive threads read consecutive words).  The
// loops stay rolled: each block runs this code once, so its size costs as
// much as its execution.
struct SmemKeys {
  const uint32_t *k;
  int npt, t;
  __device__ __forceinline__ int col(int i) const { return t * npt + i; }
  template <typename F>
  __device__ __forceinline__ void each(F f) const {
#pragma unroll 1
    for (int i = 0; i < npt; ++i) f(k[i * kT + t], i);
  }
};

// Keys of a score row read from global memory: thread t's element i is
// column t * npt + i (columns >= n absent).
struct RowKeys {
  const float *row;
  int n, npt, t;
  __device__ __forceinline__ int col(int i) const { return t * npt + i; }
  template <typename F>
  __device__ __forceinline__ void each(F f) const {
#pragma unroll 1
    for (int i = 0; i < npt; ++i) {
      const int c = t * npt + i;
      f(c < n ? skey(__ldcg(row + c)) : 0u, i);
    }
  }
};

// NS (1 or 2) radix selections over the same keys: selection s finds the
// k[s]-th largest present key.  Afterwards sm.rule[s] decides every key.
template <int NS, typename Keys>
__device__ void radix_select(const Keys &keys, const int *k, SelSmem &sm, int tid, int lane, int warp) {
  // present keys
  int mine = 0;
  keys.each([&](uint32_t key, int) { mine += key != 0u; });
  const unsigned long long ex = block_scan((unsigned long long)mine, sm.red, lane, warp);
  (void)ex;
  if (tid < NS) {
    const int present = (int)sm.red[kW - 1];
    sm.prefix[tid] = 0u;
    sm.mask[tid] = 0u;
    sm.need[tid] = k[tid];
    sm.done[tid] = present <= k[tid];
    sm.rule[tid].kthr = 0u;        // take every present key
    sm.rule[tid].cthr = 0;
    sm.rule[tid].take_eq = 0;
    sm.rule[tid].cmode = 0;
    if (tid == 0) sm.n_present = present;
  }
  __syncthreads();
#pragma unroll 1
  for (int shift = 24; shift >= 0; shift -= 8) {
    if (sm.done[0] && (NS == 1 || sm.done[1])) break;   // block-uniform
    if (tid < 256 * NS) (&sm.hist[0][0])[tid] = 0u;
    __syncthreads();
    uint32_t pf[NS], mk[NS];
    bool act[NS];
#pragma unroll
    for (int s = 0; s < NS; ++s) { pf[s] = sm.prefix[s]; mk[s] = sm.mask[s]; act[s] = !sm.done[s]; }
    keys.each([&](uint32_t key, int) {
#pragma unroll
      for (int s = 0; s < NS; ++s) {
        const bool in = act[s] && key != 0u && (key & mk[s]) == pf[s];
        const int bin = in ? (int)((key >> shift) & 255u) : -1;
        const uint32_t peers = __match_any_sync(0xffffffffu, bin);
        if (in && (__ffs(peers) - 1) == lane) atomicAdd(&sm.hist[s][bin], (uint32_t)__popc(peers));
      }
    });
    __syncthreads();
    if (warp < NS && !sm.done[warp]) {   // warp s: the bin holding the need-th largest key
      const int s = warp;
      uint32_t v[8];
      uint32_t lsum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) { v[i] = sm.hist[s][255 - 8 * lane - i]; lsum += v[i]; }
      uint32_t cum = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, cum, o);
        if (lane >= o) cum += y;
      }
      const int need = sm.need[s];
      const uint32_t before = cum - lsum;
      if ((int)before < need && (int)cum >= need) {   // exactly one lane
        uint32_t acc = before;
        int bin = 0;
        uint32_t cnt = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if ((int)(acc + v[i]) >= need) { bin = 255 - 8 * lane - i; cnt = v[i]; break; }
          acc += v[i];
        }
        const int need2 = need - (int)acc;   // 1 <= need2 <= cnt
        const uint32_t prefix = sm.prefix[s] | ((uint32_t)bin << shift);
        sm.prefix[s] = prefix;
        sm.mask[s] |= 0xFFu << shift;
        sm.need[s] = need2;
        if ((int)cnt == need2) {            // every key of the bin is taken
          sm.rule[s].kthr = prefix;
          sm.rule[s].take_eq = 0x7FFFFFFF;
          sm.rule[s].cmode = 0;
          sm.done[s] = 1;
        } else if (shift == 0) {            // one key value: need2 of its ties, in column order
          sm.rule[s].kthr = prefix;
          sm.rule[s].take_eq = need2;
          sm.rule[s].cmode = 0;
          sm.done[s] = 1;
        }
      }
    }
    __syncthreads();
  }
}

// Keys taken whatever their rank among ties, and keys among which the rank
// decides (ties of a take_eq rule).
__device__ __forceinline__ bool strictly_taken(uint32_t key, int col, const SelRule &r) {
  return key != 0u && (key > r.kthr || (r.cmode && key == r.kthr && col <= r.cthr));
}
__device__ __forceinline__ bool tie(uint32_t key, const SelRule &r) { return !r.cmode && key != 0u && key == r.kthr; }

// Output positions of this thread's taken keys: the number of taken keys in
// earlier columns.  Returns (position of my first taken key, ties before me).
template <typename Keys>
__device__ void taken_offsets(const Keys &keys, const SelRule &rule, unsigned long long *red, int lane, int warp,
                              int &pos, int &ties_before) {
  int st = 0, tt = 0;
  keys.each([&](uint32_t key, int i) {
    st += strictly_taken(key, keys.col(i), rule);
    tt += tie(key, rule);
  });
  const unsigned long long ex = block_scan(((unsigned long long)tt << 32) | (unsigned long long)st, red, lane, warp);
  ties_before = (int)(ex >> 32);
  pos = (int)(ex & 0xFFFFFFFFull) + min(ties_before, rule.take_eq);
}

// Visits this thread's taken keys in column order: f(key, i, position).
template <typename Keys, typename F>
__device__ void for_taken(const Keys &keys, const SelRule &rule, unsigned long long *red, int lane, int warp, F f) {
  int pos, tb;
  taken_offsets(keys, rule, red, lane, warp, pos, tb);
  keys.each([&](uint32_t key, int i) {
    const bool tk = strictly_taken(key, keys.col(i), rule) || (tie(key, rule) && tb < rule.take_eq);
    tb += tie(key, rule);
    if (tk) f(key, i, pos++);
  });
}

__device__ __forceinline__ int vbin(uint32_t key, float vlo, float inv) {
  const int b = (int)((kval(key) - vlo) * inv);
  return b < 0 ? 0 : (b > 255 ? 255 : b);
}

// NS selections over the same keys (see the file comment): selection s finds
// the k[s]-th largest present key; afterwards sm.rule[s] decides every key.
template <int NS, typename Keys>
__device__ void vselect(const Keys &keys, const int *k, SelSmem &sm, int tid, int lane, int warp) {
  // present count, smallest and largest key
  uint32_t mn = 0xFFFFFFFFu, mx = 0u;
  int mine = 0;
  keys.each([&](uint32_t key, int) {
    if (key) { mn = min(mn, key); mx = max(mx, key); ++mine; }
  });
  mn = __reduce_min_sync(0xffffffffu, mn);
  mx = __reduce_max_sync(0xffffffffu, mx);
  if (tid == 0) { sm.kmin = 0xFFFFFFFFu; sm.kmax = 0u; }
  block_scan((unsigned long long)mine, sm.red, lane, warp);   // its barriers order the resets above
  if (lane == 0) { atomicMin(&sm.kmin, mn); atomicMax(&sm.kmax, mx); }
  for (int i = tid; i < 256 * 8; i += kT) (&sm.vhist[0][0])[i] = 0u;
  if (tid < NS) {
    const int present = (int)sm.red[kW - 1];
    sm.done[tid] = present <= k[tid];
    sm.rule[tid].kthr = 0u;        // take every present key
    sm.rule[tid].cthr = 0;
    sm.rule[tid].take_eq = 0;
    sm.rule[tid].cmode = 0;
    sm.fallback[tid] = 0;
    sm.n_coll[tid] = 0;
    if (tid == 0) sm.n_present = present;
  }
  __syncthreads();
  if (sm.done[0] && (NS == 1 || sm.done[1])) return;
  const float vlo = kval(sm.kmin), span = kval(sm.kmax) - vlo;
  const float inv = 256.0f / span;
  const bool ok = span > 0.f && isfinite(span) && isfinite(inv);
  if (ok) {   // value-bin histogram (one for every selection)
    keys.each([&](uint32_t key, int) {
      if (key) atomicAdd(&sm.vhist[vbin(key, vlo, inv)][lane & 7], 1u);
    });
  }
  __syncthreads();
  if (warp < NS && !sm.done[warp]) {   // warp s: the value bin holding the k-th largest key
    const int s = warp;
    if (!ok) {
      if (lane == 0) sm.fallback[s] = 1;
    } else {
      uint32_t v[8], lsum = 0;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 c0 = *reinterpret_cast<const uint4 *>(&sm.vhist[255 - 8 * lane - i][0]);
        const uint4 c1 = *reinterpret_cast<const uint4 *>(&sm.vhist[255 - 8 * lane - i][4]);
        v[i] = c0.x + c0.y + c0.z + c0.w + c1.x + c1.y + c1.z + c1.w;
        lsum += v[i];
      }
      uint32_t cum = lsum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, cum, o);
        if (lane >= o) cum += y;
      }
      const int need = k[s];
      const uint32_t before = cum - lsum;
      if ((int)before < need && (int)cum >= need) {
        uint32_t acc = before;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if ((int)(acc + v[i]) >= need) {
            sm.T[s] = 255 - 8 * lane - i;
            sm.cnt[s] = (int)v[i];
            sm.need[s] = need - (int)acc;   // 1 <= need <= cnt
            sm.fallback[s] = (int)v[i] > kColl;
            break;
          }
          acc += v[i];
        }
      }
    }
  }
  __syncthreads();
  // collect the threshold bin's (key, column) pairs
  if (ok) {
    keys.each([&](uint32_t key, int i) {
      if (key) {
        const int bb = vbin(key, vlo, inv);
#pragma unroll
        for (int s = 0; s < NS; ++s) {
          if (!sm.done[s] && !sm.fallback[s] && bb == sm.T[s]) {
            const int slot = atomicAdd(&sm.n_coll[s], 1);
            sm.coll[s][slot] = make_uint2(key, (uint32_t)keys.col(i));
          }
        }
      }
    });
  }
  __syncthreads();
  // rank them exactly (key desc, column asc); the need-th one sets the rule
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    if (sm.done[s] || sm.fallback[s]) continue;
    const int n = sm.n_coll[s];
    for (int i = tid; i < n; i += kT) {
      const uint2 me = sm.coll[s][i];
      int rank = 0;
      for (int j = 0; j < n; ++j) {
        const uint2 o = sm.coll[s][j];
        rank += (o.x > me.x) || (o.x == me.x && o.y < me.y);
      }
      if (rank == sm.need[s] - 1) {   // exactly one pair
        sm.rule[s].kthr = me.x;
        sm.rule[s].cthr = (int)me.y;
        sm.rule[s].take_eq = 0;
        sm.rule[s].cmode = 1;
      }
    }
  }
  __syncthreads();
  // rare: a bin too large to rank (or no usable value range) -> key-bit radix
#pragma unroll
  for (int s = 0; s < NS; ++s) {
    if (sm.done[s] || !sm.fallback[s]) continue;   // block-uniform
    const int kk[1] = {k[s]};
    SelRule keep[2] = {sm.rule[0], sm.rule[1]};
    radix_select<1>(keys, kk, sm, tid, lane, warp);
    const SelRule r = sm.rule[0];
    __syncthreads();
    if (tid == 0) {
      sm.rule[0] = keep[0];
      sm.rule[1] = keep[1];
      sm.rule[s] = r;
    }
    __syncthreads();
  }
}

}  // namespace

__global__ void __launch_bounds__(kT, 1) topk_bmax_kernel(const TopkBmaxArgs a) {
  extern __shared__ uint8_t smem_raw[];
  Smem &sh = *reinterpret_cast<Smem *>(smem_raw);
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();
  pdl_wait();
  int n = a.n_valid ? a.n_valid[row] : a.n_cols;
  if (n > a.n_cols) n = a.n_cols;
  if (n < 0) n = 0;
  const int nb = (n + 7) / 8;
  const float *bm = a.bmax + (size_t)row * a.ld_b;
  const float *sc = a.scores + (size_t)row * a.ld;
  int32_t *out = a.out_idx + (size_t)row * a.K;

  // ---- block-maximum keys, 32 consecutive blocks per thread
#pragma unroll 1
  for (int i = 0; i < kBpt; i += 4) {
    const int b0 = tid * kBpt + i;
    float4 v = make_float4(NAN, NAN, NAN, NAN);
    if (b0 + 3 < nb) v = __ldcg(reinterpret_cast<const float4 *>(bm + b0));
    else {
      if (b0 < nb) v.x = __ldcg(bm + b0);
      if (b0 + 1 < nb) v.y = __ldcg(bm + b0 + 1);
      if (b0 + 2 < nb) v.z = __ldcg(bm + b0 + 2);
    }
    sh.bkey[i * kT + tid] = skey(v.x);
    sh.bkey[(i + 1) * kT + tid] = skey(v.y);
    sh.bkey[(i + 2) * kT + tid] = skey(v.z);
    sh.bkey[(i + 3) * kT + tid] = skey(v.w);
  }
  const SmemKeys bk{sh.bkey, kBpt, tid};   // each thread reads only its own keys

  // ---- pool (selection 1, when asked) and tau (selection 0)
  const int ks[2] = {a.K, a.P_out};
  if (a.P_out > 0) vselect<2>(bk, ks, sh.sel, tid, lane, warp);
  else vselect<1>(bk, ks, sh.sel, tid, lane, warp);
  const SelRule tau = sh.sel.rule[0];
  const bool few_blocks = sh.sel.n_present <= a.K;   // every present block is a candidate
  if (a.P_out > 0) {
    const SelRule pr = sh.sel.rule[1];
    const int n_pool = min(sh.sel.n_present, a.P_out);
    int32_t *op = a.out_pool + (size_t)row * a.P_out;
    float *ops = a.out_pool_scores ? a.out_pool_scores + (size_t)row * a.P_out : nullptr;
    for_taken(bk, pr, sh.sel.red, lane, warp, [&](uint32_t key, int i, int pos) {
      if (pos < a.P_out) {
        op[pos] = bk.col(i);
        if (ops) ops[pos] = kval(key);
      }
    });
    for (int i = n_pool + tid; i < a.P_out; i += kT) {
      op[i] = -1;
      if (ops) ops[i] = -INFINITY;
    }
  }

  // ---- candidate blocks: maximum >= tau (every present block when fewer than K)
  const uint32_t tkey = few_blocks ? 1u : tau.kthr;
  int mine = 0;
  bk.each([&](uint32_t key, int) { mine += key != 0u && key >= tkey; });
  const int cb0 = (int)block_scan((unsigned long long)mine, sh.sel.red, lane, warp);
  const int n_cb = (int)sh.sel.red[kW - 1];
  int K_take;
  float *osc = a.out_scores ? a.out_scores + (size_t)row * a.K : nullptr;
  if (n_cb * 8 <= kCap) {
    // the candidate blocks in ascending order, then their scores loaded by
    // all threads at once; entries below tau (or beyond the row) cannot be
    // selected.  Candidate position j (column order) is element j % kCpt of
    // thread j / kCpt.
    int slot = cb0;
    bk.each([&](uint32_t key, int i) {
      if (key != 0u && key >= tkey) sh.cand_blk[slot++] = bk.col(i);
    });
    __syncthreads();
#pragma unroll 1
    for (int j = tid; j < kCap; j += kT) {
      uint32_t key = 0u;
      if (j < n_cb * 8) {
        const int col = sh.cand_blk[j >> 3] * 8 + (j & 7);
        key = col < n ? skey(__ldcg(sc + col)) : 0u;
      }
      sh.cand_key[(j % kCpt) * kT + j / kCpt] = key >= tkey ? key : 0u;
    }
    __syncthreads();
    const SmemKeys cks{sh.cand_key, kCpt, tid};
    vselect<1>(cks, ks, sh.sel, tid, lane, warp);
    const SelRule rule = sh.sel.rule[0];
    K_take = min(sh.sel.n_present, a.K);
    for_taken(cks, rule, sh.sel.red, lane, warp, [&](uint32_t key, int i, int pos) {
      if (pos < a.K) {
        const int j = cks.col(i);
        out[pos] = sh.cand_blk[j >> 3] * 8 + (j & 7);
        if (osc) osc[pos] = kval(key);
      }
    });
  } else {
    // heavy ties at tau: select over the whole row
    const RowKeys rk{sc, n, (n + kT - 1) / kT, tid};
    radix_select<1>(rk, ks, sh.sel, tid, lane, warp);
    const SelRule rule = sh.sel.rule[0];
    K_take = min(sh.sel.n_present, a.K);
    for_taken(rk, rule, sh.sel.red, lane, warp, [&](uint32_t key, int i, int pos) {
      if (pos < a.K) {
        out[pos] = rk.col(i);
        if (osc) osc[pos] = kval(key);
      }
    });
  }
  for (int i = K_take + tid; i < a.K; i += kT) {
    out[i] = -1;
    if (osc) osc[i] = -INFINITY;
  }
}

// ---------------------------------------------------------------------------
// Merge of per-shard selections (a context split over several GPUs): row r's
// candidates are G segments of n_seg (score, id) pairs, segment g at
// [g][rows][n_seg]; candidate (g, i) stands for entry ids[g][r][i] +
// seg_base[g] (ids < 0: none).  The K best by (score desc, entry asc), listed
// ascending, -1 / -inf padded.  Each segment's ids ascend and the segments'
// entry ranges ascend with g, so candidate order is entry order and the
// selection's column tie rule is the entry tie rule.
__global__ void __launch_bounds__(kT, 1) topk_merge_kernel(const TopkMergeArgs a) {
  extern __shared__ uint8_t smem_raw[];
  MergeSmem &ms = *reinterpret_cast<MergeSmem *>(smem_raw);
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();
  pdl_wait();
  const int n = a.G * a.n_seg;
  // candidate j (segment-major order = entry order) is element j % kBpt of thread j / kBpt
#pragma unroll 1
  for (int j = tid; j < kBpt * kT; j += kT) {
    uint32_t key = 0u;
    if (j < n) {
      const int g = j / a.n_seg, c = j % a.n_seg;
      const size_t at = ((size_t)g * a.rows + row) * a.n_seg + c;
      if (a.ids[at] >= 0) key = skey(a.scores[at]);
    }
    ms.key[(j % kBpt) * kT + j / kBpt] = key;
  }
  __syncthreads();
  const SmemKeys ks{ms.key, kBpt, tid};
  const int k[1] = {a.K};
  vselect<1>(ks, k, ms.sel, tid, lane, warp);
  const SelRule rule = ms.sel.rule[0];
  const int K_take = min(ms.sel.n_present, a.K);
  int32_t *out = a.out_ids + (size_t)row * a.K;
  float *osc = a.out_scores ? a.out_scores + (size_t)row * a.K : nullptr;
  for_taken(ks, rule, ms.sel.red, lane, warp, [&](uint32_t kk, int i, int pos) {
    if (pos < a.K) {
      const int j = ks.col(i), g = j / a.n_seg, c = j % a.n_seg;
      out[pos] = a.ids[((size_t)g * a.rows + row) * a.n_seg + c] + a.seg_base[g];
      if (osc) osc[pos] = kval(kk);
    }
  });
  for (int i = K_take + tid; i < a.K; i += kT) {
    out[i] = -1;
    if (osc) osc[i] = -INFINITY;
  }
}

cudaError_t launch_topk_merge(const TopkMergeArgs &a, cudaStream_t s) {
  const size_t smem = sizeof(MergeSmem);
  cudaError_t e = cudaFuncSetAttribute(topk_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_merge_kernel, dim3(a.rows), dim3(kT), smem, s, dim3(1, 1, 1), a);
}

size_t topk_bmax_smem() { return sizeof(Smem); }

cudaError_t launch_topk_bmax(const TopkBmaxArgs &a, cudaStream_t s) {
  const size_t smem = sizeof(Smem);
  cudaError_t e = cudaFuncSetAttribute(topk_bmax_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  return launch_pdl(topk_bmax_kernel, dim3(a.rows), dim3(kT), smem, s, dim3(1, 1, 1), a);
}

}  // namespace csa2
