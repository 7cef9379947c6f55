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
// One 1024-thread block per row.  Thread t holds the keys of blocks
// 16t .. 16t+15 (order-preserving 32-bit keys of the block maxima, 0 =
// absent).  Two radix selections run side by side over them, 8 key bits per
// round (histograms in shared memory, warp-aggregated atomics):
//   * the pool: the P_out blocks with the largest maxima;
//   * tau: the K-th largest block maximum.
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

constexpr int kT = 1024;
constexpr int kW = kT / 32;
constexpr int kBpt = 16;           // block maxima per thread: rows of up to 16,384 blocks
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

// Final rule of a selection: take key if key > kthr, or key == kthr and its
// rank among the keys equal to kthr (in column order) is below take_eq.
struct SelRule {
  uint32_t kthr;
  int take_eq;
};

struct SelSmem {
  uint32_t hist[2][256];
  uint32_t prefix[2], mask[2];
  int need[2], done[2];
  SelRule rule[2];
  unsigned long long red[kW];
  int n_present;
};

struct Smem {
  SelSmem sel;
  uint32_t cand_key[kCap];
  int32_t cand_col[kCap];
  int n_cand_blocks;
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

// Keys held in registers: thread t's element i is column t * N + i.
template <int N>
struct RegKeys {
  const uint32_t *k;
  template <typename F>
  __device__ __forceinline__ void each(F f) const {
#pragma unroll
    for (int i = 0; i < N; ++i) f(k[i], i);
  }
};

// Keys of a score row read from global memory: thread t's element i is
// column t * npt + i (columns >= n absent).
struct RowKeys {
  const float *row;
  int n, npt, t;
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
    sm.rule[tid].take_eq = 0;
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
          sm.done[s] = 1;
        } else if (shift == 0) {            // one key value: need2 of its ties, in column order
          sm.rule[s].kthr = prefix;
          sm.rule[s].take_eq = need2;
          sm.done[s] = 1;
        }
      }
    }
    __syncthreads();
  }
}

__device__ __forceinline__ bool strictly_taken(uint32_t key, const SelRule &r) { return key != 0u && key > r.kthr; }
__device__ __forceinline__ bool tie(uint32_t key, const SelRule &r) { return key != 0u && key == r.kthr; }

// Output positions of this thread's taken keys: the number of taken keys in
// earlier columns.  Returns (position of my first taken key, ties before me).
template <typename Keys>
__device__ void taken_offsets(const Keys &keys, const SelRule &rule, unsigned long long *red, int lane, int warp,
                              int &pos, int &ties_before) {
  int st = 0, tt = 0;
  keys.each([&](uint32_t key, int) {
    st += strictly_taken(key, rule);
    tt += tie(key, rule);
  });
  const unsigned long long ex = block_scan(((unsigned long long)tt << 32) | (unsigned long long)st, red, lane, warp);
  ties_before = (int)(ex >> 32);
  pos = (int)(ex & 0xFFFFFFFFull) + min(ties_before, rule.take_eq);
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

  // ---- block-maximum keys, 16 consecutive blocks per thread
  uint32_t bkey[kBpt];
#pragma unroll
  for (int i = 0; i < kBpt; i += 4) {
    const int b0 = tid * kBpt + i;
    float4 v = make_float4(NAN, NAN, NAN, NAN);
    if (b0 + 3 < nb) v = __ldcg(reinterpret_cast<const float4 *>(bm + b0));
    else {
      if (b0 < nb) v.x = __ldcg(bm + b0);
      if (b0 + 1 < nb) v.y = __ldcg(bm + b0 + 1);
      if (b0 + 2 < nb) v.z = __ldcg(bm + b0 + 2);
    }
    bkey[i] = skey(v.x); bkey[i + 1] = skey(v.y); bkey[i + 2] = skey(v.z); bkey[i + 3] = skey(v.w);
  }
  const RegKeys<kBpt> bk{bkey};

  // ---- pool (selection 1, when asked) and tau (selection 0)
  const int ks[2] = {a.K, a.P_out};
  if (a.P_out > 0) radix_select<2>(bk, ks, sh.sel, tid, lane, warp);
  else radix_select<1>(bk, ks, sh.sel, tid, lane, warp);
  const SelRule tau = sh.sel.rule[0];
  if (a.P_out > 0) {
    const SelRule pr = sh.sel.rule[1];
    const int n_pool = min(sh.sel.n_present, a.P_out);
    int pos, tb;
    taken_offsets(bk, pr, sh.sel.red, lane, warp, pos, tb);
    int32_t *op = a.out_pool + (size_t)row * a.P_out;
#pragma unroll
    for (int i = 0; i < kBpt; ++i) {
      const uint32_t key = bkey[i];
      const bool tk = strictly_taken(key, pr) || (tie(key, pr) && tb < pr.take_eq);
      tb += tie(key, pr);
      if (tk) {
        if (pos < a.P_out) {
          op[pos] = tid * kBpt + i;
          if (a.out_pool_scores) a.out_pool_scores[(size_t)row * a.P_out + pos] = kval(key);
        }
        ++pos;
      }
    }
    for (int i = n_pool + tid; i < a.P_out; i += kT) {
      op[i] = -1;
      if (a.out_pool_scores) a.out_pool_scores[(size_t)row * a.P_out + i] = -INFINITY;
    }
  }

  // ---- candidate blocks: maximum >= tau (every block when fewer than K are present)
  const uint32_t tkey = sh.sel.n_present <= a.K ? 1u : tau.kthr;
  int mine = 0;
#pragma unroll
  for (int i = 0; i < kBpt; ++i) mine += bkey[i] != 0u && bkey[i] >= tkey;
  const int cb0 = (int)block_scan((unsigned long long)mine, sh.sel.red, lane, warp);
  const int n_cb = (int)sh.sel.red[kW - 1];
  int K_take = a.K;
  SelRule rule;
  if (n_cb * 8 <= kCap) {
    // gather the candidate blocks' scores in column order; entries below tau
    // (or beyond the row) are absent
    int slot = cb0 * 8;
#pragma unroll
    for (int i = 0; i < kBpt; ++i) {
      if (bkey[i] != 0u && bkey[i] >= tkey) {
        const int c0 = (tid * kBpt + i) * 8;
        const float4 x = __ldcg(reinterpret_cast<const float4 *>(sc + c0));
        const float4 y = __ldcg(reinterpret_cast<const float4 *>(sc + c0) + 1);
        const float v[8] = {x.x, x.y, x.z, x.w, y.x, y.y, y.z, y.w};
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const uint32_t key = c0 + j < n ? skey(v[j]) : 0u;
          sh.cand_key[slot + j] = key >= tkey ? key : 0u;
          sh.cand_col[slot + j] = c0 + j;
        }
        slot += 8;
      }
    }
    for (int i = n_cb * 8 + tid; i < kCap; i += kT) sh.cand_key[i] = 0u;
    __syncthreads();
    uint32_t ck[kCpt];
#pragma unroll
    for (int i = 0; i < kCpt; ++i) ck[i] = sh.cand_key[tid * kCpt + i];
    const RegKeys<kCpt> cks{ck};
    radix_select<1>(cks, ks, sh.sel, tid, lane, warp);
    rule = sh.sel.rule[0];
    K_take = min(sh.sel.n_present, a.K);
    int pos, tb;
    taken_offsets(cks, rule, sh.sel.red, lane, warp, pos, tb);
#pragma unroll
    for (int i = 0; i < kCpt; ++i) {
      const uint32_t key = ck[i];
      const bool tk = strictly_taken(key, rule) || (tie(key, rule) && tb < rule.take_eq);
      tb += tie(key, rule);
      if (tk) {
        if (pos < a.K) {
          out[pos] = sh.cand_col[tid * kCpt + i];
          if (a.out_scores) a.out_scores[(size_t)row * a.K + pos] = kval(key);
        }
        ++pos;
      }
    }
  } else {
    // heavy ties at tau: select over the whole row
    const RowKeys rk{sc, n, (n + kT - 1) / kT, tid};
    radix_select<1>(rk, ks, sh.sel, tid, lane, warp);
    rule = sh.sel.rule[0];
    K_take = min(sh.sel.n_present, a.K);
    int pos, tb;
    taken_offsets(rk, rule, sh.sel.red, lane, warp, pos, tb);
    rk.each([&](uint32_t key, int i) {
      const bool tk = strictly_taken(key, rule) || (tie(key, rule) && tb < rule.take_eq);
      tb += tie(key, rule);
      if (tk) {
        if (pos < a.K) {
          out[pos] = tid * rk.npt + i;
          if (a.out_scores) a.out_scores[(size_t)row * a.K + pos] = kval(key);
        }
        ++pos;
      }
    });
  }
  for (int i = K_take + tid; i < a.K; i += kT) {
    out[i] = -1;
    if (a.out_scores) a.out_scores[(size_t)row * a.K + i] = -INFINITY;
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
  SelSmem &sel = *reinterpret_cast<SelSmem *>(smem_raw);
  const int row = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_launch_dependents();
  pdl_wait();
  const int n = a.G * a.n_seg;
  uint32_t key[kBpt];
  int32_t gid[kBpt];
#pragma unroll
  for (int i = 0; i < kBpt; ++i) {
    const int j = tid * kBpt + i;
    key[i] = 0u;
    gid[i] = -1;
    if (j < n) {
      const int g = j / a.n_seg, c = j % a.n_seg;
      const size_t at = ((size_t)g * a.rows + row) * a.n_seg + c;
      const int id = a.ids[at];
      if (id >= 0) {
        key[i] = skey(a.scores[at]);
        gid[i] = id + a.seg_base[g];
      }
    }
  }
  const RegKeys<kBpt> ks{key};
  const int k[1] = {a.K};
  radix_select<1>(ks, k, sel, tid, lane, warp);
  const SelRule rule = sel.rule[0];
  const int K_take = min(sel.n_present, a.K);
  int pos, tb;
  taken_offsets(ks, rule, sel.red, lane, warp, pos, tb);
  int32_t *out = a.out_ids + (size_t)row * a.K;
#pragma unroll
  for (int i = 0; i < kBpt; ++i) {
    const bool tk = strictly_taken(key[i], rule) || (tie(key[i], rule) && tb < rule.take_eq);
    tb += tie(key[i], rule);
    if (tk) {
      if (pos < a.K) {
        out[pos] = gid[i];
        if (a.out_scores) a.out_scores[(size_t)row * a.K + pos] = kval(key[i]);
      }
      ++pos;
    }
  }
  for (int i = K_take + tid; i < a.K; i += kT) {
    out[i] = -1;
    if (a.out_scores) a.out_scores[(size_t)row * a.K + i] = -INFINITY;
  }
}

cudaError_t launch_topk_merge(const TopkMergeArgs &a, cudaStream_t s) {
  const size_t smem = sizeof(SelSmem);
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
