// Top-K selection and hierarchical pool for rows of up to 65,536 columns in
// one launch: a thread-block cluster of 8 blocks per row.
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2": Top-512 per
//   Full/Reindex layer; the first Full decoder layer's pool of 2,048 blocks
//   x 8 positions (paper sec. 2.3.2, 4.2.1, Fig. 5).
// Same contract as the multi-kernel path in topk.cu (score descending, ties
// -> smaller column, non-finite = absent, ascending output, -1 padding,
// block score = max of its present columns), without a workspace.
//
// Block r of the cluster owns columns [8192r, 8192(r+1)); thread t keeps the
// order-preserving keys of columns 8t..8t+7 of that slice in registers, and
// their maximum, the key of one 8-column pool block.  The K-th largest key is
// found by levels of 512-bin histograms:
//   * level 0 bins by VALUE, linearly between the row's smallest and largest
//     score, so scores concentrated in a few binades still spread over many
//     bins;
//   * a bin holding the K-th key with at most 256 keys is resolved exactly:
//     its keys are collected in block 0 and ranked (score desc, column asc);
//     as the bins are monotone in the key, that key and its column decide
//     every column of the row;
//   * a larger level-0 bin is turned into an exact key interval by a 32-way
//     search over keys, and further levels bin by key bits inside it;
//   * a single-valued bin with more keys shares its ties out in column order.
// Per level the block histograms are pushed into the owning block's slice
// (block r owns bins [64r, 64r+64)) with distributed-shared-memory atomics
// and read back after ONE cluster barrier; slices rotate over 3 buffers so no
// second barrier is needed before they are reused.  The two selections
// (entries, pool blocks) run side by side in the two halves of the block.
// Loops stay rolled and the state lives in shared memory: the kernel runs
// once per row, so the code it fetches is as much a cost as what it executes.
#include <cooperative_groups.h>

#include "common.cuh"
#include "kernels.h"

namespace cg = cooperative_groups;

namespace csa2 {

namespace {

constexpr int kCl = 8;            // blocks per row
constexpr int kT = 1024;          // threads per block
constexpr int kN = 8;             // columns per thread (= one pool block)
constexpr int kSpan = kT * kN;    // columns per block
constexpr int kBins = 512;        // bins per selection (kT = 2 * kBins)
constexpr int kSeg = kBins / kCl; // bins owned by one block
constexpr int kCand = 256;        // largest bin resolved by exact ranking

static_assert(kT == 2 * kBins, "one thread per (selection, bin)");

__device__ __forceinline__ uint32_t ckey(float f) {
  if (!isfinite(f)) return 0u;   // absent
  if (f == 0.0f) f = 0.0f;       // -0 == +0
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}
__device__ __forceinline__ float kval(uint32_t k) {
  return __uint_as_float((k & 0x80000000u) ? (k & 0x7FFFFFFFu) : ~k);
}

enum : int { kActive = 0, kCollect = 1, kDone = 2 };

// State of one selection, kept in shared memory and written by one thread.
struct Sel {
  int state;
  bool vs;            // the current level bins by value (level 0)
  bool vreg;          // the region is value bin T0 (else the key interval [lo, hi])
  int T0;
  float v_lo, inv;    // value bin = clamp((v - v_lo) * inv)
  uint32_t g_lo, g_hi;
  uint32_t lo, hi;    // key interval of the current level's region
  int shift;          // key bin = (key - lo) >> shift
  int need;           // keys still to take inside the region
  int cnt;            // keys in the region (when collecting)
  // final rule: key > kthr, or key == kthr and (cmode ? column <= cthr : tie rank < take_eq)
  uint32_t kthr;
  int cthr;
  bool cmode;
  int take_eq;
};

// Value bin of key k: (v - v_lo) * inv rounded to the nearest integer by
// adding 1.5 * 2^23 (the FP32 adder rounds it into the low mantissa bits: a
// full-rate add instead of a quarter-rate float-to-int conversion), clamped to
// [0, kBins).  Explicit roundings keep every call site the same function; the
// levels rely only on it being monotone in the key.
__device__ __forceinline__ int vbin(float v_lo, float inv, uint32_t k) {
  const float t = __fmul_rn(__fsub_rn(kval(k), v_lo), inv);   // in [0, kBins] up to rounding
  const int b = __float_as_int(__fadd_rn(t, 12582912.0f)) - 0x4B400000;
  return b < 0 ? 0 : (b > kBins - 1 ? kBins - 1 : b);
}
__device__ __forceinline__ int key_shift(uint32_t lo, uint32_t hi) {
  const uint32_t span = hi - lo;
  return span >= (uint32_t)kBins ? (32 - __clz(span)) - 9 : 0;
}

// Smallest key in (lo, hi] whose value bin is >= T, given vbin(lo) < T <= vbin(hi);
// one 32-way step per iteration, every lane of the warp takes part.
__device__ uint32_t first_key_of_bin(float v_lo, float inv, uint32_t lo, uint32_t hi, int T, int lane) {
#pragma unroll 1
  while (hi - lo > 1u) {
    const uint32_t step = (uint32_t)(((uint64_t)(hi - lo) + 31u) >> 5);
    const uint64_t p = (uint64_t)lo + (uint64_t)step * (uint32_t)(lane + 1);
    const bool ge = p >= hi || vbin(v_lo, inv, (uint32_t)p) >= T;
    const int j = __ffs(__ballot_sync(0xffffffffu, ge)) - 1;   // lane 31 always probes >= hi
    const uint64_t pj = __shfl_sync(0xffffffffu, p, j);
    const uint64_t pp = __shfl_sync(0xffffffffu, p, j > 0 ? j - 1 : 0);
    const uint32_t nhi = pj >= hi ? hi : (uint32_t)pj;
    lo = j > 0 ? (uint32_t)pp : lo;
    hi = nhi;
  }
  return hi;
}

template <typename T>
__device__ __forceinline__ T warp_incl_scan(T v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const T y = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += y;
  }
  return v;
}

// Exclusive block scan; afterwards red[w] holds the inclusive sum of warps 0..w
// (valid until the next scan).
template <typename T>
__device__ __forceinline__ T block_scan(T v, T *red, int lane, int warp) {
  const T incl = warp_incl_scan(v, lane);
  __syncthreads();   // the previous scan's readers of red are done
  if (lane == 31) red[warp] = incl;
  __syncthreads();
  if (warp == 0) red[lane] = warp_incl_scan(red[lane], lane);
  __syncthreads();
  return (warp ? red[warp - 1] : T(0)) + incl - v;
}

struct Shared {
  uint32_t hist[2][kBins];        // this block's histogram of the current level
  uint32_t hsum[3][2][kSeg];      // cluster histogram, the bins this block owns
  uint2 cand[2][kCand];           // collected (key, column) pairs (block 0's are used)
  uint2 loc[2][kCand];            // local copy of block 0's pairs
  unsigned long long red[32];
  uint32_t wst[2][3][32];         // per-warp min, max, count
  uint32_t stat[2][3];            // this block: min key, max key, present count
  uint32_t cand_n[2];
  int cnt[4];                     // this block: ties / strict (entries), ties / strict (blocks)
  int th[2][3];                   // threshold bin, keys above it, keys in it
  int base[2], allow[2], total[2];
  Sel sel[2];
};

// Relaxed: every remote access a thread makes before its final arrive has
// completed by then (remote reads were consumed, remote writes were released
// by an earlier cluster barrier), so the arrive needs no release fence.
__device__ __forceinline__ void cluster_arrive_relaxed() {
  asm volatile("barrier.cluster.arrive.relaxed.aligned;" ::: "memory");
}
__device__ __forceinline__ void cluster_wait() {
  asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory");
}

}  // namespace

__global__ void __cluster_dims__(kCl, 1, 1) __launch_bounds__(kT, 1) topk_cluster_kernel(const TopkArgs a) {
  __shared__ Shared sh;
  cg::cluster_group cl = cg::this_cluster();
  const int r = (int)cl.block_rank();
  const int row = blockIdx.y, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int c0 = r * kSpan + tid * kN;   // this thread's first column
  const int blk = c0 >> 3;               // its pool block
  const int nsel = a.P_out > 0 ? 2 : 1;
  pdl_launch_dependents();
  pdl_wait();
  int ncol = a.n_cols;
  if (a.n_valid) {
    const int v = a.n_valid[row];
    if (v < ncol) ncol = v < 0 ? 0 : v;
  }

  // ---- keys (both 16-byte loads are issued before either is used)
  uint32_t key[kN];
  {
    const float *src = a.scores + (size_t)row * a.ld + c0;
    float v[kN];
    if (c0 + kN <= ncol && (a.ld & 3) == 0 && (reinterpret_cast<uintptr_t>(a.scores) & 15u) == 0) {
      const float4 x = __ldcs(reinterpret_cast<const float4 *>(src));
      const float4 y = __ldcs(reinterpret_cast<const float4 *>(src) + 1);
      v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w; v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
    } else {
#pragma unroll
      for (int k = 0; k < kN; ++k) v[k] = c0 + k < ncol ? src[k] : __int_as_float(0x7fc00000);
    }
#pragma unroll
    for (int k = 0; k < kN; ++k) key[k] = ckey(v[k]);
  }
  uint32_t bkey = 0u;
#pragma unroll
  for (int k = 0; k < kN; ++k) bkey = max(bkey, key[k]);

  // ---- zero the histograms, the round-0 slices and the collect counters
  (&sh.hist[0][0])[tid] = 0u;
  if (tid < 2 * kSeg) (&sh.hsum[0][0][0])[tid] = 0u;
  if (tid < 2) sh.cand_n[tid] = 0u;

  // ---- key range and count: warp, block, cluster
  {
    uint32_t mn = 0xFFFFFFFFu, mx = 0u, c = 0u;
#pragma unroll
    for (int k = 0; k < kN; ++k)
      if (key[k]) { mn = min(mn, key[k]); mx = max(mx, key[k]); ++c; }
    const uint32_t bmn = bkey ? bkey : 0xFFFFFFFFu, bc = bkey ? 1u : 0u;
    mn = __reduce_min_sync(0xffffffffu, mn);
    mx = __reduce_max_sync(0xffffffffu, mx);
    c = __reduce_add_sync(0xffffffffu, c);
    const uint32_t bmn2 = __reduce_min_sync(0xffffffffu, bmn);
    const uint32_t bc2 = __reduce_add_sync(0xffffffffu, bc);
    if (lane == 0) {
      sh.wst[0][0][warp] = mn; sh.wst[0][1][warp] = mx; sh.wst[0][2][warp] = c;
      sh.wst[1][0][warp] = bmn2; sh.wst[1][1][warp] = mx; sh.wst[1][2][warp] = bc2;
    }
  }
  __syncthreads();
  if (warp < 2) {   // warp s combines selection s
    const uint32_t mn = __reduce_min_sync(0xffffffffu, sh.wst[warp][0][lane]);
    const uint32_t mx = __reduce_max_sync(0xffffffffu, sh.wst[warp][1][lane]);
    const uint32_t c = __reduce_add_sync(0xffffffffu, sh.wst[warp][2][lane]);
    if (lane == 0) { sh.stat[warp][0] = mn; sh.stat[warp][1] = mx; sh.stat[warp][2] = c; }
  }
  cl.sync();
  if (warp < 2) {
    const int s = warp;
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
    if (lane == 0) {
      Sel &l = sh.sel[s];
      const int Kt = s == 0 ? a.K : a.P_out;
      l.g_lo = l.lo = mn;
      l.g_hi = l.hi = mx;
      l.need = Kt;
      l.cnt = 0;
      l.kthr = 0u;   // with cmode and cthr = -1: every present key
      l.cthr = -1;
      l.cmode = true;
      l.take_eq = 0;
      l.vs = false;
      l.vreg = false;
      l.T0 = 0;
      l.v_lo = 0.f;
      l.inv = 0.f;
      l.shift = 0;
      if (s >= nsel || (int)c <= Kt) {
        l.state = kDone;
      } else {
        l.state = kActive;
        const float vlo = kval(mn), vhi = kval(mx);
        const float span = vhi - vlo;
        const float inv = (float)kBins / span;
        if (span > 0.f && isfinite(span) && isfinite(inv)) {
          l.vs = true;
          l.v_lo = vlo;
          l.inv = inv;
        } else {
          l.shift = key_shift(mn, mx);
        }
      }
    }
  }
  __syncthreads();

  // ---- levels
#pragma unroll 1
  for (int round = 0;; ++round) {
    if (sh.sel[0].state == kDone && sh.sel[1].state == kDone) break;   // cluster-uniform
    const int buf = round % 3;
    // 1. this block's histogram; zero the owned slices of round + 1
#pragma unroll 1
    for (int s = 0; s < 2; ++s) {
      const Sel &l = sh.sel[s];
      if (l.state != kActive) continue;
      const bool vs = l.vs;
      const float v_lo = l.v_lo, inv = l.inv;
      const uint32_t lo = l.lo, hi = l.hi;
      const int shift = l.shift;
#pragma unroll
      for (int k = 0; k < kN; ++k) {
        const uint32_t kk = s == 0 ? key[k] : (k == 0 ? bkey : 0u);
        if (kk && (vs || (kk >= lo && kk <= hi)))
          atomicAdd(&sh.hist[s][vs ? vbin(v_lo, inv, kk) : (int)((kk - lo) >> shift)], 1u);
      }
    }
    if (tid < 2 * kSeg) (&sh.hsum[(round + 1) % 3][0][0])[tid] = 0u;
    __syncthreads();
    // 2. thread (s, bin) pushes its bin into the owner's slice and re-zeroes it
    {
      const int s = tid / kBins, b = tid % kBins;
      const uint32_t h = sh.hist[s][b];
      if (h) {
        sh.hist[s][b] = 0u;
        atomicAdd(cl.map_shared_rank(&sh.hsum[buf][s][b % kSeg], b / kSeg), h);
      }
    }
    cl.sync();
    // 3. thread (s, bin) reads the bin's cluster count; a scan over the bins
    // finds the one holding the need-th largest key
    {
      const int s = tid / kBins, b = tid % kBins;
      const bool act = sh.sel[s].state == kActive;
      const int h = act ? (int)*cl.map_shared_rank(&sh.hsum[buf][s][b % kSeg], b / kSeg) : 0;
      uint32_t *red32 = reinterpret_cast<uint32_t *>(sh.red);   // counts of a row fit 32 bits
      const int pre = (int)block_scan<uint32_t>((uint32_t)h, red32, lane, warp);
      const int h0 = (int)red32[kBins / 32 - 1], tot = (int)red32[31];
      const int above = s == 0 ? h0 - pre - h : tot - pre - h;   // keys in higher bins
      const int need = sh.sel[s].need;
      if (act && above < need && above + h >= need) {
        sh.th[s][0] = b;
        sh.th[s][1] = above;
        sh.th[s][2] = h;
      }
    }
    __syncthreads();
    // 4. warp s decides the next level of selection s
    if (warp < 2 && sh.sel[warp].state == kActive) {
      Sel &l = sh.sel[warp];
      const int T = sh.th[warp][0], cntT = sh.th[warp][2];
      const int need2 = l.need - sh.th[warp][1];   // 1 <= need2 <= cntT
      if (l.vs && cntT <= kCand) {
        // rank the keys of value bin T exactly (no key interval needed: the
        // bins are monotone in the key, so the need2-th key of the bin and its
        // column decide every key of the row)
        if (lane == 0) { l.vreg = true; l.T0 = T; l.need = need2; l.cnt = cntT; l.state = kCollect; }
      } else {
        uint32_t lo_T, hi_T;
        if (l.vs) {   // exact key interval of value bin T
          lo_T = T == 0 ? l.g_lo : first_key_of_bin(l.v_lo, l.inv, l.g_lo, l.g_hi, T, lane);
          hi_T = T == kBins - 1 ? l.g_hi : first_key_of_bin(l.v_lo, l.inv, l.g_lo, l.g_hi, T + 1, lane) - 1u;
        } else {
          lo_T = l.lo + ((uint32_t)T << l.shift);
          const uint32_t w1 = (1u << l.shift) - 1u;
          hi_T = (l.hi - lo_T > w1) ? lo_T + w1 : l.hi;
        }
        if (lane == 0) {
          if (cntT == need2) {                 // every key of the bin is taken
            l.kthr = lo_T - 1u; l.cthr = -1; l.cmode = true; l.state = kDone;
          } else if (cntT <= kCand) {          // rank the bin's keys exactly
            l.lo = lo_T; l.hi = hi_T; l.need = need2; l.cnt = cntT; l.vs = false; l.state = kCollect;
          } else if (!l.vs && l.shift == 0) {  // one key value: need2 of its ties, in column order
            l.kthr = lo_T; l.cmode = false; l.take_eq = need2; l.state = kDone;
          } else {                             // next level inside the bin
            l.lo = lo_T; l.hi = hi_T; l.shift = key_shift(lo_T, hi_T); l.need = need2; l.vs = false;
          }
        }
      }
    }
    __syncthreads();
    if (sh.sel[0].state != kCollect && sh.sel[1].state != kCollect) continue;   // cluster-uniform

    // 5. collect the region's keys in block 0 and rank them;
    // both selections in one pass: one warp scan of (entries | blocks << 16),
    // the two slot reservations in block 0 in flight together
    {
      const auto in_region = [&](const Sel &l, uint32_t kk) {
        return l.state == kCollect && kk &&
               (l.vreg ? vbin(l.v_lo, l.inv, kk) == l.T0 : (kk >= l.lo && kk <= l.hi));
      };
      const Sel &l0 = sh.sel[0], &l1 = sh.sel[1];
      bool in[kN];
      int m0 = 0;
#pragma unroll
      for (int k = 0; k < kN; ++k) {
        in[k] = in_region(l0, key[k]);
        m0 += in[k];
      }
      const int m1 = in_region(l1, bkey) ? 1 : 0;
      const uint32_t mm = (uint32_t)m0 | ((uint32_t)m1 << 16);   // a warp holds at most 256 entries
      const uint32_t incl = warp_incl_scan(mm, lane);
      const uint32_t wtot = __shfl_sync(0xffffffffu, incl, 31);
      uint32_t wb0 = 0u, wb1 = 0u;
      if (lane == 31) {
        if (wtot & 0xFFFFu) wb0 = atomicAdd(cl.map_shared_rank(&sh.cand_n[0], 0), wtot & 0xFFFFu);
        if (wtot >> 16) wb1 = atomicAdd(cl.map_shared_rank(&sh.cand_n[1], 0), wtot >> 16);
      }
      int pos = (int)__shfl_sync(0xffffffffu, wb0, 31) + (int)(incl & 0xFFFFu) - m0;
      const int pos1 = (int)__shfl_sync(0xffffffffu, wb1, 31) + (int)(incl >> 16) - m1;
      uint2 *dst = cl.map_shared_rank(&sh.cand[0][0], 0);
#pragma unroll
      for (int k = 0; k < kN; ++k) {
        if (in[k]) {
          if (pos < kCand) dst[pos] = make_uint2(key[k], (uint32_t)(c0 + k));
          ++pos;
        }
      }
      if (m1 && pos1 < kCand) cl.map_shared_rank(&sh.cand[1][0], 0)[pos1] = make_uint2(bkey, (uint32_t)blk);
    }
    cl.sync();
    {
      const int s = tid / kBins, i = tid % kBins;
      if (sh.sel[s].state == kCollect && i < sh.sel[s].cnt) sh.loc[s][i] = cl.map_shared_rank(&sh.cand[s][0], 0)[i];
    }
    __syncthreads();
    {
      const int s = tid / kBins, i = tid % kBins;
      const int n = sh.sel[s].cnt;
      if (sh.sel[s].state == kCollect && i < n) {
        const uint2 me = sh.loc[s][i];
        int rank = 0;
#pragma unroll 1
        for (int j = 0; j < n; j += 4) {   // four pairs in flight
          uint2 o[4];
#pragma unroll
          for (int u = 0; u < 4; ++u) o[u] = sh.loc[s][j + u < n ? j + u : j];
#pragma unroll
          for (int u = 0; u < 4; ++u) rank += j + u < n && ((o[u].x > me.x) || (o[u].x == me.x && o[u].y < me.y));
        }
        if (rank == sh.sel[s].need - 1) {   // exactly one pair
          sh.sel[s].kthr = me.x;
          sh.sel[s].cthr = (int)me.y;
        }
      }
    }
    __syncthreads();
    if (tid < 2 && sh.sel[tid].state == kCollect) {
      sh.sel[tid].cmode = true;
      sh.sel[tid].state = kDone;
    }
    __syncthreads();
  }

  // ---- per-block counts -> output offsets (one exchange)
  const uint32_t kthr0 = sh.sel[0].kthr, kthr1 = sh.sel[1].kthr;
  const int cthr0 = sh.sel[0].cthr, cthr1 = sh.sel[1].cthr;
  const bool cm0 = sh.sel[0].cmode, cm1 = sh.sel[1].cmode;
  int tie_base0, tie_base1, pos0, pos1;
  {
    int t0 = 0, s0 = 0;
#pragma unroll
    for (int k = 0; k < kN; ++k) {
      const uint32_t kk = key[k];
      s0 += kk && (kk > kthr0 || (cm0 && kk == kthr0 && c0 + k <= cthr0));
      t0 += kk && !cm0 && kk == kthr0;
    }
    const int t1 = nsel > 1 && bkey && !cm1 && bkey == kthr1;
    const int s1 = nsel > 1 && bkey && (bkey > kthr1 || (cm1 && bkey == kthr1 && blk <= cthr1));
    if (cm0 && cm1) {   // no ties shared by count (block-uniform): the two strict counts in 32 bits
      uint32_t *red32 = reinterpret_cast<uint32_t *>(sh.red);
      const uint32_t ex = block_scan<uint32_t>((uint32_t)s0 | ((uint32_t)s1 << 16), red32, lane, warp);
      tie_base0 = tie_base1 = 0;
      pos0 = (int)(ex & 0xFFFFu);
      pos1 = (int)(ex >> 16);
      if (tid == 0) {
        const uint32_t tot = red32[31];
        sh.cnt[0] = 0;
        sh.cnt[1] = (int)(tot & 0xFFFFu);
        sh.cnt[2] = 0;
        sh.cnt[3] = (int)(tot >> 16);
      }
    } else {
      const unsigned long long v = (unsigned long long)t0 | ((unsigned long long)s0 << 16) |
                                   ((unsigned long long)t1 << 32) | ((unsigned long long)s1 << 48);
      const unsigned long long ex = block_scan<unsigned long long>(v, sh.red, lane, warp);
      tie_base0 = (int)(ex & 0xFFFFu);
      tie_base1 = (int)((ex >> 32) & 0xFFFFu);
      pos0 = (int)((ex >> 16) & 0xFFFFu);   // the output positions when no tie is shared by count
      pos1 = (int)((ex >> 48) & 0xFFFFu);
      if (tid == 0) {
        const unsigned long long tot = sh.red[31];
        sh.cnt[0] = (int)(tot & 0xFFFFu);
        sh.cnt[1] = (int)((tot >> 16) & 0xFFFFu);
        sh.cnt[2] = (int)((tot >> 32) & 0xFFFFu);
        sh.cnt[3] = (int)((tot >> 48) & 0xFFFFu);
      }
    }
  }
  cl.sync();
  if (warp < 2) {   // warp s: offsets of selection s
    const int s = warp;
    int tt = 0, st = 0;
    if (lane < kCl) {
      const int *rc = cl.map_shared_rank(&sh.cnt[0], lane);
      tt = rc[2 * s];
      st = rc[2 * s + 1];
    }
    const int ties_before = warp_incl_scan(tt, lane) - tt;
    const int take_eq = sh.sel[s].take_eq;
    int al = take_eq - ties_before;
    al = al < 0 ? 0 : (al > tt ? tt : al);
    const int chosen = st + al;
    const int cinc = warp_incl_scan(chosen, lane);
    const int ctot = __shfl_sync(0xffffffffu, cinc, kCl - 1);
    if (lane == r) {
      sh.base[s] = cinc - chosen;
      sh.allow[s] = take_eq - ties_before;
      sh.total[s] = ctot;
    }
  }
  cluster_arrive_relaxed();   // no remote shared memory is read after this point
  __syncthreads();

  // ---- write the chosen columns in order
  {
    const int allow0 = sh.allow[0], allow1 = sh.allow[1];
    int n0 = 0, tr = tie_base0;
#pragma unroll
    for (int k = 0; k < kN; ++k) {
      const uint32_t kk = key[k];
      const bool tie = kk && !cm0 && kk == kthr0;
      n0 += (kk && (kk > kthr0 || (cm0 && kk == kthr0 && c0 + k <= cthr0))) || (tie && tr < allow0);
      tr += tie;
    }
    const bool tie1 = nsel > 1 && bkey && !cm1 && bkey == kthr1;
    const bool take1 = (nsel > 1 && bkey && (bkey > kthr1 || (cm1 && bkey == kthr1 && blk <= cthr1))) ||
                       (tie1 && tie_base1 < allow1);
    if (!(cm0 && cm1)) {   // ties shared by count: positions from the final counts (block-uniform)
      const uint32_t ex = block_scan<uint32_t>((uint32_t)n0 | ((uint32_t)take1 << 16),
                                               reinterpret_cast<uint32_t *>(sh.red), lane, warp);
      pos0 = (int)(ex & 0xFFFFu);
      pos1 = (int)(ex >> 16);
    }
    int o = sh.base[0] + pos0;
    int32_t *out = a.out_idx + (size_t)row * a.K;
    const int32_t *pb = a.pool_blocks ? a.pool_blocks + (size_t)row * (a.n_cols / 8) : nullptr;
    tr = tie_base0;
#pragma unroll
    for (int k = 0; k < kN; ++k) {
      const uint32_t kk = key[k];
      const bool tie = kk && !cm0 && kk == kthr0;
      const bool take = (kk && (kk > kthr0 || (cm0 && kk == kthr0 && c0 + k <= cthr0))) || (tie && tr < allow0);
      tr += tie;
      if (take) {
        if (o < a.K) out[o] = pb ? pb[blk] * 8 + k : c0 + k;
        ++o;
      }
    }
    if (take1) {
      const int o1 = sh.base[1] + pos1;
      if (o1 < a.P_out) a.out_pool[(size_t)row * a.P_out + o1] = blk;
    }
    if (r == kCl - 1) {
      for (int i = sh.total[0] + tid; i < a.K; i += kT) out[i] = -1;
      if (nsel > 1)
        for (int i = sh.total[1] + tid; i < a.P_out; i += kT) a.out_pool[(size_t)row * a.P_out + i] = -1;
    }
  }
  cluster_wait();   // no block leaves while another may still read its shared memory
}

// Rows of up to kCl * kSpan columns go through the cluster kernel.
bool topk_cluster_fits(int n_cols) { return n_cols <= kCl * kSpan; }

cudaError_t launch_topk_cluster(const TopkArgs &a, cudaStream_t s) {
  return launch_pdl(topk_cluster_kernel, dim3(kCl, a.rows), dim3(kT), 0, s, dim3(1, 1, 1), a);
}

}  // namespace csa2
