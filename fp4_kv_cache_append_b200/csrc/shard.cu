// Context sharding across GPUs: copies of the entries a step selected from one
// shard of a long context, for the rank that runs the attention.
//   DeepSeek-V4.1-Flash (jaehun.me review), section "2) CSA2" and Fig. 2: the
//   decode cost of a 1M-token context is dominated by the Full scan, which
//   splits by entry range; every other step works on the <= 512 selected
//   entries.  With the context split by contiguous entry ranges over G GPUs,
//   each rank scans and selects its range, the per-rank (score, entry) lists
//   are exchanged and merged (topk_merge_kernel), and each rank copies out the
//   merged selection's entries it holds: one block per sequence writes, for
//   selection slot k, the FP4 codes and scales of entry ids[b][k] if the shard
//   holds it, else zeros, so that the ranks' buffers sum (bytewise, one
//   nonzero contributor per slot) to the compact cache of the selection.
#include "common.cuh"
#include "kernels.h"

namespace csa2 {

__global__ void __launch_bounds__(256) gather_entries_kernel(const GatherArgs a) {
  pdl_launch_dependents();
  pdl_wait();
  const int b = blockIdx.x, D = a.D;
  const int cw = D / 32;                          // 16-byte pieces of an entry's codes (D/2 bytes)
  const int per = cw + (D >= 256 ? D / 256 : 1);  // + pieces of its scales (D/16 bytes; 8 bytes when D = 128)
  for (int i = threadIdx.x; i < a.K * per; i += blockDim.x) {
    const int k = i / per, p = i % per;
    const int id = a.ids[(size_t)b * a.K + k];
    const int e = id - a.lo;
    const bool mine = id >= 0 && e >= 0 && e < a.cap;
    if (p < cw) {
      uint4 v = make_uint4(0, 0, 0, 0);
      if (mine) v = __ldg(reinterpret_cast<const uint4 *>(a.codes + ((size_t)b * a.cap + e) * (D / 2)) + p);
      reinterpret_cast<uint4 *>(a.out_codes + ((size_t)b * a.out_cap + k) * (D / 2))[p] = v;
    } else if (D >= 256) {       // scales in 16-byte pieces
      const int q = p - cw;
      uint4 v = make_uint4(0, 0, 0, 0);
      if (mine) v = __ldg(reinterpret_cast<const uint4 *>(a.scales + ((size_t)b * a.cap + e) * (D / 16)) + q);
      reinterpret_cast<uint4 *>(a.out_scales + ((size_t)b * a.out_cap + k) * (D / 16))[q] = v;
    } else {                     // D = 128: 8 scale bytes
      uint2 v = make_uint2(0, 0);
      if (mine) v = *reinterpret_cast<const uint2 *>(a.scales + ((size_t)b * a.cap + e) * (D / 16));
      *reinterpret_cast<uint2 *>(a.out_scales + ((size_t)b * a.out_cap + k) * (D / 16)) = v;
    }
    if (p == 0 && a.out_pos) a.out_pos[(size_t)b * a.K + k] = id >= 0 ? k : -1;
  }
}

cudaError_t launch_gather_entries(const GatherArgs &a, cudaStream_t s) {
  return launch_pdl(gather_entries_kernel, dim3(a.B), dim3(256), 0, s, dim3(1, 1, 1), a);
}

}  // namespace csa2
