// Host-side launchers of the libcsa2 kernels (internal; the public ABI is
// include/csa2.h).  Each returns the cudaError_t of its launch.
#pragma once
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/csa2.h"

namespace csa2 {

// Preparation of a scan's indexer query (one warp per head): per head E4M3
// codes with scale amax/448 in the scan's B-operand layout (64 rows x dI
// bytes, K-major, swizzled) and the head weights w_h * s_q,h.
constexpr int kIndexHeads = 64;   // N of the scan's MMA (indexer heads, zero padded)
struct QueryPrep {
  const uint16_t *q_idx;  // [rows][H_I][dI] bf16
  const float *w;         // [rows][H_I]
  int rows, H_I, dI;      // rows == 0: nothing to prepare
  uint8_t *q8;            // [rows][64*dI]
  float *wq;              // [rows][64]
};

struct AppendArgs {
  // main cache (codes == nullptr: no main part)
  uint8_t *codes, *scales, *ik;
  float *ik_scale;
  int32_t *n_entries;
  uint16_t *pending_kv, *pending_gate;
  int B, cap, D, dI, m;
  const uint16_t *kv, *gate, *w_ik;
  // window cache (rows == nullptr: no window part)
  uint8_t *swa_rows;
  float s_swa;
  int W_cap;
  const uint16_t *kv_swa;
  const int32_t *pos0;
  int T;
  int main_blocks_per_seq, swa_blocks_per_seq;
  int entries_per_block;   // 1, 8 or 32
  unsigned int *status;
  QueryPrep prep;          // optional: the following scan's query, 8 blocks per row
};
cudaError_t launch_append(const AppendArgs &a, cudaStream_t s);
// Indexer keys of entries already stored as FP4 (after the projected append):
// one block per group of entries_per_block new entries of a sequence.
cudaError_t launch_append_keys(const AppendArgs &a, cudaStream_t s);

// CED decoder-KV producer: codes/scales of kv = H W_KV (m = 1), token row
// r = b * T + t -> entry pos0[b] + t.
struct ProjectArgs {
  uint8_t *codes, *scales;
  int32_t *n_entries;
  int B, cap, D;
  const int32_t *pos0;
  int T, d;              // tokens per sequence, d_model
  unsigned int *status;
};
cudaError_t launch_project(const CUtensorMap &h_map, const CUtensorMap &w_map, const ProjectArgs &a, cudaStream_t s);

struct IndexArgs {
  const float *ik_scale;
  const int32_t *n_entries;
  int B, cap, m, dI;
  const uint16_t *q_idx;  // [B][T_q][H_I][dI]
  const float *w;         // [B][T_q][H_I]
  const int32_t *q_pos;   // [B][T_q]
  int T_q, H_I;
  float *scores;          // [B*T_q][ld]
  int64_t ld;
  int32_t *n_valid;       // full mode, optional
  const int32_t *pool;    // reindex mode: [B*T_q][P]
  int P;
  int tiles_per_row;      // reindex: P/16; full: cap/128 (the visible count is found in the kernel)
  int ctas_per_row;       // blocks sharing one row's tiles
  float *bmax;            // full mode, optional: [B*T_q][ld_b] maximum score of each block of 8 entries
  int64_t ld_b;
  uint8_t *q8;            // workspace: [B*T_q][64*dI] prepared FP8 query (MMA layout)
  float *wq;              // workspace: [B*T_q][64] w_h * s_q,h
  bool prepared;          // q8/wq already hold the query (no preparation kernel)
  unsigned int *status;
  uint32_t inject_polls;  // diagnostic: > 0 makes the MMA issuer first wait this many polls on a
                          // barrier nothing arrives on (a wait that runs out, then the abort path)
};
uint32_t injected_timeout_polls();   // csa2_debug_inject_timeout's setting (0 = off)
size_t index_workspace_bytes(int rows, int dI);
int index_rows_per_block(int T_q, bool reindex);   // query rows sharing one scan block (1, 2 or 4)
cudaError_t launch_index(const CUtensorMap &ik_map, const IndexArgs &a, bool reindex, int sms,
                         cudaStream_t s);

// Launch with programmatic stream serialisation (and an optional cluster
// shape): the kernel may start while the stream's previous kernel drains and
// synchronises with it through pdl_wait().
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                              dim3 cluster, Args &&...args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  int n = 1;
  if (cluster.x * cluster.y * cluster.z > 1) {
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = cluster.x;
    attr[1].val.clusterDim.y = cluster.y;
    attr[1].val.clusterDim.z = cluster.z;
    n = 2;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

struct TopkArgs {
  const float *scores;
  int rows;
  int64_t ld;
  int n_cols;
  const int32_t *n_valid;
  const int32_t *pool_blocks;
  int K;
  int32_t *out_idx;
  int P_out;
  int32_t *out_pool;
  void *ws;
};
struct TopkPlan {
  int nchunks;        // column chunks per row (histogram / filter blocks)
  int nb;             // blocks of 8 columns per row
  size_t off_hist, off_histb, off_cnt, off_range, off_sel, off_cand, off_selb, off_candb;
  size_t zero_bytes;  // [0, zero_bytes) is cleared at the start of every call
  size_t bytes;       // workspace bytes
};
TopkPlan plan_topk(int rows, int n_cols, int K, int P_out);
cudaError_t launch_topk(const TopkArgs &a, const TopkPlan &p, cudaStream_t s);
bool topk_cluster_fits(int n_cols);                              // one cluster per row, no workspace
cudaError_t launch_topk_cluster(const TopkArgs &a, cudaStream_t s);

// Top-K and pool from the block maxima a Full scan wrote (one block per row).
struct TopkBmaxArgs {
  const float *scores;    // [rows][ld]
  int64_t ld;
  const float *bmax;      // [rows][ld_b]
  int64_t ld_b;
  int rows, n_cols;
  const int32_t *n_valid; // [rows] or nullptr
  int K;
  int32_t *out_idx;       // [rows][K]
  int P_out;
  int32_t *out_pool;      // [rows][P_out]
  float *out_scores;      // [rows][K] or nullptr: the selected entries' scores
  float *out_pool_scores; // [rows][P_out] or nullptr: the pool blocks' maxima
};
constexpr int kTopkBmaxMaxBlocks = 16384;   // blocks of 8 columns per row (131,072 columns)
cudaError_t launch_topk_bmax(const TopkBmaxArgs &a, cudaStream_t s);

// Merge of G per-shard selections of one row each (see topk_merge_kernel).
constexpr int kMergeMaxShards = 16;
struct TopkMergeArgs {
  const float *scores;    // [G][rows][n_seg]
  const int32_t *ids;     // [G][rows][n_seg]
  int G, rows, n_seg;
  int seg_base[kMergeMaxShards];
  int K;
  int32_t *out_ids;       // [rows][K]
  float *out_scores;      // [rows][K] or nullptr
};
cudaError_t launch_topk_merge(const TopkMergeArgs &a, cudaStream_t s);

// Copies of selected entries of a context shard (entries lo .. lo + cap - 1
// of each sequence) into a compact cache of one row per sequence.
struct GatherArgs {
  const uint8_t *codes, *scales;   // shard planes [B][cap][D/2], [B][cap][D/16]
  int B, cap, D, lo;
  const int32_t *ids;              // [B][K] global entry ids, -1 = none
  int K;
  uint8_t *out_codes, *out_scales; // [B][out_cap][D/2], [B][out_cap][D/16]
  int out_cap;
  int32_t *out_pos;                // [B][K] k where ids >= 0, else -1 (or nullptr)
};
cudaError_t launch_gather_entries(const GatherArgs &a, cudaStream_t s);

struct AttnArgs {
  const uint8_t *codes, *scales;
  int cap, D;
  const uint8_t *swa_rows;
  float s_swa;
  int W_cap, window;
  const uint16_t *q;      // [B][T_q][H][D]
  const int32_t *q_pos;   // [B][T_q]
  int B, T_q, H;
  const int32_t *idx;     // [B][T_q][K]
  int K;
  float scale;
  uint16_t *out;          // [B][T_q][H][D]
  float *ws;              // split partials (nullptr when unsplit)
  int nsplit, chunks_per_split;
  int csplit;             // 2: a pair of blocks per split, each with half of the O channels
  int latency_form;       // attn_lat.cu: every block resident at once, one 128-key tile per block
  unsigned int *status;
};
struct AttnPlan {
  int nsplit, chunks_per_split, csplit;
  int latency_form;       // rows x nsplit x csplit blocks fit on the SMs and each split is one tile
  size_t bytes;
};
AttnPlan plan_attn(int B, int T_q, int H, int D, int K, int window, int sms);
// Launches the latency form (attn_lat.cu) when a.latency_form, else the pipelined form.
cudaError_t launch_attn(const AttnArgs &a, cudaStream_t s);
cudaError_t launch_attn_lat(const AttnArgs &a, cudaStream_t s);

}  // namespace csa2
