/*
 * csa2.h -- C ABI of libcsa2: CSA2 sparse attention over an FP4 KV cache on
 * NVIDIA B200 (sm_100a).
 *
 * The method is the CSA2 step of "DeepSeek-V4.1-Flash: Pushing the Limits of
 * KV Cache Compression" (arXiv 2609.19969) as described by the jaehun.me
 * review, sections "2) CSA2" (paper sec. 2.3, 2.3.1, 2.3.2, Fig. 4-5) and
 * "3) FP4 main KV + SWA Bounded Replay" (paper sec. 2.4.4), and by its worked
 * example of the Full / Reuse / Reindex modes (paper sec. 2.3.1, 4.2.1).
 *
 * Conventions (all entry points):
 *  - Every pointer argument is caller-owned memory; pointers into tensors are
 *    DEVICE pointers unless stated otherwise.  The library never allocates,
 *    frees or synchronises; scratch space is a caller buffer whose size the
 *    *_workspace_size functions return.
 *  - Calls are asynchronous on the given stream (NULL = legacy default
 *    stream) and return a csa2_status.  Host-side validation happens before
 *    anything is enqueued; on error nothing is enqueued and
 *    csa2_last_error() (thread-local) describes it.
 *  - Kernels are launched with programmatic dependent launch: a kernel may
 *    start while the library's previous kernel on the stream is still
 *    running, and reads what that kernel (or any earlier one) wrote only
 *    after it has completed.  Before that point a kernel reads only inputs
 *    that no kernel of the library writes (new tokens and their window
 *    copies, W_ik, positions, indexer queries and head weights, attention
 *    queries) and stores nothing; whatever wrote those inputs must precede
 *    the call in stream order, as it does for any kernel or copy that is not
 *    one of the library's.
 *  - bf16 tensors are passed as their 16-bit patterns (uint16_t).
 *  - Device pointers must be 16-byte aligned.
 *  - In-kernel anomalies (an index outside the cache, a ring position below
 *    zero, a bounded wait that ran out) never trap: the offending item is
 *    masked and a bit is set in the library's device status word, read with
 *    csa2_device_status().
 *  - Inputs with NaN or Inf are not supported (results unspecified, no trap).
 *  - The library looks up, once per device, the device addresses of its own
 *    global arrays (the status word; entry 6's scratch).  A process that
 *    resets a device (cudaDeviceReset) must not call the library on that
 *    device afterwards: those addresses belong to the context it destroyed.
 */
#ifndef CSA2_H
#define CSA2_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Exported symbols of the shared library. */
#if defined(__GNUC__)
#define CSA2_API __attribute__((visibility("default")))
#else
#define CSA2_API
#endif

/* Same type as cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st *csa2_stream_t;

typedef enum {
    CSA2_OK = 0,
    CSA2_ERR_INVALID_ARG = 1,        /* null/misaligned pointer, bad size            */
    CSA2_ERR_UNSUPPORTED_SHAPE = 2,  /* a dimension outside the supported set        */
    CSA2_ERR_CUDA = 3,               /* a CUDA runtime call failed                    */
    CSA2_ERR_DEVICE_CHECK = 4,       /* returned by csa2_device_status when flagged   */
    CSA2_ERR_WORKSPACE = 5           /* workspace too small                           */
} csa2_status;

/* Bits of the device status word. */
#define CSA2_DEV_INDEX_RANGE   0x1u  /* a selected index >= cap or a pool block beyond cap (masked) */
#define CSA2_DEV_TIMEOUT       0x2u  /* a bounded pipeline wait gave up (tile skipped)              */
#define CSA2_DEV_APPEND_RANGE  0x4u  /* an appended entry fell beyond cap (not written)             */
#define CSA2_DEV_BAD_POSITION  0x8u  /* a negative token position (item skipped)                    */

/*
 * Main (global) FP4 KV cache of one CSA2 layer group [jaehun "3) FP4 ...":
 * E2M1 values with one E4M3 scale per 16 channels; jaehun "2) CSA2": the
 * indexer key is projected from the main KV].  Shared by the group's Full or
 * Reindex layer and its Reuse layers.
 *   codes     [B][cap][D/2]  u8  E2M1 pairs, byte i = code(ch 2i) | code(ch 2i+1) << 4
 *   scales    [B][cap][D/16] u8  E4M3 scale of channels 16g..16g+15
 *   ik        [B][cap][d_I]  u8  E4M3 indexer key
 *   ik_scale  [B][cap]       f32 indexer key scale (value = E4M3 * ik_scale)
 *   n_entries [B]            i32 entries written so far (updated by append)
 *   pending_kv, pending_gate [B][D] bf16: the token that opened an incomplete
 *                            pair (m = 2 only; may be NULL when m = 1)
 *   m: tokens pooled per entry, 1 (decoder) or 2 (encoder).
 * Supported: D in {128, 256, 512}, d_I in {64, 128}, cap a multiple of 128.
 */
typedef struct {
    uint8_t  *codes;
    uint8_t  *scales;
    uint8_t  *ik;
    float    *ik_scale;
    int32_t  *n_entries;
    uint16_t *pending_kv;
    uint16_t *pending_gate;
    int32_t B, cap, D, d_I, m;
} csa2_main_cache;

/*
 * Sliding-window cache of one layer [jaehun "3) FP4 ...": the window KV stays
 * FP8; n_win = 128].  Token p lives in ring slot p mod W_cap.
 *   rows [B][W_cap][D] u8 E4M3; value = E4M3 * scale.
 *   window: tokens attended (t-window+1 .. t); W_cap >= window, and a prefill
 *   chunk of T tokens needs W_cap >= T + window - 1.
 */
typedef struct {
    uint8_t *rows;
    float    scale;
    int32_t  B, W_cap, D, window;
} csa2_swa_cache;

/*
 * 1. Append T tokens per sequence  [jaehun "2) CSA2": m tokens -> one entry,
 *    no overlap, no absolute-position term; "3) FP4 ...": FP4 main KV, FP8
 *    window KV].
 *  main   (may be NULL: Reindex/Reuse layers append their window rows only)
 *  kv     [B][T][D] bf16 main-KV rows of the new tokens (ignored if main NULL)
 *  gate   [B][T][D] bf16 gate logits (m = 2), NULL when m = 1
 *  w_ik   [D][d_I]  bf16 indexer projection
 *  swa    (may be NULL) window cache of this layer
 *  kv_swa [B][T][D] bf16 window rows of the new tokens
 *  pos0   [B] i32 DEVICE: position of each sequence's first new token
 * Entry e (tokens m*e .. m*e+m-1) is written when its last token arrives:
 * pooled (m = 2: per-channel softmax of the pair's gate logits), quantised
 * per 16 channels (scale = E4M3(amax/6), codes = E2M1(x/scale), round to
 * nearest even), and its indexer key k = W_ik^T x^ (x^ = the dequantised
 * entry) is stored as E4M3 with scale amax(k)/448.  n_entries[b] becomes
 * floor((pos0[b]+T)/m).  The window cache receives E4M3(x/scale) of the last
 * min(T, W_cap) tokens.
 */
CSA2_API csa2_status csa2_append_quant(const csa2_main_cache *main, const uint16_t *kv,
                              const uint16_t *gate, const uint16_t *w_ik,
                              const csa2_swa_cache *swa, const uint16_t *kv_swa,
                              const int32_t *pos0, int T, csa2_stream_t stream);

/*
 * 1b. Append, and prepare the indexer query of the scan that follows, in one
 *     launch: csa2_append_quant plus, for each of the B*T_q query rows, the
 *     query preparation csa2_index_full performs (per head E4M3 codes with
 *     scale amax/448 and the weights w_h * s_q,h) written into ws, for
 *     csa2_index_full_prepared.  Saves the scan a launch in a decode step.
 *  main  required (its d_I sets the layout); T may be 0 (preparation only)
 *  q_idx [B][T_q][H_I][d_I] bf16, w [B][T_q][H_I] f32 (as for csa2_index_full)
 *  ws, ws_bytes: csa2_index_workspace_size(B*T_q, d_I) bytes, kept by the
 *         caller until the prepared scan has run
 */
CSA2_API csa2_status csa2_append_quant_ex(const csa2_main_cache *main, const uint16_t *kv,
                              const uint16_t *gate, const uint16_t *w_ik,
                              const csa2_swa_cache *swa, const uint16_t *kv_swa,
                              const int32_t *pos0, int T, const uint16_t *q_idx, const float *w,
                              int T_q, int H_I, void *ws, size_t ws_bytes, csa2_stream_t stream);

/*
 * 1c. Projected append: the CED decoder-KV producer  [jaehun "1) CED": the
 *     decoder's global KV is the final encoder hidden state projected by each
 *     decoder layer's W_KV^l (the flowchart edge "project W_KV^l, W_Z^l"; the
 *     equation was lost, so this is the plain linear projection; W_Z can only
 *     gate an m >= 2 pooling and the decoder caches are m = 1)].
 *  main   m = 1 cache, D a multiple of 256
 *  h      [B][T][d_model] bf16 hidden states of the new tokens
 *  w_kv   [d_model][D] bf16 projection W_KV^l
 *  w_ik   [D][d_I] bf16 indexer projection
 *  pos0   [B] i32 DEVICE: position (= entry) of each sequence's first new token
 * kv = h W_kv is accumulated in fp32 on the tensor cores and quantised in the
 * same kernel to the FP4 entry (scale = E4M3(amax/6), codes = E2M1(x/scale));
 * the indexer key of each new entry then follows from the stored bytes as in
 * csa2_append_quant, and n_entries[b] becomes pos0[b] + T.  No window rows
 * (a layer's window KV is appended with csa2_append_quant, main = NULL).
 * The fp32 accumulation order is the tensor core's: an FP4 byte can differ
 * from the correctly rounded projection's only where that value lies within
 * the accumulation error of a rounding boundary of the quantiser.
 * Supported: 64 <= d_model <= 32768, d_model a multiple of 64.
 */
CSA2_API csa2_status csa2_append_project(const csa2_main_cache *main, const uint16_t *h, int d_model,
                                         const uint16_t *w_kv, const uint16_t *w_ik, const int32_t *pos0, int T,
                                         csa2_stream_t stream);

/*
 * 2. Full indexer scoring  [jaehun "2) CSA2": a Full layer scores all entries
 *    with its own indexer; score_j = sum_h w_h ReLU(q_h . k_j) as an FP8
 *    contraction].
 *  q_idx  [B][T_q][H_I][d_I] bf16 indexer queries (quantised in-kernel per
 *         head to E4M3 with scale amax/448)
 *  w      [B][T_q][H_I] f32 head weights
 *  q_pos  [B][T_q] i32 token position of each query
 *  scores [B*T_q][ld] f32 out: scores[r][j] for j < n_vis(r), where
 *         n_vis = min(n_entries[b], floor((q_pos+1)/m)); columns >= n_vis are
 *         not written
 *  n_valid [B*T_q] i32 out (may be NULL): n_vis of each row
 *  ws, ws_bytes: workspace of csa2_index_workspace_size(B*T_q, d_I) bytes
 *         (holds each row's prepared FP8 query)
 * Supported: 1 <= H_I <= 64, ld >= cap.
 */
CSA2_API csa2_status csa2_index_full(const csa2_main_cache *main, const uint16_t *q_idx,
                            const float *w, const int32_t *q_pos, int T_q, int H_I,
                            float *scores, int64_t ld, int32_t *n_valid,
                            void *ws, size_t ws_bytes, csa2_stream_t stream);
CSA2_API size_t csa2_index_workspace_size(int rows, int d_I);

/*
 * 2b. Full indexer scoring with the query already prepared in ws by
 *     csa2_append_quant_ex (same rows, same T_q); otherwise as
 *     csa2_index_full.
 */
CSA2_API csa2_status csa2_index_full_prepared(const csa2_main_cache *main, const int32_t *q_pos, int T_q,
                              float *scores, int64_t ld, int32_t *n_valid,
                              const void *ws, size_t ws_bytes, csa2_stream_t stream);

/*
 * 2c. Full scoring fused with the first level of the Top-K and pool selection
 *     [jaehun "2) CSA2": the Full layer scans every entry, keeps the Top-512
 *     and builds the 2,048 blocks x 8 positions pool (paper sec. 2.3.2,
 *     Fig. 5)].  The scan's epilogue writes, with the scores, the maximum of
 *     every block of 8 entries; the selection reads those maxima (not the
 *     scores) to pick the pool and the K-th largest block maximum tau, and
 *     then only the scores of the blocks whose maximum is >= tau (every Top-K
 *     entry lies in one).  Results are those of csa2_index_full followed by
 *     csa2_topk(scores, ..., n_valid, NULL, K, out_idx, P_out, out_pool).
 *  q_idx, w  as for csa2_index_full; both NULL: the query was prepared in ws
 *            by csa2_append_quant_ex (then ws starts with that preparation)
 *  scores [B*T_q][ld] f32 out (ld >= cap, a multiple of 4), n_valid as for
 *            csa2_index_full (may be NULL)
 *  K, out_idx, P_out, out_pool as for csa2_topk
 *  out_scores [B*T_q][K] f32 out (may be NULL): the score of each selected
 *            entry (-inf where out_idx is -1); out_pool_scores [B*T_q][P_out]
 *            (may be NULL): each pool block's maximum (-inf padded) -- what a
 *            context shard sends to the merge (entry 2d)
 *  ws, ws_bytes: csa2_index_topk_workspace_size(B*T_q, cap, d_I) bytes
 * Supported: cap <= 131,072 (rows of more entries: csa2_index_full +
 * csa2_topk), 1 <= K <= 2048, 0 <= P_out <= 4096.
 */
CSA2_API csa2_status csa2_index_topk(const csa2_main_cache *main, const uint16_t *q_idx, const float *w,
                                     const int32_t *q_pos, int T_q, int H_I, float *scores, int64_t ld,
                                     int32_t *n_valid, int K, int32_t *out_idx, int P_out, int32_t *out_pool,
                                     float *out_scores, float *out_pool_scores, void *ws, size_t ws_bytes,
                                     csa2_stream_t stream);
CSA2_API size_t csa2_index_topk_workspace_size(int rows, int cap, int d_I);

/*
 * 2d. Context sharding across GPUs  [jaehun "2) CSA2" and Fig. 2: a long
 *     context's decode cost is the Full scan over all entries, which splits by
 *     entry range; the selection keeps <= 512 entries and 2,048 blocks].  With
 *     a sequence's entries split by contiguous ranges over G GPUs, each rank
 *     runs csa2_index_topk on its range (with out_scores / out_pool_scores),
 *     the ranks exchange those (score, id) lists (an all-gather), and
 *     csa2_topk_merge selects the global Top-K (and, with block ids, the pool)
 *     from them: every global Top-K entry is in its own range's Top-K, so the
 *     merge is exact.  csa2_gather_entries then copies, on each rank, the
 *     merged selection's entries that rank holds into a compact cache (zeros
 *     for the others); the ranks' buffers summed bytewise (one contributor
 *     per slot) form the cache the attention runs on.
 *
 * csa2_topk_merge: per row, the K best of G segments of n_seg candidates.
 *  scores, ids [G][rows][n_seg] f32 / i32 (DEVICE): segment g of row r is
 *         rank g's list; candidate (g, i) is entry ids[g][r][i] + seg_base[g]
 *         (ids < 0: none).  Each segment's ids ascend, and the segments'
 *         entry ranges ascend with g (so ties go to the smaller entry).
 *  seg_base [G] i32 HOST array: first entry of each rank's range
 *  out_ids [rows][K] i32 out: the K best entries (score desc, entry asc),
 *         ascending, -1 padded; out_scores [rows][K] f32 out (may be NULL)
 * Supported: 1 <= G <= 16, G * n_seg <= 16,384, 1 <= K <= 4096.
 */
CSA2_API csa2_status csa2_topk_merge(const float *scores, const int32_t *ids, int G, int rows, int n_seg,
                                     const int32_t *seg_base, int K, int32_t *out_ids, float *out_scores,
                                     csa2_stream_t stream);

/*
 * csa2_gather_entries: the selected entries a shard holds, in selection order.
 *  shard  the rank's main cache: its entry e is entry lo + e of the sequence
 *  ids    [B][K] i32 global entry ids of the merged selection (-1 = none)
 *  out_codes [B][out_cap][D/2], out_scales [B][out_cap][D/16] u8 out: slot k
 *         holds entry ids[b][k] when lo <= ids[b][k] < lo + cap, else zeros
 *  out_pos [B][K] i32 out (may be NULL): k where ids[b][k] >= 0, else -1 --
 *         the selection as slots of the compact cache
 * Supported: K <= out_cap, K <= 4096.
 */
CSA2_API csa2_status csa2_gather_entries(const csa2_main_cache *shard, int lo, const int32_t *ids, int K,
                                         uint8_t *out_codes, uint8_t *out_scales, int out_cap, int32_t *out_pos,
                                         csa2_stream_t stream);

/*
 * 3. Reindex scoring  [jaehun "2) CSA2": later Reindex layers rescore only the
 *    <= 2,048 blocks x 8 positions pool built by the first Full layer; the toy
 *    example: KV reused, indices recomputed with the layer's own indexer Q].
 *  pool_blocks [B*T_q][P] i32 block ids (block g = entries 8g..8g+7), -1 = none
 *  pool_scores [B*T_q][P*8] f32 out: column c scores entry pool[c/8]*8 + c%8,
 *              -inf when the block is -1 or the entry is not visible
 *  ws, ws_bytes: as for csa2_index_full
 * Supported: P a multiple of 16, 16 <= P <= 4096.
 */
CSA2_API csa2_status csa2_index_reindex(const csa2_main_cache *main, const uint16_t *q_idx,
                               const float *w, const int32_t *q_pos, int T_q, int H_I,
                               const int32_t *pool_blocks, int P, float *pool_scores,
                               void *ws, size_t ws_bytes, csa2_stream_t stream);

/*
 * 4. Top-K selection and the hierarchical candidate pool  [jaehun "2) CSA2":
 *    Top-512 per Full/Reindex layer; the first Full layer builds the pool of
 *    2,048 blocks x 8 positions].
 *  scores [rows][ld] f32; columns 0..n_cols-1 are candidates, further limited
 *         per row to n_valid[r] when n_valid is not NULL; -inf/NaN = absent
 *  pool_blocks [rows][n_cols/8] i32 (may be NULL): maps column c to entry
 *         pool_blocks[r][c/8]*8 + c%8 (Reindex); NULL = column is the entry
 *  out_idx [rows][K] i32 out: the K best columns (ties -> smaller column),
 *         listed in ascending column order, -1 padded
 *  out_pool [rows][P_out] i32 out (P_out > 0, pool_blocks NULL): the P_out
 *         blocks of 8 columns with the largest block maximum (ties -> smaller
 *         block), ascending, -1 padded
 *  ws, ws_bytes: workspace of csa2_topk_workspace_size(rows, n_cols, K, P_out);
 *         none (size 0, ws may be NULL) for rows of at most 65,536 columns
 *         (one thread-block cluster per row) and for 128 or more rows of at
 *         most 131,072 columns without a pool (one block per row, the row
 *         re-read from L2: prefill chunks)
 * Supported: 1 <= K <= 2048, 0 <= P_out <= 4096, n_cols <= 2^20.
 */
CSA2_API csa2_status csa2_topk(const float *scores, int rows, int64_t ld, int n_cols,
                      const int32_t *n_valid, const int32_t *pool_blocks, int K,
                      int32_t *out_idx, int P_out, int32_t *out_pool,
                      void *ws, size_t ws_bytes, csa2_stream_t stream);
CSA2_API size_t csa2_topk_workspace_size(int rows, int n_cols, int K, int P_out);

/*
 * 5. Sparse MQA attention  [jaehun "2) CSA2": global sparse retrieval plus the
 *    128-token local window in one attention; "3) FP4 ...": FP4 main KV, FP8
 *    window].  H query heads share one KV (K = V).
 *  q     [B][T_q][H][D] bf16
 *  q_pos [B][T_q] i32 token position t of each query
 *  idx   [B][T_q][K] i32 selected entries (-1 = none); may be NULL when K = 0
 *  K     selected entries per query; K = 0 attends to the window rows only,
 *        the SWA-only layers of the encoder [jaehun "새로운 접근법" and its
 *        flowchart: layers 1-2 use sliding-window attention only]
 *  out   [B][T_q][H][D] bf16: softmax over {idx != -1} U {window rows of
 *        tokens max(0,t-window+1)..t} of scale * q . x^, FP32 accumulation;
 *        zeros when that set is empty
 *  ws, ws_bytes: workspace of csa2_attn_workspace_size(...); with a smaller
 *        workspace (or none) the kernel runs unsplit
 * Supported: D in {128, 256, 512}, 1 <= H <= 64, 0 <= K <= 2048, window <= 1024.
 */
CSA2_API csa2_status csa2_sparse_attn_decode(const csa2_main_cache *main, const csa2_swa_cache *swa,
                                    const uint16_t *q, const int32_t *q_pos, int T_q, int H,
                                    const int32_t *idx, int K, float softmax_scale,
                                    uint16_t *out, void *ws, size_t ws_bytes,
                                    csa2_stream_t stream);
CSA2_API size_t csa2_attn_workspace_size(int B, int T_q, int H, int D, int K, int window);

/*
 * 6. Top-K selection without a caller workspace.  (No counterpart in the
 *    paper: this is a deployment variant of entry point 4.)
 *  For callers that cannot allocate device memory when they call the
 *  library -- e.g. a plugin inside another framework's engine whose memory
 *  is planned and owned by that framework, or code that must not allocate
 *  on its serving path.  Same arguments, outputs and results as csa2_topk,
 *  without ws/ws_bytes: the scratch is a 4 MiB array in device global memory
 *  built into the library (present on every GPU that loads it, until the
 *  process exits).
 *  - Selections needing more scratch than that (see
 *    csa2_topk_workspace_size) return CSA2_ERR_WORKSPACE, nothing enqueued.
 *  - All calls share the array: calls whose kernels may overlap on the GPU
 *    (unordered streams) race and give undefined results; calls on one
 *    stream are safe.  Nothing in the array needs to start at zero.
 *  - The first call on a device looks up the array's device address; make
 *    it before any stream capture on that device.
 */
CSA2_API csa2_status csa2_topk_noalloc(const float *scores, int rows, int64_t ld, int n_cols,
                                       const int32_t *n_valid, const int32_t *pool_blocks, int K,
                                       int32_t *out_idx, int P_out, int32_t *out_pool,
                                       csa2_stream_t stream);

/* Diagnostic: with polls > 0, the MMA-issuing warp of every later indexer
 * scan (csa2_index_full, _prepared, _topk, _reindex) first waits `polls`
 * polls on a barrier that nothing arrives on.  That wait runs out, and the
 * scan takes the path of any wait that gives up: it sets CSA2_DEV_TIMEOUT,
 * stops every role, waits (bounded) for its issued copies and MMAs, frees its
 * tensor memory and returns, leaving its scores incomplete.  polls = 0 (the
 * default) switches it off.  Process-wide; for tests of the give-up path. */
CSA2_API void csa2_debug_inject_timeout(uint32_t polls);

/* Thread-local description of the last error of this thread ("" if none). */
CSA2_API const char *csa2_last_error(void);

/* Reads the device status word of the current device (a stream-ordered copy
 * followed by a synchronisation of that stream) into *flags; clears it when
 * clear != 0.  Returns CSA2_ERR_DEVICE_CHECK when any bit is set. */
CSA2_API csa2_status csa2_device_status(csa2_stream_t stream, uint32_t *flags, int clear);

/* ABI version: (major << 16) | minor. */
CSA2_API int csa2_version(void);

#ifdef __cplusplus
}
#endif
#endif /* CSA2_H */
