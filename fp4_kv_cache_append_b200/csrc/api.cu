// C ABI of libcsa2 (declared in include/csa2.h): argument validation, TMA
// descriptor encoding, launch planning.  Nothing here allocates device memory.
#include <atomic>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <mutex>
#include <string>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.h"

namespace csa2 {

// Device status word: in-kernel anomalies set bits here (never trap).
__device__ unsigned int g_status;

namespace {

thread_local std::string t_err;
std::atomic<uint32_t> g_inject_polls{0};

// An NVTX range named after the entry point for the duration of the call
// (host side: validation and launches), visible in Nsight timelines.
struct NvtxRange {
  explicit NvtxRange(const char *name) { nvtxRangePushA(name); }
  ~NvtxRange() { nvtxRangePop(); }
};

csa2_status fail(csa2_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  t_err = buf;
  return st;
}

csa2_status cuda_fail(cudaError_t e, const char *where) {
  return fail(CSA2_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

struct DeviceState {
  unsigned int *status = nullptr;
  int sms = 0;
};
std::mutex g_mu;
DeviceState g_dev[64];

// Per-device set-up on first use (the status word's device address and the
// SM count); call before any stream capture begins.
csa2_status device_state(DeviceState **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= 64) return fail(CSA2_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceState &d = g_dev[dev];
  if (!d.status) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_status);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetSymbolAddress(status)");
    e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    d.status = static_cast<unsigned int *>(p);
  }
  *out = &d;
  return CSA2_OK;
}

using EncodeTiled = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                 const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                 CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

csa2_status get_encoder(EncodeTiled *fn) {
  static EncodeTiled cached = nullptr;
  static std::once_flag once;
  static cudaError_t err = cudaSuccess;
  std::call_once(once, [] {
    void *p = nullptr;
    cudaDriverEntryPointQueryResult q;
    err = cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q);
    if (err == cudaSuccess && q == cudaDriverEntryPointSuccess) cached = reinterpret_cast<EncodeTiled>(p);
  });
  if (!cached) return fail(CSA2_ERR_CUDA, "cuTensorMapEncodeTiled unavailable (%s)", cudaGetErrorString(err));
  *fn = cached;
  return CSA2_OK;
}

// 2D map over the indexer-key plane [B*cap][d_I] (u8), boxes of `box_rows`
// rows x d_I bytes (128: a whole Full tile per copy; 8: one pool block),
// swizzled to the d_I-byte pattern of the MMA's shared-memory descriptors.
csa2_status encode_ik_map(const csa2_main_cache *m, CUtensorMap *map, int box_rows) {
  EncodeTiled enc = nullptr;
  csa2_status st = get_encoder(&enc);
  if (st != CSA2_OK) return st;
  cuuint64_t dims[2] = {(cuuint64_t)m->d_I, (cuuint64_t)m->B * (cuuint64_t)m->cap};
  cuuint64_t strides[1] = {(cuuint64_t)m->d_I};
  cuuint32_t box[2] = {(cuuint32_t)m->d_I, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, m->ik, dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE,
                   m->d_I == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA2_ERR_INVALID_ARG, "cuTensorMapEncodeTiled failed (%d)", (int)r);
  return CSA2_OK;
}

// 2D map over a row-major bf16 matrix [rows][cols] with boxes of box_rows x 64
// elements (128 bytes) in the 128B swizzle.
csa2_status encode_bf16_map(const void *base, int64_t rows, int64_t cols, int box_rows, CUtensorMap *map) {
  EncodeTiled enc = nullptr;
  csa2_status st = get_encoder(&enc);
  if (st != CSA2_OK) return st;
  cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
  cuuint64_t strides[1] = {(cuuint64_t)cols * 2};
  cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(CSA2_ERR_INVALID_ARG, "cuTensorMapEncodeTiled (bf16) failed (%d)", (int)r);
  return CSA2_OK;
}

csa2_status check_main(const csa2_main_cache *m, bool need_pending) {
  if (!m) return fail(CSA2_ERR_INVALID_ARG, "main cache is NULL");
  if (!m->codes || !m->scales || !m->ik || !m->ik_scale || !m->n_entries)
    return fail(CSA2_ERR_INVALID_ARG, "main cache has a NULL plane");
  if (!aligned16(m->codes) || !aligned16(m->scales) || !aligned16(m->ik) || !aligned16(m->ik_scale) ||
      !aligned16(m->n_entries))
    return fail(CSA2_ERR_INVALID_ARG, "main cache planes must be 16-byte aligned");
  if (m->B <= 0 || m->cap <= 0) return fail(CSA2_ERR_INVALID_ARG, "main cache B=%d cap=%d", m->B, m->cap);
  if (m->cap % 128) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "cap=%d must be a multiple of 128", m->cap);
  if ((int64_t)m->B * m->cap >= (int64_t)1 << 31)
    return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "B*cap must be < 2^31");
  if (m->D != 128 && m->D != 256 && m->D != 512) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "D=%d not in {128,256,512}", m->D);
  if (m->d_I != 64 && m->d_I != 128) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "d_I=%d not in {64,128}", m->d_I);
  if (m->m != 1 && m->m != 2) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "m=%d not in {1,2}", m->m);
  if (need_pending && m->m == 2 && (!m->pending_kv || !m->pending_gate))
    return fail(CSA2_ERR_INVALID_ARG, "m=2 needs the pending buffers");
  return CSA2_OK;
}

csa2_status check_swa(const csa2_swa_cache *s) {
  if (!s->rows) return fail(CSA2_ERR_INVALID_ARG, "window cache rows is NULL");
  if (!aligned16(s->rows)) return fail(CSA2_ERR_INVALID_ARG, "window rows must be 16-byte aligned");
  if (s->B <= 0 || s->W_cap <= 0 || s->window < 0 || s->window > s->W_cap || s->window > 1024)
    return fail(CSA2_ERR_INVALID_ARG, "window cache B=%d W_cap=%d window=%d", s->B, s->W_cap, s->window);
  if (s->D != 128 && s->D != 256 && s->D != 512) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "window D=%d", s->D);
  if (!(s->scale > 0.0f) || s->scale != s->scale) return fail(CSA2_ERR_INVALID_ARG, "window scale must be > 0");
  return CSA2_OK;
}

}  // namespace

void set_last_error_message(const char *msg) { t_err = msg; }

uint32_t injected_timeout_polls() { return g_inject_polls.load(std::memory_order_relaxed); }

}  // namespace csa2

using namespace csa2;

extern "C" {

int csa2_version(void) { return (1 << 16) | 0; }

const char *csa2_last_error(void) { return t_err.c_str(); }

void csa2_debug_inject_timeout(uint32_t polls) { g_inject_polls.store(polls, std::memory_order_relaxed); }

csa2_status csa2_device_status(csa2_stream_t stream, uint32_t *flags, int clear) {
  if (!flags) return fail(CSA2_ERR_INVALID_ARG, "flags is NULL");
  DeviceState *d;
  csa2_status st = device_state(&d);
  if (st != CSA2_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyAsync(&v, d->status, sizeof v, cudaMemcpyDeviceToHost, s);
  if (e == cudaSuccess) e = cudaStreamSynchronize(s);
  if (e == cudaSuccess && clear) e = cudaMemsetAsync(d->status, 0, sizeof v, s);
  if (e == cudaSuccess && clear) e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "csa2_device_status");
  *flags = v;
  return v ? CSA2_ERR_DEVICE_CHECK : CSA2_OK;
}

static csa2_status append_impl(const csa2_main_cache *main, const uint16_t *kv, const uint16_t *gate,
                               const uint16_t *w_ik, const csa2_swa_cache *swa, const uint16_t *kv_swa,
                               const int32_t *pos0, int T, const QueryPrep *prep, csa2_stream_t stream) {
  if (!main && !swa) return fail(CSA2_ERR_INVALID_ARG, "append needs a main or a window cache");
  if (T < 0) return fail(CSA2_ERR_INVALID_ARG, "T=%d", T);
  if (!pos0 || !aligned16(pos0)) return fail(CSA2_ERR_INVALID_ARG, "pos0 must be a 16-byte aligned device pointer");
  csa2_status st;
  int B = 0, D = 0;
  if (main) {
    if ((st = check_main(main, true)) != CSA2_OK) return st;
    if (T > 0 && (!kv || !w_ik || !aligned16(kv) || !aligned16(w_ik)))
      return fail(CSA2_ERR_INVALID_ARG, "kv and w_ik must be 16-byte aligned device pointers");
    if (T > 0 && main->m == 2 && (!gate || !aligned16(gate))) return fail(CSA2_ERR_INVALID_ARG, "m=2 needs gate");
    if (main->m == 2 && (!aligned16(main->pending_kv) || !aligned16(main->pending_gate)))
      return fail(CSA2_ERR_INVALID_ARG, "pending buffers must be 16-byte aligned");
    B = main->B;
    D = main->D;
  }
  if (swa) {
    if ((st = check_swa(swa)) != CSA2_OK) return st;
    if (T > 0 && (!kv_swa || !aligned16(kv_swa)))
      return fail(CSA2_ERR_INVALID_ARG, "kv_swa must be a 16-byte aligned device pointer");
    if (main && (swa->B != B || swa->D != D)) return fail(CSA2_ERR_INVALID_ARG, "window and main cache disagree on B or D");
    B = swa->B;
    D = swa->D;
  }
  if (T == 0 && !prep) return CSA2_OK;
  DeviceState *d;
  if ((st = device_state(&d)) != CSA2_OK) return st;
  AppendArgs a{};
  if (prep) a.prep = *prep;
  if (main) {
    a.codes = main->codes; a.scales = main->scales; a.ik = main->ik; a.ik_scale = main->ik_scale;
    a.n_entries = main->n_entries; a.pending_kv = main->pending_kv; a.pending_gate = main->pending_gate;
    a.cap = main->cap; a.dI = main->d_I; a.m = main->m;
    a.kv = kv; a.gate = gate; a.w_ik = w_ik;
    const int max_new = T == 0 ? 0 : (main->m == 1 ? T : T / 2 + 1);   // upper bound of complete entries
    a.entries_per_block = max_new >= 256 ? 32 : (max_new >= 64 ? 8 : 1);
    a.main_blocks_per_seq = (max_new + a.entries_per_block - 1) / a.entries_per_block;
  }
  if (!main) a.entries_per_block = 1;
  a.B = B; a.D = D;
  if (swa) {
    a.swa_rows = swa->rows; a.s_swa = swa->scale; a.W_cap = swa->W_cap; a.kv_swa = kv_swa;
    a.swa_blocks_per_seq = T < swa->W_cap ? T : swa->W_cap;
  }
  a.pos0 = pos0; a.T = T; a.status = d->status;
  if ((int64_t)B * (a.main_blocks_per_seq + a.swa_blocks_per_seq) >= (int64_t)1 << 31)
    return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "too many append blocks");
  cudaError_t e = launch_append(a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "append launch");
}

csa2_status csa2_append_quant(const csa2_main_cache *main, const uint16_t *kv, const uint16_t *gate,
                              const uint16_t *w_ik, const csa2_swa_cache *swa, const uint16_t *kv_swa,
                              const int32_t *pos0, int T, csa2_stream_t stream) {
  t_err.clear();
  NvtxRange nvtx("csa2_append_quant");
  return append_impl(main, kv, gate, w_ik, swa, kv_swa, pos0, T, nullptr, stream);
}

csa2_status csa2_append_quant_ex(const csa2_main_cache *main, const uint16_t *kv, const uint16_t *gate,
                                 const uint16_t *w_ik, const csa2_swa_cache *swa, const uint16_t *kv_swa,
                                 const int32_t *pos0, int T, const uint16_t *q_idx, const float *w, int T_q,
                                 int H_I, void *ws, size_t ws_bytes, csa2_stream_t stream) {
  t_err.clear();
  NvtxRange nvtx("csa2_append_quant_ex");
  if (!main) return fail(CSA2_ERR_INVALID_ARG, "preparing a scan's query needs the main cache (its d_I)");
  if (!q_idx || !w || !aligned16(q_idx) || !aligned16(w))
    return fail(CSA2_ERR_INVALID_ARG, "q_idx and w must be 16-byte aligned device pointers");
  if (T_q <= 0 || (int64_t)main->B * T_q > 65535) return fail(CSA2_ERR_INVALID_ARG, "T_q=%d", T_q);
  if (H_I < 1 || H_I > 64) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "H_I=%d not in [1,64]", H_I);
  if (main->d_I != 64 && main->d_I != 128) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "d_I=%d", main->d_I);
  const int rows = main->B * T_q;
  const size_t need = index_workspace_bytes(rows, main->d_I);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return fail(CSA2_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, ws_bytes);
  QueryPrep p{};
  p.q_idx = q_idx; p.w = w; p.rows = rows; p.H_I = H_I; p.dI = main->d_I;
  p.q8 = static_cast<uint8_t *>(ws);
  p.wq = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) + (((size_t)rows * 64 * main->d_I + 15) & ~size_t(15)));
  return append_impl(main, kv, gate, w_ik, swa, kv_swa, pos0, T, &p, stream);
}

csa2_status csa2_append_project(const csa2_main_cache *main, const uint16_t *h, int d_model, const uint16_t *w_kv,
                                const uint16_t *w_ik, const int32_t *pos0, int T, csa2_stream_t stream) {
  t_err.clear();
  NvtxRange nvtx("csa2_append_project");
  csa2_status st;
  if ((st = check_main(main, false)) != CSA2_OK) return st;
  if (main->m != 1) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "the projected append serves m = 1 caches (m=%d)", main->m);
  if (main->D % 256) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "D=%d must be a multiple of 256", main->D);
  if (d_model < 64 || d_model > 32768 || d_model % 64)
    return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "d_model=%d must be a multiple of 64 in [64, 32768]", d_model);
  if (T < 0) return fail(CSA2_ERR_INVALID_ARG, "T=%d", T);
  if (!pos0 || !aligned16(pos0)) return fail(CSA2_ERR_INVALID_ARG, "pos0 must be a 16-byte aligned device pointer");
  if (T == 0) return CSA2_OK;
  if (!h || !w_kv || !w_ik || !aligned16(h) || !aligned16(w_kv) || !aligned16(w_ik))
    return fail(CSA2_ERR_INVALID_ARG, "h, w_kv and w_ik must be 16-byte aligned device pointers");
  if ((int64_t)main->B * T >= (int64_t)1 << 31) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "B*T must be < 2^31");
  DeviceState *d;
  if ((st = device_state(&d)) != CSA2_OK) return st;
  CUtensorMap hm, wm;
  if ((st = encode_bf16_map(h, (int64_t)main->B * T, d_model, 128, &hm)) != CSA2_OK) return st;
  if ((st = encode_bf16_map(w_kv, d_model, main->D, 64, &wm)) != CSA2_OK) return st;
  ProjectArgs p{};
  p.codes = main->codes; p.scales = main->scales; p.n_entries = main->n_entries;
  p.B = main->B; p.cap = main->cap; p.D = main->D; p.pos0 = pos0; p.T = T; p.d = d_model; p.status = d->status;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_project(hm, wm, p, s);
  if (e != cudaSuccess) return cuda_fail(e, "projection launch");
  AppendArgs a{};
  a.codes = main->codes; a.scales = main->scales; a.ik = main->ik; a.ik_scale = main->ik_scale;
  a.n_entries = main->n_entries; a.B = main->B; a.cap = main->cap; a.D = main->D; a.dI = main->d_I; a.m = 1;
  a.w_ik = w_ik; a.pos0 = pos0; a.T = T; a.status = d->status;
  a.entries_per_block = T >= 256 ? 32 : 8;
  a.main_blocks_per_seq = (T + a.entries_per_block - 1) / a.entries_per_block;
  e = launch_append_keys(a, s);
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "key projection launch");
}

// Blocks per row of a scan: about four resident blocks per SM in one wave,
// the row's tiles split evenly over them.
static int index_ctas_per_row(int tiles_per_row, int rows, int sms) {
  int64_t c = (int64_t)sms * 4 / rows;
  if (c < 1) c = 1;
  if (c > tiles_per_row) c = tiles_per_row;
  return (int)c;
}

static csa2_status index_common(const csa2_main_cache *main, const uint16_t *q_idx, const float *w,
                                const int32_t *q_pos, int T_q, int H_I, float *scores, void *ws, size_t ws_bytes,
                                IndexArgs *a, CUtensorMap *map, int box_rows, bool prepared = false) {
  csa2_status st;
  if ((st = check_main(main, false)) != CSA2_OK) return st;
  if (!prepared && (!q_idx || !w)) return fail(CSA2_ERR_INVALID_ARG, "NULL argument");
  if (!q_pos || !scores) return fail(CSA2_ERR_INVALID_ARG, "NULL argument");
  if ((!prepared && (!aligned16(q_idx) || !aligned16(w))) || !aligned16(q_pos) || !aligned16(scores))
    return fail(CSA2_ERR_INVALID_ARG, "pointers must be 16-byte aligned");
  if (T_q <= 0) return fail(CSA2_ERR_INVALID_ARG, "T_q=%d", T_q);
  if (!prepared && (H_I < 1 || H_I > 64)) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "H_I=%d not in [1,64]", H_I);
  if ((int64_t)main->B * T_q > 65535) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "B*T_q must be <= 65535");
  const size_t need = index_workspace_bytes(main->B * T_q, main->d_I);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return fail(CSA2_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, ws_bytes);
  if ((st = encode_ik_map(main, map, box_rows)) != CSA2_OK) return st;
  *a = IndexArgs{};
  a->q8 = static_cast<uint8_t *>(ws);
  a->wq = reinterpret_cast<float *>(static_cast<uint8_t *>(ws) +
                                    (((size_t)main->B * T_q * 64 * main->d_I + 15) & ~size_t(15)));
  a->ik_scale = main->ik_scale; a->n_entries = main->n_entries;
  a->B = main->B; a->cap = main->cap; a->m = main->m; a->dI = main->d_I;
  a->q_idx = q_idx; a->w = w; a->q_pos = q_pos; a->T_q = T_q; a->H_I = H_I; a->scores = scores;
  a->prepared = prepared;
  a->inject_polls = injected_timeout_polls();
  return CSA2_OK;
}

size_t csa2_index_workspace_size(int rows, int d_I) {
  if (rows <= 0 || (d_I != 64 && d_I != 128)) return 0;
  return index_workspace_bytes(rows, d_I);
}

static csa2_status index_full_impl(const csa2_main_cache *main, const uint16_t *q_idx, const float *w,
                                   const int32_t *q_pos, int T_q, int H_I, float *scores, int64_t ld,
                                   int32_t *n_valid, void *ws, size_t ws_bytes, bool prepared, csa2_stream_t stream,
                                   float *bmax = nullptr, int64_t ld_b = 0) {
  IndexArgs a;
  CUtensorMap map;
  csa2_status st = index_common(main, q_idx, w, q_pos, T_q, H_I, scores, ws, ws_bytes, &a, &map, 128, prepared);
  if (st != CSA2_OK) return st;
  if (ld < main->cap) return fail(CSA2_ERR_INVALID_ARG, "ld=%lld < cap=%d", (long long)ld, main->cap);
  if (n_valid && !aligned16(n_valid)) return fail(CSA2_ERR_INVALID_ARG, "n_valid must be 16-byte aligned");
  DeviceState *d;
  if ((st = device_state(&d)) != CSA2_OK) return st;
  a.ld = ld; a.n_valid = n_valid; a.status = d->status;
  a.bmax = bmax; a.ld_b = ld_b;
  a.tiles_per_row = main->cap / 128;
  const int R = index_rows_per_block(T_q, false);
  if (R == 1) {
    a.ctas_per_row = index_ctas_per_row(a.tiles_per_row, main->B * T_q, d->sms);
  } else {   // R rows per block, 4/R blocks per SM
    const int64_t groups = (int64_t)main->B * T_q / R;
    int64_t c = (int64_t)d->sms * (4 / R) / groups;
    if (c < 1) c = 1;
    if (c > a.tiles_per_row) c = a.tiles_per_row;
    a.ctas_per_row = (int)c;
  }
  cudaError_t e = launch_index(map, a, false, d->sms, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "index_full launch");
}

csa2_status csa2_index_full(const csa2_main_cache *main, const uint16_t *q_idx, const float *w,
                            const int32_t *q_pos, int T_q, int H_I, float *scores, int64_t ld,
                            int32_t *n_valid, void *ws, size_t ws_bytes, csa2_stream_t stream) {
  t_err.clear();
  NvtxRange nvtx("csa2_index_full");
  return index_full_impl(main, q_idx, w, q_pos, T_q, H_I, scores, ld, n_valid, ws, ws_bytes, false, stream);
}

csa2_status csa2_index_full_prepared(const csa2_main_cache *main, const int32_t *q_pos, int T_q, float *scores,
                                     int64_t ld, int32_t *n_valid, const void *ws, size_t ws_bytes,
                                     csa2_stream_t stream) {
  t_err.clear();
  NvtxRange nvtx("csa2_index_full_prepared");
  return index_full_impl(main, nullptr, nullptr, q_pos, T_q, 64, scores, ld, n_valid, const_cast<void *>(ws),
                         ws_bytes, true, stream);
}

// Workspace of csa2_index_topk: the prepared query (as for csa2_index_full),
// then the block maxima [rows][cap/8] f32, then n_valid [rows] i32.
static size_t index_topk_offsets(int rows, int cap, int d_I, size_t *off_b, size_t *off_nv) {
  const size_t q = (index_workspace_bytes(rows, d_I) + 15) & ~size_t(15);
  const size_t b = ((size_t)rows * (cap / 8) * 4 + 15) & ~size_t(15);
  *off_b = q;
  *off_nv = q + b;
  return q + b + (((size_t)rows * 4 + 15) & ~size_t(15));
}

size_t csa2_index_topk_workspace_size(int rows, int cap, int d_I) {
  if (rows <= 0 || cap <= 0 || cap % 128 || (d_I != 64 && d_I != 128)) return 0;
  size_t ob, onv;
  return index_topk_offsets(rows, cap, d_I, &ob, &onv);
}

csa2_status csa2_index_topk(const csa2_main_cache *main, const uint16_t *q_idx, const float *w,
                            const int32_t *q_pos, int T_q, int H_I, float *scores, int64_t ld, int32_t *n_valid,
                            int K, int32_t *out_idx, int P_out, int32_t *out_pool, float *out_scores,
                            float *out_pool_scores, void *ws, size_t ws_bytes, csa2_stream_t stream) {
  t_err.clear();
  NvtxRange nvtx("csa2_index_topk");
  csa2_status st;
  if ((st = check_main(main, false)) != CSA2_OK) return st;
  const bool prepared = !q_idx && !w;
  if (main->cap > kTopkBmaxMaxBlocks * 8)
    return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "cap=%d above %d (use csa2_index_full + csa2_topk)", main->cap,
                kTopkBmaxMaxBlocks * 8);
  if (K < 1 || K > 2048) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "K=%d not in [1,2048]", K);
  if (P_out < 0 || P_out > 4096) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "P_out=%d not in [0,4096]", P_out);
  if (!out_idx || !aligned16(out_idx)) return fail(CSA2_ERR_INVALID_ARG, "out_idx must be a 16-byte aligned device pointer");
  if (P_out > 0 && (!out_pool || !aligned16(out_pool))) return fail(CSA2_ERR_INVALID_ARG, "out_pool needed");
  if (ld % 4) return fail(CSA2_ERR_INVALID_ARG, "ld=%lld must be a multiple of 4", (long long)ld);
  if ((out_scores && !aligned16(out_scores)) || (out_pool_scores && !aligned16(out_pool_scores)))
    return fail(CSA2_ERR_INVALID_ARG, "out_scores / out_pool_scores must be 16-byte aligned");
  if (T_q <= 0 || (int64_t)main->B * T_q > 65535) return fail(CSA2_ERR_INVALID_ARG, "T_q=%d", T_q);
  const int rows = main->B * T_q;
  size_t off_b, off_nv;
  const size_t need = index_topk_offsets(rows, main->cap, main->d_I, &off_b, &off_nv);
  if (!ws || ws_bytes < need || !aligned16(ws))
    return fail(CSA2_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", need, ws_bytes);
  uint8_t *wb = static_cast<uint8_t *>(ws);
  float *bmax = reinterpret_cast<float *>(wb + off_b);
  int32_t *nv = n_valid ? n_valid : reinterpret_cast<int32_t *>(wb + off_nv);
  st = index_full_impl(main, q_idx, w, q_pos, T_q, prepared ? 64 : H_I, scores, ld, nv, ws, ws_bytes, prepared,
                       stream, bmax, main->cap / 8);
  if (st != CSA2_OK) return st;
  TopkBmaxArgs t{scores, ld, bmax, main->cap / 8, rows, main->cap, nv, K, out_idx, P_out, out_pool,
                 out_scores, P_out > 0 ? out_pool_scores : nullptr};
  cudaError_t e = launch_topk_bmax(t, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "topk_bmax launch");
}

csa2_status csa2_topk_merge(const float *scores, const int32_t *ids, int G, int rows, int n_seg,
                            const int32_t *seg_base, int K, int32_t *out_ids, float *out_scores,
                            csa2_stream_t stream) {
  t_err.clear();
  NvtxRange nvtx("csa2_topk_merge");
  if (!scores || !ids || !out_ids || !aligned16(scores) || !aligned16(ids) || !aligned16(out_ids))
    return fail(CSA2_ERR_INVALID_ARG, "scores/ids/out_ids must be 16-byte aligned device pointers");
  if (out_scores && !aligned16(out_scores)) return fail(CSA2_ERR_INVALID_ARG, "out_scores alignment");
  if (!seg_base) return fail(CSA2_ERR_INVALID_ARG, "seg_base (host array of G ints) is NULL");
  if (G < 1 || G > kMergeMaxShards) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "G=%d not in [1,%d]", G, kMergeMaxShards);
  if (rows < 1 || rows > 65535 || n_seg < 1) return fail(CSA2_ERR_INVALID_ARG, "rows=%d n_seg=%d", rows, n_seg);
  if ((int64_t)G * n_seg > kTopkBmaxMaxBlocks)
    return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "G*n_seg=%lld above %d", (long long)G * n_seg, kTopkBmaxMaxBlocks);
  if (K < 1 || K > 4096) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "K=%d not in [1,4096]", K);
  TopkMergeArgs a{};
  a.scores = scores; a.ids = ids; a.G = G; a.rows = rows; a.n_seg = n_seg;
  for (int g = 0; g < G; ++g) a.seg_base[g] = seg_base[g];
  a.K = K; a.out_ids = out_ids; a.out_scores = out_scores;
  cudaError_t e = launch_topk_merge(a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "topk_merge launch");
}

csa2_status csa2_gather_entries(const csa2_main_cache *shard, int lo, const int32_t *ids, int K,
                                uint8_t *out_codes, uint8_t *out_scales, int out_cap, int32_t *out_pos,
                                csa2_stream_t stream) {
  t_err.clear();
  NvtxRange nvtx("csa2_gather_entries");
  csa2_status st;
  if ((st = check_main(shard, false)) != CSA2_OK) return st;
  if (!ids || !out_codes || !out_scales || !aligned16(ids) || !aligned16(out_codes) || !aligned16(out_scales))
    return fail(CSA2_ERR_INVALID_ARG, "ids/out_codes/out_scales must be 16-byte aligned device pointers");
  if (out_pos && !aligned16(out_pos)) return fail(CSA2_ERR_INVALID_ARG, "out_pos alignment");
  if (lo < 0) return fail(CSA2_ERR_INVALID_ARG, "lo=%d", lo);
  if (K < 1 || K > 4096 || out_cap < K) return fail(CSA2_ERR_INVALID_ARG, "K=%d out_cap=%d", K, out_cap);
  GatherArgs a{};
  a.codes = shard->codes; a.scales = shard->scales; a.B = shard->B; a.cap = shard->cap; a.D = shard->D; a.lo = lo;
  a.ids = ids; a.K = K; a.out_codes = out_codes; a.out_scales = out_scales; a.out_cap = out_cap; a.out_pos = out_pos;
  cudaError_t e = launch_gather_entries(a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "gather_entries launch");
}

csa2_status csa2_index_reindex(const csa2_main_cache *main, const uint16_t *q_idx, const float *w,
                               const int32_t *q_pos, int T_q, int H_I, const int32_t *pool_blocks, int P,
                               float *pool_scores, void *ws, size_t ws_bytes, csa2_stream_t stream) {
  t_err.clear();
  NvtxRange nvtx("csa2_index_reindex");
  IndexArgs a;
  CUtensorMap map;
  csa2_status st = index_common(main, q_idx, w, q_pos, T_q, H_I, pool_scores, ws, ws_bytes, &a, &map, 8);
  if (st != CSA2_OK) return st;
  if (!pool_blocks || !aligned16(pool_blocks)) return fail(CSA2_ERR_INVALID_ARG, "pool_blocks must be a 16-byte aligned device pointer");
  if (P < 16 || P > 4096 || P % 16) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "P=%d must be a multiple of 16 in [16,4096]", P);
  DeviceState *d;
  if ((st = device_state(&d)) != CSA2_OK) return st;
  a.ld = (int64_t)P * 8; a.pool = pool_blocks; a.P = P; a.status = d->status;
  a.tiles_per_row = P / 16;
  a.ctas_per_row = index_ctas_per_row(a.tiles_per_row, main->B * T_q, d->sms);
  cudaError_t e = launch_index(map, a, true, d->sms, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "index_reindex launch");
}

size_t csa2_topk_workspace_size(int rows, int n_cols, int K, int P_out) {
  if (rows <= 0 || n_cols < 0 || K <= 0) return 0;
  return plan_topk(rows, n_cols, K, P_out).bytes;
}

csa2_status csa2_topk(const float *scores, int rows, int64_t ld, int n_cols, const int32_t *n_valid,
                      const int32_t *pool_blocks, int K, int32_t *out_idx, int P_out, int32_t *out_pool,
                      void *ws, size_t ws_bytes, csa2_stream_t stream) {
  t_err.clear();
  NvtxRange nvtx("csa2_topk");
  if (!scores || !out_idx || !aligned16(scores) || !aligned16(out_idx))
    return fail(CSA2_ERR_INVALID_ARG, "scores/out_idx must be 16-byte aligned device pointers");
  if (rows <= 0 || rows > 65535) return fail(CSA2_ERR_INVALID_ARG, "rows=%d", rows);
  if (n_cols < 0 || n_cols > (1 << 20) || ld < n_cols) return fail(CSA2_ERR_INVALID_ARG, "n_cols=%d ld=%lld", n_cols, (long long)ld);
  if (K < 1 || K > 2048) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "K=%d not in [1,2048]", K);
  if (P_out < 0 || P_out > 4096) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "P_out=%d not in [0,4096]", P_out);
  if (P_out > 0 && (!out_pool || !aligned16(out_pool))) return fail(CSA2_ERR_INVALID_ARG, "out_pool needed");
  if (P_out > 0 && pool_blocks) return fail(CSA2_ERR_INVALID_ARG, "a pool is built from entry scores only");
  if (pool_blocks && (!aligned16(pool_blocks) || n_cols % 8)) return fail(CSA2_ERR_INVALID_ARG, "pool_blocks alignment / n_cols%%8");
  if (n_valid && !aligned16(n_valid)) return fail(CSA2_ERR_INVALID_ARG, "n_valid alignment");
  const TopkPlan p = plan_topk(rows, n_cols, K, P_out);
  if (p.bytes > 0 && (!ws || ws_bytes < p.bytes || !aligned16(ws)))
    return fail(CSA2_ERR_WORKSPACE, "workspace of %zu bytes needed (got %zu)", p.bytes, ws_bytes);
  TopkArgs a{scores, rows, ld, n_cols, n_valid, pool_blocks, K, out_idx, P_out, out_pool, ws};
  cudaError_t e = launch_topk(a, p, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "topk launch");
}

size_t csa2_attn_workspace_size(int B, int T_q, int H, int D, int K, int window) {
  if (B <= 0 || T_q <= 0) return 0;
  DeviceState *d;
  int sms = 148;
  if (device_state(&d) == CSA2_OK) sms = d->sms;
  return plan_attn(B, T_q, H, D, K, window, sms).bytes;
}

csa2_status csa2_sparse_attn_decode(const csa2_main_cache *main, const csa2_swa_cache *swa, const uint16_t *q,
                                    const int32_t *q_pos, int T_q, int H, const int32_t *idx, int K,
                                    float softmax_scale, uint16_t *out, void *ws, size_t ws_bytes,
                                    csa2_stream_t stream) {
  t_err.clear();
  NvtxRange nvtx("csa2_sparse_attn_decode");
  csa2_status st;
  if ((st = check_main(main, false)) != CSA2_OK) return st;
  if (!swa) return fail(CSA2_ERR_INVALID_ARG, "window cache is NULL");
  if ((st = check_swa(swa)) != CSA2_OK) return st;
  if (swa->B != main->B || swa->D != main->D) return fail(CSA2_ERR_INVALID_ARG, "window and main cache disagree");
  if (!q || !q_pos || !out || !aligned16(q) || !aligned16(q_pos) || !aligned16(out))
    return fail(CSA2_ERR_INVALID_ARG, "q/q_pos/out must be 16-byte aligned device pointers");
  if (K < 0 || K > 2048) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "K=%d not in [0,2048]", K);
  if (K > 0 && (!idx || !aligned16(idx)))
    return fail(CSA2_ERR_INVALID_ARG, "idx must be a 16-byte aligned device pointer when K > 0");
  if (T_q <= 0 || (int64_t)main->B * T_q > 65535) return fail(CSA2_ERR_INVALID_ARG, "T_q=%d", T_q);
  if (H < 1 || H > 64) return fail(CSA2_ERR_UNSUPPORTED_SHAPE, "H=%d not in [1,64]", H);
  DeviceState *d;
  if ((st = device_state(&d)) != CSA2_OK) return st;
  AttnPlan p = plan_attn(main->B, T_q, H, main->D, K, swa->window, d->sms);
  if (p.nsplit > 1 && (!ws || ws_bytes < p.bytes || !aligned16(ws))) {   // no workspace: one block per row
    p.nsplit = 1;
    p.chunks_per_split = 1 << 20;
    p.csplit = 1;
    p.latency_form = ((int64_t)main->B * T_q <= d->sms && K <= 128 && swa->window <= 128 && (K == 0 || swa->window == 0))
                         ? 1 : 0;   // one 128-key tile per row
  }
  AttnArgs a{};
  a.codes = main->codes; a.scales = main->scales; a.cap = main->cap; a.D = main->D;
  a.swa_rows = swa->rows; a.s_swa = swa->scale; a.W_cap = swa->W_cap; a.window = swa->window;
  a.q = q; a.q_pos = q_pos; a.B = main->B; a.T_q = T_q; a.H = H; a.idx = K > 0 ? idx : nullptr; a.K = K;
  a.scale = softmax_scale; a.out = out;
  a.ws = p.nsplit > 1 ? static_cast<float *>(ws) : nullptr;
  a.nsplit = p.nsplit; a.chunks_per_split = p.chunks_per_split; a.csplit = p.csplit; a.latency_form = p.latency_form;
  a.status = d->status;
  cudaError_t e = launch_attn(a, reinterpret_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? CSA2_OK : cuda_fail(e, "attention launch");
}

}  // extern "C"
