// csa2_topk_noalloc: the Top-K / candidate-pool selection of csa2_topk for
// callers that cannot allocate device memory when they call the library.
//
// Some callers have no way to obtain a scratch buffer at call time: a plugin
// running inside another framework's execution engine, whose device memory is
// planned ahead and owned by that framework, or code that must not allocate
// because an allocation would disturb what it is doing (a latency-critical
// serving loop, a region being captured into a CUDA graph by someone else).
// This variant takes the same inputs and outputs as csa2_topk but keeps its
// scratch in a fixed array in device global memory that is part of the
// library itself.
//
// Costs and rules of that choice:
//  - The array (kNoallocScratchBytes = 4 MiB) exists on every GPU that loads
//    the library, from module load until process exit.
//  - Calls whose scratch need (csa2_topk_workspace_size) exceeds it are
//    rejected with CSA2_ERR_WORKSPACE; nothing is enqueued.
//  - Every call uses the same array.  Two calls whose kernels can overlap on
//    the GPU (different streams without ordering between them) race on it and
//    give undefined results; calls on one stream are safe.
//  - The array keeps the contents of the previous call.  Nothing in it has
//    to start at zero: the first kernel writes every slot the second reads.
//  - The first call on a device looks up the array's device address (host
//    code only sees a host-side stand-in for the array's name).  Make that
//    first call before any stream capture on that device.  The address is
//    kept for the life of the process: after a cudaDeviceReset it would point
//    into the destroyed context, so a process that resets a device must not
//    call this entry point on it again.
#include <cstdarg>
#include <cstdio>
#include <mutex>

#include <nvtx3/nvToolsExt.h>

#include "common.cuh"
#include "kernels.h"

namespace csa2 {

// Sets the message csa2_last_error() returns on this thread (defined in api.cu).
void set_last_error_message(const char *msg);

namespace {

constexpr size_t kNoallocScratchBytes = size_t(4) << 20;

// The scratch itself (device global memory, 256-byte aligned).
static __device__ __align__(256) unsigned char g_topk_scratch[kNoallocScratchBytes];

std::mutex g_noalloc_mu;
void *g_noalloc_ptr[64];   // device address of g_topk_scratch, per device ordinal

csa2_status noalloc_fail(csa2_status st, const char *fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof buf, fmt, ap);
  va_end(ap);
  set_last_error_message(buf);
  return st;
}

bool noalloc_aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Once per device, with that device current: the device address of the array.
csa2_status scratch_address(void **out) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(CSA2_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= 64) return noalloc_fail(CSA2_ERR_CUDA, "device ordinal %d out of range", dev);
  std::lock_guard<std::mutex> lk(g_noalloc_mu);
  if (!g_noalloc_ptr[dev]) {
    void *p = nullptr;
    e = cudaGetSymbolAddress(&p, g_topk_scratch);
    if (e != cudaSuccess)
      return noalloc_fail(CSA2_ERR_CUDA, "cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
    g_noalloc_ptr[dev] = p;
  }
  *out = g_noalloc_ptr[dev];
  return CSA2_OK;
}

}  // namespace
}  // namespace csa2

using namespace csa2;

static csa2_status topk_noalloc_impl(const float *scores, int rows, int64_t ld, int n_cols, const int32_t *n_valid,
                                     const int32_t *pool_blocks, int K, int32_t *out_idx, int P_out,
                                     int32_t *out_pool, csa2_stream_t stream);

extern "C" CSA2_API csa2_status csa2_topk_noalloc(const float *scores, int rows, int64_t ld, int n_cols,
                                                  const int32_t *n_valid, const int32_t *pool_blocks, int K,
                                                  int32_t *out_idx, int P_out, int32_t *out_pool,
                                                  csa2_stream_t stream) {
  set_last_error_message("");
  nvtxRangePushA("csa2_topk_noalloc");
  const csa2_status st = topk_noalloc_impl(scores, rows, ld, n_cols, n_valid, pool_blocks, K, out_idx, P_out, out_pool,
                                           stream);
  nvtxRangePop();
  return st;
}

static csa2_status topk_noalloc_impl(const float *scores, int rows, int64_t ld, int n_cols, const int32_t *n_valid,
                                     const int32_t *pool_blocks, int K, int32_t *out_idx, int P_out,
                                     int32_t *out_pool, csa2_stream_t stream) {
  if (!scores || !out_idx || !noalloc_aligned16(scores) || !noalloc_aligned16(out_idx))
    return noalloc_fail(CSA2_ERR_INVALID_ARG, "scores/out_idx must be 16-byte aligned device pointers");
  if (rows <= 0 || rows > 65535) return noalloc_fail(CSA2_ERR_INVALID_ARG, "rows=%d", rows);
  if (n_cols < 0 || n_cols > (1 << 20) || ld < n_cols)
    return noalloc_fail(CSA2_ERR_INVALID_ARG, "n_cols=%d ld=%lld", n_cols, (long long)ld);
  if (K < 1 || K > 2048) return noalloc_fail(CSA2_ERR_UNSUPPORTED_SHAPE, "K=%d not in [1,2048]", K);
  if (P_out < 0 || P_out > 4096) return noalloc_fail(CSA2_ERR_UNSUPPORTED_SHAPE, "P_out=%d not in [0,4096]", P_out);
  if (P_out > 0 && (!out_pool || !noalloc_aligned16(out_pool)))
    return noalloc_fail(CSA2_ERR_INVALID_ARG, "out_pool needed");
  if (P_out > 0 && pool_blocks) return noalloc_fail(CSA2_ERR_INVALID_ARG, "a pool is built from entry scores only");
  if (pool_blocks && (!noalloc_aligned16(pool_blocks) || n_cols % 8))
    return noalloc_fail(CSA2_ERR_INVALID_ARG, "pool_blocks alignment / n_cols%%8");
  if (n_valid && !noalloc_aligned16(n_valid)) return noalloc_fail(CSA2_ERR_INVALID_ARG, "n_valid alignment");
  const TopkPlan p = plan_topk(rows, n_cols, K, P_out);
  if (p.bytes > kNoallocScratchBytes)
    return noalloc_fail(CSA2_ERR_WORKSPACE,
                        "this selection needs %zu bytes of scratch; the built-in scratch of csa2_topk_noalloc "
                        "holds %zu bytes (use csa2_topk with a caller workspace)",
                        p.bytes, kNoallocScratchBytes);
  void *ws = nullptr;
  csa2_status st = scratch_address(&ws);
  if (st != CSA2_OK) return st;
  TopkArgs a{scores, rows, ld, n_cols, n_valid, pool_blocks, K, out_idx, P_out, out_pool, ws};
  cudaError_t e = launch_topk(a, p, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return noalloc_fail(CSA2_ERR_CUDA, "topk_noalloc launch: %s", cudaGetErrorString(e));
  return CSA2_OK;
}
