// Decode attention for callers that cannot allocate device memory.
//
// tq_attend_decode needs a caller-provided workspace for the rotated queries, the
// S-projected queries and the per-split partial results.  Some callers have no way to
// provide one: a plugin running inside a host runtime that owns the whole device memory
// pool and hands out no allocator, or a serving loop whose memory was planned once at
// start-up and which must not call cudaMalloc (an allocation can block on the device and
// stall every stream) in the middle of a decode step.  For them this file keeps the
// workspace in a fixed array in device global memory, defined at file scope, and passes
// its address to the unchanged decode kernels.
//
// The array costs kScratchBytes of device memory on every GPU that loads this library,
// held until the process exits.  All calls on a device share it, so two calls whose
// kernels overlap in time (different streams, or different host threads without
// ordering) race on it and their results are undefined; order them on one stream.  The
// decode kernels write every scratch byte they later read (rotated queries, S-projected
// queries and every (row, split) partial), so nothing has to be cleared between calls.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "tq.h"
#include "tq_internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;  // 8 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

std::mutex g_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// The array's name is only a host-side handle; the device address has to be looked up
// once per device with that device current.
tq_status scratch_address(void** out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return tqi::fail(TQ_ERR_CUDA, "tq_attend_decode_noalloc: cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices)
    return tqi::fail(TQ_ERR_UNSUPPORTED, "tq_attend_decode_noalloc: device ordinal above 63");
  std::lock_guard<std::mutex> lock(g_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_decode_scratch);
    if (e != cudaSuccess || p == nullptr) {
      char buf[256];
      std::snprintf(buf, sizeof(buf), "tq_attend_decode_noalloc: cudaGetSymbolAddress failed: %s",
                    cudaGetErrorString(e));
      return tqi::fail(TQ_ERR_CUDA, buf);
    }
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return TQ_OK;
}

}  // namespace

extern "C" tq_status tq_attend_decode_noalloc(const tq_config* cfg, const tq_params* params,
                                              const tq_cache* cache, int32_t layer, const void* q,
                                              int32_t q_dtype, int32_t q_heads, int32_t seq_q,
                                              const int32_t* seq_lens, int32_t n_splits, float* out,
                                              int32_t* dev_status, tq_stream_t stream) {
  tqi::clear_error();
  if (!cfg || !cache) return tqi::fail(TQ_ERR_INVALID_ARG, "tq_attend_decode_noalloc: config or cache is NULL");
  const size_t need = tq_decode_workspace_bytes(cfg, cache->batch, q_heads, seq_q, n_splits);
  if (need == 0)
    return tqi::fail(TQ_ERR_INVALID_ARG,
                     "tq_attend_decode_noalloc: invalid config, batch, q_heads, seq_q or n_splits");
  if (need > kScratchBytes) {
    char buf[320];
    std::snprintf(buf, sizeof(buf),
                  "tq_attend_decode_noalloc: these sizes need %zu bytes of scratch but the built-in "
                  "buffer holds %zu (8 MiB); use fewer splits, fewer query rows, or "
                  "tq_attend_decode with a caller workspace",
                  need, kScratchBytes);
    return tqi::fail(TQ_ERR_UNSUPPORTED, buf);
  }
  void* ws = nullptr;
  const tq_status st = scratch_address(&ws);
  if (st != TQ_OK) return st;
  return tq_attend_decode(cfg, params, cache, layer, q, q_dtype, q_heads, seq_q, seq_lens, n_splits, ws,
                          kScratchBytes, out, dev_status, stream);
}
