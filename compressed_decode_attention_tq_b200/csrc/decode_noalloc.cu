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
// The array costs kScratchBytes of device memory in every CUDA context that loads this
// file's module, held until the context ends.  With lazy module loading (the CUDA default
// since 11.7) the module, and with it the array, is loaded on a device at the first call
// of this entry point there, not at library load: that first call is where the 8 MiB are
// taken, so a caller whose pool is claimed later makes it at start-up.  All calls on a
// device share it, so two calls whose
// kernels overlap in time (different streams, or different host threads without
// ordering) race on it and their results are undefined; order them on one stream.  The
// decode kernels write every scratch byte they later read (rotated queries, S-projected
// queries, the merge counters and every (row, split) partial), so nothing has to be
// cleared between calls.
#include <cuda_runtime.h>

#include <cstdio>
#include <mutex>

#include "tq.h"
#include "tq_internal.h"

namespace {

constexpr size_t kScratchBytes = size_t(8) << 20;  // 8 MiB
constexpr int kMaxContexts = 64;

static __device__ __align__(256) unsigned char g_decode_scratch[kScratchBytes];

// The array's name is only a host-side handle: its device address belongs to the module
// loaded in one CUDA context, and it has to be looked up with that context current.  The
// lookup is repeated on every call made outside stream capture (a host-side table lookup
// once the module is loaded), so a context that was destroyed and re-created (after
// cudaDeviceReset, say) never reuses an address of the old one.  Calls made while the
// stream is being captured cannot make that lookup (it may load the module, which capture
// forbids) and reuse the address last found for the same context.
typedef int (*CtxGetCurrentFn)(void**);

std::mutex g_mutex;
struct Entry {
  void* ctx;
  void* addr;
};
Entry g_entries[kMaxContexts] = {};
CtxGetCurrentFn g_ctx_get = nullptr;
bool g_ctx_get_resolved = false;

// The current driver context, read through the driver entry point the runtime hands out
// (the library does not link the driver library directly); null if it cannot be read.
void* current_context() {
  if (!g_ctx_get_resolved) {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &fn, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_ctx_get = reinterpret_cast<CtxGetCurrentFn>(fn);
    g_ctx_get_resolved = true;
  }
  void* ctx = nullptr;
  if (g_ctx_get == nullptr || g_ctx_get(&ctx) != 0) return nullptr;
  return ctx;
}

tq_status scratch_address(cudaStream_t stream, void** out) {
  std::lock_guard<std::mutex> lock(g_mutex);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  cudaError_t e = cudaStreamIsCapturing(stream, &cap);
  if (e != cudaSuccess) return tqi::fail(TQ_ERR_CUDA, "tq_attend_decode_noalloc: cudaStreamIsCapturing failed");
  if (cap != cudaStreamCaptureStatusNone) {
    void* ctx = current_context();
    for (int i = 0; i < kMaxContexts && ctx != nullptr; ++i) {
      if (g_entries[i].ctx == ctx) {
        *out = g_entries[i].addr;
        return TQ_OK;
      }
    }
    return tqi::fail(TQ_ERR_INVALID_ARG,
                     "tq_attend_decode_noalloc: the first call in a CUDA context must come before "
                     "stream capture begins (it looks up the scratch array's address)");
  }
  // outside capture: look the address up in the current context (this also brings up the
  // runtime's context and loads the module when this is the first use)
  void* p = nullptr;
  e = cudaGetSymbolAddress(&p, g_decode_scratch);
  if (e != cudaSuccess || p == nullptr) {
    char buf[256];
    std::snprintf(buf, sizeof(buf), "tq_attend_decode_noalloc: cudaGetSymbolAddress failed: %s",
                  cudaGetErrorString(e));
    return tqi::fail(TQ_ERR_CUDA, buf);
  }
  void* ctx = current_context();
  if (ctx != nullptr) {
    int slot = -1;
    for (int i = 0; i < kMaxContexts && slot < 0; ++i)
      if (g_entries[i].ctx == ctx) slot = i;
    for (int i = 0; i < kMaxContexts && slot < 0; ++i)
      if (g_entries[i].ctx == nullptr) slot = i;
    if (slot < 0) slot = 0;  // more contexts than entries: reuse the first
    g_entries[slot].ctx = ctx;
    g_entries[slot].addr = p;
  }
  *out = p;
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
  const tq_status st = scratch_address(reinterpret_cast<cudaStream_t>(stream), &ws);
  if (st != TQ_OK) return st;
  return tq_attend_decode(cfg, params, cache, layer, q, q_dtype, q_heads, seq_q, seq_lens, n_splits, ws,
                          kScratchBytes, out, dev_status, stream);
}
