// The C ABI of include/tq.h: argument checks on the host, then kernel launches.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstdlib>
#include <cstring>

#include <nvtx3/nvToolsExt.h>

#include "tq.h"
#include "tq_internal.h"
#include "tq_kernels.h"

namespace {
// One NVTX range per device-side API call, named after the call (visible in Nsight Systems
// and in ncu's NVTX filters; the calls cost next to nothing when no tool is attached).
struct CallRange {
  explicit CallRange(const char* name) { nvtxRangePushA(name); }
  ~CallRange() { nvtxRangePop(); }
  CallRange(const CallRange&) = delete;
  CallRange& operator=(const CallRange&) = delete;
};
}  // namespace

namespace tqi {

static thread_local char g_last_error[512] = "";

tq_status fail(tq_status st, const char* msg) {
  std::snprintf(g_last_error, sizeof(g_last_error), "%s", msg);
  return st;
}

void clear_error() { g_last_error[0] = 0; }

static tq_status cuda_fail(cudaError_t e, const char* where) {
  char buf[400];
  std::snprintf(buf, sizeof(buf), "%s: %s", where, cudaGetErrorString(e));
  return fail(TQ_ERR_CUDA, buf);
}

static tq_status check_config(const tq_config* cfg) {
  if (!cfg) return fail(TQ_ERR_INVALID_ARG, "config is NULL");
  if (cfg->head_dim != tqk::D) return fail(TQ_ERR_UNSUPPORTED, "head_dim must be 128");
  if (cfg->qjl_m != tqk::QM) return fail(TQ_ERR_UNSUPPORTED, "qjl_m must be 128");
  if (cfg->page_tokens != tqk::PT) return fail(TQ_ERR_UNSUPPORTED, "page_tokens must be 256");
  if (cfg->key_bits < 1 || cfg->key_bits > 4) return fail(TQ_ERR_UNSUPPORTED, "key_bits must be in 1..4");
  if (cfg->value_bits < 1 || cfg->value_bits > 4)
    return fail(TQ_ERR_UNSUPPORTED, "value_bits must be in 1..4");
  if (cfg->key_qjl != 0 && cfg->key_qjl != 1) return fail(TQ_ERR_INVALID_ARG, "key_qjl must be 0 or 1");
  if (cfg->value_qjl != 0 && cfg->value_qjl != 1) return fail(TQ_ERR_INVALID_ARG, "value_qjl must be 0 or 1");
  if (cfg->rotation != TQ_ROT_HADAMARD && cfg->rotation != TQ_ROT_DENSE)
    return fail(TQ_ERR_INVALID_ARG, "unknown rotation kind");
  if (cfg->dither != 0 && cfg->dither != 1) return fail(TQ_ERR_INVALID_ARG, "dither must be 0 or 1");
  if (cfg->dither && cfg->rotation != TQ_ROT_HADAMARD)
    return fail(TQ_ERR_UNSUPPORTED, "dither needs TQ_ROT_HADAMARD");
  if (cfg->key_corrected_norm != 0 && cfg->key_corrected_norm != 1)
    return fail(TQ_ERR_INVALID_ARG, "key_corrected_norm must be 0 or 1");
  return TQ_OK;
}

static tq_status check_params(const tq_config* cfg, const tq_params* p, bool need_s) {
  if (!p) return fail(TQ_ERR_INVALID_ARG, "params is NULL");
  if (cfg->rotation == TQ_ROT_HADAMARD && !p->signs) return fail(TQ_ERR_INVALID_ARG, "params.signs is NULL");
  if (cfg->rotation == TQ_ROT_DENSE && !p->pi) return fail(TQ_ERR_INVALID_ARG, "params.pi is NULL");
  if (need_s && (cfg->key_qjl || cfg->value_qjl) && !p->s) return fail(TQ_ERR_INVALID_ARG, "params.s is NULL");
  if (!p->k_centroids || !p->v_centroids) return fail(TQ_ERR_INVALID_ARG, "centroid pointer is NULL");
  return TQ_OK;
}

static tq_status check_cache(const tq_cache* c, int32_t layer) {
  if (!c) return fail(TQ_ERR_INVALID_ARG, "cache is NULL");
  if (!c->pages || !c->block_table) return fail(TQ_ERR_INVALID_ARG, "cache.pages or block_table is NULL");
  if (c->batch < 1 || c->kv_heads < 1 || c->num_layers < 1 || c->num_pages < 1 || c->max_pages < 1)
    return fail(TQ_ERR_INVALID_ARG, "cache sizes must be >= 1");
  if (layer < 0 || layer >= c->num_layers) return fail(TQ_ERR_INVALID_ARG, "layer out of range");
  if ((size_t)c->batch * c->max_pages > (size_t)1 << 31) return fail(TQ_ERR_INVALID_ARG, "block table too large");
  return TQ_OK;
}

static tqk::CacheRef cache_ref(const tq_config* cfg, const tq_cache* c, int32_t layer) {
  tqk::CacheRef r;
  r.pages = static_cast<uint8_t*>(c->pages);
  r.block_table = c->block_table;
  r.num_pages = c->num_pages;
  r.max_pages = c->max_pages;
  r.batch = c->batch;
  r.kv_heads = c->kv_heads;
  r.layer = layer;
  r.L = tqk::make_layout(cfg->key_bits, cfg->key_qjl, cfg->value_bits, cfg->value_qjl, cfg->dither);
  return r;
}

}  // namespace tqi

using namespace tqi;

extern "C" {

int32_t tq_version(void) { return 102; }

const char* tq_status_str(tq_status st) {
  switch (st) {
    case TQ_OK: return "TQ_OK";
    case TQ_ERR_INVALID_ARG: return "TQ_ERR_INVALID_ARG";
    case TQ_ERR_UNSUPPORTED: return "TQ_ERR_UNSUPPORTED";
    case TQ_ERR_CUDA: return "TQ_ERR_CUDA";
    case TQ_ERR_OVERFLOW: return "TQ_ERR_OVERFLOW";
    case TQ_ERR_TIMEOUT: return "TQ_ERR_TIMEOUT";
    case TQ_ERR_BOUNDS: return "TQ_ERR_BOUNDS";
  }
  return "TQ_ERR_UNKNOWN";
}

const char* tq_last_error(void) { return g_last_error; }

tq_status tq_check(const int32_t* dev_status_host_copy) {
  clear_error();
  if (!dev_status_host_copy) return fail(TQ_ERR_INVALID_ARG, "tq_check: dev_status_host_copy is NULL");
  const int32_t v = *dev_status_host_copy;
  if (v < TQ_OK || v > TQ_ERR_BOUNDS) {
    char buf[96];
    std::snprintf(buf, sizeof(buf), "tq_check: %d is not a status code", (int)v);
    return fail(TQ_ERR_INVALID_ARG, buf);
  }
  const tq_status st = static_cast<tq_status>(v);
  switch (st) {
    case TQ_OK: break;
    case TQ_ERR_OVERFLOW: fail(st, "device: a norm does not fit in fp16"); break;
    case TQ_ERR_TIMEOUT: fail(st, "device: a bounded wait inside a kernel gave up"); break;
    case TQ_ERR_BOUNDS: fail(st, "device: a sequence length or page id is outside the cache"); break;
    case TQ_ERR_INVALID_ARG: fail(st, "device: a parameter failed a device-side check"); break;
    default: fail(st, "device: error recorded"); break;
  }
  return st;
}

tq_status tq_validate_config(const tq_config* cfg) {
  clear_error();
  return check_config(cfg);
}

size_t tq_page_bytes(const tq_config* cfg) {
  if (check_config(cfg) != TQ_OK) return 0;
  return (size_t)tqk::make_layout(cfg->key_bits, cfg->key_qjl, cfg->value_bits, cfg->value_qjl, cfg->dither)
      .bytes;
}

static tq_status compress_common(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                                 int32_t layer, const void* k, const void* v, const float* k_offsets,
                                 const float* v_offsets, int32_t in_dtype, int32_t max_len,
                                 const int32_t* seq_lens, int32_t* dev_status, tq_stream_t stream) {
  tq_status st;
  if ((st = check_config(cfg)) != TQ_OK) return st;
  if ((st = check_params(cfg, params, true)) != TQ_OK) return st;
  if ((st = check_cache(cache, layer)) != TQ_OK) return st;
  if (!params->k_boundaries || !params->v_boundaries) return fail(TQ_ERR_INVALID_ARG, "boundary pointer is NULL");
  if (!k || !v || !seq_lens) return fail(TQ_ERR_INVALID_ARG, "k, v or seq_lens is NULL");
  if (in_dtype != TQ_F16 && in_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "in_dtype must be TQ_F16 or TQ_F32");
  if (max_len < 0) return fail(TQ_ERR_INVALID_ARG, "max_len must be >= 0");
  tqk::CompressArgs a;
  a.cache = cache_ref(cfg, cache, layer);
  a.k = k;
  a.v = v;
  a.in_dtype = in_dtype;
  a.max_len = max_len;
  a.qjl = cfg->key_qjl;
  a.dense = cfg->rotation == TQ_ROT_DENSE;
  a.key_corr = cfg->key_corrected_norm;
  a.k_off = k_offsets;
  a.v_off = v_offsets;
  a.seq_lens = seq_lens;
  a.signs = params->signs;
  a.pi = params->pi;
  a.s = params->s;
  a.k_centroids = params->k_centroids;
  a.k_boundaries = params->k_boundaries;
  a.v_centroids = params->v_centroids;
  a.v_boundaries = params->v_boundaries;
  a.operands = params->operands;
  if (a.operands && (reinterpret_cast<uintptr_t>(a.operands) & 15))
    return fail(TQ_ERR_INVALID_ARG, "params->operands must be 16-byte aligned");
  a.status = dev_status;
  cudaError_t e = tqk::launch_compress(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_compress_kv launch");
  return TQ_OK;
}

tq_status tq_compress_kv(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                         int32_t layer, const void* k, const void* v, int32_t in_dtype, int32_t max_len,
                         const int32_t* seq_lens, int32_t* dev_status, tq_stream_t stream) {
  CallRange range("tq_compress_kv");
  clear_error();
  if (cfg && cfg->dither)
    return fail(TQ_ERR_INVALID_ARG, "a dithered configuration is compressed by tq_compress_kv_dithered");
  return compress_common(cfg, params, cache, layer, k, v, nullptr, nullptr, in_dtype, max_len, seq_lens,
                         dev_status, stream);
}

tq_status tq_compress_kv_dithered(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                                  int32_t layer, const void* k, const void* v, const float* k_offsets,
                                  const float* v_offsets, int32_t in_dtype, int32_t max_len,
                                  const int32_t* seq_lens, int32_t* dev_status, tq_stream_t stream) {
  CallRange range("tq_compress_kv_dithered");
  clear_error();
  if (!cfg || !cfg->dither) return fail(TQ_ERR_INVALID_ARG, "tq_compress_kv_dithered needs cfg->dither = 1");
  if (!k_offsets || !v_offsets) return fail(TQ_ERR_INVALID_ARG, "k_offsets or v_offsets is NULL");
  return compress_common(cfg, params, cache, layer, k, v, k_offsets, v_offsets, in_dtype, max_len, seq_lens,
                         dev_status, stream);
}

size_t tq_operand_bytes(const tq_config* cfg) {
  if (check_config(cfg) != TQ_OK) return 0;
  return tqk::operand_bytes(cfg->rotation == TQ_ROT_DENSE);
}

tq_status tq_prepare_operands(const tq_config* cfg, const tq_params* params, void* operands, tq_stream_t stream) {
  CallRange range("tq_prepare_operands");
  clear_error();
  tq_status st;
  if ((st = check_config(cfg)) != TQ_OK) return st;
  if (!operands || (reinterpret_cast<uintptr_t>(operands) & 15))
    return fail(TQ_ERR_INVALID_ARG, "operands must be a 16-byte aligned device pointer");
  cudaError_t e;
  if (cfg->rotation == TQ_ROT_DENSE) {
    if (!params || !params->pi) return fail(TQ_ERR_INVALID_ARG, "params or params->pi is NULL");
    e = tqk::launch_prepare_dense(params->pi, operands, reinterpret_cast<cudaStream_t>(stream));
  } else {
    if (!params || !params->signs) return fail(TQ_ERR_INVALID_ARG, "params or params->signs is NULL");
    const int qjl = cfg->key_qjl || cfg->value_qjl;
    if (qjl && !params->s) return fail(TQ_ERR_INVALID_ARG, "params->s is NULL");
    e = tqk::launch_prepare_operands(params->signs, params->s, qjl, operands, reinterpret_cast<cudaStream_t>(stream));
  }
  if (e != cudaSuccess) return cuda_fail(e, "tq_prepare_operands launch");
  return TQ_OK;
}

size_t tq_decode_workspace_bytes(const tq_config* cfg, int32_t batch, int32_t q_heads, int32_t seq_q,
                                 int32_t n_splits) {
  if (check_config(cfg) != TQ_OK || batch < 1 || q_heads < 1 || seq_q < 1 || n_splits < 1) return 0;
  return tqk::decode_workspace(batch, q_heads, seq_q, n_splits, cfg->value_qjl).total;
}

// A test of the device's bounded waits: TQ_DEBUG_BOUNDED_WAIT_US=<n> (1..1000000) makes one
// consumer warp of the tensor-core split kernel wait n microseconds on a barrier nothing
// arrives on and report TQ_ERR_TIMEOUT; the call's results are unaffected.  Read on every
// call.
static int debug_wait_ns() {
  const char* v = std::getenv("TQ_DEBUG_BOUNDED_WAIT_US");
  if (!v || !*v) return 0;
  const long us = std::strtol(v, nullptr, 10);
  if (us <= 0 || us > 1000000) return 0;
  return (int)(us * 1000);
}

// SMs of the current device (looked up once per device)
static int sm_count() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return 148;
  if (dev < 64 && cached[dev] > 0) return cached[dev];
  int n = 0;
  if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
  if (dev < 64) cached[dev] = n;
  return n;
}

static tq_status decode_common(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                               int32_t layer, const void* q, int32_t q_dtype, int32_t q_heads,
                               int32_t seq_q, const int32_t* seq_lens, int32_t n_splits, void* workspace,
                               size_t workspace_bytes, tqk::DecodeArgs& a) {
  tq_status st;
  if ((st = check_config(cfg)) != TQ_OK) return st;
  if ((st = check_params(cfg, params, true)) != TQ_OK) return st;
  if ((st = check_cache(cache, layer)) != TQ_OK) return st;
  if (!q || !seq_lens || !workspace) return fail(TQ_ERR_INVALID_ARG, "q, seq_lens or workspace is NULL");
  if (q_dtype != TQ_F16 && q_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "q_dtype must be TQ_F16 or TQ_F32");
  if (q_heads < 1 || q_heads % cache->kv_heads != 0)
    return fail(TQ_ERR_INVALID_ARG, "q_heads must be a positive multiple of kv_heads");
  if (seq_q < 1) return fail(TQ_ERR_INVALID_ARG, "seq_q must be >= 1");
  const int group = q_heads / cache->kv_heads;
  if (group * seq_q > 32) return fail(TQ_ERR_UNSUPPORTED, "q_heads/kv_heads * seq_q must be <= 32");
  if (n_splits < 1 || n_splits > 1024) return fail(TQ_ERR_INVALID_ARG, "n_splits must be in 1..1024");
  if ((reinterpret_cast<uintptr_t>(workspace) & 255) != 0)
    return fail(TQ_ERR_INVALID_ARG, "workspace must be 256-byte aligned");
  const tqk::DecodeWorkspace w = tqk::decode_workspace(cache->batch, q_heads, seq_q, n_splits, cfg->value_qjl);
  if (workspace_bytes < w.total) return fail(TQ_ERR_INVALID_ARG, "workspace too small");
  char* ws = static_cast<char*>(workspace);
  a.cache = cache_ref(cfg, cache, layer);
  a.q = q;
  a.q_dtype = q_dtype;
  a.q_heads = q_heads;
  a.seq_q = seq_q;
  a.group = group;
  a.rows = group * seq_q;
  a.n_splits = n_splits;
  a.qjl = cfg->key_qjl;
  a.dense = cfg->rotation == TQ_ROT_DENSE;
  a.key_corr = cfg->key_corrected_norm;
  a.seq_lens = seq_lens;
  a.signs = params->signs;
  a.pi = params->pi;
  a.s = params->s;
  a.k_centroids = params->k_centroids;
  a.v_centroids = params->v_centroids;
  a.qrot = reinterpret_cast<float*>(ws + w.qrot);
  a.sq = reinterpret_cast<float*>(ws + w.sq);
  a.part_acc = reinterpret_cast<float*>(ws + w.part_acc);
  a.part_ml = reinterpret_cast<float*>(ws + w.part_ml);
  a.part_sig = cfg->value_qjl ? reinterpret_cast<float*>(ws + w.part_sig) : nullptr;
  a.sq_int = reinterpret_cast<int16_t*>(ws + w.sq_int);
  a.sq_scale = reinterpret_cast<float*>(ws + w.sq_scale);
  a.sq_sum = reinterpret_cast<int*>(ws + w.sq_sum);
  a.q8 = reinterpret_cast<int8_t*>(ws + w.q8);
  a.q8_scale = reinterpret_cast<float*>(ws + w.q8_scale);
  a.counter = reinterpret_cast<unsigned int*>(ws + w.counter);
  a.ready = reinterpret_cast<unsigned int*>(ws + w.ready);
  a.fast_query = 0;
  a.target_ctas = 2 * sm_count();
  a.out = nullptr;
  a.scores = nullptr;
  a.max_len = 0;
  a.k_new = nullptr;
  a.v_new = nullptr;
  a.new_dtype = TQ_F16;
  a.n_new = 0;
  a.k_boundaries = params->k_boundaries;
  a.v_boundaries = params->v_boundaries;
  a.k_new_off = nullptr;
  a.v_new_off = nullptr;
  a.debug_wait_ns = debug_wait_ns();
  return TQ_OK;
}

// Checks of the appended tokens' arguments shared by tq_append_kv and tq_append_attend_decode.
static tq_status check_append(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                              const void* k_new, const void* v_new, int32_t in_dtype, int32_t n_new,
                              const float* k_off, const float* v_off, bool dithered_call) {
  if (cfg->dither && !dithered_call)
    return fail(TQ_ERR_UNSUPPORTED, "a dithered configuration appends with the _dithered calls (offsets)");
  if (dithered_call && !cfg->dither) return fail(TQ_ERR_INVALID_ARG, "the _dithered appends need cfg->dither = 1");
  if (dithered_call && (!k_off || !v_off)) return fail(TQ_ERR_INVALID_ARG, "k_offsets or v_offsets is NULL");
  if (!params->k_boundaries || !params->v_boundaries) return fail(TQ_ERR_INVALID_ARG, "boundary pointer is NULL");
  if (!k_new || !v_new) return fail(TQ_ERR_INVALID_ARG, "k_new or v_new is NULL");
  if (in_dtype != TQ_F16 && in_dtype != TQ_F32) return fail(TQ_ERR_INVALID_ARG, "in_dtype must be TQ_F16 or TQ_F32");
  if (n_new < 1) return fail(TQ_ERR_INVALID_ARG, "n_new must be >= 1");
  if ((int64_t)cache->batch * cache->kv_heads * n_new > (int64_t)1 << 30)
    return fail(TQ_ERR_INVALID_ARG, "batch * kv_heads * n_new too large");
  if ((cfg->key_qjl || cfg->value_qjl) && (reinterpret_cast<uintptr_t>(params->s) & 15))
    return fail(TQ_ERR_INVALID_ARG, "params->s must be 16-byte aligned");
  if (cfg->rotation == TQ_ROT_DENSE && (reinterpret_cast<uintptr_t>(params->pi) & 15))
    return fail(TQ_ERR_INVALID_ARG, "params->pi must be 16-byte aligned");
  return TQ_OK;
}

tq_status tq_attend_decode(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                           int32_t layer, const void* q, int32_t q_dtype, int32_t q_heads, int32_t seq_q,
                           const int32_t* seq_lens, int32_t n_splits, void* workspace,
                           size_t workspace_bytes, float* out, int32_t* dev_status, tq_stream_t stream) {
  CallRange range("tq_attend_decode");
  clear_error();
  tqk::DecodeArgs a;
  tq_status st = decode_common(cfg, params, cache, layer, q, q_dtype, q_heads, seq_q, seq_lens, n_splits,
                               workspace, workspace_bytes, a);
  if (st != TQ_OK) return st;
  if (!out) return fail(TQ_ERR_INVALID_ARG, "out is NULL");
  a.out = out;
  a.status = dev_status;
  cudaError_t e = tqk::launch_decode(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_attend_decode launch");
  return TQ_OK;
}

static tq_status append_attend_common(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                                      int32_t layer, const void* k_new, const void* v_new, const float* k_off,
                                      const float* v_off, bool dithered_call, int32_t in_dtype, int32_t n_new,
                                      const void* q, int32_t q_dtype, int32_t q_heads, int32_t seq_q,
                                      const int32_t* seq_lens, int32_t n_splits, void* workspace,
                                      size_t workspace_bytes, float* out, int32_t* dev_status, tq_stream_t stream) {
  tqk::DecodeArgs a;
  tq_status st = decode_common(cfg, params, cache, layer, q, q_dtype, q_heads, seq_q, seq_lens, n_splits,
                               workspace, workspace_bytes, a);
  if (st != TQ_OK) return st;
  if ((st = check_append(cfg, params, cache, k_new, v_new, in_dtype, n_new, k_off, v_off, dithered_call)) != TQ_OK)
    return st;
  if (!out) return fail(TQ_ERR_INVALID_ARG, "out is NULL");
  if ((int64_t)cache->batch * q_heads * seq_q + (int64_t)cache->batch * cache->kv_heads * n_new > (int64_t)1 << 30)
    return fail(TQ_ERR_INVALID_ARG, "too many query rows and appended tokens");
  a.k_new = k_new;
  a.v_new = v_new;
  a.k_new_off = k_off;
  a.v_new_off = v_off;
  a.new_dtype = in_dtype;
  a.n_new = n_new;
  a.out = out;
  a.status = dev_status;
  cudaError_t e = tqk::launch_decode(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_append_attend_decode launch");
  return TQ_OK;
}

tq_status tq_append_attend_decode(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                                  int32_t layer, const void* k_new, const void* v_new, int32_t in_dtype,
                                  int32_t n_new, const void* q, int32_t q_dtype, int32_t q_heads,
                                  int32_t seq_q, const int32_t* seq_lens, int32_t n_splits, void* workspace,
                                  size_t workspace_bytes, float* out, int32_t* dev_status,
                                  tq_stream_t stream) {
  CallRange range("tq_append_attend_decode");
  clear_error();
  return append_attend_common(cfg, params, cache, layer, k_new, v_new, nullptr, nullptr, false, in_dtype, n_new, q,
                              q_dtype, q_heads, seq_q, seq_lens, n_splits, workspace, workspace_bytes, out,
                              dev_status, stream);
}

tq_status tq_append_attend_decode_dithered(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                                           int32_t layer, const void* k_new, const void* v_new,
                                           const float* k_offsets, const float* v_offsets, int32_t in_dtype,
                                           int32_t n_new, const void* q, int32_t q_dtype, int32_t q_heads,
                                           int32_t seq_q, const int32_t* seq_lens, int32_t n_splits,
                                           void* workspace, size_t workspace_bytes, float* out,
                                           int32_t* dev_status, tq_stream_t stream) {
  CallRange range("tq_append_attend_decode_dithered");
  clear_error();
  return append_attend_common(cfg, params, cache, layer, k_new, v_new, k_offsets, v_offsets, true, in_dtype,
                              n_new, q, q_dtype, q_heads, seq_q, seq_lens, n_splits, workspace, workspace_bytes,
                              out, dev_status, stream);
}

static tq_status append_common(const tq_config* cfg, const tq_params* params, const tq_cache* cache, int32_t layer,
                               const void* k_new, const void* v_new, const float* k_off, const float* v_off,
                               bool dithered_call, int32_t in_dtype, int32_t n_new, const int32_t* seq_lens,
                               int32_t* dev_status, tq_stream_t stream) {
  tq_status st;
  if ((st = check_config(cfg)) != TQ_OK) return st;
  if ((st = check_params(cfg, params, true)) != TQ_OK) return st;
  if ((st = check_cache(cache, layer)) != TQ_OK) return st;
  if (!seq_lens) return fail(TQ_ERR_INVALID_ARG, "seq_lens is NULL");
  if ((st = check_append(cfg, params, cache, k_new, v_new, in_dtype, n_new, k_off, v_off, dithered_call)) != TQ_OK)
    return st;
  tqk::DecodeArgs a = {};
  a.cache = cache_ref(cfg, cache, layer);
  a.qjl = cfg->key_qjl;
  a.dense = cfg->rotation == TQ_ROT_DENSE;
  a.key_corr = cfg->key_corrected_norm;
  a.seq_lens = seq_lens;
  a.signs = params->signs;
  a.pi = params->pi;
  a.s = params->s;
  a.k_centroids = params->k_centroids;
  a.v_centroids = params->v_centroids;
  a.k_boundaries = params->k_boundaries;
  a.v_boundaries = params->v_boundaries;
  a.k_new = k_new;
  a.v_new = v_new;
  a.k_new_off = k_off;
  a.v_new_off = v_off;
  a.new_dtype = in_dtype;
  a.n_new = n_new;
  a.status = dev_status;
  cudaError_t e = tqk::launch_append(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_append_kv launch");
  return TQ_OK;
}

tq_status tq_append_kv(const tq_config* cfg, const tq_params* params, const tq_cache* cache, int32_t layer,
                       const void* k_new, const void* v_new, int32_t in_dtype, int32_t n_new,
                       const int32_t* seq_lens, int32_t* dev_status, tq_stream_t stream) {
  CallRange range("tq_append_kv");
  clear_error();
  return append_common(cfg, params, cache, layer, k_new, v_new, nullptr, nullptr, false, in_dtype, n_new, seq_lens,
                       dev_status, stream);
}

tq_status tq_append_kv_dithered(const tq_config* cfg, const tq_params* params, const tq_cache* cache, int32_t layer,
                                const void* k_new, const void* v_new, const float* k_offsets, const float* v_offsets,
                                int32_t in_dtype, int32_t n_new, const int32_t* seq_lens, int32_t* dev_status,
                                tq_stream_t stream) {
  CallRange range("tq_append_kv_dithered");
  clear_error();
  return append_common(cfg, params, cache, layer, k_new, v_new, k_offsets, v_offsets, true, in_dtype, n_new,
                       seq_lens, dev_status, stream);
}

tq_status tq_decode_scores(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                           int32_t layer, const void* q, int32_t q_dtype, int32_t q_heads, int32_t seq_q,
                           const int32_t* seq_lens, int32_t max_len, void* workspace,
                           size_t workspace_bytes, float* scores, int32_t* dev_status, tq_stream_t stream) {
  CallRange range("tq_decode_scores");
  clear_error();
  tqk::DecodeArgs a;
  tq_status st = decode_common(cfg, params, cache, layer, q, q_dtype, q_heads, seq_q, seq_lens, 1,
                               workspace, workspace_bytes, a);
  if (st != TQ_OK) return st;
  if (!scores) return fail(TQ_ERR_INVALID_ARG, "scores is NULL");
  if (max_len < 0) return fail(TQ_ERR_INVALID_ARG, "max_len must be >= 0");
  a.scores = scores;
  a.max_len = max_len;
  a.status = dev_status;
  cudaError_t e = tqk::launch_decode_scores(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_decode_scores launch");
  return TQ_OK;
}

tq_status tq_decompress(const tq_config* cfg, const tq_params* params, const tq_cache* cache, int32_t layer,
                        const int32_t* seq_lens, int32_t max_len, float* k_hat, float* v_hat,
                        int32_t* dev_status, tq_stream_t stream) {
  CallRange range("tq_decompress");
  clear_error();
  tq_status st;
  if ((st = check_config(cfg)) != TQ_OK) return st;
  if ((st = check_params(cfg, params, false)) != TQ_OK) return st;
  if ((st = check_cache(cache, layer)) != TQ_OK) return st;
  if (!seq_lens) return fail(TQ_ERR_INVALID_ARG, "seq_lens is NULL");
  if (max_len < 0) return fail(TQ_ERR_INVALID_ARG, "max_len must be >= 0");
  tqk::DecompressArgs a;
  a.cache = cache_ref(cfg, cache, layer);
  a.seq_lens = seq_lens;
  a.max_len = max_len;
  a.dense = cfg->rotation == TQ_ROT_DENSE;
  a.signs = params->signs;
  a.pi = params->pi;
  a.k_centroids = params->k_centroids;
  a.v_centroids = params->v_centroids;
  a.k_hat = k_hat;
  a.v_hat = v_hat;
  a.status = dev_status;
  cudaError_t e = tqk::launch_decompress(a, reinterpret_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return cuda_fail(e, "tq_decompress launch");
  return TQ_OK;
}

}  // extern "C"
