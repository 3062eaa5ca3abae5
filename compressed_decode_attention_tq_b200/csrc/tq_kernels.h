// Kernel argument blocks and launchers (internal to the library).
#pragma once
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "tq_device.cuh"

namespace tqk {

// The prologue of the tensor-core split kernel forms each query row's terms in this many
// parts (thread blocks), each announced by its own ready word.
constexpr int kQueryParts = 4;

struct CompressArgs {
  CacheRef cache;
  const void* k;
  const void* v;
  int in_dtype, max_len, qjl, dense;
  int key_corr;                  // keys store the corrected norm ||k|| / ||y_hat||
  int tok_per_block;             // CUDA-core compress: tokens per thread block (set at launch)
  const float *k_off, *v_off;    // dithered: the offsets [batch][kv_heads][max_len], else null
  const int32_t* seq_lens;
  const float *signs, *pi, *s, *k_centroids, *k_boundaries, *v_centroids, *v_boundaries;
  const void* operands;  // prepared tensor-core operands (B = H D, S D H hi / lo; or sqrt(d) Pi hi / lo) or null
  int32_t* status;
};

struct DecodeArgs {
  CacheRef cache;
  const void* q;
  int q_dtype, q_heads, seq_q, group, rows, n_splits, qjl, dense;
  int key_corr;  // appended keys store the corrected norm
  const float *k_new_off, *v_new_off;  // dithered appends: the new tokens' offsets [B][H][n_new]
  const int32_t* seq_lens;
  const float *signs, *pi, *s, *k_centroids, *v_centroids;
  float* qrot;      // [B*Hq*seq_q][D]  workspace
  float* sq;        // [B*Hq*seq_q][QM] workspace
  float* part_acc;  // [B*Hq*seq_q][n_splits][D] workspace
  float* part_ml;   // [B*Hq*seq_q][n_splits][2] workspace
  float* part_sig;  // [B*Hq*seq_q][n_splits][QM] workspace (values with QJL): sum_t p_t ||r_v|| (2 sigma - 1)
  int16_t* sq_int;  // [B*Hq*seq_q][QM] workspace: S q in 16-bit fixed point
  float* sq_scale;  // [B*Hq*seq_q] workspace: S q ~= sq_int * sq_scale (a power of two)
  int* sq_sum;      // [B*Hq*seq_q] workspace: sum_i sq_int
  int8_t* q8;       // [B*Hq*seq_q][D] workspace: R q in int8 (scaled by q8_scale)
  float* q8_scale;  // [B*Hq*seq_q] workspace
  unsigned int* counter;  // workspace (sized B*Hq*seq_q): finished splits per (sequence, kv head,
                          // run of up to four query rows)
  unsigned int* ready;    // workspace [B*Hq*seq_q][kQueryParts]: 1 once the prologue has written that
                          // part of the row's terms
  float* out;       // [B*Hq*seq_q][D]
  float* scores;    // score-only mode: [B*Hq*seq_q][max_len]
  int max_len;
  // tokens appended before attending (n_new = 0: none): k_new, v_new [B][Hkv][n_new][D] of
  // element type new_dtype go to positions seq_lens[b] - n_new .. seq_lens[b] - 1
  const void* k_new;
  const void* v_new;
  int new_dtype, n_new;
  const float *k_boundaries, *v_boundaries;
  // > 0: a test of the bounded waits (one consumer warp of the first thread block of the
  // fast split kernel waits this many nanoseconds on a barrier nothing arrives on and
  // reports TQ_ERR_TIMEOUT; the results are computed as usual)
  int debug_wait_ns;
  // the tensor-core split kernel's wave: thread blocks resident at once (two per SM); a batch
  // of different lengths sizes its splits from it
  int target_ctas;
  // 1: the prologue forms the query terms in kQueryParts parts per row for the tensor-core split
  // kernel (fp32 S q, ready word per part); 0: one block per row for the general kernels
  int fast_query;
  int32_t* status;
};

struct DecompressArgs {
  CacheRef cache;
  const int32_t* seq_lens;
  int max_len, dense;
  const float *signs, *pi, *k_centroids, *v_centroids;
  float *k_hat, *v_hat;
  int32_t* status;
};

size_t compress_smem_bytes(int qjl, int dense);
cudaError_t launch_compress(const CompressArgs& a, cudaStream_t stream);
bool compress_tc_supported(const CompressArgs& a);
cudaError_t launch_compress_tc(const CompressArgs& a, cudaStream_t stream);
// Tensor-core operands of the compress kernel for a Hadamard rotation (and with QJL the
// sketch): three canonical 128 x 128 fp16 tiles, B = H D, then S D H as hi and lo parts.
size_t operand_bytes(bool dense);
cudaError_t launch_prepare_operands(const float* signs, const float* s, int qjl, void* ops, cudaStream_t stream);
cudaError_t launch_prepare_dense(const float* pi, void* ops, cudaStream_t stream);

// Workspace layout of decode, all offsets 256-byte aligned.
struct DecodeWorkspace {
  size_t qrot, sq, part_acc, part_ml, part_sig, sq_int, sq_scale, sq_sum, q8, q8_scale, counter, ready, total;
};
DecodeWorkspace decode_workspace(int batch, int q_heads, int seq_q, int n_splits, int vqjl);

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream);
bool fast_decode_supported(const DecodeArgs& a);
size_t fast_decode_smem_bytes();
cudaError_t launch_fast_split(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decode_scores(const DecodeArgs& a, cudaStream_t stream);
// the append alone: a.n_new tokens per (sequence, kv head), no query
cudaError_t launch_append(const DecodeArgs& a, cudaStream_t stream);
cudaError_t launch_decompress(const DecompressArgs& a, cudaStream_t stream);

}  // namespace tqk
