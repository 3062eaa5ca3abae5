/*
 * tq.h - C ABI of the TurboQuant compressed-KV decode library for NVIDIA B200 (sm_100a).
 *
 * The library compresses a KV cache with TurboQuant and runs decode attention
 * directly on the packed, paged cache.  What it computes follows these pages:
 *
 *   [CUTILE]  "turboquant_cutile" function list (codehub.bot, DevTechJr/turboquant_cutile):
 *             compress K -> dict (MSE + 1-bit QJL), compress V -> dict (MSE only),
 *             asymmetric estimator = MSE dot + QJL correction, full pipeline
 *             scores -> softmax -> weighted V sum, decompression
 *             indices -> centroids -> un-rotate -> rescale, codebook as sorted
 *             float32 (centroids (2^b,), boundaries (2^b - 1,)).
 *   [MOBILINT] "TurboQuant explained: near-optimal KV cache compression and why
 *             the theory breaks down in practice" (Mobilint blog): sections
 *             "How JL Matrices Evolved" (HD rotation), "QJL: Inner Product Recovery
 *             from a Single Sign Bit", "Coordinates Become Predictable After
 *             Rotation" (Beta density), "Designing the Optimal Codebook Without
 *             Data" (Lloyd-Max), "Two-Stage Approach: MSE Approximation + QJL
 *             Correction", "Practical Issues Found in Implementation" (fused
 *             kernels, no dense K/V round trip).
 *   [TQKV]    "tq-kv" crate documentation (docs.rs): pre-rotated query, centroid
 *             table scoring without decompression, incremental cache.
 *   [LIMITS]  "TurboQuant Limits And Assumptions" (ginkgoq): vLLM-style packed
 *             paged decode; storage claims count every byte.
 *
 * Conventions for every call below:
 *   - The library allocates nothing.  Every buffer is owned by the caller and
 *     passed as a plain pointer; "device" pointers are CUDA device memory of the
 *     current device, "host" pointers are ordinary host memory.
 *   - Device calls are asynchronous on the given stream (a cudaStream_t; NULL is
 *     the legacy default stream).  They return after enqueueing.
 *   - Host-side argument errors are returned as a tq_status and nothing is
 *     enqueued; tq_last_error() then describes the failing argument.
 *   - Errors found on the device (norm overflow, page table out of range, a
 *     parameter the device checks) are written to the caller's int32 dev_status
 *     word (device memory, must start at 0): the first error code wins and the
 *     affected output is left unspecified.  Read it after a stream sync.
 *   - Arrays are row-major and contiguous with the shapes given.
 *   - Supported: head_dim = 128, qjl_m = 128, page_tokens = 256, key/value
 *     bits in 1..4.  Other values return TQ_ERR_UNSUPPORTED.
 *
 * Packed cache format (one block per (layer, physical page, kv head); the cache
 * buffer is [num_layers][num_pages][kv_heads][tq_page_bytes(cfg)] bytes):
 *
 *   region  content                                   bytes (P = page_tokens)
 *   KN      stored ||k|| (fp16) per token              2P
 *   KR      stored ||r|| (fp16) per token, QJL keys    2P
 *   VN      stored ||v|| (fp16) per token              2P
 *   KC      key codes, key_bits*d/8 bytes per token    key_bits*16*P  (merged keys: 64*P)
 *   KS      QJL sign bits, m/8 bytes per token          16*P   (QJL keys, not merged)
 *   VC      value codes                               value_bits*16*P
 *   VS      QJL sign bits of the value residual        16*P   (value_qjl)
 *   VR      stored ||r_v|| (fp16) per token            2P     (value_qjl)
 *   KD      key dither offset xi (fp16) per token      2P     (dither)
 *   VD      value dither offset xi (fp16) per token    2P     (dither)
 *
 *   A code region stores each token's bytes as 16-byte chunks, chunk-major:
 *   chunk c of slot t is at region byte (c*P + t)*16.  A token's chunks,
 *   concatenated, form its bit string; bit k is bit (k mod 8) of byte k/8.
 *   Index idx in [0, 2^b) of coordinate j is stored in sign-magnitude form,
 *   h = 2^(b-1): s = [idx >= h], r = idx - h if s else h - 1 - idx, so that
 *   c[idx] = (s ? +1 : -1) * c[h + r] for the (symmetric) codebook c:
 *     b = 1: bit j = s
 *     b = 2: bits 2j, 2j+1 = r, s
 *     b = 3: bits 2j, 2j+1 = r (2 bits); the sign plane starts at bit 2d and,
 *            for j = 32q + 8a + 4u + t (a < 4, u < 2, t < 4), holds s at plane bit
 *            32q + 4a + t + 16u
 *     b = 4: bits 4j..4j+2 = r (3 bits), bit 4j + 3 = s
 *   Merged keys (key_bits = 3 with QJL): bits 4j..4j+3 = r0, r1, s, sigma_j, where
 *   sigma_i = [(S r)_i >= 0] (sign(0) is stored as +1); there is no KS region.
 *   Other QJL keys: bit i of the KS chunk = sigma_i.
 *   Values with QJL: bit i of the VS chunk = [(S r_v)_i >= 0], r_v = v - v_mse.
 *   Dithered configurations: a vector is coded as idx = Quant(y - xi) and read back as
 *   n R^T (c[idx] + xi), xi its stored offset.
 *   Slots past a sequence's length are never read and their bytes unspecified.
 *
 * [DITHER]  "Minimum Distortion Quantization with Specified Output Distribution"
 *           (thelatestinai.com), third abstract: dithered TurboQuant, one randomized
 *           Hadamard transform and a random scalar offset subtracted before the scalar
 *           quantizer; unbiased, MSE (pi sqrt(3)/2 + o(1)) 4^-b.  This library reads the
 *           quantizer as a uniform grid (tq_dither_codebook) with subtractive dither.
 */
#ifndef TQ_H_
#define TQ_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define TQ_API __attribute__((visibility("default")))
#else
#define TQ_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t, without pulling in the CUDA headers. */
typedef struct CUstream_st* tq_stream_t;

typedef enum tq_status {
  TQ_OK = 0,
  TQ_ERR_INVALID_ARG = 1,  /* null pointer, inconsistent sizes, bad parameter values   */
  TQ_ERR_UNSUPPORTED = 2,  /* a size or mode outside what this library supports        */
  TQ_ERR_CUDA = 3,         /* a CUDA runtime call or a kernel launch failed            */
  TQ_ERR_OVERFLOW = 4,     /* a norm does not fit in fp16 (device)                     */
  TQ_ERR_TIMEOUT = 5,      /* a bounded wait inside a kernel gave up (device)          */
  TQ_ERR_BOUNDS = 6        /* sequence longer than its page-table row, or page id out
                              of range (device)                                        */
} tq_status;

typedef enum tq_density { TQ_DENSITY_BETA = 0, TQ_DENSITY_GAUSS = 1 } tq_density;
typedef enum tq_rotation_kind { TQ_ROT_HADAMARD = 0, TQ_ROT_DENSE = 1 } tq_rotation_kind;
typedef enum tq_dtype { TQ_F16 = 0, TQ_F32 = 1 } tq_dtype;

/* Configuration of one cache ([TQKV] TurboQuantConfig: bits, rotation, QJL mode).
 * Callers set every field (value_qjl = 0 for the format of version 1.00). */
typedef struct tq_config {
  int32_t head_dim;     /* d, must be 128                                             */
  int32_t key_bits;     /* b_k: bits of the key MSE stage, 1..4                        */
  int32_t key_qjl;      /* 1: keys carry the 1-bit QJL sketch of the residual and ||r|| */
  int32_t qjl_m;        /* m: rows of S, must be 128                                   */
  int32_t value_bits;   /* b_v: bits of the value MSE stage, 1..4                      */
  int32_t page_tokens;  /* P: tokens per page, must be 256                             */
  int32_t rotation;     /* tq_rotation_kind                                            */
  int32_t value_qjl;    /* 1: values carry the 1-bit QJL sketch of their residual and
                           ||r_v|| (TurboQuant_prod on the value cache, [MOBILINT]
                           "Two-Stage Approach": the value is reconstructed as
                           v_mse + sqrt(pi/2)/m ||r_v|| S^T (2 sigma_v - 1))        */
  int32_t dither;       /* 1: dithered HD ([DITHER]): every key and value is coded as
                           Quant(y - xi) with its own offset xi, stored in KD / VD and added
                           back at reconstruction; needs TQ_ROT_HADAMARD and the uniform
                           grids of tq_dither_codebook; compressed by
                           tq_compress_kv_dithered                                    */
  int32_t key_corrected_norm; /* 1: keys store the corrected norm ([TQKV]
                           compress_single_key returns "corrected_norm"): ||k|| / ||y_hat||
                           with y_hat = c[idx] (+ xi), so that the reconstruction has the
                           key's norm (0 for y_hat = 0); the decoder is unchanged. With
                           QJL the residual is taken against this reconstruction.      */
} tq_config;

/* Random inputs of the method and the codebooks, all device memory, fp32.
 * [MOBILINT] "How JL Matrices Evolved": R = H D (H the normalized Sylvester
 * Walsh-Hadamard matrix, D a +-1 diagonal); [CUTILE]: the dense option is a
 * Haar orthogonal Pi.  [MOBILINT] "QJL": S is an m x d Gaussian matrix. */
typedef struct tq_params {
  const float* signs;         /* [d] +-1 diagonal of D (TQ_ROT_HADAMARD), else unused     */
  const float* pi;            /* [d*d] Pi, row-major, y = Pi u (TQ_ROT_DENSE), else unused */
  const float* s;             /* [m*d] S, row-major; unused unless key_qjl or value_qjl.  When
                                 tq_compress_kv forms its operands itself (operands
                                 NULL), every entry must be exactly representable in
                                 fp16 (checked on the device, TQ_ERR_INVALID_ARG)      */
  const float* k_centroids;   /* [2^key_bits] sorted, symmetric (c_i = -c_{n-1-i})      */
  const float* k_boundaries;  /* [2^key_bits - 1] sorted, symmetric, middle one 0        */
  const float* v_centroids;   /* [2^value_bits]                                          */
  const float* v_boundaries;  /* [2^value_bits - 1]                                      */
  const void* operands;       /* NULL, or device memory of tq_operand_bytes() bytes (16-byte
                                 aligned) that tq_prepare_operands filled for these signs
                                 and s (or this pi): tq_compress_kv then copies its
                                 tensor-core operands from it instead of forming them in
                                 every thread block.  Read only by tq_compress_kv.  With
                                 TQ_ROT_DENSE, compression runs on the tensor cores only
                                 when these operands are given (and keys and values carry
                                 no QJL sketch); otherwise on the CUDA cores.          */
} tq_params;

/* A paged cache ([LIMITS] vLLM-style packed paged cache). */
typedef struct tq_cache {
  void* pages;                 /* device [num_layers][num_pages][kv_heads][page bytes]     */
  const int32_t* block_table;  /* device [batch][max_pages]: physical page of each logical
                                  page of each sequence                                   */
  int32_t num_pages;           /* physical pages per layer                                */
  int32_t max_pages;           /* length of one block-table row                           */
  int32_t batch;
  int32_t kv_heads;
  int32_t num_layers;
} tq_cache;

/* Library version (major*10000 + minor*100 + patch). */
TQ_API int32_t tq_version(void);

/* Human-readable name of a status code (static string). */
TQ_API const char* tq_status_str(tq_status st);

/* Status of the device work of earlier calls, from the caller's host copy of their
 * dev_status word (copy it back after synchronising the stream the calls ran on).
 *   dev_status_host_copy  host pointer to that int32 value
 * Returns the recorded code (TQ_OK when the word is 0) and describes it in
 * tq_last_error(); TQ_ERR_INVALID_ARG for a NULL pointer or a value that is no
 * status code.  The word itself is not changed: the caller resets it to 0 before the
 * next calls that should be checked on their own. */
TQ_API tq_status tq_check(const int32_t* dev_status_host_copy);

/* Detail of the last host-side error on the calling thread (static per-thread
 * buffer, empty string if none). */
TQ_API const char* tq_last_error(void);

/* Checks a configuration; TQ_OK if this library supports it. */
TQ_API tq_status tq_validate_config(const tq_config* cfg);

/* Bytes of one (layer, page, kv head) block for cfg; 0 if cfg is invalid. */
TQ_API size_t tq_page_bytes(const tq_config* cfg);

/* Lloyd-Max codebook ([MOBILINT] "Designing the Optimal Codebook Without Data",
 * steps 1-3, on the density of "Coordinates Become Predictable After Rotation";
 * [CUTILE] codebook function; [TQKV] module codebook for the Gaussian variant).
 * HOST call, synchronous.
 *   bits        1..8
 *   head_dim    d >= 3; the density is f_X(t) ~ (1 - t^2)^((d-3)/2) on [-1, 1]
 *               (TQ_DENSITY_BETA) or N(0, 1/d) (TQ_DENSITY_GAUSS)
 *   centroids   host float[2^bits], written sorted ascending
 *   boundaries  host float[2^bits - 1], the fp32 rounding of the midpoints of the
 *               double-precision centroids
 * The iteration starts from linspace(-2/sqrt(d), 2/sqrt(d), 2^bits), runs until
 * the centroids move by less than 1e-13, and symmetrises the result. */
TQ_API tq_status tq_codebook(int32_t bits, int32_t head_dim, int32_t density, float* centroids,
                      float* boundaries);

/* Uniform codebook of the dithered quantizer ([DITHER]; HOST call, synchronous):
 * centroids c_j = (j - (2^b - 1)/2) delta, boundaries at their midpoints (the middle one
 * 0), each rounded to fp32 from double.  delta minimises the expected squared error of a
 * coordinate with density f_X (as for tq_codebook) under subtractive dither, xi uniform
 * on [-delta/2, delta/2):  D(delta) = delta^2/12 + 2 int_A^inf (t - A)^2 f_X(t) dt,
 * A = (2^b - 1) delta / 2; it is the root of dD/d delta (increasing in delta), found by
 * bisection on the closed-form tail moments.  Arguments as for tq_codebook. */
TQ_API tq_status tq_dither_codebook(int32_t bits, int32_t head_dim, int32_t density, float* centroids,
                                    float* boundaries);

/* Compress K and V into the packed cache ([CUTILE] compress K (MSE + QJL) and
 * compress V (MSE only); [MOBILINT] "Two-Stage Approach": per vector n = ||x||,
 * u = x/n, y = R u, idx_j = #{i : beta_i < y_j}, stored fp16(n); for keys with
 * QJL, k_mse = fp16(n) R^T c[idx], r = k - k_mse, sign bits [(S r)_i >= 0] and
 * fp16(||r||)).
 *   layer      0..num_layers-1
 *   k, v       device [batch][kv_heads][max_len][d], element type in_dtype
 *   seq_lens   device int32 [batch]; tokens 0..seq_lens[b]-1 of each (b, head) are
 *              written to slots via the block table (logical page t/P, slot t%P)
 *   dev_status device int32; TQ_ERR_OVERFLOW, TQ_ERR_BOUNDS, TQ_ERR_INVALID_ARG
 * Pages not covered by a sequence are not touched.  A dithered configuration returns
 * TQ_ERR_INVALID_ARG (its offsets come through tq_compress_kv_dithered). */
TQ_API tq_status tq_compress_kv(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                         int32_t layer, const void* k, const void* v, int32_t in_dtype,
                         int32_t max_len, const int32_t* seq_lens, int32_t* dev_status,
                         tq_stream_t stream);

/* tq_compress_kv for a dithered configuration (cfg->dither = 1, [DITHER]): every vector
 * x = k or v of token t is coded with its own offset xi = fp16(offsets[b][h][t]) (RNE):
 * y = H D x / ||x||, idx = #{i : beta_i < y_j - xi}, xi stored in KD / VD.  The caller
 * draws the offsets (uniform on [-delta/2, delta/2), delta = c[1] - c[0] of the
 * tq_dither_codebook grid, makes the reconstruction unbiased inside the grid's range).
 *   k_offsets, v_offsets  device float [batch][kv_heads][max_len]
 * Everything else as for tq_compress_kv; TQ_ERR_INVALID_ARG for a configuration that is
 * not dithered. */
TQ_API tq_status tq_compress_kv_dithered(const tq_config* cfg, const tq_params* params,
                                         const tq_cache* cache, int32_t layer, const void* k,
                                         const void* v, const float* k_offsets, const float* v_offsets,
                                         int32_t in_dtype, int32_t max_len, const int32_t* seq_lens,
                                         int32_t* dev_status, tq_stream_t stream);

/* Bytes of the prepared tensor-core operands of tq_compress_kv for cfg (96 KiB for a
 * TQ_ROT_HADAMARD configuration, 64 KiB for TQ_ROT_DENSE; 0 if cfg is invalid). */
TQ_API size_t tq_operand_bytes(const tq_config* cfg);

/* Prepare the operands tq_compress_kv uses on the tensor cores for the rotation
 * R = H D / sqrt(d) ([MOBILINT] "How JL Matrices Evolved") and, with key_qjl, the QJL
 * sketch taken in the rotated domain ([MOBILINT] "QJL: Inner Product Recovery from a
 * Single Sign Bit": S r = (S D H) (H D r) / d): three 128 x 128 fp16 tiles in the
 * tensor cores' canonical K-major layout, B = H D (entries +-1, exact), then S D H
 * (formed in fp32) as a high fp16 part and the fp16 rounding of the remainder.  For
 * TQ_ROT_DENSE ([CUTILE]: Haar Pi), two tiles: sqrt(d) Pi (row i, column k = Pi_ik,
 * formed in fp32) as a high fp16 part and the fp16 rounding of the remainder.
 *   params    signs (and s with key_qjl) as for tq_compress_kv, or pi for TQ_ROT_DENSE;
 *             S need not be fp16-exact on this path
 *   operands  device, tq_operand_bytes(cfg) bytes, 16-byte aligned; written
 *             asynchronously on stream; owned by the caller, who passes it in
 *             tq_params.operands while signs and s stay unchanged
 * Errors: TQ_ERR_INVALID_ARG for NULL or misaligned pointers. */
TQ_API tq_status tq_prepare_operands(const tq_config* cfg, const tq_params* params, void* operands,
                                     tq_stream_t stream);

/* Workspace bytes tq_attend_decode and tq_decode_scores need for these sizes. */
TQ_API size_t tq_decode_workspace_bytes(const tq_config* cfg, int32_t batch, int32_t q_heads,
                                 int32_t seq_q, int32_t n_splits);

/* Decode attention over the packed cache ([CUTILE] full pipeline with the
 * asymmetric estimator and fused on-chip V dequantisation; [MOBILINT] "How is this
 * different from PolarQuant's reconstruction?": <q, R^T c> = <R q, c>, so R q is
 * formed once per query; [TQKV] pre_rotate_query / fused_attention_scores).
 * For query row (b, h, p), kv head g = h / (q_heads / kv_heads):
 *   score_t = ( ||k||_t <R q, c_k[idx_t]>
 *               + [QJL] ||r||_t sqrt(pi/2)/m <S q, 2 sigma_t - 1> ) / sqrt(d)
 *   out     = R^T sum_t softmax(score)_t ||v||_t c_v[idx_v,t]
 *             [+ with value_qjl: sqrt(pi/2)/m S^T sum_t softmax(score)_t ||r_v||_t (2 sigma_v,t - 1)]
 * over t < seq_lens[b] (no causal mask between the seq_q rows; an empty sequence
 * gives 0).  The sequence is cut into at most n_splits contiguous ranges processed in
 * parallel and merged by their log-sum-exp: n_splits when every sequence of the batch
 * has the same length; when the lengths differ, the tensor-core kernel sizes the ranges
 * from the batch's total work, so that shorter sequences take fewer of them.
 *   q          device [batch][q_heads][seq_q][d], element type q_dtype
 *   q_heads    multiple of kv_heads; q_heads/kv_heads * seq_q <= 32
 *   n_splits   1..1024
 *   workspace  device, >= tq_decode_workspace_bytes(...) bytes, 256-byte aligned;
 *              scratch only, contents on return unspecified
 *   out        device float [batch][q_heads][seq_q][d]
 * A test of the device's bounded waits: with the environment variable
 * TQ_DEBUG_BOUNDED_WAIT_US set to n (1..1000000) when the call is made, one warp of the
 * tensor-core split kernel (keys 2- or 3-bit with QJL or 4-bit without, values 2- or
 * 3-bit) waits n microseconds on a barrier that nothing completes and writes
 * TQ_ERR_TIMEOUT to dev_status; the results are computed as usual. */
TQ_API tq_status tq_attend_decode(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                           int32_t layer, const void* q, int32_t q_dtype, int32_t q_heads,
                           int32_t seq_q, const int32_t* seq_lens, int32_t n_splits,
                           void* workspace, size_t workspace_bytes, float* out,
                           int32_t* dev_status, tq_stream_t stream);

/* Incremental append ([TQKV] incremental cache: CompressedKeys::append_raw and
 * compress_single_key_with_signs; [LIMITS] packed page update): compresses n_new new
 * tokens of every (sequence, kv head) exactly as tq_compress_kv would and writes them to
 * their slots, leaving every other slot of the cache untouched (a token's bytes are
 * independent of its neighbours' in the packed format above).
 *   k_new, v_new  device [batch][kv_heads][n_new][d], element type in_dtype
 *   n_new         >= 1 (batch * kv_heads * n_new <= 2^30)
 *   seq_lens      device int32 [batch]: the lengths AFTER the append; new token n of
 *                 sequence b goes to position seq_lens[b] - n_new + n (logical page
 *                 pos / P, slot pos % P of the block table)
 *   dev_status    TQ_ERR_BOUNDS when seq_lens[b] < n_new, seq_lens[b] exceeds the
 *                 block-table row or a page id is out of range (that token is skipped);
 *                 TQ_ERR_OVERFLOW as for tq_compress_kv
 * params.s (with key_qjl) and params.pi (TQ_ROT_DENSE) must be 16-byte aligned; S is
 * used in fp32 as given (no fp16 requirement).  One thread block per new token.
 * Dithered configurations return TQ_ERR_UNSUPPORTED: their appends take the new tokens'
 * offsets through tq_append_kv_dithered. */
TQ_API tq_status tq_append_kv(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                              int32_t layer, const void* k_new, const void* v_new, int32_t in_dtype,
                              int32_t n_new, const int32_t* seq_lens, int32_t* dev_status,
                              tq_stream_t stream);

/* One decode step with its append fused in: the effect of tq_append_kv(k_new, v_new,
 * n_new, seq_lens) followed by tq_attend_decode(q, seq_lens), so the new tokens are
 * attended to by the query rows of the same step (seq_lens are the lengths after the
 * append).  The new tokens are encoded by extra thread blocks of the decode's query
 * prologue; the attention kernels copy a page range holding a new token only after the
 * prologue has finished.  Arguments, errors and workspace as for the two calls. */
TQ_API tq_status tq_append_attend_decode(const tq_config* cfg, const tq_params* params,
                                         const tq_cache* cache, int32_t layer, const void* k_new,
                                         const void* v_new, int32_t in_dtype, int32_t n_new,
                                         const void* q, int32_t q_dtype, int32_t q_heads,
                                         int32_t seq_q, const int32_t* seq_lens, int32_t n_splits,
                                         void* workspace, size_t workspace_bytes, float* out,
                                         int32_t* dev_status, tq_stream_t stream);

/* The two appends for a dithered configuration (cfg->dither = 1, [DITHER]): new token n of
 * (sequence b, head h) is coded with the offsets xi = fp16(k_offsets[b][h][n]) and
 * fp16(v_offsets[b][h][n]) exactly as tq_compress_kv_dithered codes it, the offsets stored
 * in its KD / VD slots.
 *   k_offsets, v_offsets  device float [batch][kv_heads][n_new]
 * Everything else as for tq_append_kv and tq_append_attend_decode; TQ_ERR_INVALID_ARG for a
 * configuration that is not dithered or NULL offsets. */
TQ_API tq_status tq_append_kv_dithered(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                                       int32_t layer, const void* k_new, const void* v_new,
                                       const float* k_offsets, const float* v_offsets, int32_t in_dtype,
                                       int32_t n_new, const int32_t* seq_lens, int32_t* dev_status,
                                       tq_stream_t stream);
TQ_API tq_status tq_append_attend_decode_dithered(const tq_config* cfg, const tq_params* params,
                                                  const tq_cache* cache, int32_t layer, const void* k_new,
                                                  const void* v_new, const float* k_offsets,
                                                  const float* v_offsets, int32_t in_dtype, int32_t n_new,
                                                  const void* q, int32_t q_dtype, int32_t q_heads,
                                                  int32_t seq_q, const int32_t* seq_lens, int32_t n_splits,
                                                  void* workspace, size_t workspace_bytes, float* out,
                                                  int32_t* dev_status, tq_stream_t stream);

/* Decode attention for callers that cannot allocate device memory (no counterpart on
 * the source pages; it exists for users of this library).  Same computation, arguments
 * and results as tq_attend_decode, minus the workspace: a plugin inside a runtime that
 * owns all device memory, or a serving loop that must not call cudaMalloc mid-step, can
 * call this instead.  The scratch lives in a built-in 8 MiB array in device global
 * memory, held until the CUDA context ends.
 *   - Sizes whose tq_decode_workspace_bytes(...) exceeds 8 MiB return
 *     TQ_ERR_UNSUPPORTED with an explanation in tq_last_error(); nothing is enqueued.
 *   - Under lazy module loading (the CUDA default) the array's 8 MiB are reserved on a
 *     device by the first call there, not when the library is loaded: make that first
 *     call at start-up, before the caller's runtime claims the device memory pool.
 *   - Every call made outside stream capture looks up the array's device address in the
 *     current context (so a context that was reset gets its own address); a call made
 *     while its stream is being captured reuses the address its context found before and
 *     returns TQ_ERR_INVALID_ARG if there is none: make the first call in each context
 *     before any stream capture begins.
 *   - All calls on a device share the one array: calls whose kernels can overlap in
 *     time race and give undefined results.  Order them on a single stream.
 *   - Nothing in the array needs clearing between calls (every byte read is first
 *     written by the same call).
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library call. */
TQ_API tq_status tq_attend_decode_noalloc(const tq_config* cfg, const tq_params* params,
                                          const tq_cache* cache, int32_t layer, const void* q,
                                          int32_t q_dtype, int32_t q_heads, int32_t seq_q,
                                          const int32_t* seq_lens, int32_t n_splits, float* out,
                                          int32_t* dev_status, tq_stream_t stream);

/* Score-only decode ([CUTILE] "Score-only kernel ... streams over KV"): writes the
 * scaled scores score_t above for every query row and t < seq_lens[b]; entries with
 * t >= seq_lens[b] are left untouched.
 *   scores     device float [batch][q_heads][seq_q][max_len]
 *   workspace  as for tq_attend_decode with n_splits = 1 */
TQ_API tq_status tq_decode_scores(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                           int32_t layer, const void* q, int32_t q_dtype, int32_t q_heads,
                           int32_t seq_q, const int32_t* seq_lens, int32_t max_len,
                           void* workspace, size_t workspace_bytes, float* scores,
                           int32_t* dev_status, tq_stream_t stream);

/* Decompress ([CUTILE] "indices -> centroids -> un-rotate -> rescale"):
 * k_hat = ||k|| R^T c_k[idx] (the MSE part k_mse for QJL keys) and
 * v_hat = ||v|| R^T c_v[idx_v] (the MSE part for values with QJL), c[idx] + xi for
 * dithered configurations, with the stored (possibly corrected) norms, for tokens
 * t < seq_lens[b]; rows past the
 * length are left untouched.
 *   k_hat, v_hat  device float [batch][kv_heads][max_len][d] (either may be NULL) */
TQ_API tq_status tq_decompress(const tq_config* cfg, const tq_params* params, const tq_cache* cache,
                        int32_t layer, const int32_t* seq_lens, int32_t max_len, float* k_hat,
                        float* v_hat, int32_t* dev_status, tq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* TQ_H_ */
