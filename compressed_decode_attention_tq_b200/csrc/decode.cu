// Decode attention directly over the packed cache (split-KV, flash-decoding style).
//
// "turboquant_cutile" function list: asymmetric estimator = MSE dot + QJL correction;
// full pipeline scores -> softmax -> weighted V sum; fused attention + online softmax
// with V decompressed on chip; scores scaled by 1/sqrt(d).
// "TurboQuant explained" (Mobilint blog), section "How is this different from
// PolarQuant's reconstruction?": <q, Pi^T c> = <Pi q, c>, so the rotated query is
// formed once and each cached token costs an O(d) centroid-table product; section
// "Practical Issues Found in Implementation": dequantisation must be fused with the
// attention, never materialising dense K/V in HBM.
// "tq-kv" crate documentation: pre_rotate_query, fused_attention_scores.
//
// Kernels: prologue (R q and S q per query row), split (online softmax over one
// contiguous range of pages, partial (m, l, acc) in rotated space), combine
// (log-sum-exp merge, divide by l, un-rotate with R^T).
#include <cuda_fp16.h>
#include <math_constants.h>

#include "tq_device.cuh"
#include "tq_kernels.h"

namespace tqk {

namespace {

constexpr int kRowsMax = 32;
constexpr int kTile = 128;  // tokens per tile (half a page)
constexpr float kInvSqrtD = 0.08838834764831845f;
constexpr float kQjlScale = 1.2533141373155003f / QM;  // sqrt(pi/2)/m

size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ---------------------------------------------------------------------------
// append: one CTA of 128 threads per new token of one (sequence, kv head); thread i owns
// coordinate i, warp w the coordinates 32w..32w+31.  The same encoding as the compress
// kernels ("TurboQuant explained", section "Two-Stage Approach: MSE Approximation + QJL
// Correction"; "tq-kv" crate documentation, incremental cache: a new token is compressed
// and appended to its page without touching the tokens already stored).
// ---------------------------------------------------------------------------
constexpr int kMergedNibble = 0;  // pack_code's `bits` for a merged key nibble, passed whole in r

struct __align__(16) AppendShared {
  float xs[D];          // the vector being transformed
  float tab[4][16];     // k centroids, k boundaries, v centroids, v boundaries
  float red[4];
  uint32_t kw[16], ksw[4], vw[16], vsw[4];
};

__device__ __forceinline__ float block_sum128(float v, float* red, int lane, int warp) {
  v = warp_sum(v);
  __syncthreads();  // red may still be read by an earlier sum
  if (lane == 0) red[warp] = v;
  __syncthreads();
  return (red[0] + red[1]) + (red[2] + red[3]);
}

// y = R x / n for thread i's coordinate (x_i in x): H D through the warp-level transform
// in warp 0, or a row of Pi.
__device__ __forceinline__ float rotate_coord(const DecodeArgs& a, AppendShared& sh, float x, float inv,
                                              int i, int lane, int warp) {
  float y;
  if (!a.dense) {
    sh.xs[i] = x * a.signs[i];
    __syncthreads();
    if (warp == 0) {
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = sh.xs[lane + 32 * e];
      fwht128_warp(v, lane);
#pragma unroll
      for (int e = 0; e < 4; ++e) sh.xs[lane + 32 * e] = v[e];
    }
    __syncthreads();
    y = sh.xs[i] * (inv * kInvSqrtD);
  } else {
    sh.xs[i] = x * inv;
    __syncthreads();
    const float4* prow = reinterpret_cast<const float4*>(a.pi + (size_t)i * D);
    float acc = 0.f;
#pragma unroll 8
    for (int k = 0; k < D / 4; ++k) {
      const float4 p = prow[k];
      acc = fmaf(p.x, sh.xs[4 * k], acc);
      acc = fmaf(p.y, sh.xs[4 * k + 1], acc);
      acc = fmaf(p.z, sh.xs[4 * k + 2], acc);
      acc = fmaf(p.w, sh.xs[4 * k + 3], acc);
    }
    y = acc;
  }
  __syncthreads();  // xs is free again
  return y;
}

// Code words of one token for `bits` from this thread's (s, r); warp w writes the words
// that hold coordinates 32w..32w+31 (the stored layout of the cache format).
__device__ __forceinline__ void pack_code(int s, int r, int bits, int lane, int warp, uint32_t* w) {
  const int e = warp;
  if (bits == 1) {
    const uint32_t b = __ballot_sync(FULL, s);
    if (lane == 0) w[e] = b;
  } else if (bits == 2 || bits == 3) {
    const uint32_t f = bits == 2 ? (uint32_t)(r | (s << 1)) : (uint32_t)r;
    const uint32_t sh = f << (2 * (lane & 15));
    const uint32_t lo = __reduce_or_sync(FULL, lane < 16 ? sh : 0u);
    const uint32_t hi = __reduce_or_sync(FULL, lane < 16 ? 0u : sh);
    const uint32_t sp = bits == 3 ? __reduce_or_sync(FULL, (uint32_t)s << (sign_plane_pos(lane) & 31)) : 0u;
    if (lane == 0) {
      w[2 * e] = lo;
      w[2 * e + 1] = hi;
      if (bits == 3) w[8 + e] = sp;
    }
  } else {
    // 4-bit fields (r in bits 0..2, s in bit 3), or a merged key nibble (r0, r1, s, sigma)
    const uint32_t f = bits == kMergedNibble ? (uint32_t)r : (uint32_t)(r | (s << 3));
    const uint32_t sh = f << (4 * (lane & 7));
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t v = __reduce_or_sync(FULL, (lane >> 3) == q ? sh : 0u);
      if (lane == 0) w[4 * e + q] = v;
    }
  }
}

// Encodes thread i's coordinate of one vector: stored norm, index, (s, r); returns y.
// xi: the vector's dither offset (0 when not dithered): idx = Quant(y - xi).  cent
// non-null: store the corrected norm n / ||c[idx] + xi|| ("tq-kv" documentation:
// corrected_norm) instead of n.
__device__ __forceinline__ float encode_coord(const DecodeArgs& a, AppendShared& sh, float x, const float* bnd,
                                              int bits, int i, int lane, int warp, __half& nh, int& idx,
                                              int& s, int& r, const float* cent = nullptr, float xi = 0.f) {
  const float n = sqrtf(block_sum128(x * x, sh.red, lane, warp));
  const float y = rotate_coord(a, sh, x, n > 0.f ? 1.0f / n : 0.0f, i, lane, warp);
  const int nb = (1 << bits) - 1, h = 1 << (bits - 1);
  const float yq = y - xi;
  idx = 0;
  for (int k = 0; k < nb; ++k) idx += (yq > bnd[k]) ? 1 : 0;
  s = idx >= h;
  r = s ? idx - h : h - 1 - idx;
  float stored = n;
  if (cent) {
    const float c = cent[idx] + xi;
    const float yn = sqrtf(block_sum128(c * c, sh.red, lane, warp));
    stored = yn > 0.f ? n / yn : 0.f;
  }
  nh = __float2half_rn(stored);
  if (__hisinf(nh) && i == 0) report(a.status, TQ_ERR_OVERFLOW);
  return y;
}

// Residual of thread i's coordinate in the original space, r = x - fp16(n) R^T c[idx] (c_i:
// the centroid of its index), its stored norm fp16(||r||) (returned), and the sign
// sigma = [(S r)_i >= 0] of row i of S (sign(0) stored as +1).
__device__ __forceinline__ __half append_qjl(const DecodeArgs& a, AppendShared& sh, float x, __half nh, float c_i,
                                             int i, int lane, int warp, int& sigma) {
  float z;
  sh.xs[i] = c_i;
  __syncthreads();
  if (!a.dense) {
    if (warp == 0) {
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = sh.xs[lane + 32 * e];
      fwht128_warp(v, lane);
#pragma unroll
      for (int e = 0; e < 4; ++e) sh.xs[lane + 32 * e] = v[e];
    }
    __syncthreads();
    z = sh.xs[i] * kInvSqrtD * a.signs[i];
  } else {
    float acc = 0.f;
#pragma unroll 8
    for (int k = 0; k < D; ++k) acc = fmaf(a.pi[(size_t)k * D + i], sh.xs[k], acc);  // (Pi^T z)_i
    z = acc;
  }
  __syncthreads();
  const float res = x - __half2float(nh) * z;
  const __half rho = __float2half_rn(sqrtf(block_sum128(res * res, sh.red, lane, warp)));
  sh.xs[i] = res;
  __syncthreads();
  // (S r)_o for the 32 rows o of this warp: lanes read 4 consecutive entries of row o
  const float4 r4 = reinterpret_cast<const float4*>(sh.xs)[lane];
  float sr = 0.f;
#pragma unroll 8
  for (int u = 0; u < 32; ++u) {
    const float4 p = reinterpret_cast<const float4*>(a.s + (size_t)(32 * warp + u) * D)[lane];
    float t = p.x * r4.x;
    t = fmaf(p.y, r4.y, t);
    t = fmaf(p.z, r4.z, t);
    t = fmaf(p.w, r4.w, t);
    t = warp_sum(t);
    if (lane == u) sr = t;
  }
  sigma = sr >= 0.f;
  __syncthreads();  // xs is free again
  return rho;
}

template <typename T>
__device__ __forceinline__ float ld_new(const void* p, size_t i) {
  return (float)reinterpret_cast<const T*>(p)[i];
}

// Token job = ((b * kv_heads + h) * n_new + n) goes to position seq_lens[b] - n_new + n.
__device__ void append_token(const DecodeArgs& a, int job) {
  __shared__ AppendShared sh;
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  const int n = job % a.n_new, h = (job / a.n_new) % a.cache.kv_heads, b = job / (a.n_new * a.cache.kv_heads);
  const Layout& L = a.cache.L;
  const int nk = 1 << L.kbits, nv = 1 << L.vbits;
  if (i < nk) sh.tab[0][i] = a.k_centroids[i];
  if (i < nk - 1) sh.tab[1][i] = a.k_boundaries[i];
  if (i < nv) sh.tab[2][i] = a.v_centroids[i];
  if (i < nv - 1) sh.tab[3][i] = a.v_boundaries[i];
  const int len = a.seq_lens[b];
  const int pos = len - a.n_new + n;
  if (len < a.n_new || len > a.cache.max_pages * PT) {
    if (i == 0) report(a.status, TQ_ERR_BOUNDS);
    return;
  }
  const int phys = a.cache.block_table[(size_t)b * a.cache.max_pages + pos / PT];
  if (phys < 0 || phys >= a.cache.num_pages) {
    if (i == 0) report(a.status, TQ_ERR_BOUNDS);
    return;
  }
  uint8_t* blk = a.cache.block(phys, h);
  const int slot = pos % PT;
  const size_t src = (size_t)job * D + i;
  // dithered: the token's offsets, used and stored as fp16
  __half kxi16 = __float2half_rn(0.f), vxi16 = kxi16;
  if (L.dither) {
    kxi16 = __float2half_rn(a.k_new_off[job]);
    vxi16 = __float2half_rn(a.v_new_off[job]);
    if (i == 0) {
      reinterpret_cast<__half*>(blk + L.kd)[slot] = kxi16;
      reinterpret_cast<__half*>(blk + L.vd)[slot] = vxi16;
    }
  }
  const float kxi = __half2float(kxi16), vxi = __half2float(vxi16);
  __syncthreads();

  // ---- key: norm, rotation, quantisation
  const float x = a.new_dtype == TQ_F16 ? __half2float(reinterpret_cast<const __half*>(a.k_new)[src])
                                        : ld_new<float>(a.k_new, src);
  __half nh;
  int idx, s, r;
  encode_coord(a, sh, x, sh.tab[1], L.kbits, i, lane, warp, nh, idx, s, r, a.key_corr ? sh.tab[0] : nullptr, kxi);
  if (!L.kmerged) pack_code(s, r, L.kbits, lane, warp, sh.kw);
  if (a.qjl) {
    int sigma;
    const __half rho = append_qjl(a, sh, x, nh, sh.tab[0][idx] + kxi, i, lane, warp, sigma);
    if (L.kmerged) {
      pack_code(s, r | (s << 2) | (sigma << 3), kMergedNibble, lane, warp, sh.kw);
    } else {
      const uint32_t bw = __ballot_sync(FULL, sigma);
      if (lane == 0) sh.ksw[warp] = bw;
    }
    if (i == 0) reinterpret_cast<__half*>(blk + L.kr)[slot] = rho;
  }
  __syncthreads();
  if (i < L.kchunks)
    reinterpret_cast<uint4*>(blk + L.kc)[i * PT + slot] = reinterpret_cast<const uint4*>(sh.kw)[i];
  if (a.qjl && !L.kmerged && i == 0)
    reinterpret_cast<uint4*>(blk + L.ks)[slot] = reinterpret_cast<const uint4*>(sh.ksw)[0];
  if (i == 0) reinterpret_cast<__half*>(blk + L.kn)[slot] = nh;

  // ---- value
  const float xv = a.new_dtype == TQ_F16 ? __half2float(reinterpret_cast<const __half*>(a.v_new)[src])
                                         : ld_new<float>(a.v_new, src);
  __half nv16;
  encode_coord(a, sh, xv, sh.tab[3], L.vbits, i, lane, warp, nv16, idx, s, r, nullptr, vxi);
  pack_code(s, r, L.vbits, lane, warp, sh.vw);
  if (L.vqjl) {
    // values with QJL: the same sketch of the value residual, signs in VS, norm in VR
    int sigma;
    const __half rho = append_qjl(a, sh, xv, nv16, sh.tab[2][idx] + vxi, i, lane, warp, sigma);
    const uint32_t bw = __ballot_sync(FULL, sigma);
    if (lane == 0) sh.vsw[warp] = bw;
    if (i == 0) reinterpret_cast<__half*>(blk + L.vr)[slot] = rho;
  }
  __syncthreads();
  if (i < L.vbits)
    reinterpret_cast<uint4*>(blk + L.vc)[i * PT + slot] = reinterpret_cast<const uint4*>(sh.vw)[i];
  if (L.vqjl && i == 0)
    reinterpret_cast<uint4*>(blk + L.vs)[slot] = reinterpret_cast<const uint4*>(sh.vsw)[0];
  if (i == 0) reinterpret_cast<__half*>(blk + L.vn)[slot] = nv16;
}

// ---------------------------------------------------------------------------
// prologue: one CTA of 128 threads per query row.  Thread i owns coordinate i.
//   qrot = R q (fp32), q8 = int8 rounding of qrot * 127 / max|qrot| (with its scale),
//   sq = S q (fp32), sq_int = S q in 16-bit fixed point with a power-of-two scale, sum.
// A row's terms are published through its ready word: zeroed before the CTA lets the split
// kernel start, set (release) once every term of the row is written.  The tensor-core split
// kernel acquires the words of its rows instead of waiting for this whole grid to finish.
// ---------------------------------------------------------------------------

// Before launch_dependents: the row's terms of an earlier call are no longer announced (its
// kQueryParts ready words, threads 0 .. kQueryParts - 1).
__device__ __forceinline__ void unpublish_row(const DecodeArgs& a, int row) {
  if (threadIdx.x < kQueryParts) {
    const unsigned int* rw = a.ready + (size_t)row * kQueryParts + threadIdx.x;
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(rw), "r"(0u) : "memory");
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
  }
  __syncthreads();
}

// After every term of the row is written: the barrier orders the block's writes before the
// release stores that set the ready words.
__device__ __forceinline__ void publish_row(const DecodeArgs& a, int row) {
  __syncthreads();
  if (threadIdx.x < kQueryParts)
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(a.ready + (size_t)row * kQueryParts + threadIdx.x),
                 "r"(1u)
                 : "memory");
}

// The merge counter of the tensor-core split kernel's run of query rows that starts at this
// row (runs of four, or eight when a KV head has more than four rows): zero at every call,
// zeroed before the row's terms are announced
__device__ __forceinline__ void zero_run_counter(const DecodeArgs& a, int row) {
  const int nr = a.rows > 4 ? 8 : 4, local = row % a.rows;
  TQ_DCHECK(a.status, (row / a.rows) * ((a.rows + nr - 1) / nr) + local / nr < a.cache.batch * a.q_heads * a.seq_q);
  if (threadIdx.x == 0 && local % nr == 0) a.counter[(row / a.rows) * ((a.rows + nr - 1) / nr) + local / nr] = 0u;
}

__device__ __forceinline__ void query_row(const DecodeArgs& a, int row) {
  __shared__ __align__(16) float qs[D];
  __shared__ float ys[D];
  __shared__ float red[2][4];
  __shared__ int ired[4];
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  zero_run_counter(a, row);
  // the rows of S this warp needs, requested before the query (they do not depend on it)
  float4 p[32];
  if (a.qjl) {
#pragma unroll
    for (int u = 0; u < 32; ++u) p[u] = reinterpret_cast<const float4*>(a.s + (size_t)(32 * warp + u) * D)[lane];
  }
  const float x = a.q_dtype == TQ_F16 ? __half2float(reinterpret_cast<const __half*>(a.q)[(size_t)row * D + i])
                                      : reinterpret_cast<const float*>(a.q)[(size_t)row * D + i];
  qs[i] = x;
  __syncthreads();
  float y;
  if (!a.dense) {
    // y = H D q / sqrt(d): the warp-level transform in warp 0
    if (warp == 0) {
      float v[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) v[e] = qs[lane + 32 * e] * a.signs[lane + 32 * e];
      fwht128_warp(v, lane);
#pragma unroll
      for (int e = 0; e < 4; ++e) ys[lane + 32 * e] = v[e] * kInvSqrtD;
    }
    __syncthreads();
    y = ys[i];
  } else {
    const float4* prow = reinterpret_cast<const float4*>(a.pi + (size_t)i * D);
    float acc = 0.f;
#pragma unroll 8
    for (int k = 0; k < D / 4; ++k) {
      const float4 p = prow[k];
      acc = fmaf(p.x, qs[4 * k], acc);
      acc = fmaf(p.y, qs[4 * k + 1], acc);
      acc = fmaf(p.z, qs[4 * k + 2], acc);
      acc = fmaf(p.w, qs[4 * k + 3], acc);
    }
    y = acc;
  }
  a.qrot[(size_t)row * D + i] = y;
  float sq = 0.f;
  if (a.qjl) {
    // (S q)_o for the 32 outputs o of this warp: lanes read 4 consecutive entries of row o
    // (coalesced), then a warp sum; all 32 row loads are in flight together
    const float4 q4 = reinterpret_cast<const float4*>(qs)[lane];
#pragma unroll
    for (int u = 0; u < 32; ++u) {
      float t = p[u].x * q4.x;
      t = fmaf(p[u].y, q4.y, t);
      t = fmaf(p[u].z, q4.z, t);
      t = fmaf(p[u].w, q4.w, t);
      t = warp_sum(t);
      if (lane == u) sq = t;
    }
    a.sq[(size_t)row * QM + i] = sq;
  }
  // maxima of |R q| and |S q| over the row
  float my = fabsf(y), ms = fabsf(sq);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    my = fmaxf(my, __shfl_xor_sync(FULL, my, o));
    ms = fmaxf(ms, __shfl_xor_sync(FULL, ms, o));
  }
  if (lane == 0) {
    red[0][warp] = my;
    red[1][warp] = ms;
  }
  __syncthreads();
  const float ym = fmaxf(fmaxf(red[0][0], red[0][1]), fmaxf(red[0][2], red[0][3]));
  const float lam = ym > 0.f ? 127.f / ym : 0.f;
  a.q8[(size_t)row * D + i] = (int8_t)__float2int_rn(y * lam);
  if (i == 0) a.q8_scale[row] = lam;
  if (a.qjl) {
    const float mx = fmaxf(fmaxf(red[1][0], red[1][1]), fmaxf(red[1][2], red[1][3]));
    // 16-bit fixed point with a power-of-two scale: |sq_int| <= 32000
    int ex = 0;
    if (mx > 0.f) {
      frexpf(32000.f / mx, &ex);
      ex -= 1;  // 2^ex <= 32000 / mx
    }
    const int v = __float2int_rn(sq * ldexpf(1.f, ex));
    a.sq_int[(size_t)row * QM + i] = (int16_t)v;
    int sum = v;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum += __shfl_xor_sync(FULL, sum, o);
    if (lane == 0) ired[warp] = sum;
    __syncthreads();
    if (i == 0) {
      a.sq_scale[row] = ldexpf(1.f, -ex);
      a.sq_sum[row] = ired[0] + ired[1] + ired[2] + ired[3];
    }
  }
}

// Before launch_dependents: this part's terms of an earlier call are no longer announced.
__device__ __forceinline__ void unpublish_part(const DecodeArgs& a, int blk) {
  if (threadIdx.x == 0) {
    asm volatile("st.relaxed.gpu.global.u32 [%0], %1;" ::"l"(a.ready + blk), "r"(0u) : "memory");
    asm volatile("fence.acq_rel.gpu;" ::: "memory");
  }
  __syncthreads();
}

// Part blk % kQueryParts of query row blk / kQueryParts (after unpublish_part and the launch
// of the dependents).
__device__ __forceinline__ void query_part(const DecodeArgs& a, int blk) {
  const int row = blk / kQueryParts, part = blk % kQueryParts;
  TQ_DCHECK(a.status, row < a.cache.batch * a.q_heads * a.seq_q);
  const unsigned int* rw = a.ready + blk;
  __shared__ __align__(16) float qs[D];
  __shared__ float ys[D];
  __shared__ float red[4];
  const int i = threadIdx.x, lane = i & 31, warp = i >> 5;
  // the rows of S of this warp's outputs o = 32 part + 8 warp + j, requested before the query
  // (they do not depend on it); lane l holds entries 4 l .. 4 l + 3 of each
  const int o0 = 32 * part + 8 * warp;
  float4 p[8];
  if (a.qjl) {
#pragma unroll
    for (int j = 0; j < 8; ++j) p[j] = reinterpret_cast<const float4*>(a.s + (size_t)(o0 + j) * D)[lane];
  }
  qs[i] = a.q_dtype == TQ_F16 ? __half2float(reinterpret_cast<const __half*>(a.q)[(size_t)row * D + i])
                              : reinterpret_cast<const float*>(a.q)[(size_t)row * D + i];
  if (part == 0) zero_run_counter(a, row);
  __syncthreads();
  if (part == 0) {
    float y;
    if (!a.dense) {
      // y = H D q / sqrt(d): the warp-level transform in warp 0
      if (warp == 0) {
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) v[e] = qs[lane + 32 * e] * a.signs[lane + 32 * e];
        fwht128_warp(v, lane);
#pragma unroll
        for (int e = 0; e < 4; ++e) ys[lane + 32 * e] = v[e] * kInvSqrtD;
      }
      __syncthreads();
      y = ys[i];
    } else {
      const float4* prow = reinterpret_cast<const float4*>(a.pi + (size_t)i * D);
      float acc = 0.f;
#pragma unroll 8
      for (int k = 0; k < D / 4; ++k) {
        const float4 m = prow[k];
        acc = fmaf(m.x, qs[4 * k], acc);
        acc = fmaf(m.y, qs[4 * k + 1], acc);
        acc = fmaf(m.z, qs[4 * k + 2], acc);
        acc = fmaf(m.w, qs[4 * k + 3], acc);
      }
      y = acc;
    }
    a.qrot[(size_t)row * D + i] = y;
    float my = warp_max(fabsf(y));
    if (lane == 0) red[warp] = my;
    __syncthreads();
    my = fmaxf(fmaxf(red[0], red[1]), fmaxf(red[2], red[3]));
    const float lam = my > 0.f ? 127.f / my : 0.f;
    a.q8[(size_t)row * D + i] = (int8_t)__float2int_rn(y * lam);
    if (i == 0) a.q8_scale[row] = lam;
  }
  if (a.qjl) {
    const float4 q4 = reinterpret_cast<const float4*>(qs)[lane];
    float t[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      float v = p[j].x * q4.x;
      v = fmaf(p[j].y, q4.y, v);
      v = fmaf(p[j].z, q4.z, v);
      t[j] = fmaf(p[j].w, q4.w, v);
    }
    // sum over the lanes: within each group of eight lanes a reduce-scatter (after the step
    // over lane bit h a lane keeps the half of its sums whose output index has that bit, plus
    // the partner's copy of that half), so lane l holds output l & 7 of its group; then the
    // four groups are added
#pragma unroll
    for (int h = 4; h >= 1; h >>= 1) {
#pragma unroll
      for (int j = 0; j < h; ++j) {
        const bool upper = lane & h;
        const float send = upper ? t[j] : t[j + h];
        const float keep = upper ? t[j + h] : t[j];
        t[j] = keep + __shfl_xor_sync(FULL, send, h);
      }
    }
    float v = t[0];
    v += __shfl_xor_sync(FULL, v, 8);
    v += __shfl_xor_sync(FULL, v, 16);
    if (lane < 8) a.sq[(size_t)row * QM + o0 + lane] = v;
  }
  __syncthreads();
  if (threadIdx.x == 0) asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(rw), "r"(1u) : "memory");
}

// The query terms for the tensor-core split kernel, kQueryParts thread blocks of 128 threads
// per query row.  Part c forms outputs 32 c .. 32 c + 31 of S q in fp32 (the split kernel
// takes them to fixed point), 8 per warp; part 0 also R q and its int8 copy with the scale,
// and zeroes the merge counter of a run that starts at this row.  Each part announces its
// terms through its own ready word.  Few registers: a block waiting for its predecessor stays
// resident beside two split-kernel blocks of the previous call.
__global__ void __launch_bounds__(128) query_kernel(DecodeArgs a) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  unpublish_part(a, blockIdx.x);
  asm volatile("griddepcontrol.launch_dependents;");
  query_part(a, blockIdx.x);
}

// Query rows (thread blocks 0 .. q_blocks - 1), then one thread block per appended token.
// With fast_query the query blocks are the tensor-core split kernel's kQueryParts parts per
// row (as query_kernel), otherwise one block per row with the general kernels' terms.
__global__ void __launch_bounds__(128) prologue_kernel(DecodeArgs a, int q_blocks) {
  asm volatile("griddepcontrol.wait;" ::: "memory");
  const int blk = blockIdx.x;
  if (blk < q_blocks) {
    if (a.fast_query) unpublish_part(a, blk);
    else unpublish_row(a, blk);
  }
  asm volatile("griddepcontrol.launch_dependents;");
  if (blk >= q_blocks) {
    // thread blocks past the query rows append the new tokens (none unless a.n_new > 0)
    if (a.n_new > 0 && blk - q_blocks < a.cache.batch * a.cache.kv_heads * a.n_new) append_token(a, blk - q_blocks);
    return;
  }
  if (a.fast_query) {
    query_part(a, blk);
    return;
  }
  query_row(a, blk);
  publish_row(a, blk);
}

// ---------------------------------------------------------------------------
// split kernel: grid (n_splits, kv_heads, batch), 128 threads
// ---------------------------------------------------------------------------
struct SmemSplit {
  float qrot[kRowsMax][D];
  float sq[kRowsMax][QM];
  float p[kRowsMax][kTile];
  uint32_t vcode[kTile][17];  // up to 16 words per token (+1 pad)
  float vnorm[kTile];
  float vxi[kTile];           // dithered values: the offset of each token
  uint32_t vsig[kTile][4];    // values with QJL: the residual's sign bits
  float vrho[kTile];          // and its stored norm
  float kmag[8], vmag[8];
  float sqsum[kRowsMax];
  float qsum[kRowsMax];  // dithered keys: sum_i (R q)_i, the weight of a key's offset
  float m[kRowsMax], l[kRowsMax], alpha[kRowsMax];
};

// Key formats of the split kernel's template: b-bit codes (1..4) or the merged 3-bit + QJL
// nibbles; RB: the smallest of 4, 8, 32 at least R (the per-row loops run to RB).
constexpr int kKeyMerged = 5;

template <bool kScoresOnly, int KF, int RB>
__global__ void __launch_bounds__(128) split_kernel(DecodeArgs a) {
  static_assert(QM == D, "the QJL sum shares the coordinate loop");
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SmemSplit& sm = *reinterpret_cast<SmemSplit*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
  const Layout& L = a.cache.L;
  const int R = a.rows;
  const size_t row0 = ((size_t)b * a.q_heads + (size_t)g * a.group) * a.seq_q;
  const int hk = 1 << (L.kbits - 1), hv = 1 << (L.vbits - 1);
  if (tid < hk) sm.kmag[tid] = a.k_centroids[hk + tid];
  if (tid < hv) sm.vmag[tid] = a.v_centroids[hv + tid];
  for (int i = tid; i < R * D; i += blockDim.x) sm.qrot[i / D][i % D] = a.qrot[row0 * D + i];
  if (L.qjl)
    for (int i = tid; i < R * QM; i += blockDim.x) sm.sq[i / QM][i % QM] = a.sq[row0 * QM + i];
  if (tid < R) {
    sm.m[tid] = -CUDART_INF_F;
    sm.l[tid] = 0.f;
  }
  __syncthreads();
  if (L.qjl && tid < R) {
    float t = 0.f;
    for (int i = 0; i < QM; ++i) t += sm.sq[tid][i];
    sm.sqsum[tid] = t;
  }
  if (L.dither && tid < R) {
    // <R q, c[idx] + xi 1> = <R q, c[idx]> + xi sum_i (R q)_i
    float t = 0.f;
    for (int i = 0; i < D; ++i) t += sm.qrot[tid][i];
    sm.qsum[tid] = t;
  }
  const int len = a.seq_lens[b];
  const bool bad_len = len < 0 || len > a.cache.max_pages * PT || (kScoresOnly && len > a.max_len);
  if (bad_len && tid == 0 && split == 0) report(a.status, TQ_ERR_BOUNDS);
  const int n_eff = bad_len ? 0 : len;
  const int npages = (n_eff + PT - 1) / PT;
  const int cp = (npages + a.n_splits - 1) / a.n_splits;
  TQ_DCHECK(a.status, R >= 1 && R <= kRowsMax && split < a.n_splits);
  const int t_begin = min(n_eff, split * cp * PT);
  const int t_end = min(n_eff, (split + 1) * cp * PT);
  float acc[RB];
#pragma unroll
  for (int r = 0; r < RB; ++r) acc[r] = 0.f;
  // values with QJL: thread i also sums p_t ||r_v||_t (2 sigma_t,i - 1) over the tokens, the
  // sign-space half of the value reconstruction (S^T is applied once, after the merge)
  float accs[RB];
#pragma unroll
  for (int r = 0; r < RB; ++r) accs[r] = 0.f;
  __syncthreads();

  for (int tile0 = t_begin; tile0 < t_end; tile0 += kTile) {
    // ---- phase A: thread = token, scores for all rows
    const int t = tile0 + tid;
    float vn = 0.f;
    bool valid = t < t_end;
    uint8_t* blk = nullptr;
    int slot = 0;
    if (valid) {
      const int phys = a.cache.block_table[(size_t)b * a.cache.max_pages + t / PT];
      if (phys < 0 || phys >= a.cache.num_pages) {
        report(a.status, TQ_ERR_BOUNDS);
        valid = false;
      } else {
        blk = a.cache.block(phys, g);
        slot = t % PT;
      }
    }
    if (valid) {
      // the token's key, 32 coordinates at a time: the words holding coordinates
      // 32q..32q+31 sit in registers and every field below has a constant position
      float dot[RB], qj[RB];
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        dot[r] = 0.f;
        qj[r] = 0.f;
      }
      const uint8_t* kcb = blk + L.kc + (size_t)slot * 16;
      const bool qjl = L.qjl != 0;
#pragma unroll 1
      for (int q = 0; q < 4; ++q) {
        uint32_t g[4] = {0u, 0u, 0u, 0u}, sp = 0u, sgw = 0u;
        if constexpr (KF == 1) {
          g[0] = *reinterpret_cast<const uint32_t*>(kcb + 4 * q);
        } else if constexpr (KF == 2 || KF == 3) {
          const uint2 v2 = *reinterpret_cast<const uint2*>(kcb + (q >> 1) * PT * 16 + (q & 1) * 8);
          g[0] = v2.x;
          g[1] = v2.y;
          if constexpr (KF == 3) sp = *reinterpret_cast<const uint32_t*>(kcb + 2 * PT * 16 + 4 * q);
        } else {
          const uint4 v4 = *reinterpret_cast<const uint4*>(kcb + q * PT * 16);
          g[0] = v4.x; g[1] = v4.y; g[2] = v4.z; g[3] = v4.w;
        }
        if (KF != kKeyMerged && qjl) sgw = *reinterpret_cast<const uint32_t*>(blk + L.ks + (size_t)slot * 16 + 4 * q);
#pragma unroll
        for (int jj = 0; jj < 32; ++jj) {
          int s, rk, sig;
          if constexpr (KF == 1) {
            s = (g[0] >> jj) & 1;
            rk = 0;
          } else if constexpr (KF == 2) {
            const uint32_t f = (g[jj >> 4] >> ((jj & 15) * 2)) & 3u;
            rk = f & 1;
            s = f >> 1;
          } else if constexpr (KF == 3) {
            rk = (g[jj >> 4] >> ((jj & 15) * 2)) & 3u;
            s = (sp >> (sign_plane_pos(jj) & 31)) & 1;
          } else if constexpr (KF == 4) {
            const uint32_t f = (g[jj >> 3] >> ((jj & 7) * 4)) & 15u;
            rk = f & 7;
            s = f >> 3;
          } else {
            const uint32_t f = (g[jj >> 3] >> ((jj & 7) * 4)) & 15u;
            rk = f & 3;
            s = (f >> 2) & 1;
          }
          if constexpr (KF == kKeyMerged)
            sig = (g[jj >> 3] >> ((jj & 7) * 4 + 3)) & 1;
          else
            sig = (sgw >> jj) & 1;
          const int j = 32 * q + jj;
          const float val = s ? sm.kmag[rk] : -sm.kmag[rk];
#pragma unroll
          for (int r = 0; r < RB; ++r)
            if (r < R) dot[r] = fmaf(sm.qrot[r][j], val, dot[r]);
          if (qjl && sig) {
#pragma unroll
            for (int r = 0; r < RB; ++r)
              if (r < R) qj[r] += sm.sq[r][j];
          }
        }
      }
      const float kn = __half2float(reinterpret_cast<const __half*>(blk + L.kn)[slot]);
      const float rho = qjl ? __half2float(reinterpret_cast<const __half*>(blk + L.kr)[slot]) : 0.f;
      const float kxi = L.dither ? __half2float(reinterpret_cast<const __half*>(blk + L.kd)[slot]) : 0.f;
#pragma unroll
      for (int r = 0; r < RB; ++r) {
        if (r < R) {
          float sc = kn * (L.dither ? fmaf(kxi, sm.qsum[r], dot[r]) : dot[r]);
          if (L.qjl) sc = fmaf(rho * kQjlScale, 2.f * qj[r] - sm.sqsum[r], sc);
          sc *= kInvSqrtD;
          if (kScoresOnly)
            a.scores[(row0 + r) * (size_t)a.max_len + t] = sc;
          else
            sm.p[r][tid] = sc;
        }
      }
      if (!kScoresOnly) {
        for (int c = 0; c < L.vbits; ++c) {
          const uint4 v4 = reinterpret_cast<const uint4*>(blk + L.vc)[c * PT + slot];
          sm.vcode[tid][4 * c] = v4.x; sm.vcode[tid][4 * c + 1] = v4.y;
          sm.vcode[tid][4 * c + 2] = v4.z; sm.vcode[tid][4 * c + 3] = v4.w;
        }
        vn = __half2float(reinterpret_cast<const __half*>(blk + L.vn)[slot]);
        if (L.dither) sm.vxi[tid] = __half2float(reinterpret_cast<const __half*>(blk + L.vd)[slot]);
        if (L.vqjl) {
          const uint4 s4 = reinterpret_cast<const uint4*>(blk + L.vs)[slot];
          sm.vsig[tid][0] = s4.x; sm.vsig[tid][1] = s4.y; sm.vsig[tid][2] = s4.z; sm.vsig[tid][3] = s4.w;
          sm.vrho[tid] = __half2float(reinterpret_cast<const __half*>(blk + L.vr)[slot]);
        }
      }
    } else if (!kScoresOnly) {
      for (int r = 0; r < R; ++r) sm.p[r][tid] = -CUDART_INF_F;
    }
    if (kScoresOnly) continue;
    sm.vnorm[tid] = valid ? vn : 0.f;
    if (L.dither && !valid) sm.vxi[tid] = 0.f;
    if (L.vqjl && !valid) sm.vrho[tid] = 0.f;
    __syncthreads();
    // ---- phase B: online softmax bookkeeping, warp per row
    for (int r = warp; r < R; r += 4) {
      float v[4], mx = -CUDART_INF_F;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[e] = sm.p[r][lane + 32 * e];
        mx = fmaxf(mx, v[e]);
      }
      mx = warp_max(mx);
      const float m_old = sm.m[r];
      const float m_new = fmaxf(m_old, mx);
      float ps = 0.f;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float p = (m_new == -CUDART_INF_F) ? 0.f : __expf(v[e] - m_new);
        sm.p[r][lane + 32 * e] = p;
        ps += p;
      }
      ps = warp_sum(ps);
      if (lane == 0) {
        const float al = (m_new == -CUDART_INF_F) ? 1.f : __expf(m_old - m_new);
        sm.alpha[r] = al;
        sm.l[r] = sm.l[r] * al + ps;
        sm.m[r] = m_new;
      }
    }
    __syncthreads();
    // ---- phase C: thread = coordinate j, V accumulation in rotated space
    const int j = tid;
#pragma unroll
    for (int r = 0; r < RB; ++r)
      if (r < R) acc[r] *= sm.alpha[r];
    const int nt = min(kTile, t_end - tile0);
    for (int tt = 0; tt < nt; ++tt) {
      int s, rk;
      code_fields(sm.vcode[tt], L.vbits, j, s, rk);
      float c = s ? sm.vmag[rk] : -sm.vmag[rk];
      if (L.dither) c += sm.vxi[tt];
      const float val = c * sm.vnorm[tt];
#pragma unroll
      for (int r = 0; r < RB; ++r)
        if (r < R) acc[r] = fmaf(sm.p[r][tt], val, acc[r]);
    }
    if (L.vqjl) {
      // thread j holds sign index i = j (m = d = blockDim)
#pragma unroll
      for (int r = 0; r < RB; ++r)
        if (r < R) accs[r] *= sm.alpha[r];
      for (int tt = 0; tt < nt; ++tt) {
        const float sv = ((sm.vsig[tt][j >> 5] >> (j & 31)) & 1u) ? sm.vrho[tt] : -sm.vrho[tt];
#pragma unroll
        for (int r = 0; r < RB; ++r)
          if (r < R) accs[r] = fmaf(sm.p[r][tt], sv, accs[r]);
      }
    }
    __syncthreads();
  }
  // ---- partials (the score-only variant stops with the scores)
  if constexpr (!kScoresOnly) {
#pragma unroll
    for (int r = 0; r < RB; ++r) {
      if (r < R) {
        const size_t pr = (row0 + r) * a.n_splits + split;
        a.part_acc[pr * D + tid] = acc[r];
        if (L.vqjl) a.part_sig[pr * QM + tid] = accs[r];
        if (tid == 0) {
          a.part_ml[pr * 2] = sm.m[r];
          a.part_ml[pr * 2 + 1] = sm.l[r];
        }
      }
    }
  }
}

// ---------------------------------------------------------------------------
// combine: one CTA of 128 threads per query row, thread j owns coordinate j
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128) combine_kernel(DecodeArgs a, int total_rows) {
  // wait for the split kernel (launched as our programmatic predecessor) to finish
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float os[D], ss[QM];
  const int j = threadIdx.x;
  const int row = blockIdx.x;
  if (row >= total_rows) return;
  const bool vqjl = a.cache.L.vqjl != 0;
  TQ_DCHECK(a.status, row < a.cache.batch * a.q_heads * a.seq_q);
  const float* ml = a.part_ml + (size_t)row * a.n_splits * 2;
  const float* pa = a.part_acc + (size_t)row * a.n_splits * D;
  const float* ps = vqjl ? a.part_sig + (size_t)row * a.n_splits * QM : nullptr;
  float M = -CUDART_INF_F;
  for (int s = 0; s < a.n_splits; ++s) M = fmaxf(M, ml[2 * s]);
  float l = 0.f, o = 0.f, osig = 0.f;
  if (M != -CUDART_INF_F) {
    for (int s = 0; s < a.n_splits; ++s) {
      const float ms = ml[2 * s];
      if (ms == -CUDART_INF_F) continue;
      const float wgt = __expf(ms - M);
      l = fmaf(wgt, ml[2 * s + 1], l);
      o = fmaf(wgt, pa[(size_t)s * D + j], o);
      if (vqjl) osig = fmaf(wgt, ps[(size_t)s * QM + j], osig);
    }
  }
  o = l > 0.f ? o / l : 0.f;
  osig = l > 0.f ? osig / l : 0.f;
  float y;
  if (!a.dense) {
    // R^T = D H: butterflies in shared memory, then the sign flips
    os[j] = o;
    __syncthreads();
#pragma unroll
    for (int h = 1; h < D; h <<= 1) {
      const float u = os[j], v = os[j ^ h];
      __syncthreads();
      os[j] = (j & h) ? (v - u) : (u + v);
      __syncthreads();
    }
    y = os[j] * kInvSqrtD * a.signs[j];
  } else {
    os[j] = o;
    __syncthreads();
    float acc = 0.f;
    for (int i = 0; i < D; ++i) acc = fmaf(a.pi[(size_t)i * D + j], os[i], acc);
    y = acc;
  }
  if (vqjl) {
    // values with QJL: + sqrt(pi/2)/m S^T (sum_t p_t ||r_v||_t (2 sigma_t - 1)) / l
    ss[j] = osig;
    __syncthreads();
    float acc = 0.f;
    for (int i = 0; i < QM; ++i) acc = fmaf(a.s[(size_t)i * D + j], ss[i], acc);
    y = fmaf(kQjlScale, acc, y);
  }
  a.out[(size_t)row * D + j] = y;
}

}  // namespace

DecodeWorkspace decode_workspace(int batch, int q_heads, int seq_q, int n_splits, int vqjl) {
  const size_t rows = (size_t)batch * q_heads * seq_q;
  DecodeWorkspace w;
  size_t off = 0;
  w.qrot = off; off = align256(off + rows * D * sizeof(float));
  w.sq = off; off = align256(off + rows * QM * sizeof(float));
  w.part_acc = off; off = align256(off + rows * (size_t)n_splits * D * sizeof(float));
  w.part_ml = off; off = align256(off + rows * (size_t)n_splits * 2 * sizeof(float));
  w.part_sig = off; off = align256(off + (vqjl ? rows * (size_t)n_splits * QM * sizeof(float) : 0));
  w.sq_int = off; off = align256(off + rows * QM * sizeof(int16_t));
  w.sq_scale = off; off = align256(off + rows * sizeof(float));
  w.sq_sum = off; off = align256(off + rows * sizeof(int));
  w.q8 = off; off = align256(off + rows * D);
  w.q8_scale = off; off = align256(off + rows * sizeof(float));
  // one counter per (sequence, kv head, run of up to four query rows): at most one per query row
  w.counter = off; off = align256(off + rows * sizeof(unsigned int));
  // kQueryParts ready words per query row
  w.ready = off; off = align256(off + rows * kQueryParts * sizeof(unsigned int));
  w.total = off;
  return w;
}

template <bool kScoresOnly, int KF>
static void (*split_for_rows(int rows))(DecodeArgs) {
  if (rows <= 4) return split_kernel<kScoresOnly, KF, 4>;
  if (rows <= 8) return split_kernel<kScoresOnly, KF, 8>;
  return split_kernel<kScoresOnly, KF, kRowsMax>;
}

template <bool kScoresOnly>
static void (*split_for(const Layout& L, int rows))(DecodeArgs) {
  if (L.kmerged) return split_for_rows<kScoresOnly, kKeyMerged>(rows);
  switch (L.kbits) {
    case 1: return split_for_rows<kScoresOnly, 1>(rows);
    case 2: return split_for_rows<kScoresOnly, 2>(rows);
    case 3: return split_for_rows<kScoresOnly, 3>(rows);
    default: return split_for_rows<kScoresOnly, 4>(rows);
  }
}

static cudaError_t launch_split(const DecodeArgs& a, cudaStream_t stream, bool scores_only) {
  const size_t smem = sizeof(SmemSplit);
  dim3 grid(scores_only ? 1 : a.n_splits, a.cache.kv_heads, a.cache.batch);
  void (*k)(DecodeArgs) = scores_only ? split_for<true>(a.cache.L, a.rows) : split_for<false>(a.cache.L, a.rows);
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  k<<<grid, 128, smem, stream>>>(a);
  return cudaGetLastError();
}

// Launch with programmatic stream serialization: the kernel may start while its
// predecessor on the stream is still running and waits (griddepcontrol.wait) before it
// reads the predecessor's results.
template <typename... Args>
static cudaError_t launch_pdl(void (*k)(Args...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                              Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, args...);
}

cudaError_t launch_decode(const DecodeArgs& a, cudaStream_t stream) {
  const int total_rows = a.cache.batch * a.q_heads * a.seq_q;
  // the prologue's grid: one thread block per query row, then one per appended token
  const int blocks = total_rows + (a.n_new > 0 ? a.cache.batch * a.cache.kv_heads * a.n_new : 0);
  if (fast_decode_supported(a)) {
    // query transforms (and zeroed merge counters), then the split kernel, whose last
    // split per (sequence, kv head) merges the partials: two launches
    DecodeArgs f = a;
    f.fast_query = 1;
    const int qb = total_rows * kQueryParts;
    cudaError_t e = a.n_new > 0 ? launch_pdl(prologue_kernel, dim3(qb + blocks - total_rows), dim3(128), 0, stream, f, qb)
                                : launch_pdl(query_kernel, dim3(qb), dim3(128), 0, stream, f);
    if (e != cudaSuccess) return e;
    return launch_fast_split(f, stream);
  }
  // the split kernel is an ordinary launch: it starts once the prologue (and any append)
  // has finished
  cudaError_t e = launch_pdl(prologue_kernel, dim3(blocks), dim3(128), 0, stream, a, total_rows);
  if (e != cudaSuccess) return e;
  e = launch_split(a, stream, false);
  if (e != cudaSuccess) return e;
  e = launch_pdl(combine_kernel, dim3(total_rows), dim3(128), 0, stream, a, total_rows);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

cudaError_t launch_append(const DecodeArgs& a, cudaStream_t stream) {
  const int blocks = a.cache.batch * a.cache.kv_heads * a.n_new;
  if (blocks == 0) return cudaSuccess;
  return launch_pdl(prologue_kernel, dim3(blocks), dim3(128), 0, stream, a, 0);
}

cudaError_t launch_decode_scores(const DecodeArgs& a, cudaStream_t stream) {
  const int total_rows = a.cache.batch * a.q_heads * a.seq_q;
  cudaError_t e = launch_pdl(prologue_kernel, dim3(total_rows), dim3(128), 0, stream, a, total_rows);
  if (e != cudaSuccess) return e;
  return launch_split(a, stream, true);
}

}  // namespace tqk
