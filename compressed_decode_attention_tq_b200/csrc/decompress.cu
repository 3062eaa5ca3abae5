// Decompression of the packed cache to dense fp32 K_hat / V_hat.
//
// "turboquant_cutile" function list: "indices -> centroids -> un-rotate -> rescale"
// (4-level and 8-level decompress kernels); dithered codes add their stored offset to the
// centroids before un-rotating.  For keys with QJL this returns the MSE
// part k_mse = ||k|| R^T c[idx] ("k_mse should be a reasonable approximation of K").
// One warp per (token, kv head), lane l holds coordinates l + 32 e.
#include <cuda_fp16.h>

#include "tq_device.cuh"
#include "tq_kernels.h"

namespace tqk {

namespace {

constexpr float kInvSqrtD = 0.08838834764831845f;

__device__ void decode_vector(const uint8_t* blk, int code_off, int norm_off, int off_off, int bits,
                              int merged, int slot, const float* cent, const float* signs,
                              const float* pi, float* stage, int lane, float* dst) {
  uint32_t w[16];
  const int chunks = merged ? 4 : bits;
  for (int c = 0; c < chunks; ++c) {
    const uint4 v4 = reinterpret_cast<const uint4*>(blk + code_off)[c * PT + slot];
    w[4 * c] = v4.x; w[4 * c + 1] = v4.y; w[4 * c + 2] = v4.z; w[4 * c + 3] = v4.w;
  }
  const int h = 1 << (bits - 1);
  float z[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    int s, r;
    if (merged) {
      const int j = lane + 32 * e;
      const uint32_t f = (w[j >> 3] >> ((j & 7) * 4)) & 15u;
      r = f & 3;
      s = (f >> 2) & 1;
    } else {
      code_fields(w, bits, lane + 32 * e, s, r);
    }
    z[e] = s ? cent[h + r] : -cent[h + r];
  }
  if (off_off >= 0) {
    // dithered: c[idx] + xi
    const float xi = __half2float(reinterpret_cast<const __half*>(blk + off_off)[slot]);
#pragma unroll
    for (int e = 0; e < 4; ++e) z[e] += xi;
  }
  const float n = __half2float(reinterpret_cast<const __half*>(blk + norm_off)[slot]);
  if (pi == nullptr) {
    fwht128_warp(z, lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) dst[lane + 32 * e] = n * (z[e] * kInvSqrtD * signs[lane + 32 * e]);
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) stage[lane + 32 * e] = z[e];
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float acc = 0.f;
      for (int i = 0; i < D; ++i) acc = fmaf(pi[(size_t)i * D + lane + 32 * e], stage[i], acc);
      dst[lane + 32 * e] = n * acc;
    }
    __syncwarp();
  }
}

__global__ void decompress_kernel(DecompressArgs a) {
  __shared__ float stage[4][D];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int t = blockIdx.x * 4 + w;
  const int h = blockIdx.y, b = blockIdx.z;
  const int len = a.seq_lens[b];
  if (len < 0 || len > a.max_len || len > a.cache.max_pages * PT) {
    if (lane == 0 && blockIdx.x == 0 && w == 0) report(a.status, TQ_ERR_BOUNDS);
    return;
  }
  if (t >= len) return;
  const int phys = a.cache.block_table[(size_t)b * a.cache.max_pages + t / PT];
  if (phys < 0 || phys >= a.cache.num_pages) {
    if (lane == 0) report(a.status, TQ_ERR_BOUNDS);
    return;
  }
  const uint8_t* blk = a.cache.block(phys, h);
  const int slot = t % PT;
  TQ_DCHECK(a.status, t < a.max_len && t / PT < a.cache.max_pages && slot < PT);
  const size_t row = (((size_t)b * a.cache.kv_heads + h) * a.max_len + t) * D;
  const Layout& L = a.cache.L;
  const float* pi = a.dense ? a.pi : nullptr;
  if (a.k_hat)
    decode_vector(blk, L.kc, L.kn, L.dither ? L.kd : -1, L.kbits, L.kmerged, slot, a.k_centroids, a.signs, pi,
                  stage[w], lane, a.k_hat + row);
  if (a.v_hat)
    decode_vector(blk, L.vc, L.vn, L.dither ? L.vd : -1, L.vbits, 0, slot, a.v_centroids, a.signs, pi,
                  stage[w], lane, a.v_hat + row);
}

}  // namespace

cudaError_t launch_decompress(const DecompressArgs& a, cudaStream_t stream) {
  dim3 grid((a.max_len + 3) / 4, a.cache.kv_heads, a.cache.batch);
  if (grid.x == 0) return cudaSuccess;
  decompress_kernel<<<grid, 128, 0, stream>>>(a);
  return cudaGetLastError();
}

}  // namespace tqk
