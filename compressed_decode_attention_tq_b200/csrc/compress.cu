// Compression of K and V into the packed paged cache.
//
// "turboquant_cutile" function list: compress K -> MSE indices + 1-bit QJL
// (2-bit + 1, 3-bit + 1), compress V -> MSE only.
// "TurboQuant explained" (Mobilint blog):
//   section "Coordinates Become Predictable After Rotation": quantize the unit vector
//     x/||x|| after a random rotation;
//   section "How JL Matrices Evolved": the rotation H D (signs, then Walsh-Hadamard
//     butterflies, O(d log d)); the dense option Pi;
//   section "Two-Stage Approach: MSE Approximation + QJL Correction":
//     x_mse = DeQuant(Quant(x)), r = x - x_mse, store sign(S r) and ||r||.
//
// One warp per token: lane l holds coordinates j = l + 32 e, e = 0..3.
#include <cuda_fp16.h>

#include "tq_device.cuh"
#include "tq_kernels.h"

namespace tqk {

namespace {

constexpr int kWarps = 8;
constexpr int kTokPerBlockMax = 64;  // tokens per thread block (fewer when the grid would not fill the GPU)
constexpr int kPad = D + 1;  // padded row stride of S / Pi in shared memory (bank-conflict free)

struct SmemCompress {
  float kc[16], kb[16], vc[16], vb[16], signs[D];
  float stage[kWarps][D];
  uint32_t words[kWarps][16];
};

// Stored code bit string of one token for `bits`, from this lane's (s, r) of its four
// coordinates; the words land in `wout` (16 words max).
__device__ __forceinline__ void pack_words(const int (&s)[4], const int (&r)[4], int bits, int lane,
                                           uint32_t* wout) {
  const bool lo16 = lane < 16;
  switch (bits) {
    case 1:
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t w = __ballot_sync(FULL, s[e]);
        if (lane == 0) wout[e] = w;
      }
      break;
    case 2:
    case 3:
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t f = bits == 2 ? (uint32_t)(r[e] | (s[e] << 1)) : (uint32_t)r[e];
        const uint32_t sh = f << (2 * (lane & 15));
        const uint32_t lo = __reduce_or_sync(FULL, lo16 ? sh : 0u);
        const uint32_t hi = __reduce_or_sync(FULL, lo16 ? 0u : sh);
        if (lane == 0) {
          wout[2 * e] = lo;
          wout[2 * e + 1] = hi;
        }
        if (bits == 3) {
          const uint32_t w = __reduce_or_sync(FULL, (uint32_t)s[e] << (sign_plane_pos(lane) & 31));
          if (lane == 0) wout[8 + e] = w;
        }
      }
      break;
    default:
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t f = (uint32_t)(r[e] | (s[e] << 3));
        const uint32_t sh = f << (4 * (lane & 7));
        const int g = lane >> 3;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint32_t w = __reduce_or_sync(FULL, g == q ? sh : 0u);
          if (lane == 0) wout[4 * e + q] = w;
        }
      }
      break;
  }
}

// Merged 3-bit key fields (r0, r1, s, sigma) as 4-bit nibbles, nibble j at bit 4j.
__device__ __forceinline__ void pack_merged(const int (&s)[4], const int (&r)[4], const int (&sg)[4],
                                            int lane, uint32_t* wout) {
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const uint32_t f = (uint32_t)(r[e] | (s[e] << 2) | (sg[e] << 3));
    const uint32_t sh = f << (4 * (lane & 7));
    const int g = lane >> 3;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t w = __reduce_or_sync(FULL, g == q ? sh : 0u);
      if (lane == 0) wout[4 * e + q] = w;
    }
  }
}

struct VecOut {
  __half norm;
  int idx[4];
  int s[4], r[4];
};

// norm, rotation, quantization, packing of one vector (x already loaded).  xi: the
// vector's dither offset (0 when not dithered): idx = Quant(y - xi).  corr: store the
// corrected norm n / ||c[idx] + xi|| ("tq-kv" documentation: corrected_norm) instead of n.
__device__ __forceinline__ void encode_vector(const float (&x)[4], int bits, const float* cent,
                                              const float* bnd, const float* signs, const float* pi_s,
                                              float* stage, int lane, uint32_t* wbuf, VecOut& out,
                                              int32_t* status, bool defer_pack = false, float xi = 0.f,
                                              bool corr = false) {
  float ss = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) ss = fmaf(x[e], x[e], ss);
  ss = warp_sum(ss);
  const float n = sqrtf(ss);
  const float inv = n > 0.f ? 1.0f / n : 0.0f;
  float y[4];
  if (pi_s == nullptr) {
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] = x[e] * signs[lane + 32 * e];
    fwht128_warp(y, lane);
    const float sc = inv * 0.08838834764831845f;  // 1/sqrt(128)
#pragma unroll
    for (int e = 0; e < 4; ++e) y[e] *= sc;
  } else {
#pragma unroll
    for (int e = 0; e < 4; ++e) stage[lane + 32 * e] = x[e] * inv;
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float* row = pi_s + (lane + 32 * e) * kPad;
      float acc = 0.f;
      for (int k = 0; k < D; ++k) acc = fmaf(row[k], stage[k], acc);
      y[e] = acc;
    }
    __syncwarp();
  }
  const int nb = (1 << bits) - 1;
  const int h = 1 << (bits - 1);
  int s[4], r[4];
  float yy = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float yq = y[e] - xi;
    int idx = 0;
    for (int i = 0; i < nb; ++i) idx += (yq > bnd[i]) ? 1 : 0;
    out.idx[e] = idx;
    s[e] = idx >= h;
    r[e] = s[e] ? idx - h : h - 1 - idx;
    out.s[e] = s[e];
    out.r[e] = r[e];
    const float yh = cent[idx] + xi;
    yy = fmaf(yh, yh, yy);
  }
  float stored = n;
  if (corr) {
    const float yn = sqrtf(warp_sum(yy));
    stored = yn > 0.f ? n / yn : 0.f;
  }
  out.norm = __float2half_rn(stored);
  if (__hisinf(out.norm) && lane == 0) report(status, TQ_ERR_OVERFLOW);
  if (!defer_pack) pack_words(s, r, bits, lane, wbuf);
}

// QJL sketch of the residual in the original space, r = x - fp16(n) R^T (c[idx] + xi)
// ("TurboQuant explained", section "Two-Stage Approach"): returns fp16(||r||) and the signs
// sg[e] = [(S r)_j >= 0] of the lane's rows j = lane + 32 e (sign(0) stored as +1).
__device__ __forceinline__ __half qjl_residual_signs(const float (&x)[4], const int (&idx)[4], __half norm,
                                                     const float* cent, const float* signs,
                                                     const float* pi_s, const float* s_s, float* stage,
                                                     int lane, int (&sg)[4], float xi = 0.f) {
  float z[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) z[e] = cent[idx[e]] + xi;
  if (pi_s == nullptr) {
    fwht128_warp(z, lane);
#pragma unroll
    for (int e = 0; e < 4; ++e) z[e] *= 0.08838834764831845f * signs[lane + 32 * e];
  } else {
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 4; ++e) stage[lane + 32 * e] = z[e];
    __syncwarp();
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float acc = 0.f;
      for (int i = 0; i < D; ++i) acc = fmaf(pi_s[i * kPad + lane + 32 * e], stage[i], acc);
      z[e] = acc;
    }
  }
  const float nh = __half2float(norm);
  float rr[4], r2 = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    rr[e] = x[e] - nh * z[e];
    r2 = fmaf(rr[e], rr[e], r2);
  }
  r2 = warp_sum(r2);
  const __half rho = __float2half_rn(sqrtf(r2));
  __syncwarp();
#pragma unroll
  for (int e = 0; e < 4; ++e) stage[lane + 32 * e] = rr[e];
  __syncwarp();
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float* srow = s_s + (lane + 32 * e) * kPad;
    float acc = 0.f;
    for (int k = 0; k < D; ++k) acc = fmaf(srow[k], stage[k], acc);
    sg[e] = acc >= 0.f;
  }
  __syncwarp();
  return rho;
}

template <typename T>
__device__ __forceinline__ float ld_in(const T* p) { return (float)p[0]; }
template <>
__device__ __forceinline__ float ld_in<__half>(const __half* p) { return __half2float(p[0]); }

template <typename T>
__global__ void __launch_bounds__(kWarps * 32) compress_kernel(CompressArgs a) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SmemCompress& sm = *reinterpret_cast<SmemCompress*>(smem_raw);
  float* s_s = reinterpret_cast<float*>(smem_raw + sizeof(SmemCompress));  // [QM][kPad] if qjl
  const bool sketch = a.qjl || a.cache.L.vqjl;                               // S is used
  float* pi_s = s_s + (sketch ? QM * kPad : 0);                              // [D][kPad] if dense
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int b = blockIdx.z, h = blockIdx.y;
  const Layout& L = a.cache.L;
  const int nk = 1 << L.kbits, nv = 1 << L.vbits;
  if (tid < nk) sm.kc[tid] = a.k_centroids[tid];
  if (tid < nk - 1) sm.kb[tid] = a.k_boundaries[tid];
  if (tid < nv) sm.vc[tid] = a.v_centroids[tid];
  if (tid < nv - 1) sm.vb[tid] = a.v_boundaries[tid];
  if (!a.dense)
    for (int i = tid; i < D; i += blockDim.x) sm.signs[i] = a.signs[i];
  if (sketch) {
    for (int i = tid; i < QM * D; i += blockDim.x) {
      const float v = a.s[i];
      if (__half2float(__float2half_rn(v)) != v) report(a.status, TQ_ERR_INVALID_ARG);
      s_s[(i / D) * kPad + (i % D)] = v;
    }
  }
  if (a.dense)
    for (int i = tid; i < D * D; i += blockDim.x) pi_s[(i / D) * kPad + (i % D)] = a.pi[i];
  __syncthreads();
  if (tid == 0 && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0) {
    for (int i = 0; i < nk; ++i)
      if (sm.kc[i] != -sm.kc[nk - 1 - i]) report(a.status, TQ_ERR_INVALID_ARG);
    for (int i = 0; i < nv; ++i)
      if (sm.vc[i] != -sm.vc[nv - 1 - i]) report(a.status, TQ_ERR_INVALID_ARG);
  }
  const int len = a.seq_lens[b];
  if (len < 0 || len > a.max_len || len > a.cache.max_pages * PT) {
    if (tid == 0 && blockIdx.x == 0) report(a.status, TQ_ERR_BOUNDS);
    return;
  }
  const size_t head_off = ((size_t)b * a.cache.kv_heads + h) * (size_t)a.max_len;
  const T* kin = reinterpret_cast<const T*>(a.k);
  const T* vin = reinterpret_cast<const T*>(a.v);
  float* stage = sm.stage[warp];
  uint32_t* wbuf = sm.words[warp];
  const float* pis = a.dense ? pi_s : nullptr;
  for (int tt = warp; tt < a.tok_per_block; tt += kWarps) {
    const int t = blockIdx.x * a.tok_per_block + tt;
    if (t >= len) break;
    const int phys = a.cache.block_table[(size_t)b * a.cache.max_pages + t / PT];
    if (phys < 0 || phys >= a.cache.num_pages) {
      if (lane == 0) report(a.status, TQ_ERR_BOUNDS);
      continue;
    }
    uint8_t* blk = a.cache.block(phys, h);
    const int slot = t % PT;
    const size_t row = (head_off + t) * D;
    TQ_DCHECK(a.status, t < a.max_len && t / PT < a.cache.max_pages);
    // dithered: the vectors' offsets, used and stored as fp16
    __half kxi = __float2half_rn(0.f), vxi = kxi;
    if (L.dither) {
      kxi = __float2half_rn(a.k_off[head_off + t]);
      vxi = __float2half_rn(a.v_off[head_off + t]);
      if (lane == 0) {
        reinterpret_cast<__half*>(blk + L.kd)[slot] = kxi;
        reinterpret_cast<__half*>(blk + L.vd)[slot] = vxi;
      }
    }
    // ---- key
    float x[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = ld_in<T>(kin + row + lane + 32 * e);
    VecOut ko;
    encode_vector(x, L.kbits, sm.kc, sm.kb, sm.signs, pis, stage, lane, wbuf, ko, a.status,
                  L.kmerged != 0, __half2float(kxi), a.key_corr != 0);
    __syncwarp();
    if (!L.kmerged && lane < L.kbits)
      reinterpret_cast<uint4*>(blk + L.kc)[lane * PT + slot] = reinterpret_cast<const uint4*>(wbuf)[lane];
    if (lane == 0) reinterpret_cast<__half*>(blk + L.kn)[slot] = ko.norm;
    if (a.qjl) {
      int sg[4];
      const __half rho =
          qjl_residual_signs(x, ko.idx, ko.norm, sm.kc, sm.signs, pis, s_s, stage, lane, sg, __half2float(kxi));
      if (L.kmerged) {
        pack_merged(ko.s, ko.r, sg, lane, wbuf);
        __syncwarp();
        if (lane < 4)
          reinterpret_cast<uint4*>(blk + L.kc)[lane * PT + slot] = reinterpret_cast<const uint4*>(wbuf)[lane];
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t w = __ballot_sync(FULL, sg[e]);
          if (lane == 0) wbuf[e] = w;
        }
        __syncwarp();
        if (lane == 0) reinterpret_cast<uint4*>(blk + L.ks)[slot] = reinterpret_cast<const uint4*>(wbuf)[0];
      }
      if (lane == 0) reinterpret_cast<__half*>(blk + L.kr)[slot] = rho;
      __syncwarp();
    }
    // ---- value
#pragma unroll
    for (int e = 0; e < 4; ++e) x[e] = ld_in<T>(vin + row + lane + 32 * e);
    VecOut vo;
    __syncwarp();
    encode_vector(x, L.vbits, sm.vc, sm.vb, sm.signs, pis, stage, lane, wbuf, vo, a.status, false,
                  __half2float(vxi));
    __syncwarp();
    if (lane < L.vbits)
      reinterpret_cast<uint4*>(blk + L.vc)[lane * PT + slot] = reinterpret_cast<const uint4*>(wbuf)[lane];
    if (lane == 0) reinterpret_cast<__half*>(blk + L.vn)[slot] = vo.norm;
    __syncwarp();
    if (L.vqjl) {
      // values with QJL: the same sketch of the value residual, signs in VS, norm in VR
      int sg[4];
      const __half rho =
          qjl_residual_signs(x, vo.idx, vo.norm, sm.vc, sm.signs, pis, s_s, stage, lane, sg, __half2float(vxi));
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t w = __ballot_sync(FULL, sg[e]);
        if (lane == 0) wbuf[e] = w;
      }
      __syncwarp();
      if (lane == 0) {
        reinterpret_cast<uint4*>(blk + L.vs)[slot] = reinterpret_cast<const uint4*>(wbuf)[0];
        reinterpret_cast<__half*>(blk + L.vr)[slot] = rho;
      }
      __syncwarp();
    }
  }
}

}  // namespace

size_t compress_smem_bytes(int qjl, int dense) {
  return sizeof(SmemCompress) + (qjl ? QM * kPad * sizeof(float) : 0) +
         (dense ? D * kPad * sizeof(float) : 0);
}

cudaError_t launch_compress(const CompressArgs& a, cudaStream_t stream) {
  if (compress_tc_supported(a)) {
    const cudaError_t e = launch_compress_tc(a, stream);
    if (e != cudaErrorInvalidValue) return e;  // otherwise fall through to the CUDA-core kernel
  }
  const size_t smem = compress_smem_bytes(a.qjl || a.cache.L.vqjl, a.dense);
  // tokens per thread block: 64, or fewer (a multiple of the warp count, at least one token
  // per warp) so that a small input still spreads over about two thread blocks per SM
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const long long heads = (long long)a.cache.kv_heads * a.cache.batch;
  long long tpb = heads > 0 ? ((long long)a.max_len * heads + 2LL * sms - 1) / (2LL * sms) : kTokPerBlockMax;
  tpb = ((tpb + kWarps - 1) / kWarps) * kWarps;
  CompressArgs b = a;
  b.tok_per_block = (int)(tpb < kWarps ? kWarps : (tpb > kTokPerBlockMax ? kTokPerBlockMax : tpb));
  dim3 grid((a.max_len + b.tok_per_block - 1) / b.tok_per_block, a.cache.kv_heads, a.cache.batch);
  if (grid.x == 0) return cudaSuccess;
  if (a.in_dtype == TQ_F16) {
    auto k = compress_kernel<__half>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, kWarps * 32, smem, stream>>>(b);
  } else {
    auto k = compress_kernel<float>;
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    k<<<grid, kWarps * 32, smem, stream>>>(b);
  }
  return cudaGetLastError();
}

}  // namespace tqk
