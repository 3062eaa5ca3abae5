// Device-side helpers shared by the kernels (not part of the ABI).
#pragma once
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "tq.h"

namespace tqk {

constexpr int D = 128;      // head_dim supported by the kernels
constexpr int QM = 128;     // rows of S
constexpr int PT = 256;     // tokens per page
constexpr unsigned FULL = 0xffffffffu;

// Byte offsets of the regions of one (layer, page, kv head) block; the format is
// stated in tq.h.
struct Layout {
  int kn, kr, vn, kc, ks, vc, bytes;
  int kbits, vbits, qjl;
  int kmerged;  // 3-bit keys with QJL: one 4-bit field (r0, r1, s, sigma) per coordinate
  int kchunks;  // 16-byte chunks of one token's key bit string
  int vqjl;     // values carry the QJL signs of their residual (VS) and its norm (VR)
  int vs, vr;
  int dither;   // dithered: each vector's offset xi (fp16) in KD (keys) and VD (values)
  int kd, vd;
};

__host__ __device__ inline Layout make_layout(int kbits, int qjl, int vbits, int vqjl = 0, int dither = 0) {
  Layout L;
  L.kbits = kbits;
  L.vbits = vbits;
  L.qjl = qjl;
  L.vqjl = vqjl;
  L.dither = dither;
  L.kmerged = (qjl && kbits == 3) ? 1 : 0;
  L.kchunks = L.kmerged ? 4 : kbits;
  int off = 0;
  L.kn = off; off += 2 * PT;
  L.kr = off; off += qjl ? 2 * PT : 0;
  L.vn = off; off += 2 * PT;
  L.kc = off; off += L.kchunks * 16 * PT;
  L.ks = off; off += (qjl && !L.kmerged) ? (QM / 8) * PT : 0;
  L.vc = off; off += vbits * (D / 8) * PT;
  L.vs = off; off += vqjl ? (QM / 8) * PT : 0;
  L.vr = off; off += vqjl ? 2 * PT : 0;
  L.kd = off; off += dither ? 2 * PT : 0;
  L.vd = off; off += dither ? 2 * PT : 0;
  L.bytes = off;
  return L;
}

// Position of coordinate j's sign inside the 3-bit sign plane: j = 32q + 8a + 4h + t
// sits at 32q + 4a + t + 16h.
__host__ __device__ __forceinline__ int sign_plane_pos(int j) {
  const int e = j & 31;
  return (j & ~31) + 4 * (e >> 3) + (e & 3) + 16 * ((e >> 2) & 1);
}

// Everything a kernel needs to find a block of the cache.
struct CacheRef {
  uint8_t* pages;
  const int32_t* block_table;
  int num_pages, max_pages, batch, kv_heads, layer;
  Layout L;
  __device__ __forceinline__ uint8_t* block(int page, int head) const {
    return pages + ((size_t)((size_t)layer * num_pages + page) * kv_heads + head) * (size_t)L.bytes;
  }
};

// First error wins.
__device__ __forceinline__ void report(int32_t* st, int code) {
  if (st) atomicCAS(st, 0, code);
}

// Index checks of the debug build (compiled with -DTQ_DEBUG, libtq_debug.so): a check that
// fails records TQ_ERR_BOUNDS in the status word and the kernel carries on (no trap, so the
// context stays usable); the release build compiles them away.
#ifdef TQ_DEBUG
#define TQ_DCHECK(status, cond)                    \
  do {                                             \
    if (!(cond)) report((status), TQ_ERR_BOUNDS);  \
  } while (0)
#else
#define TQ_DCHECK(status, cond) \
  do {                          \
  } while (0)
#endif

// Stored-code magnitude table: mag[r] = c[h + r] with h = 2^(b-1).
// Value of stored (s, r): s ? mag[r] : -mag[r].

// Field extraction from a token's code bit string, given as 32-bit words (little endian).
// Returns (s, r) of coordinate j.
__device__ __forceinline__ void code_fields(const uint32_t* w, int bits, int j, int& s, int& r) {
  switch (bits) {
    case 1:
      s = (w[j >> 5] >> (j & 31)) & 1;
      r = 0;
      break;
    case 2: {
      const uint32_t f = (w[j >> 4] >> ((j & 15) * 2)) & 3u;
      r = f & 1;
      s = f >> 1;
      break;
    }
    case 3: {
      r = (w[j >> 4] >> ((j & 15) * 2)) & 3u;
      const int p = sign_plane_pos(j);
      s = (w[8 + (p >> 5)] >> (p & 31)) & 1;
      break;
    }
    default: {
      const uint32_t f = (w[j >> 3] >> ((j & 7) * 4)) & 15u;
      r = f & 7;
      s = f >> 3;
      break;
    }
  }
}

// Key fields of coordinate j: merged keys carry sigma_j in the same nibble.
__device__ __forceinline__ void key_fields(const uint32_t* w, const Layout& L, int j, int& s, int& r,
                                           int& sigma) {
  if (L.kmerged) {
    const uint32_t f = (w[j >> 3] >> ((j & 7) * 4)) & 15u;
    r = f & 3;
    s = (f >> 2) & 1;
    sigma = f >> 3;
  } else {
    code_fields(w, L.kbits, j, s, r);
    sigma = 0;
  }
}

// Normalized Walsh-Hadamard butterflies on 128 values held as 4 per lane,
// element j = lane + 32*e.  Output in natural (Sylvester) order, unnormalized
// (the caller scales by 1/sqrt(128)).
__device__ __forceinline__ void fwht128_warp(float (&x)[4], int lane) {
#pragma unroll
  for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const float o = __shfl_xor_sync(FULL, x[e], h);
      x[e] = (lane & h) ? (o - x[e]) : (x[e] + o);
    }
  }
  // strides 32 and 64: within the lane
  float a0 = x[0] + x[1], a1 = x[0] - x[1], a2 = x[2] + x[3], a3 = x[2] - x[3];
  x[0] = a0 + a2;
  x[1] = a1 + a3;
  x[2] = a0 - a2;
  x[3] = a1 - a3;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(FULL, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(FULL, v, o));
  return v;
}

}  // namespace tqk
