// Compression on the tensor cores (tcgen05 + TMEM + TMA), randomized-Hadamard rotation.
//
// What is computed is the same as compress.cu ("TurboQuant explained", sections "How JL
// Matrices Evolved", "Coordinates Become Predictable After Rotation" and "Two-Stage
// Approach: MSE Approximation + QJL Correction"; "turboquant_cutile" function list:
// compress K = MSE + 1-bit QJL, compress V = MSE only).  The dense contractions run on
// the 5th-generation tensor cores:
//
//  * y' = (H D) x for a tile of 128 tokens: A = the fp16 input tile (exact), B = H D with
//    +-1 entries (exact), fp32 accumulation in tensor memory.  y = y' / ||y'||.
//  * QJL sketch in the rotated domain: with R = H D / sqrt(d) orthogonal,
//      S r = S R^T R r = (S D H) r_rot' / d,   r_rot' = y' - sqrt(d) fp16(||x||) c[idx],
//    so sign(S r) = sign((S D H) a r_rot') for any a > 0.  S D H is formed once per CTA
//    and held as an fp16 hi + lo pair; a r_rot' (scaled to O(1)) is split hi + lo as
//    well; three MMAs (hi.hi, hi.lo, lo.hi) give the projections to ~2^-22 relative.
//
// Quantisation works on y' directly: |y| > beta  <=>  |y'| > beta ||y'||, so each token
// scales its boundaries once instead of normalising every coordinate, and the rank is a
// sum of comparison masks (the boundaries are sorted) that also drive the centroid
// select of the residual.
//
// One persistent CTA per SM: 16 compute warps and one producer warp.  Compute warp w
// reads tensor-memory lane quadrant w % 4 (tokens 32 (w % 4) .. + 31) and coordinates
// 32 (w / 4) .. + 31, so four warps share a token; their per-token sums (norms, residual
// norm) meet in spare tensor-memory columns behind a 128-thread named barrier.  The
// producer warp issues the TMA copies (two K/V tile stages), the MMAs and their commits;
// the compute warps hand tensor-memory columns back through two mbarriers.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tq_device.cuh"
#include "tq_kernels.h"

namespace tqk {

namespace {

constexpr int TT = 128;                      // tokens per tile
constexpr int kComputeWarps = 16;
constexpr int kThreadsTC = (kComputeWarps + 1) * 32;
constexpr int kTileBytes = TT * D * 2;       // one 128 x 128 fp16 operand
// tensor-memory columns: y'_K, y'_V, A = residual hi / lo, S = sketch (and exchange slots)
constexpr uint32_t kColK = 0, kColV = 128, kColAhi = 256, kColAlo = 320, kColS = 384;
constexpr uint32_t kColNormX = kColS, kColRrX = kColS + 8;
constexpr uint32_t kTmemCols = 512;
// instruction descriptor: D f32, A and B f16, both K-major, N = 128, M = 128
constexpr uint32_t kIdesc = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr unsigned long long kWaitNs = 1000000000ull;  // a wait gives up after 1 s
constexpr float kSqrtD = 11.313708498984761f;
constexpr float kResidScale = 256.f;         // residual scaled to ~O(1) before the fp16 split

struct SmemTC {
  unsigned char x[2][2][kTileBytes];  // [stage][K, V] input tiles (canonical layout)
  unsigned char bhd[kTileBytes];      // B = H D
  unsigned char bshi[kTileBytes];     // B = S D H, fp16 hi part
  unsigned char bslo[kTileBytes];     // fp16 lo part
  unsigned long long bar_load[2], bar_fwd, bar_sig, kv_free, a_ready;
  uint32_t tmem_base;
  int bad_s;
};
constexpr size_t kSmemTC = sizeof(SmemTC) + 128;  // + base alignment slack

// Canonical no-swizzle K-major offset of element (row, k) of a 128 x 128 fp16 tile:
// 16-byte core-matrix rows, 8-row groups 128 B apart, 8-element K chunks 2048 B apart.
__device__ __forceinline__ int canon(int row, int k) {
  return (k >> 3) * 2048 + (row >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}

__device__ __forceinline__ uint32_t s_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint64_t smem_desc(const void* base, int ks) {
  const uint32_t addr = s_u32(base) + ks * 4096;
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)(2048 >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
         (1ull << 46);
}

__device__ __forceinline__ void bar_init(unsigned long long* b, int n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(s_u32(b)), "r"(n));
}

__device__ __forceinline__ bool bar_try(uint32_t addr, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(addr), "r"(parity)
      : "memory");
  return done != 0;
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Wait for the phase with the given parity to complete; false after kWaitNs (or 2^24
// polls, whichever comes first) without completion.
__device__ __forceinline__ bool bar_wait(unsigned long long* b, uint32_t parity) {
  const uint32_t addr = s_u32(b);
  if (bar_try(addr, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (int it = 0; it < (1 << 18); ++it) {
#pragma unroll 1
    for (int k = 0; k < 64; ++k)
      if (bar_try(addr, parity)) return true;
    if (global_ns() - t0 > kWaitNs) break;
  }
  return false;
}

__device__ __forceinline__ void bar_arrive(unsigned long long* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(s_u32(b)) : "memory");
}

// 128-thread barrier of the four compute warps that share a tensor-memory lane quadrant
__device__ __forceinline__ void quad_sync(int qd) {
  asm volatile("bar.sync %0, 128;" ::"r"(1 + qd) : "memory");
}

__device__ __forceinline__ void tma_load_tile(void* dst, const CUtensorMap* map, int row0,
                                              unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(s_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(row0), "r"(0), "r"(s_u32(bar))
      : "memory");
}

__device__ __forceinline__ void mma_ss(uint32_t d, uint64_t a, uint64_t b, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(a), "l"(b), "r"(kIdesc), "r"(acc));
}

__device__ __forceinline__ void mma_ts(uint32_t d, uint32_t a, uint64_t b, uint32_t acc) {
  asm volatile(
      "{\n .reg .pred p;\n setp.ne.b32 p, %4, 0;\n"
      " tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d),
      "r"(a), "l"(b), "r"(kIdesc), "r"(acc));
}

__device__ __forceinline__ void mma_commit(unsigned long long* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(s_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }
__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 consecutive tensor-memory columns of this warp's 32 lanes (one per thread).
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%18,%"
      "19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
        "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
        "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
        "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&v)[4]) {
  uint32_t r[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
      : "memory");
}

__device__ __forceinline__ void tmem_st2(uint32_t taddr, float a, float b) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x2.b32 [%0], {%1,%2};" ::"r"(taddr), "r"(__float_as_uint(a)),
               "r"(__float_as_uint(b))
               : "memory");
}

__device__ __forceinline__ void tmem_st1(uint32_t taddr, float a) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x1.b32 [%0], {%1};" ::"r"(taddr), "r"(__float_as_uint(a))
               : "memory");
}

// all-ones when a > b (a >= b), zero otherwise and for NaN
__device__ __forceinline__ uint32_t gt_mask(float a, float b) {
  uint32_t m;
  asm("set.gt.u32.f32 %0, %1, %2;" : "=r"(m) : "f"(a), "f"(b));
  return m;
}
__device__ __forceinline__ uint32_t ge_mask(float a, float b) {
  uint32_t m;
  asm("set.ge.u32.f32 %0, %1, %2;" : "=r"(m) : "f"(a), "f"(b));
  return m;
}

// sum of squares of 32 values, two lanes of packed fp32 at a time
__device__ __forceinline__ float sumsq32(const float (&v)[32]) {
  unsigned long long acc = 0;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    unsigned long long p;
    asm("mov.b64 %0, {%1, %2};" : "=l"(p) : "f"(v[i]), "f"(v[i + 1]));
    asm("fma.rn.f32x2 %0, %1, %1, %0;" : "+l"(acc) : "l"(p));
  }
  float lo, hi;
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(acc));
  return lo + hi;
}

// Bit of coordinate e (0..31) of a 32-coordinate group in the sign plane of 3-bit codes
// (the permutation of sign_plane_pos, which the decode's byte tables read).
__host__ __device__ constexpr int plane_bit(int e) { return 4 * (e >> 3) + (e & 3) + 16 * ((e >> 2) & 1); }

// Thermometer masks of |y'| against the scaled positive boundaries; returns the rank
// r = number of boundaries below |y'|.
template <int NB>
__device__ __forceinline__ uint32_t rank_masks(float y, const float (&thr)[8], uint32_t (&m)[8]) {
  const float ay = fabsf(y);
  uint32_t sum = 0;
#pragma unroll
  for (int k = 0; k < NB; ++k) {
    m[k] = gt_mask(ay, thr[k]);
    sum += m[k];
  }
  return 0u - sum;
}

// Code words of this thread's 32 coordinates for the b-bit field layouts without a QJL
// sign: pack (r, s) of coordinate i into w[].
//   b = 2: 2-bit r | s << 1, two words;  b = 3: 2-bit r in two words + one word of the
//   permuted sign plane;  b = 4: r | s << 3, four words.
template <int B>
__device__ __forceinline__ void pack_plain(uint32_t (&w)[4], int i, uint32_t r, uint32_t smask) {
  if constexpr (B == 2) {
    w[i >> 4] += r << (2 * (i & 15));
    w[i >> 4] |= smask & (2u << (2 * (i & 15)));
  } else if constexpr (B == 3) {
    w[i >> 4] += r << (2 * (i & 15));
    w[2] |= smask & (1u << plane_bit(i));
  } else {
    w[i >> 3] += r << (4 * (i & 7));
    w[i >> 3] |= smask & (8u << (4 * (i & 7)));
  }
}

// Store the words of pack_plain for one token slot (plane p = 16 bytes per slot; this
// thread's coordinates 32 part .. 32 part + 31).
template <int B>
__device__ __forceinline__ void store_plain(uint8_t* base, int part, int slot, const uint32_t (&w)[4]) {
  if constexpr (B == 2) {
    *reinterpret_cast<uint2*>(base + ((size_t)(part >> 1) * PT + slot) * 16 + 8 * (part & 1)) = make_uint2(w[0], w[1]);
  } else if constexpr (B == 3) {
    *reinterpret_cast<uint2*>(base + ((size_t)(part >> 1) * PT + slot) * 16 + 8 * (part & 1)) = make_uint2(w[0], w[1]);
    *reinterpret_cast<uint32_t*>(base + ((size_t)2 * PT + slot) * 16 + 4 * part) = w[2];
  } else {
    *reinterpret_cast<uint4*>(base + ((size_t)part * PT + slot) * 16) = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <int KB, int KQ, int VB>
__global__ void __launch_bounds__(kThreadsTC, 1)
    compress_tc_kernel(CompressArgs a, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const uint32_t pad = (128u - (s_u32(smem_raw) & 127u)) & 127u;
  SmemTC& sm = *reinterpret_cast<SmemTC*>(smem_raw + pad);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = warp == kComputeWarps;
  const int qd = warp & 3;           // tensor-memory lane quadrant
  const int part = (warp >> 2) & 3;  // coordinates 32 part .. 32 part + 31
  const int row = 32 * qd + lane;    // token within the tile
  const Layout& L = a.cache.L;
  constexpr int HK = 1 << (KB - 1), HV = 1 << (VB - 1);
  constexpr bool kMerged = KQ && KB == 3;

  const int tiles_per_head = (a.max_len + TT - 1) / TT;
  const int total = a.cache.batch * a.cache.kv_heads * tiles_per_head;
  const int my_tiles = (int)blockIdx.x < total ? (total - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  auto tile_coords = [&](int j, int& b, int& h, int& t0) {
    const int t = blockIdx.x + j * gridDim.x;
    t0 = (t % tiles_per_head) * TT;
    h = (t / tiles_per_head) % a.cache.kv_heads;
    b = t / (tiles_per_head * a.cache.kv_heads);
  };
  auto issue_load = [&](int j) {
    int b, h, t0;
    tile_coords(j, b, h, t0);
    const int row0 = (int)(((size_t)b * a.cache.kv_heads + h) * a.max_len + t0);
    unsigned long long* bar = &sm.bar_load[j & 1];
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(s_u32(bar)), "r"(2 * kTileBytes)
                 : "memory");
    tma_load_tile(sm.x[j & 1][0], &tmk, row0, bar);
    tma_load_tile(sm.x[j & 1][1], &tmv, row0, bar);
  };

  // ---------------- set-up ----------------
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s_u32(&sm.tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    bar_init(&sm.bar_load[0], 1);
    bar_init(&sm.bar_load[1], 1);
    bar_init(&sm.bar_fwd, 1);
    bar_init(&sm.bar_sig, 1);
    bar_init(&sm.kv_free, kComputeWarps);
    bar_init(&sm.a_ready, kComputeWarps);
    sm.bad_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // tile 0 streams in while the rotation operands are built (stage 1 is set-up scratch)
  if (producer && lane == 0 && my_tiles > 0) issue_load(0);
  __syncwarp();
  if (tid == 0 && blockIdx.x == 0) {
    for (int i = 0; i < 2 * HK; ++i)
      if (a.k_centroids[i] != -a.k_centroids[2 * HK - 1 - i]) report(a.status, TQ_ERR_INVALID_ARG);
    for (int i = 0; i < 2 * HV; ++i)
      if (a.v_centroids[i] != -a.v_centroids[2 * HV - 1 - i]) report(a.status, TQ_ERR_INVALID_ARG);
    // the rank rule reads only the positive boundaries: they must mirror, middle one 0
    for (int i = 0; i < 2 * HK - 1; ++i)
      if (a.k_boundaries[i] != -a.k_boundaries[2 * HK - 2 - i]) report(a.status, TQ_ERR_INVALID_ARG);
    for (int i = 0; i < 2 * HV - 1; ++i)
      if (a.v_boundaries[i] != -a.v_boundaries[2 * HV - 2 - i]) report(a.status, TQ_ERR_INVALID_ARG);
  }
  if (!producer) {
    // B = H D: row i, column k = (-1)^popcount(i & k) D_k
    for (int c = tid; c < D * 16; c += kComputeWarps * 32) {
      const int i = c & 127, ch = c >> 7;
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k0 = ch * 8 + 2 * e;
        const float s0 = a.signs[k0], s1 = a.signs[k0 + 1];
        const float v0 = (__popc(i & k0) & 1) ? -s0 : s0;
        const float v1 = (__popc(i & (k0 + 1)) & 1) ? -s1 : s1;
        const __half2 h = __floats2half2_rn(v0, v1);
        w[e] = *reinterpret_cast<const uint32_t*>(&h);
      }
      *reinterpret_cast<uint4*>(sm.bhd + canon(i, ch * 8)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (KQ) {
      // B = S D H: thread (n, p) transforms coordinates 32p .. 32p + 31 of row n of S D in
      // registers (butterfly spans 1..16); the spans 32 and 64 meet through scratch.
      const int n = tid & 127, p = tid >> 7;
      float v[32];
      const float4* srow = reinterpret_cast<const float4*>(a.s + (size_t)n * D + 32 * p);
      int bad = 0;
#pragma unroll
      for (int i4 = 0; i4 < 8; ++i4) {
        const float4 q = srow[i4];
        const float e[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int i = 4 * i4 + u;
          if (__half2float(__float2half_rn(e[u])) != e[u]) bad = 1;
          v[i] = e[u] * a.signs[32 * p + i];
        }
      }
      if (bad) sm.bad_s = 1;
#pragma unroll
      for (int hs = 1; hs < 32; hs <<= 1) {
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          if (i & hs) continue;
          const float u = v[i], w = v[i + hs];
          v[i] = u + w;
          v[i + hs] = u - w;
        }
      }
      float* scr = reinterpret_cast<float*>(sm.x[1][0]);  // [coordinate][n], 64 KB
#pragma unroll
      for (int i = 0; i < 32; ++i) scr[(32 * p + i) * 128 + n] = v[i];
      asm volatile("bar.sync 5, 512;" ::: "memory");  // the 16 compute warps
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        float acc = 0.f;
#pragma unroll
        for (int bb = 0; bb < 4; ++bb) {
          const float t = scr[(32 * bb + i) * 128 + n];
          acc += (__popc(p & bb) & 1) ? -t : t;
        }
        v[i] = acc;
      }
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float x0 = v[8 * c + 2 * e], x1 = v[8 * c + 2 * e + 1];
          const __half2 h2 = __floats2half2_rn(x0, x1);
          const float2 hf = __half22float2(h2);
          const __half2 l2 = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
          hi[e] = *reinterpret_cast<const uint32_t*>(&h2);
          lo[e] = *reinterpret_cast<const uint32_t*>(&l2);
        }
        *reinterpret_cast<uint4*>(sm.bshi + canon(n, 32 * p + 8 * c)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(sm.bslo + canon(n, 32 * p + 8 * c)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  if (tid == 0 && sm.bad_s) report(a.status, TQ_ERR_INVALID_ARG);
  const uint32_t tmem = sm.tmem_base;

  if (producer) {
    // ---------------- producer: copies and MMAs ----------------
    if (lane == 0 && my_tiles > 0) {
      if (my_tiles > 1) issue_load(1);
      int loads_issued = my_tiles > 1 ? 2 : 1, loads_done = 0;
      int fwd_issued = 0, fwd_done = 0;
      bool ok = true;
      for (int j = 0; j < my_tiles; ++j) {
        const int st = j & 1;
        ok = bar_wait(&sm.bar_load[st], (j >> 1) & 1);
        if (!ok) break;
        ++loads_done;
        if (j > 0) {
          ok = bar_wait(&sm.kv_free, (j - 1) & 1);
          if (!ok) break;
        }
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(tmem + kColK, smem_desc(sm.x[st][0], ks), smem_desc(sm.bhd, ks), ks > 0);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(tmem + kColV, smem_desc(sm.x[st][1], ks), smem_desc(sm.bhd, ks), ks > 0);
        mma_commit(&sm.bar_fwd);
        ++fwd_issued;
        ok = bar_wait(&sm.bar_fwd, j & 1);
        if (!ok) break;
        ++fwd_done;
        // stage st is consumed: stream tile j + 2 into it
        if (j + 2 < my_tiles) {
          issue_load(j + 2);
          ++loads_issued;
        }
        if (KQ) {
          ok = bar_wait(&sm.a_ready, j & 1);
          if (!ok) break;
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            mma_ts(tmem + kColS, tmem + kColAhi + 8 * ks, smem_desc(sm.bshi, ks), ks > 0);
            mma_ts(tmem + kColS, tmem + kColAhi + 8 * ks, smem_desc(sm.bslo, ks), 1);
            mma_ts(tmem + kColS, tmem + kColAlo + 8 * ks, smem_desc(sm.bshi, ks), 1);
          }
          mma_commit(&sm.bar_sig);  // the compute warps wait for this one
        }
      }
      if (!ok) {
        report(a.status, TQ_ERR_TIMEOUT);
        // drain what is still in flight before the shared and tensor memory go away
        while (loads_done < loads_issued) {
          bar_wait(&sm.bar_load[loads_done & 1], (loads_done >> 1) & 1);
          ++loads_done;
        }
        if (fwd_done < fwd_issued) bar_wait(&sm.bar_fwd, fwd_done & 1);
      }
    }
    __syncwarp();
  } else {
    // ---------------- compute warps ----------------
    float kpos[8], vpos[8], kmag[8], vmag[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      kpos[i] = (i < HK - 1) ? a.k_boundaries[HK + i] : 0.f;
      vpos[i] = (i < HV - 1) ? a.v_boundaries[HV + i] : 0.f;
      kmag[i] = (i < HK) ? a.k_centroids[HK + i] : 0.f;
      vmag[i] = (i < HV) ? a.v_centroids[HV + i] : 0.f;
    }
    const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
    bool failed = false;
    for (int j = 0; j < my_tiles; ++j) {
      int b, h, t0;
      tile_coords(j, b, h, t0);
      const int len = a.seq_lens[b];
      const int tok = t0 + row;
      const bool bad_len = len < 0 || len > a.max_len || len > a.cache.max_pages * PT;
      bool valid = !bad_len && tok < len;
      if (bad_len && tid == 0 && t0 == 0) report(a.status, TQ_ERR_BOUNDS);
      uint8_t* blk = nullptr;
      const int slot = tok % PT;
      if (valid) {
        const int phys = a.cache.block_table[(size_t)b * a.cache.max_pages + tok / PT];
        if (phys < 0 || phys >= a.cache.num_pages) {
          if (part == 0) report(a.status, TQ_ERR_BOUNDS);
          valid = false;
        } else {
          blk = a.cache.block(phys, h);
        }
      }

      // ---- forward result, per-token norms ----
      if (!failed && !bar_wait(&sm.bar_fwd, j & 1)) failed = true;
      __syncwarp();
      tc_fence_after();
      float y[32];
      tmem_ld32(tmem + lane_base + kColK + 32 * part, y);
      float z[32];
      tmem_ld32(tmem + lane_base + kColV + 32 * part, z);
      tmem_wait_ld();
      const float ssk = sumsq32(y), ssv = sumsq32(z);
      // every warp of the quadrant is past its reads of the previous tile's sketch
      tc_fence_before();
      quad_sync(qd);
      tc_fence_after();
      tmem_st2(tmem + lane_base + kColNormX + 2 * part, ssk, ssv);
      tmem_wait_st();
      tc_fence_before();
      quad_sync(qd);
      tc_fence_after();
      float nx[8];
      tmem_ld8(tmem + lane_base + kColNormX, nx);
      tmem_wait_ld();
      const float nyk = sqrtf((nx[0] + nx[2]) + (nx[4] + nx[6]));  // ||y'_K|| = sqrt(d) ||k||
      const float nyv = sqrtf((nx[1] + nx[3]) + (nx[5] + nx[7]));

      // ---- keys ----
      const __half nk16 = __float2half_rn(nyk * (1.0f / kSqrtD));
      if (valid && part == 0 && __hisinf(nk16)) report(a.status, TQ_ERR_OVERFLOW);
      float thr[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) thr[k] = kpos[k] * nyk;
      const float alpha = nyk > 0.f ? kResidScale / nyk : 1.f;
      float am[8];
      const float csa = alpha * kSqrtD * __half2float(nk16);
#pragma unroll
      for (int k = 0; k < 8; ++k) am[k] = csa * kmag[k];
      uint32_t kw[4] = {0, 0, 0, 0};
      float rr = 0.f;
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        uint32_t m[8];
        const uint32_t r = rank_masks<HK - 1>(y[i], thr, m);
        const uint32_t smask = gt_mask(y[i], 0.f);
        if constexpr (kMerged) {
          kw[i >> 3] += r << (4 * (i & 7));
          kw[i >> 3] |= smask & (4u << (4 * (i & 7)));
        } else {
          pack_plain<KB>(kw, i, r, smask);
        }
        if constexpr (KQ) {
          // signed centroid a cs c[idx] from the masks, then the scaled residual
          uint32_t c = __float_as_uint(am[0]);
#pragma unroll
          for (int k = 1; k < HK; ++k) c = (m[k - 1] & __float_as_uint(am[k])) | (~m[k - 1] & c);
          c ^= ~smask & 0x80000000u;
          const float rv = fmaf(y[i], alpha, -__uint_as_float(c));
          y[i] = rv;
          rr = fmaf(rv, rv, rr);
        }
      }
      float rho = 0.f;
      if constexpr (KQ) {
        uint32_t hi[16], lo[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float r0 = y[2 * i], r1 = y[2 * i + 1];
          const float h0 = __uint_as_float(__float_as_uint(r0) & 0xFFFFE000u);
          const float h1 = __uint_as_float(__float_as_uint(r1) & 0xFFFFE000u);
          const __half2 hh = __floats2half2_rn(h0, h1);
          const __half2 ll = __floats2half2_rn(r0 - h0, r1 - h1);
          hi[i] = *reinterpret_cast<const uint32_t*>(&hh);
          lo[i] = *reinterpret_cast<const uint32_t*>(&ll);
        }
        tmem_st16(tmem + lane_base + kColAhi + 16 * part, hi);
        tmem_st16(tmem + lane_base + kColAlo + 16 * part, lo);
        tmem_st1(tmem + lane_base + kColRrX + part, rr);
        tmem_wait_st();
        tc_fence_before();
        quad_sync(qd);
        tc_fence_after();
        float rx[4];
        tmem_ld4(tmem + lane_base + kColRrX, rx);
        tmem_wait_ld();
        rho = sqrtf((rx[0] + rx[1]) + (rx[2] + rx[3])) / (alpha * kSqrtD);
      }
      // ---- values: re-read y'_V (its columns are released after this) ----
      tmem_ld32(tmem + lane_base + kColV + 32 * part, z);
      tmem_wait_ld();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        bar_arrive(&sm.kv_free);
        if (KQ) bar_arrive(&sm.a_ready);
      }
      const __half nv16 = __float2half_rn(nyv * (1.0f / kSqrtD));
      if (valid && part == 0 && __hisinf(nv16)) report(a.status, TQ_ERR_OVERFLOW);
#pragma unroll
      for (int k = 0; k < 8; ++k) thr[k] = vpos[k] * nyv;
      uint32_t vw[4] = {0, 0, 0, 0};
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        uint32_t m[8];
        const uint32_t r = rank_masks<HV - 1>(z[i], thr, m);
        pack_plain<VB>(vw, i, r, gt_mask(z[i], 0.f));
      }
      if (valid && !failed) {
        store_plain<VB>(blk + L.vc, part, slot, vw);
        if (part == 0) reinterpret_cast<__half*>(blk + L.vn)[slot] = nv16;
      }

      // ---- QJL signs, then the key words ----
      uint32_t sgw = 0;
      if constexpr (KQ) {
        if (!failed && !bar_wait(&sm.bar_sig, j & 1)) failed = true;
        __syncwarp();
        tc_fence_after();
        tmem_ld32(tmem + lane_base + kColS + 32 * part, z);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint32_t sg = ge_mask(z[i], 0.f);
          if constexpr (kMerged)
            kw[i >> 3] |= sg & (8u << (4 * (i & 7)));
          else
            sgw |= sg & (1u << i);
        }
      }
      if (valid && !failed) {
        if constexpr (kMerged) {
          *reinterpret_cast<uint4*>(blk + L.kc + ((size_t)part * PT + slot) * 16) =
              make_uint4(kw[0], kw[1], kw[2], kw[3]);
        } else {
          store_plain<KB>(blk + L.kc, part, slot, kw);
          if (KQ) *reinterpret_cast<uint32_t*>(blk + L.ks + (size_t)slot * 16 + 4 * part) = sgw;
        }
        if (part == 0) {
          reinterpret_cast<__half*>(blk + L.kn)[slot] = nk16;
          if (KQ) reinterpret_cast<__half*>(blk + L.kr)[slot] = __float2half_rn(rho);
        }
      }
    }
    if (failed && lane == 0) report(a.status, TQ_ERR_TIMEOUT);
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols));
  }
}

// ---------------------------------------------------------------------------
// host: tensor maps
// ---------------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// The [rows][128] fp16 input viewed as 3-D (element e < 8, row, 16-byte chunk < 16) so that
// one box of (8, 128, 16) lands as the canonical K-major tile: e*2 + row*16 + chunk*2048
// (8 rows of 16 bytes make the 128-byte core-matrix group stride).  Rows past the end of
// the input read as zero.
bool make_tile_map(CUtensorMap* m, const void* base, size_t rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {8, (cuuint64_t)rows, 16};
  const cuuint64_t strides[2] = {256, 16};  // bytes, dims 1..2
  const cuuint32_t box[3] = {8, TT, 16};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int KB, int KQ, int VB>
cudaError_t launch_tc(const CompressArgs& a, const CUtensorMap& mk, const CUtensorMap& mv, cudaStream_t stream) {
  auto k = compress_tc_kernel<KB, KQ, VB>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmemTC);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tiles = a.cache.batch * a.cache.kv_heads * ((a.max_len + TT - 1) / TT);
  const int grid = tiles < sms ? tiles : sms;
  if (grid == 0) return cudaSuccess;
  k<<<grid, kThreadsTC, kSmemTC, stream>>>(a, mk, mv);
  return cudaGetLastError();
}

}  // namespace

bool compress_tc_supported(const CompressArgs& a) {
  const Layout& L = a.cache.L;
  if (a.dense || a.in_dtype != TQ_F16) return false;
  if ((size_t)a.cache.batch * a.cache.kv_heads * a.max_len >= (1ull << 31)) return false;
  if (L.qjl && !(L.kbits == 2 || L.kbits == 3)) return false;
  if (!L.qjl && !(L.kbits >= 2 && L.kbits <= 4)) return false;
  if (!(L.vbits >= 2 && L.vbits <= 4)) return false;
  if ((reinterpret_cast<uintptr_t>(a.k) & 15) || (reinterpret_cast<uintptr_t>(a.v) & 15)) return false;
  return encode_fn() != nullptr;
}

cudaError_t launch_compress_tc(const CompressArgs& a, cudaStream_t stream) {
  const Layout& L = a.cache.L;
  const size_t rows = (size_t)a.cache.batch * a.cache.kv_heads * a.max_len;
  if (rows == 0) return cudaSuccess;
  CUtensorMap mk, mv;
  if (!make_tile_map(&mk, a.k, rows) || !make_tile_map(&mv, a.v, rows)) return cudaErrorInvalidValue;
#define TQ_TC(KB, KQ, VB) \
  if (L.kbits == KB && L.qjl == KQ && L.vbits == VB) return launch_tc<KB, KQ, VB>(a, mk, mv, stream);
#define TQ_TC_V(KB, KQ) TQ_TC(KB, KQ, 2) TQ_TC(KB, KQ, 3) TQ_TC(KB, KQ, 4)
  TQ_TC_V(3, 1)
  TQ_TC_V(2, 1)
  TQ_TC_V(2, 0)
  TQ_TC_V(3, 0)
  TQ_TC_V(4, 0)
#undef TQ_TC_V
#undef TQ_TC
  return cudaErrorInvalidValue;
}

}  // namespace tqk
