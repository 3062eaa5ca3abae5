// Compression on the tensor cores (tcgen05 + TMEM + TMA), randomized-Hadamard rotation.
//
// What is computed is the same as compress.cu ("TurboQuant explained", sections "How JL
// Matrices Evolved", "Coordinates Become Predictable After Rotation" and "Two-Stage
// Approach: MSE Approximation + QJL Correction"; "turboquant_cutile" function list:
// compress K = MSE + 1-bit QJL, compress V = MSE only).  The dense contractions run on
// the 5th-generation tensor cores:
//
//  * y' = (H D) x for a tile of 128 tokens: A = the fp16 input tile (exact), B = H D with
//    +-1 entries (exact), fp32 accumulation in tensor memory.  y = y' / (sqrt(d) ||x||).
//  * QJL sketch in the rotated domain: with R = H D / sqrt(d) orthogonal,
//      S r = S R^T R r = (S D H) r_rot' / d,   r_rot' = y' - sqrt(d) fp16(||x||) c[idx],
//    so sign(S r) = sign((S D H) r_rot').  S D H is formed once per CTA in fp64 and held
//    as an fp16 hi + lo pair; r_rot' is split hi + lo as well; three MMAs (hi.hi, hi.lo,
//    lo.hi) give the projections to ~2^-22 relative precision.
//
// One persistent CTA per SM, 256 threads: thread t and t + 128 own token t of the tile
// (coordinates 0..63 and 64..127).  Tiles arrive by one 3-D TMA copy each, landing
// directly in the canonical no-swizzle K-major layout the MMA descriptors describe.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tq_device.cuh"
#include "tq_kernels.h"

namespace tqk {

namespace {

constexpr int TT = 128;                      // tokens per tile
constexpr int kThreadsTC = 256;
constexpr int kTileBytes = TT * D * 2;       // one 128 x 128 fp16 operand
constexpr uint32_t kColK = 0, kColV = 128, kColAhi = 256, kColAlo = 320, kColS = 384;
constexpr uint32_t kTmemCols = 512;
// instruction descriptor: D f32, A and B f16, both K-major, N = 128, M = 128
constexpr uint32_t kIdesc = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr long long kWaitLimitTC = 1ll << 26;
constexpr float kSqrtD = 11.313708498984761f;

struct SmemTC {
  unsigned char xk[kTileBytes];    // K tile (canonical layout); fp64 scratch during set-up
  unsigned char xv[kTileBytes];    // V tile
  unsigned char bhd[kTileBytes];   // B = H D
  unsigned char bshi[kTileBytes];  // B = S D H, fp16 hi part
  unsigned char bslo[kTileBytes];  // fp16 lo part
  unsigned long long bar_load, bar_fwd, bar_sig;
  uint32_t tmem_base;
  float red[2][TT];                // row partial sums of the two thread halves
  float kmag[8], vmag[8], kpos[8], vpos[8];
  float signs[D];
  int bad_s;
};

// Canonical no-swizzle K-major offset of element (row, k) of a 128 x 128 fp16 tile:
// 16-byte core-matrix rows, 8-row groups 128 B apart, 8-element K chunks 2048 B apart.
__device__ __forceinline__ int canon(int row, int k) {
  return (k >> 3) * 2048 + (row >> 3) * 128 + (row & 7) * 16 + (k & 7) * 2;
}

__device__ __forceinline__ uint64_t smem_desc(const void* base, int ks) {
  const uint32_t addr = static_cast<uint32_t>(__cvta_generic_to_shared(base)) + ks * 4096;
  return (uint64_t)((addr >> 4) & 0x3FFF) | ((uint64_t)(2048 >> 4) << 16) | ((uint64_t)(128 >> 4) << 32) |
         (1ull << 46);
}

__device__ __forceinline__ uint32_t s_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void bar_init(unsigned long long* b, int n) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(s_u32(b)), "r"(n));
}

__device__ __forceinline__ bool bar_wait(unsigned long long* b, uint32_t parity) {
  const uint32_t addr = s_u32(b);
  for (long long it = 0; it < kWaitLimitTC; ++it) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    if (done) return true;
  }
  return false;
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

// 32 consecutive TMEM columns of this warp's 32 lanes.
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

__device__ __forceinline__ void tmem_wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_st32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,%17,%"
      "18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15]), "r"(r[16]),
      "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]), "r"(r[23]), "r"(r[24]),
      "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}

__device__ __forceinline__ void tmem_wait_st() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// Rank of |y| among the positive boundaries pos[0..nb-1] with the oracle's tie rule:
// idx = #{beta < y} gives r = #{pos < |y|} for y > 0 and #{pos <= |y|} for y <= 0.
template <int NB>
__device__ __forceinline__ int rank_of(float y, const float (&pos)[8], int& s) {
  s = y > 0.f;
  const int ai = (__float_as_int(y) & 0x7fffffff) + (s ? 0 : 1);
  int r = 0;
#pragma unroll
  for (int k = 0; k < NB; ++k) r += (__float_as_int(pos[k]) < ai) ? 1 : 0;
  return r;
}

template <int KB, int KQ, int VB>
__global__ void __launch_bounds__(kThreadsTC, 1)
    compress_tc_kernel(CompressArgs a, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  // the tiles start on a 1024-byte boundary whatever the base alignment the launch gives
  const uint32_t pad = (1024u - (s_u32(smem_raw) & 1023u)) & 1023u;
  SmemTC& sm = *reinterpret_cast<SmemTC*>(smem_raw + pad);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int half = tid >> 7;       // coordinates 64 half .. 64 half + 63
  const int row = tid & 127;       // token within the tile = TMEM lane
  const Layout& L = a.cache.L;
  constexpr int HK = 1 << (KB - 1), HV = 1 << (VB - 1);

  // ---------------- set-up ----------------
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s_u32(&sm.tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    bar_init(&sm.bar_load, 1);
    bar_init(&sm.bar_fwd, 1);
    bar_init(&sm.bar_sig, 1);
    sm.bad_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (tid < HK) sm.kmag[tid] = a.k_centroids[HK + tid];
  if (tid < HK - 1) sm.kpos[tid] = a.k_boundaries[HK + tid];
  if (tid < HV) sm.vmag[tid] = a.v_centroids[HV + tid];
  if (tid < HV - 1) sm.vpos[tid] = a.v_boundaries[HV + tid];
  if (tid < D) sm.signs[tid] = a.signs[tid];
  __syncthreads();
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
  // B = H D: row i, column k = (-1)^popcount(i & k) D_k
  for (int c = tid; c < D * 16; c += kThreadsTC) {
    const int i = c >> 4, ch = c & 15;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const int k0 = ch * 8 + 2 * e;
      const float v0 = (__popc(i & k0) & 1) ? -sm.signs[k0] : sm.signs[k0];
      const float v1 = (__popc(i & (k0 + 1)) & 1) ? -sm.signs[k0 + 1] : sm.signs[k0 + 1];
      const __half2 h = __floats2half2_rn(v0, v1);
      w[e] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(sm.bhd + canon(i, ch * 8)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (KQ) {
    // B = S D H, exact in fp64, in 4 groups of 32 rows (scratch in the K tile buffer)
    double* scr = reinterpret_cast<double*>(sm.xk);  // [32][128]
    for (int g0 = 0; g0 < D; g0 += 32) {
      for (int e = tid; e < 32 * D; e += kThreadsTC) {
        const int r = e >> 7, j = e & 127;
        const float v = a.s[(size_t)(g0 + r) * D + j];
        if (__half2float(__float2half_rn(v)) != v) sm.bad_s = 1;
        scr[e] = (double)v * (double)sm.signs[j];
      }
      __syncthreads();
      for (int h = 1; h < D; h <<= 1) {
        for (int e = tid; e < 32 * 64; e += kThreadsTC) {
          const int r = e >> 6, p = e & 63;
          const int lo = ((p & ~(h - 1)) << 1) | (p & (h - 1));
          const double u = scr[r * D + lo], v = scr[r * D + lo + h];
          scr[r * D + lo] = u + v;
          scr[r * D + lo + h] = u - v;
        }
        __syncthreads();
      }
      for (int c = tid; c < 32 * 16; c += kThreadsTC) {
        const int r = c >> 4, ch = c & 15;
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const double x0 = scr[r * D + ch * 8 + 2 * e], x1 = scr[r * D + ch * 8 + 2 * e + 1];
          const __half h0 = __double2half(x0), h1 = __double2half(x1);
          const __half l0 = __double2half(x0 - (double)__half2float(h0));
          const __half l1 = __double2half(x1 - (double)__half2float(h1));
          hi[e] = (uint32_t)__half_as_ushort(h0) | ((uint32_t)__half_as_ushort(h1) << 16);
          lo[e] = (uint32_t)__half_as_ushort(l0) | ((uint32_t)__half_as_ushort(l1) << 16);
        }
        *reinterpret_cast<uint4*>(sm.bshi + canon(g0 + r, ch * 8)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
        *reinterpret_cast<uint4*>(sm.bslo + canon(g0 + r, ch * 8)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
      }
      __syncthreads();
    }
  }
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  __syncthreads();
  if (tid == 0 && sm.bad_s) report(a.status, TQ_ERR_INVALID_ARG);
  const uint32_t tmem = sm.tmem_base;
  const uint32_t lane_base = (uint32_t)(32 * (warp & 3)) << 16;  // this warp's TMEM lane quadrant

  float kpos[8], vpos[8], kmag[8], vmag[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    kpos[i] = (i < HK - 1) ? sm.kpos[i] : 0.f;
    vpos[i] = (i < HV - 1) ? sm.vpos[i] : 0.f;
    kmag[i] = (i < HK) ? sm.kmag[i] : 0.f;
    vmag[i] = (i < HV) ? sm.vmag[i] : 0.f;
  }

  // ---------------- tiles ----------------
  const int tiles_per_head = (a.max_len + TT - 1) / TT;
  const int total = a.cache.batch * a.cache.kv_heads * tiles_per_head;
  uint32_t ph_load = 0, ph_fwd = 0, ph_sig = 0;
  auto tile_coords = [&](int t, int& b, int& h, int& t0) {
    t0 = (t % tiles_per_head) * TT;
    h = (t / tiles_per_head) % a.cache.kv_heads;
    b = t / (tiles_per_head * a.cache.kv_heads);
  };
  auto issue_load = [&](int t) {
    int b, h, t0;
    tile_coords(t, b, h, t0);
    const int row0 = (int)(((size_t)b * a.cache.kv_heads + h) * a.max_len + t0);
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(s_u32(&sm.bar_load)),
                 "r"(2 * kTileBytes)
                 : "memory");
    tma_load_tile(sm.xk, &tmk, row0, &sm.bar_load);
    tma_load_tile(sm.xv, &tmv, row0, &sm.bar_load);
  };
  int t = blockIdx.x;
  // outstanding asynchronous work, drained (with the same bound) if a wait gives up
  bool load_out = t < total, fwd_out = false, sig_out = false;
  if (tid == 0 && t < total) issue_load(t);
  for (; t < total; t += gridDim.x) {
    int b, h, t0;
    tile_coords(t, b, h, t0);
    const int len = a.seq_lens[b];
    if (!bar_wait(&sm.bar_load, ph_load)) {
      if (tid == 0) report(a.status, TQ_ERR_TIMEOUT);
      break;
    }
    ph_load ^= 1;
    load_out = false;
    // forward rotations of K and V
    if (tid == 0) {
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) mma_ss(tmem + kColK, smem_desc(sm.xk, ks), smem_desc(sm.bhd, ks), ks > 0);
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) mma_ss(tmem + kColV, smem_desc(sm.xv, ks), smem_desc(sm.bhd, ks), ks > 0);
      mma_commit(&sm.bar_fwd);
    }
    fwd_out = true;
    if (!bar_wait(&sm.bar_fwd, ph_fwd)) {
      if (tid == 0) report(a.status, TQ_ERR_TIMEOUT);
      break;
    }
    ph_fwd ^= 1;
    fwd_out = false;
    tc_fence_after();
    // the input tiles are consumed: prefetch the next tile
    load_out = t + (int)gridDim.x < total;
    if (tid == 0 && load_out) issue_load(t + gridDim.x);

    const int tok = t0 + row;
    const bool bad_len = len < 0 || len > a.max_len || len > a.cache.max_pages * PT;
    bool valid = !bad_len && tok < len;
    if (bad_len && tid == 0 && t0 == 0) report(a.status, TQ_ERR_BOUNDS);
    uint8_t* blk = nullptr;
    int slot = tok % PT;
    if (valid) {
      const int phys = a.cache.block_table[(size_t)b * a.cache.max_pages + tok / PT];
      if (phys < 0 || phys >= a.cache.num_pages) {
        if (half == 0) report(a.status, TQ_ERR_BOUNDS);
        valid = false;
      } else {
        blk = a.cache.block(phys, h);
      }
    }

    // ======== keys ========
    float y[64];
    {
      float v[32];
      tmem_ld32(tmem + lane_base + kColK + 64 * half, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) y[i] = v[i];
      tmem_ld32(tmem + lane_base + kColK + 64 * half + 32, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) y[32 + i] = v[i];
      tmem_wait_ld();
    }
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 64; ++i) ss = fmaf(y[i], y[i], ss);
    sm.red[half][row] = ss;
    __syncthreads();
    const float nk = sqrtf(sm.red[0][row] + sm.red[1][row]) * (1.0f / kSqrtD);
    const __half nk16 = __float2half_rn(nk);
    if (valid && half == 0 && __hisinf(nk16)) report(a.status, TQ_ERR_OVERFLOW);
    const float kinv = nk > 0.f ? 1.0f / (nk * kSqrtD) : 0.f;
    uint32_t kw[8] = {0, 0, 0, 0, 0, 0, 0, 0};  // this half's key words
    const float cs = kSqrtD * __half2float(nk16);
    float rr = 0.f;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      int s;
      const int r = rank_of<HK - 1>(y[i] * kinv, kpos, s);
      const int j = 64 * half + i;  // coordinate
      if (KQ && KB == 3) {
        kw[i >> 3] |= (uint32_t)(r | (s << 2)) << (4 * (i & 7));
      } else if (KB == 2) {
        kw[i >> 4] |= (uint32_t)(r | (s << 1)) << (2 * (i & 15));
      } else if (KB == 3) {
        kw[i >> 4] |= (uint32_t)r << (2 * (i & 15));
        const int p = sign_plane_pos(j) - 64 * half;
        kw[4 + (p >> 5)] |= (uint32_t)s << (p & 31);
      } else if (KB == 4) {
        kw[i >> 3] |= (uint32_t)(r | (s << 3)) << (4 * (i & 7));
      } else {
        kw[i >> 5] |= (uint32_t)s << (i & 31);
      }
      if (KQ) {
        float c = kmag[0];
#pragma unroll
        for (int m = 1; m < HK; ++m) c = (r == m) ? kmag[m] : c;
        const float rv = fmaf(-cs, s ? c : -c, y[i]);
        y[i] = rv;
        rr = fmaf(rv, rv, rr);
      }
    }
    if (KQ) {
      // r_rot' hi and lo halves into tensor memory (A operand of the sketch MMAs)
      uint32_t hi[32], lo[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const __half2 h2 = __floats2half2_rn(y[2 * i], y[2 * i + 1]);
        const float2 hf = __half22float2(h2);
        const __half2 l2 = __floats2half2_rn(y[2 * i] - hf.x, y[2 * i + 1] - hf.y);
        hi[i] = *reinterpret_cast<const uint32_t*>(&h2);
        lo[i] = *reinterpret_cast<const uint32_t*>(&l2);
      }
      tmem_st32(tmem + lane_base + kColAhi + 32 * half, hi);
      tmem_st32(tmem + lane_base + kColAlo + 32 * half, lo);
      tmem_wait_st();
      sm.red[half][row] = rr;
    }
    tc_fence_before();
    __syncthreads();
    float rho = 0.f;
    if (KQ) {
      rho = sqrtf(sm.red[0][row] + sm.red[1][row]) * (1.0f / kSqrtD);
      if (tid == 0) {
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          mma_ts(tmem + kColS, tmem + kColAhi + 8 * ks, smem_desc(sm.bshi, ks), ks > 0);
          mma_ts(tmem + kColS, tmem + kColAhi + 8 * ks, smem_desc(sm.bslo, ks), 1);
          mma_ts(tmem + kColS, tmem + kColAlo + 8 * ks, smem_desc(sm.bshi, ks), 1);
        }
        mma_commit(&sm.bar_sig);
      }
      sig_out = true;
    }

    // ======== values (overlaps the sketch MMAs) ========
    {
      float v[32];
      tmem_ld32(tmem + lane_base + kColV + 64 * half, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) y[i] = v[i];
      tmem_ld32(tmem + lane_base + kColV + 64 * half + 32, v);
#pragma unroll
      for (int i = 0; i < 32; ++i) y[32 + i] = v[i];
      tmem_wait_ld();
    }
    ss = 0.f;
#pragma unroll
    for (int i = 0; i < 64; ++i) ss = fmaf(y[i], y[i], ss);
    __syncthreads();  // every thread has read the key rho partials
    sm.red[half][row] = ss;
    __syncthreads();
    const float nv = sqrtf(sm.red[0][row] + sm.red[1][row]) * (1.0f / kSqrtD);
    const __half nv16 = __float2half_rn(nv);
    if (valid && half == 0 && __hisinf(nv16)) report(a.status, TQ_ERR_OVERFLOW);
    const float vinv = nv > 0.f ? 1.0f / (nv * kSqrtD) : 0.f;
    uint32_t vw[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
    for (int i = 0; i < 64; ++i) {
      int s;
      const int r = rank_of<HV - 1>(y[i] * vinv, vpos, s);
      const int j = 64 * half + i;
      if (VB == 2) {
        vw[i >> 4] |= (uint32_t)(r | (s << 1)) << (2 * (i & 15));
      } else if (VB == 3) {
        vw[i >> 4] |= (uint32_t)r << (2 * (i & 15));
        const int p = sign_plane_pos(j) - 64 * half;
        vw[4 + (p >> 5)] |= (uint32_t)s << (p & 31);
      } else if (VB == 4) {
        vw[i >> 3] |= (uint32_t)(r | (s << 3)) << (4 * (i & 7));
      } else {
        vw[i >> 5] |= (uint32_t)s << (i & 31);
      }
    }
    if (valid) {
      uint4* vc = reinterpret_cast<uint4*>(blk + L.vc);
      if (VB == 2) {
        vc[half * PT + slot] = make_uint4(vw[0], vw[1], vw[2], vw[3]);
      } else if (VB == 3) {
        vc[half * PT + slot] = make_uint4(vw[0], vw[1], vw[2], vw[3]);
        *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(vc + 2 * PT + slot) + 8 * half) = make_uint2(vw[4], vw[5]);
      } else if (VB == 4) {
        vc[(2 * half) * PT + slot] = make_uint4(vw[0], vw[1], vw[2], vw[3]);
        vc[(2 * half + 1) * PT + slot] = make_uint4(vw[4], vw[5], vw[6], vw[7]);
      } else {
        *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(vc + slot) + 8 * half) = make_uint2(vw[0], vw[1]);
      }
      if (half == 0) reinterpret_cast<__half*>(blk + L.vn)[slot] = nv16;
    }

    // ======== QJL signs, then the key words ========
    if (KQ) {
      if (!bar_wait(&sm.bar_sig, ph_sig)) {
        if (tid == 0) report(a.status, TQ_ERR_TIMEOUT);
        break;
      }
      ph_sig ^= 1;
      sig_out = false;
      tc_fence_after();
      uint32_t sgw[2] = {0, 0};
#pragma unroll
      for (int part = 0; part < 2; ++part) {
        float v[32];
        tmem_ld32(tmem + lane_base + kColS + 64 * half + 32 * part, v);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const uint32_t bit = v[i] >= 0.f ? 1u : 0u;
          const int ii = 32 * part + i;
          if (KB == 3)
            kw[ii >> 3] |= bit << (4 * (ii & 7) + 3);
          else
            sgw[part] |= bit << i;
        }
      }
      if (valid) {
        uint4* kc = reinterpret_cast<uint4*>(blk + L.kc);
        if (KB == 3) {
          kc[(2 * half) * PT + slot] = make_uint4(kw[0], kw[1], kw[2], kw[3]);
          kc[(2 * half + 1) * PT + slot] = make_uint4(kw[4], kw[5], kw[6], kw[7]);
        } else {
          kc[half * PT + slot] = make_uint4(kw[0], kw[1], kw[2], kw[3]);
          *reinterpret_cast<uint2*>(blk + L.ks + (size_t)slot * 16 + 8 * half) = make_uint2(sgw[0], sgw[1]);
        }
        if (half == 0) reinterpret_cast<__half*>(blk + L.kr)[slot] = __float2half_rn(rho);
      }
    } else if (valid) {
      uint4* kc = reinterpret_cast<uint4*>(blk + L.kc);
      if (KB == 2) {
        kc[half * PT + slot] = make_uint4(kw[0], kw[1], kw[2], kw[3]);
      } else if (KB == 3) {
        kc[half * PT + slot] = make_uint4(kw[0], kw[1], kw[2], kw[3]);
        *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(kc + 2 * PT + slot) + 8 * half) = make_uint2(kw[4], kw[5]);
      } else if (KB == 4) {
        kc[(2 * half) * PT + slot] = make_uint4(kw[0], kw[1], kw[2], kw[3]);
        kc[(2 * half + 1) * PT + slot] = make_uint4(kw[4], kw[5], kw[6], kw[7]);
      } else {
        *reinterpret_cast<uint2*>(reinterpret_cast<uint8_t*>(kc + slot) + 8 * half) = make_uint2(kw[0], kw[1]);
      }
    }
    if (valid && half == 0) reinterpret_cast<__half*>(blk + L.kn)[slot] = nk16;
    // all tensor-memory reads of this tile are done before the next tile's MMAs
    tc_fence_before();
    __syncthreads();
  }
  // normal exit leaves nothing outstanding; after a timeout, wait (bounded) for the copy
  // and the MMAs still in flight before the shared and tensor memory go away
  if (load_out) bar_wait(&sm.bar_load, ph_load);
  if (fwd_out) bar_wait(&sm.bar_fwd, ph_fwd);
  if (sig_out) bar_wait(&sm.bar_sig, ph_sig);
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
// (8 rows of 16 bytes make the 128-byte core-matrix group stride).
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
  const size_t smem = sizeof(SmemTC) + 1024;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int tiles = a.cache.batch * a.cache.kv_heads * ((a.max_len + TT - 1) / TT);
  const int grid = tiles < sms ? tiles : sms;
  if (grid == 0) return cudaSuccess;
  k<<<grid, kThreadsTC, smem, stream>>>(a, mk, mv);
  return cudaGetLastError();
}

}  // namespace

bool compress_tc_supported(const CompressArgs& a) {
  const Layout& L = a.cache.L;
  if (a.dense || a.in_dtype != TQ_F16) return false;
  if ((size_t)a.cache.batch * a.cache.kv_heads * a.max_len >= (1ull << 31)) return false;
  if (L.qjl && !(L.kbits == 2 || L.kbits == 3)) return false;
  if (!L.qjl && !(L.kbits >= 1 && L.kbits <= 4)) return false;
  if (!(L.vbits >= 2 && L.vbits <= 3)) return false;
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
  TQ_TC(3, 1, 3)
  TQ_TC(3, 1, 2)
  TQ_TC(2, 1, 2)
  TQ_TC(2, 1, 3)
  TQ_TC(1, 0, 3)
  TQ_TC(2, 0, 3)
  TQ_TC(3, 0, 3)
  TQ_TC(4, 0, 3)
  TQ_TC(1, 0, 2)
  TQ_TC(2, 0, 2)
  TQ_TC(3, 0, 2)
  TQ_TC(4, 0, 2)
#undef TQ_TC
  return cudaErrorInvalidValue;
}

}  // namespace tqk
