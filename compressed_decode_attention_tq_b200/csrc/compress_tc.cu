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
// scales its boundaries once instead of normalising every coordinate; the rank is a sum
// of saturated unit steps (the boundaries are sorted), and the residual's centroid is read
// from a table by the code field just formed.
//
// One persistent CTA per SM: 8 compute warps and a producer warpgroup.  Compute warp w
// reads tensor-memory lane quadrant w % 4 (tokens 32 (w % 4) .. + 31) and coordinates
// 64 (w / 4) .. + 63, so two warps share a token; their per-token sums (norms, residual
// norm) meet in spare tensor-memory columns behind a 64-thread named barrier.  One thread
// of the producer warpgroup issues the TMA copies (two K/V tile stages), the MMAs and their
// commits; the compute warps hand tensor-memory columns back through mbarriers.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tq_device.cuh"
#include "tq_kernels.h"

namespace tqk {

namespace {

constexpr int TT = 128;                      // tokens per tile
constexpr int kComputeWarps = 8;
constexpr int kCPT = 64;  // coordinates per compute thread
// two compute warpgroups and one producer warpgroup (one thread of which issues the copies
// and MMAs); registers move from the producer to the compute warpgroups after launch:
// launched with 384 x 168, then 128 x 72 + 256 x 216 = 64512 = 384 x 168.
constexpr int kThreadsTC = (kComputeWarps + 4) * 32;
constexpr int kRegsLaunch = 168, kRegsProducer = 72, kRegsCompute = 216;
static_assert(128 * kRegsProducer + 32 * kComputeWarps * kRegsCompute <= kThreadsTC * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr int kTileBytes = TT * D * 2;       // one 128 x 128 fp16 operand
// Tensor-memory columns.  KS[0], KS[1]: y'_K of a tile (alternate tiles, alternate
// blocks); as each 32-coordinate chunk of it is read, the chunk's scaled residual is
// written in its place as fp16 hi (first 16 columns) and lo (next 16): the sketch's A
// operand.  V: y'_V of a tile.  X: the sketch (S D H) a r_rot' of a tile, then (+0, +1) the
// residual sums of the two warps of a token.
constexpr uint32_t kColKS0 = 0, kColKS1 = 128, kColV = 256, kColX = 384;
constexpr uint32_t kTmemCols = 512;
// instruction descriptor: D f32, A and B f16, both K-major, N = 128, M = 128
constexpr uint32_t kIdesc = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr unsigned long long kWaitNs = 1000000000ull;  // a wait gives up after 1 s
constexpr float kSqrtD = 11.313708498984761f;

struct SmemTC {
  unsigned char x[2][2][kTileBytes];  // [stage][K, V] input tiles (canonical layout); S at set-up
  unsigned char bhd[kTileBytes];      // B = H D
  unsigned char bshi[kTileBytes];     // B = S D H, fp16 hi part
  unsigned char bslo[kTileBytes];     // fp16 lo part
  unsigned long long bar_load[2], stage_free[2], bar_fwdk, bar_fwdv, bar_sig, ks_free, a_ready, v_free, bar_setup;
  uint32_t tmem_base;
  int bad_s;
  float kc[16], kb[16], vc[16], vb[16];  // codebooks: centroids, boundaries
  float kcode_c[8];                      // c[idx] of a key code field r + sw s
  float2 red[TT][2];                     // per-token sums of the two warps of a token
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
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, 1000000;\n"
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

// Wait for the phase with the given parity to complete (each poll may suspend the thread
// for up to 1 ms until it does); false after kWaitNs without completion, or after 2^24
// polls.
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

// 64-thread barrier of the two compute warps that share a tensor-memory lane quadrant
__device__ __forceinline__ void pair_sync(int qd) {
  asm volatile("bar.sync %0, 64;" ::"r"(1 + qd) : "memory");
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

__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float (&v)[4]) {
  uint32_t r[4];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(taddr));
#pragma unroll
  for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}

__device__ __forceinline__ void tmem_ld2(uint32_t taddr, float (&v)[2]) {
  uint32_t r0, r1;
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x2.b32 {%0,%1}, [%2];" : "=r"(r0), "=r"(r1) : "r"(taddr));
  v[0] = __uint_as_float(r0);
  v[1] = __uint_as_float(r1);
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

// ---- packed fp32 pairs (two coordinates per instruction) and saturated steps ----
typedef unsigned long long f2_t;
__device__ __forceinline__ f2_t f2(float a, float b) {
  f2_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(a), "f"(b));
  return r;
}
__device__ __forceinline__ f2_t f2s(float a) { return f2(a, a); }
__device__ __forceinline__ void uf2(f2_t p, float& a, float& b) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(a), "=f"(b) : "l"(p));
}
__device__ __forceinline__ f2_t fma2(f2_t a, f2_t b, f2_t c) {
  f2_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}
__device__ __forceinline__ f2_t mul2(f2_t a, f2_t b) {
  f2_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f2_t add2(f2_t a, f2_t b) {
  f2_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
// clamp(a b + c, 0, 1): a unit step of a b + c once it is scaled far past 1
__device__ __forceinline__ float fma_sat(float a, float b, float c) {
  float d;
  asm("fma.rn.sat.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float mul_sat(float a, float b) {
  float d;
  asm("mul.rn.sat.f32 %0, %1, %2;" : "=f"(d) : "f"(a), "f"(b));
  return d;
}

// sum of squares of 32 values, two lanes of packed fp32 at a time
__device__ __forceinline__ float sumsq32(const float (&v)[32]) {
  f2_t acc = 0;
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const f2_t p = f2(v[i], v[i + 1]);
    acc = fma2(p, p, acc);
  }
  float lo, hi;
  uf2(acc, lo, hi);
  return lo + hi;
}

// Integer codes are assembled in the mantissa of 2^23 + code (exact for 0 <= code < 2^23)
// and shifted into place with an integer multiply-add; the 2^23 exponent bits each
// coordinate drags along are subtracted up front (mod 2^32).
constexpr float kMagic = 8388608.f;
constexpr uint32_t kMagicBits = 0x4B000000u;
__host__ __device__ constexpr uint32_t magic_at(int sh) {
  return (uint32_t)(((unsigned long long)kMagicBits << sh) & 0xFFFFFFFFull);
}

// Bit of coordinate e (0..31) of a 32-coordinate group in the sign plane of 3-bit codes
// (the permutation of sign_plane_pos, which the decode's byte tables read).
__host__ __device__ constexpr int plane_bit(int e) { return 4 * (e >> 3) + (e & 3) + 16 * ((e >> 2) & 1); }

// Where coordinate i (0..31 of one 32-coordinate chunk) of a b-bit code lands in the
// chunk's four words.  Field = r + sw * s:
//   b = 2: 2-bit r | s << 1 (words 0, 1);  b = 3: 2-bit r (words 0, 1) and s in word 2 at
//   the permuted sign-plane bit;  b = 4: r | s << 3 (words 0..3);  merged 3-bit key:
//   r | s << 2 | sigma << 3 (words 0..3).
template <int B, bool MERGED>
struct Fields {
  static constexpr bool nib = MERGED || B == 4;
  static constexpr int sw = MERGED ? 4 : (B == 2 ? 2 : (B == 3 ? 0 : 8));
  static constexpr bool plane = !MERGED && B == 3;
  __host__ __device__ static constexpr int word(int i) { return nib ? (i >> 3) : (i >> 4); }
  __host__ __device__ static constexpr int shift(int i) { return nib ? 4 * (i & 7) : 2 * (i & 15); }
  // minus the magic bits the code (and, merged, sigma) adds of every coordinate of word w
  __host__ __device__ static constexpr uint32_t init(int w) {
    uint32_t c = 0;
    for (int i = 0; i < 32; ++i) {
      if (word(i) == w) c += magic_at(shift(i)) * (MERGED ? 2u : 1u);
      if (plane && w == 2) c += magic_at(plane_bit(i));
    }
    return 0u - c;
  }
  __host__ __device__ static constexpr uint32_t sig_init() {
    uint32_t c = 0;
    for (int i = 0; i < 32; ++i) c += magic_at(i);
    return 0u - c;
  }
};

// Store the words of one chunk (coordinates 64 part + 32 c .. + 31) of a token slot
// (plane p = 16 bytes per slot).
template <int B, bool MERGED>
__device__ __forceinline__ void store_chunk(uint8_t* base, int part, int c, int slot, const uint4& w) {
  if constexpr (B == 2 || (B == 3 && !MERGED)) {
    *reinterpret_cast<uint2*>(base + ((size_t)part * PT + slot) * 16 + 8 * c) = make_uint2(w.x, w.y);
    if constexpr (B == 3) *reinterpret_cast<uint32_t*>(base + ((size_t)2 * PT + slot) * 16 + 4 * (2 * part + c)) = w.z;
  } else {
    *reinterpret_cast<uint4*>(base + ((size_t)(2 * part + c) * PT + slot) * 16) = w;
  }
}

// Boundary scales of one token: |y| > beta ||y'||  <=>  bs |y'| - bs beta ||y'|| > 0 with
// bs = 2^(40 - e) for ||y'|| ~ 2^e: one fused multiply-add of |y'| (exact product, one
// rounding, so the sign is exact), saturated to [0, 1], is a unit step outside a 2^-40
// relative band; bs y' saturated is the step s = [y' > 0].
struct TokScale {
  int e;
  float bs;
  __device__ __forceinline__ explicit TokScale(float ny) {
    e = min(max((int)((__float_as_uint(ny) >> 23) & 0xff) - 127, -40), 40);
    bs = __uint_as_float((uint32_t)(127 + 40 - e) << 23);
  }
};

// Per-token constants of the quantiser: the scaled boundaries, and with QJL the residual
// scale a = 2^(8 - e) and a sqrt(d) fp16(||x||).
template <int NB>
struct QuantConst {
  TokScale ts;
  float tb[NB > 0 ? NB : 1];  // -bs beta_k ||y'||
  float alpha, inv_alpha, csa;
  __device__ __forceinline__ QuantConst(float ny, const float* pos, float cnorm) : ts(ny) {
#pragma unroll
    for (int k = 0; k < NB; ++k) tb[k] = -(pos[k] * ny) * ts.bs;
    alpha = __uint_as_float((uint32_t)(127 + 8 - ts.e) << 23);
    inv_alpha = __uint_as_float((uint32_t)(127 - 8 + ts.e) << 23);
    csa = alpha * kSqrtD * cnorm;
  }
};

// Codes of one 32-coordinate chunk of y' into the chunk's words w; with KQ also the scaled
// residual a y' - a sqrt(d) fp16(||x||) c[idx] (c[idx] read from the table of signed
// centroids by the code just formed) split into fp16 hi / lo pairs for the sketch MMAs, and
// its sum of squares (accumulated into rr2).
template <int NB, class F, bool KQ>
__device__ __forceinline__ void quantise32(const float (&y)[32], const QuantConst<NB>& qc, const float* ctab,
                                           uint32_t (&w)[4], uint32_t (&hi)[16], uint32_t (&lo)[16], f2_t& rr2) {
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const float y0 = y[i], y1 = y[i + 1];
    f2_t sum = f2s(kMagic);
#pragma unroll
    for (int k = 0; k < NB; ++k)
      sum = add2(sum, f2(fma_sat(fabsf(y0), qc.ts.bs, qc.tb[k]), fma_sat(fabsf(y1), qc.ts.bs, qc.tb[k])));
    const f2_t S = f2(mul_sat(y0, qc.ts.bs), mul_sat(y1, qc.ts.bs));  // s = [y' > 0]
    if (F::sw) sum = fma2(S, f2s((float)F::sw), sum);
    float c0, c1;
    uf2(sum, c0, c1);
    const uint32_t code0 = __float_as_uint(c0), code1 = __float_as_uint(c1);
    w[F::word(i)] += code0 << F::shift(i);
    w[F::word(i + 1)] += code1 << F::shift(i + 1);
    if (F::plane) {
      uf2(add2(S, f2s(kMagic)), c0, c1);
      w[2] += __float_as_uint(c0) << plane_bit(i);
      w[2] += __float_as_uint(c1) << plane_bit(i + 1);
    }
    if constexpr (KQ) {
      const f2_t C = f2(ctab[code0 & 7], ctab[code1 & 7]);
      const f2_t R = fma2(C, f2s(-qc.csa), mul2(f2(y0, y1), f2s(qc.alpha)));
      rr2 = fma2(R, R, rr2);
      float r0, r1;
      uf2(R, r0, r1);
      const float h0 = __uint_as_float(__float_as_uint(r0) & 0xFFFFE000u);
      const float h1 = __uint_as_float(__float_as_uint(r1) & 0xFFFFE000u);
      float l0, l1;
      uf2(fma2(f2(h0, h1), f2s(-1.f), R), l0, l1);
      const __half2 hh = __floats2half2_rn(h0, h1);
      const __half2 ll = __floats2half2_rn(l0, l1);
      hi[i >> 1] = *reinterpret_cast<const uint32_t*>(&hh);
      lo[i >> 1] = *reinterpret_cast<const uint32_t*>(&ll);
    }
  }
}

// QJL signs sigma = [p >= 0] (1 also within 2^-40 below 0) of one 32-entry chunk of the
// sketch: merged into bit 3 of the chunk's key nibbles, or one sign-plane word.
template <bool MERGED, class F>
__device__ __forceinline__ void sigma32(const float (&p)[32], uint4& w, uint32_t& sgw) {
  uint32_t wa[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    const f2_t G = f2(fma_sat(p[i], 1099511627776.f, 1.f), fma_sat(p[i + 1], 1099511627776.f, 1.f));
    float c0, c1;
    if constexpr (MERGED) {
      uf2(fma2(G, f2s(8.f), f2s(kMagic)), c0, c1);
      wa[F::word(i)] += __float_as_uint(c0) << F::shift(i);
      wa[F::word(i + 1)] += __float_as_uint(c1) << F::shift(i + 1);
    } else {
      uf2(add2(G, f2s(kMagic)), c0, c1);
      sgw += __float_as_uint(c0) << i;
      sgw += __float_as_uint(c1) << (i + 1);
    }
  }
  w = make_uint4(wa[0], wa[1], wa[2], wa[3]);
}

// The cache block and slot of the token this thread owns in tile j (blk null when the
// token is past its sequence or its page is invalid; errors reported once, by part 0).
struct TokRef {
  uint8_t* blk;
  int slot;
};

template <int KB, int KQ, int VB>
__global__ void __launch_bounds__(kThreadsTC, 1)
    compress_tc_kernel(CompressArgs a, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const uint32_t pad = (128u - (s_u32(smem_raw) & 127u)) & 127u;
  SmemTC& sm = *reinterpret_cast<SmemTC*>(smem_raw + pad);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = warp >= kComputeWarps;  // the producer warpgroup
  const int qd = warp & 3;           // tensor-memory lane quadrant
  const int part = (warp >> 2) & 1;  // coordinates 64 part .. 64 part + 63
  const int row = 32 * qd + lane;    // token within the tile
  const Layout& L = a.cache.L;
  constexpr int HK = 1 << (KB - 1), HV = 1 << (VB - 1);
  constexpr bool kMerged = KQ && KB == 3;
  constexpr int kComputeThreads = kComputeWarps * 32;

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
    bar_init(&sm.stage_free[0], 1);
    bar_init(&sm.stage_free[1], 1);
    bar_init(&sm.bar_fwdk, 1);
    bar_init(&sm.bar_fwdv, 1);
    bar_init(&sm.bar_sig, 1);
    bar_init(&sm.ks_free, kComputeWarps);
    bar_init(&sm.a_ready, kComputeWarps);
    bar_init(&sm.v_free, kComputeWarps);
    bar_init(&sm.bar_setup, 1);
    sm.bad_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  // tile 0 streams in while the rotation operands are built (stage 1 is set-up scratch)
  if (warp == kComputeWarps + 1 && lane == 0 && my_tiles > 0) issue_load(0);
  __syncwarp();
  if (!producer) {
    // S (fp16-exact by contract) is requested first: lanes read consecutive 16-byte pieces
    // of a row (coalesced); it is converted and stored once the small tables are in
    constexpr int kSIter = QM * 16 / kComputeThreads;
    float4 sraw[KQ ? 2 * kSIter : 1];
    if (KQ) {
#pragma unroll
      for (int it = 0; it < kSIter; ++it) {
        const int c = tid + it * kComputeThreads;
        const float4* src = reinterpret_cast<const float4*>(a.s + (size_t)(c >> 4) * D + 8 * (c & 15));
        sraw[2 * it] = src[0];
        sraw[2 * it + 1] = src[1];
      }
    }
    // small inputs once into shared memory, one load per thread
    // D of the rotation, for the set-up only (in the space of the S D H operand, filled later)
    float* signs = reinterpret_cast<float*>(sm.bshi);
    if (tid < D) signs[tid] = a.signs[tid];
    if (tid < 16) {
      sm.kc[tid] = tid < 2 * HK ? a.k_centroids[tid] : 0.f;
      sm.kb[tid] = tid < 2 * HK - 1 ? a.k_boundaries[tid] : 0.f;
      sm.vc[tid] = tid < 2 * HV ? a.v_centroids[tid] : 0.f;
      sm.vb[tid] = tid < 2 * HV - 1 ? a.v_boundaries[tid] : 0.f;
    }
    asm volatile("bar.sync 5, %0;" ::"n"(kComputeThreads) : "memory");
    if (tid < 8) {
      // code field f = r + sw s (merged keys: r + 4 s; 2-bit: r + 2 s) -> c[s ? h + r : h - 1 - r]
      constexpr int sw = Fields<KB, kMerged>::sw > 0 ? Fields<KB, kMerged>::sw : HK;
      const int r = tid % sw, sg = tid / sw;
      sm.kcode_c[tid] = (sg <= 1 && r < HK) ? sm.kc[sg ? HK + r : HK - 1 - r] : 0.f;
    }
    if (tid == 0 && blockIdx.x == 0) {
      bool sym = true;
      for (int i = 0; i < 2 * HK; ++i) sym &= sm.kc[i] == -sm.kc[2 * HK - 1 - i];
      for (int i = 0; i < 2 * HV; ++i) sym &= sm.vc[i] == -sm.vc[2 * HV - 1 - i];
      // the rank rule reads only the positive boundaries: they must mirror, middle one 0
      for (int i = 0; i < 2 * HK - 1; ++i) sym &= sm.kb[i] == -sm.kb[2 * HK - 2 - i];
      for (int i = 0; i < 2 * HV - 1; ++i) sym &= sm.vb[i] == -sm.vb[2 * HV - 2 - i];
      if (!sym) report(a.status, TQ_ERR_INVALID_ARG);
    }
    // B = H D: row i, column k = (-1)^popcount(i & k) D_k
#pragma unroll
    for (int it = 0; it < D * 16 / kComputeThreads; ++it) {
      const int c = tid + it * kComputeThreads;
      const int i = c & 127, ch = c >> 7;
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k0 = ch * 8 + 2 * e;
        const float s0 = signs[k0], s1 = signs[k0 + 1];
        const float v0 = (__popc(i & k0) & 1) ? -s0 : s0;
        const float v1 = (__popc(i & (k0 + 1)) & 1) ? -s1 : s1;
        const __half2 h = __floats2half2_rn(v0, v1);
        w[e] = *reinterpret_cast<const uint32_t*>(&h);
      }
      *reinterpret_cast<uint4*>(sm.bhd + canon(i, ch * 8)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    if (KQ) {
      // S as an fp16 A operand in stage 1; S D H = S (H D)^T is then one MMA against the
      // B = H D operand above
      unsigned char* sa = sm.x[1][0];
      int bad = 0;
#pragma unroll
      for (int it = 0; it < kSIter; ++it) {
        const int c = tid + it * kComputeThreads;
        const int m = c >> 4, ch = c & 15;
        const float4 q0 = sraw[2 * it], q1 = sraw[2 * it + 1];
        const float e[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
        uint32_t w[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const __half2 h = __floats2half2_rn(e[2 * u], e[2 * u + 1]);
          const float2 hf = __half22float2(h);
          if (hf.x != e[2 * u] || hf.y != e[2 * u + 1]) bad = 1;
          w[u] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(sa + canon(m, 8 * ch)) = make_uint4(w[0], w[1], w[2], w[3]);
      }
      if (bad) sm.bad_s = 1;
    }
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  __syncthreads();
  if (tid == 0 && sm.bad_s) report(a.status, TQ_ERR_INVALID_ARG);
  const uint32_t tmem = sm.tmem_base;

  if (producer) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
    // ---------------- producer: MMAs (warp 8) and copies (warp 9) ----------------
    // MMAs of tile j: forward K into KS[j & 1] once KS[(j - 2) & 1] is released (its sketch
    // read, or without QJL its exchange done); the sketch into KS[j & 1] once the compute
    // warps have written A; forward V into V once the previous y'_V is read.  Copies: tile
    // j + 2 into stage j & 1 as soon as both forward MMAs of tile j have read it.  Each wait's
    // phase is one the other side cannot run two phases past.
    if (warp == kComputeWarps && lane == 0 && KQ) {
      // S D H into KS[1] (free until tile 1): read out by the compute warps before tile 0
      tc_fence_after();
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) mma_ss(tmem + kColKS1, smem_desc(sm.x[1][0], ks), smem_desc(sm.bhd, ks), ks > 0);
      mma_commit(&sm.bar_setup);
    }
    if (warp == kComputeWarps && lane == 0 && my_tiles > 0) {
      auto fwd = [&](int j, uint32_t dcol, int kv) {
#pragma unroll
        for (int ks = 0; ks < 8; ++ks)
          mma_ss(tmem + dcol, smem_desc(sm.x[j & 1][kv], ks), smem_desc(sm.bhd, ks), ks > 0);
      };
      bool ok = bar_wait(&sm.bar_load[0], 0);
      if (ok) {
        tc_fence_after();
        fwd(0, kColKS0, 0);
        mma_commit(&sm.bar_fwdk);
        fwd(0, kColV, 1);
        mma_commit(&sm.bar_fwdv);
        mma_commit(&sm.stage_free[0]);
      }
      for (int j = 0; j < my_tiles && ok; ++j) {
        const uint32_t ks_j = (j & 1) ? kColKS1 : kColKS0;
        if (j + 1 < my_tiles) {
          // y'_V of tile j has been read (v_free phase j arrives after each compute warp has
          // waited for it and read it): the next one may land
          if (!(ok = bar_wait(&sm.v_free, j & 1))) break;
          if (!(ok = bar_wait(&sm.bar_load[(j + 1) & 1], ((j + 1) >> 1) & 1))) break;
          tc_fence_after();
          fwd(j + 1, kColV, 1);
          mma_commit(&sm.bar_fwdv);
          // KS[(j + 1) & 1] holds tile j - 1's A: its sketch must be done with it (this thread
          // issued it and consumes each sketch commit in turn); ks_free phase j arrives after
          // every compute warp has waited for y'_K of tile j
          if (KQ && j >= 1 && !(ok = bar_wait(&sm.bar_sig, (j - 1) & 1))) break;
          if (!(ok = bar_wait(&sm.ks_free, j & 1))) break;
          tc_fence_after();
          fwd(j + 1, (j & 1) ? kColKS0 : kColKS1, 0);
          mma_commit(&sm.bar_fwdk);
          mma_commit(&sm.stage_free[(j + 1) & 1]);  // both forward MMAs of tile j + 1 read it
        }
        if (KQ) {
          // A of tile j is in KS[j & 1] and X is free (the previous sketch was read)
          if (!(ok = bar_wait(&sm.a_ready, j & 1))) break;
          tc_fence_after();
#pragma unroll
          for (int ks = 0; ks < 8; ++ks) {
            // coordinates 16 ks ..: part ks / 4, chunk (ks / 2) % 2, half ks % 2
            const uint32_t ahi = tmem + ks_j + 64 * (ks >> 2) + 32 * ((ks >> 1) & 1) + 8 * (ks & 1);
            mma_ts(tmem + kColX, ahi, smem_desc(sm.bshi, ks), ks > 0);
            mma_ts(tmem + kColX, ahi, smem_desc(sm.bslo, ks), 1);
            mma_ts(tmem + kColX, ahi + 16, smem_desc(sm.bshi, ks), 1);
          }
          mma_commit(&sm.bar_sig);
        }
      }
      if (!ok) {
        report(a.status, TQ_ERR_TIMEOUT);
        // let the MMAs already issued finish (bounded) before tensor memory is freed
        mma_commit(&sm.bar_setup);
        bar_wait(&sm.bar_setup, KQ ? 1 : 0);
      }
    } else if (warp == kComputeWarps + 1 && lane == 0 && my_tiles > 0) {
      int issued = 1;  // tile 0 went out before the set-up
      bool ok = true;
      // stage 1 holds S until the S D H MMA has read it
      if (KQ && !(ok = bar_wait(&sm.bar_setup, 0))) report(a.status, TQ_ERR_TIMEOUT);
      if (ok && my_tiles > 1) {
        issue_load(1);
        issued = 2;
      }
      for (int i = 0; ok && i + 2 < my_tiles; ++i) {
        // phase i >> 1 of stage_free[i & 1]: the forward MMAs of tile i are done with it
        if (!(ok = bar_wait(&sm.stage_free[i & 1], (i >> 1) & 1))) break;
        issue_load(i + 2);
        issued = i + 3;
      }
      if (!ok) report(a.status, TQ_ERR_TIMEOUT);
      // the last copy into each stage is that stage's final phase: wait (bounded) for both to
      // land so that no copy is still in flight when the shared memory goes away
      for (int i = (issued > 2 ? issued - 2 : 0); i < issued; ++i) bar_wait(&sm.bar_load[i & 1], (i >> 1) & 1);
    }
    __syncwarp();
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsCompute));
    // ---------------- compute warps ----------------
    typedef Fields<KB, kMerged> FK;
    typedef Fields<VB, false> FV;
    const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
    auto token_ref = [&](int j) -> TokRef {
      int b, h, t0;
      tile_coords(j, b, h, t0);
      const int len = a.seq_lens[b];
      const int tok = t0 + row;
      const bool bad_len = len < 0 || len > a.max_len || len > a.cache.max_pages * PT;
      if (bad_len && tid == 0 && t0 == 0) report(a.status, TQ_ERR_BOUNDS);
      TokRef r{nullptr, tok % PT};
      if (!bad_len && tok < len) {
        const int phys = a.cache.block_table[(size_t)b * a.cache.max_pages + tok / PT];
        if (phys < 0 || phys >= a.cache.num_pages) {
          if (part == 0) report(a.status, TQ_ERR_BOUNDS);
        } else {
          r.blk = a.cache.block(phys, h);
        }
      }
      return r;
    };
    // per-token sum over the two warps of a token, through shared memory; the barrier
    // before the write keeps the partner's reads of the previous use ahead of it
    auto pair_sum2 = [&](float u, float v) -> float2 {
      pair_sync(qd);
      sm.red[row][part] = make_float2(u, v);
      pair_sync(qd);
      const float2 a0 = sm.red[row][0], a1 = sm.red[row][1];
      return make_float2(a0.x + a1.x, a0.y + a1.y);
    };
    // key words of the previous tile, completed by its sketch signs one tile later
    TokRef prev{nullptr, 0};
    uint4 pk[2] = {make_uint4(0, 0, 0, 0), make_uint4(0, 0, 0, 0)};
    uint32_t pnorms = 0;  // fp16 ||k|| | fp16 rho << 16
    // the previous tile's signs from X, chunk by chunk, and its key words stored
    auto finish_keys = [&]() {
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float sk[32];
        tmem_ld32(tmem + lane_base + kColX + kCPT * part + 32 * c, sk);
        tmem_wait_ld();
        uint4 w = c ? pk[1] : pk[0];
        uint32_t sgw = FK::sig_init();
        sigma32<kMerged, FK>(sk, w, sgw);
        if (prev.blk != nullptr) {
          store_chunk<KB, kMerged>(prev.blk + L.kc, part, c, prev.slot, w);
          if (!kMerged) *reinterpret_cast<uint32_t*>(prev.blk + L.ks + (size_t)prev.slot * 16 + 4 * (2 * part + c)) = sgw;
        }
      }
      if (prev.blk != nullptr && part == 0) {
        reinterpret_cast<uint16_t*>(prev.blk + L.kn)[prev.slot] = (uint16_t)(pnorms & 0xffff);
        reinterpret_cast<uint16_t*>(prev.blk + L.kr)[prev.slot] = (uint16_t)(pnorms >> 16);
      }
    };
    bool failed = false;
    if constexpr (KQ) {
      // S D H (fp32 in KS[1], row = sketch index) split into the fp16 hi / lo B operands
      if (!bar_wait(&sm.bar_setup, 0)) failed = true;
      __syncwarp();
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float v[32];
        tmem_ld32(tmem + lane_base + kColKS1 + kCPT * part + 32 * c, v);
        tmem_wait_ld();
#pragma unroll
        for (int g = 0; g < 4; ++g) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = v[8 * g + 2 * e], x1 = v[8 * g + 2 * e + 1];
            const __half2 h2 = __floats2half2_rn(x0, x1);
            const float2 hf = __half22float2(h2);
            const __half2 l2 = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
            hi[e] = *reinterpret_cast<const uint32_t*>(&h2);
            lo[e] = *reinterpret_cast<const uint32_t*>(&l2);
          }
          const int k = kCPT * part + 32 * c + 8 * g;
          *reinterpret_cast<uint4*>(sm.bshi + canon(row, k)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(sm.bslo + canon(row, k)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      // visible to the sketch MMAs, which wait for a_ready after these writes
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
    }
    // the token address of the next tile is looked up one tile ahead
    TokRef next = my_tiles > 0 ? token_ref(0) : TokRef{nullptr, 0};
    for (int j = 0; j < my_tiles; ++j) {
      const TokRef cur = next;
      if (j + 1 < my_tiles) next = token_ref(j + 1);
      const uint32_t ks_j = (j & 1) ? kColKS1 : kColKS0;

      // ---- norms of y'_K and y'_V ----
      if (!failed && !bar_wait(&sm.bar_fwdk, j & 1)) failed = true;
      if (!failed && !bar_wait(&sm.bar_fwdv, j & 1)) failed = true;
      __syncwarp();
      tc_fence_after();
      if (lane == 0) bar_arrive(&sm.ks_free);  // this warp is past its wait for y'_K of tile j
      float ssk = 0.f, ssv = 0.f;
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float y[32], z[32];
        tmem_ld32(tmem + lane_base + ks_j + kCPT * part + 32 * c, y);
        tmem_ld32(tmem + lane_base + kColV + kCPT * part + 32 * c, z);
        tmem_wait_ld();
        ssk += sumsq32(y);
        ssv += sumsq32(z);
      }
      const float2 ss = pair_sum2(ssk, ssv);
      const float nyk = sqrtf(ss.x);  // ||y'_K|| = sqrt(d) ||k||
      const float nyv = sqrtf(ss.y);
      const __half nk16 = __float2half_rn(nyk * (1.0f / kSqrtD));
      const __half nv16 = __float2half_rn(nyv * (1.0f / kSqrtD));
      if (cur.blk && part == 0 && (__hisinf(nk16) || __hisinf(nv16))) report(a.status, TQ_ERR_OVERFLOW);

      // ---- values and keys, chunk by chunk; the keys' residual goes to TMEM in place ----
      const QuantConst<HK - 1> qk(nyk, sm.kb + HK, __half2float(nk16));
      const QuantConst<HV - 1> qv(nyv, sm.vb + HV, 0.f);
      f2_t rr2 = 0;
      uint4 kwc[2];
#pragma unroll 1
      for (int c = 0; c < 2; ++c) {
        float y[32], z[32];
        tmem_ld32(tmem + lane_base + ks_j + kCPT * part + 32 * c, y);
        tmem_ld32(tmem + lane_base + kColV + kCPT * part + 32 * c, z);
        tmem_wait_ld();
        constexpr uint32_t vw0 = FV::init(0), vw1 = FV::init(1), vw2 = FV::init(2), vw3 = FV::init(3);
        constexpr uint32_t kw0 = FK::init(0), kw1 = FK::init(1), kw2 = FK::init(2), kw3 = FK::init(3);
        uint32_t vw[4] = {vw0, vw1, vw2, vw3}, kw[4] = {kw0, kw1, kw2, kw3};
        uint32_t hi[16], lo[16], dh[16], dl[16];
        f2_t drr = 0;
        quantise32<HV - 1, FV, false>(z, qv, sm.kcode_c, vw, dh, dl, drr);
        quantise32<HK - 1, FK, KQ != 0>(y, qk, sm.kcode_c, kw, hi, lo, rr2);
        if (cur.blk && !failed) store_chunk<VB, false>(cur.blk + L.vc, part, c, cur.slot, make_uint4(vw[0], vw[1], vw[2], vw[3]));
        const uint4 kq = make_uint4(kw[0], kw[1], kw[2], kw[3]);
        if constexpr (KQ) {
          tmem_st16(tmem + lane_base + ks_j + kCPT * part + 32 * c, hi);
          tmem_st16(tmem + lane_base + ks_j + kCPT * part + 32 * c + 16, lo);
          if (c) kwc[1] = kq; else kwc[0] = kq;
        } else if (cur.blk && !failed) {
          store_chunk<KB, false>(cur.blk + L.kc, part, c, cur.slot, kq);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) bar_arrive(&sm.v_free);  // y'_V of tile j is read
      if (cur.blk && !failed && part == 0) {
        reinterpret_cast<__half*>(cur.blk + L.vn)[cur.slot] = nv16;
        if (!KQ) reinterpret_cast<__half*>(cur.blk + L.kn)[cur.slot] = nk16;
      }

      if constexpr (KQ) {
        // the previous tile's sketch (in X) is done: its signs complete that tile's keys
        tmem_wait_st();
        if (j > 0) {
          if (!failed && !bar_wait(&sm.bar_sig, (j - 1) & 1)) failed = true;
          __syncwarp();
          tc_fence_after();
          if (failed) prev.blk = nullptr;
          finish_keys();
        }
        float ra, rb;
        uf2(rr2, ra, rb);
        const float rho = sqrtf(pair_sum2(ra + rb, 0.f).x) * qk.inv_alpha * (1.0f / kSqrtD);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(&sm.a_ready);  // A of tile j is written and X is free
        prev = failed ? TokRef{nullptr, 0} : cur;
        pk[0] = kwc[0];
        pk[1] = kwc[1];
        pnorms = (uint32_t)__half_as_ushort(nk16) | ((uint32_t)__half_as_ushort(__float2half_rn(rho)) << 16);
      }
    }
    if constexpr (KQ) {
      // the last tile's signs
      if (my_tiles > 0) {
        if (!failed && !bar_wait(&sm.bar_sig, (my_tiles - 1) & 1)) failed = true;
        __syncwarp();
        tc_fence_after();
        if (failed) prev.blk = nullptr;
        finish_keys();
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
  // the register hand-over inside the kernel assumes the launch allocation it was built for
  cudaFuncAttributes fa;
  if (cudaFuncGetAttributes(&fa, k) != cudaSuccess || fa.numRegs != kRegsLaunch ||
      fa.maxThreadsPerBlock < kThreadsTC)
    return cudaErrorInvalidValue;
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
