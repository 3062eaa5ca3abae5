// Compression on the tensor cores (tcgen05 + TMEM + TMA), randomized-Hadamard or dense
// Haar rotation.
//
// What is computed is the same as compress.cu ("TurboQuant explained", sections "How JL
// Matrices Evolved", "Coordinates Become Predictable After Rotation" and "Two-Stage
// Approach: MSE Approximation + QJL Correction"; "turboquant_cutile" function list:
// compress K = MSE + 1-bit QJL, compress V = MSE only).  The dense contractions run on
// the 5th-generation tensor cores:
//
//  * y' = (H D) x for a tile of 128 tokens: A = the fp16 input tile (exact), B = H D with
//    +-1 entries (exact), fp32 accumulation in tensor memory.  y = y' / ||y'||.
//  * With the dense rotation Pi ("turboquant_cutile" function list: Haar matrix from the QR
//    of a Gaussian) y' = (sqrt(d) Pi) x, the same scale as (H D) x: B = sqrt(d) Pi is held
//    as an fp16 hi + lo pair (prepared once per cache by prepare_dense_kernel), and two
//    MMAs per K step (x . hi, x . lo) accumulate y' to ~2^-22 relative.  Keys without QJL
//    only: the sketch's two more operand tiles would not fit beside the input stages.
//  * QJL sketch in the rotated domain: with R = H D / sqrt(d) orthogonal,
//      S r = S R^T R r = (S D H) r_rot' / d,   r_rot' = y' - sqrt(d) fp16(||x||) c[idx],
//    so sign(S r) = sign((S D H) a r_rot') for any a > 0.  S D H is held as an fp16 hi + lo
//    pair, prepared once per cache (prepare_operands_kernel, passed in as operands) or
//    formed by one MMA in every CTA; a r_rot' (scaled to O(1)) is split hi + lo as well;
//    three MMAs (hi.hi, hi.lo, lo.hi) give the projections to ~2^-22 relative.  They are
//    issued chunk by chunk as the keys' residual is written.
//
// Quantisation works on y' directly: |y| > beta  <=>  |y'| > beta ||y'||, so each token
// scales its boundaries once instead of normalising every coordinate; the rank is formed
// from saturated unit steps (a binary search for three positive boundaries), sign bits are
// placed in the packed words by sign-replicating byte permutes, and the residual's centroid
// is read from a table at the offset the rank's code bits hold.
//
// One persistent CTA per SM: two compute groups of four warps and a producer warpgroup.
// Group g takes the CTA's tiles g, g + 2, ... (ping-pong), so that one group's waits for
// its MMAs are covered by the other group's CUDA-core work.  Each thread owns one token
// (a tensor-memory lane: warp w reads lane quadrant w % 4) and all 128 of its coordinates,
// so no per-token sum crosses threads.  Each group has its own tensor-memory columns
// (y'_K, then the sketch's A operand in place; y'_V, then the sketch output) and its own
// MMA-issuing thread; one more producer thread issues the TMA copies into two stages.
#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>

#include "tq_device.cuh"
#include "tq_kernels.h"

namespace tqk {

namespace {

constexpr int TT = 128;                      // tokens per tile
constexpr int kComputeWarps = 8;
constexpr int kGroupWarps = 4;  // warps of one compute group (one tile)
// producer warpgroup: the MMA issuers of groups 0 and 1 and the copy issuer
constexpr int kIssuerWarp0 = kComputeWarps, kLoaderWarp = kComputeWarps + 1, kIssuerWarp1 = kComputeWarps + 2;
// two compute warpgroups and one producer warpgroup; registers move from the producer to
// the compute warpgroups after launch: launched with 384 x 168, then 128 x 72 + 256 x 216
// = 64512 = 384 x 168.
constexpr int kThreadsTC = (kComputeWarps + 4) * 32;
constexpr int kRegsLaunch = 168, kRegsProducer = 72, kRegsCompute = 216;
static_assert(kComputeWarps == 2 * kGroupWarps && kGroupWarps == 4, "two groups of four lane quadrants");
static_assert(128 * kRegsProducer + 32 * kComputeWarps * kRegsCompute <= kThreadsTC * kRegsLaunch,
              "register split exceeds the launch allocation");
constexpr int kTileBytes = TT * D * 2;       // one 128 x 128 fp16 operand
// Tensor-memory columns of group g, from kColGroup g: +0 y'_K of the group's tile; as each
// 32-coordinate chunk of it is read, the chunk's scaled residual is written in its place as
// fp16 hi (first 16 columns) and lo (next 16): the sketch's A operand.  +kColV: y'_V, then
// the sketch (S D H) a r_rot' once y'_V has been read.  At set-up S D H lands in group 1's
// y'_K columns.
constexpr uint32_t kColGroup = 256, kColV = 128;
constexpr uint32_t kTmemCols = 512;
// instruction descriptor: D f32, A and B f16, both K-major, N = 128, M = 128
constexpr uint32_t kIdesc = (1u << 4) | ((128u >> 3) << 17) | ((128u >> 4) << 24);
constexpr unsigned long long kWaitNs = 1000000000ull;  // a wait gives up after 1 s
constexpr float kSqrtD = 11.313708498984761f;

struct SmemTC {
  unsigned char x[2][2][kTileBytes];  // [stage][K, V] input tiles (canonical layout); S at set-up
  unsigned char bhd[kTileBytes];      // B = H D (dense rotation: sqrt(d) Pi, fp16 hi part)
  unsigned char bshi[kTileBytes];     // B = S D H, fp16 hi part (dense rotation: sqrt(d) Pi, lo part)
  unsigned char bslo[kTileBytes];     // fp16 lo part
  // [stage]: tile landed / read by its forward MMAs; [group]: forward MMAs done, A of key
  // chunk c written (y'_V read before the first), sketch done, tensor-memory columns
  // released, error drain
  unsigned long long bar_load[2], stage_free[2], fwd_done[2], a_chunk[2][4], sig_done[2], tm_free[2], bar_drain[2];
  // set-up: B = H D built, S staged as an fp16 A operand, S D H MMA done, S D H read out
  unsigned long long hd_ready, s_ready, bar_setup, setup_read;
  unsigned long long ops_ready;  // prepared operands copied in
  uint32_t tmem_base;
  int bad_s;
  float kc[16], kb[16], vc[16], vb[16];  // codebooks: centroids, boundaries
  float kmag[8];                         // |c| of a key's magnitude rank r: c[h + r]
  // the tiles that hold tokens: sequence b's are tprefix[b] .. tprefix[b + 1] - 1 (batches of
  // at most kMaxCompact sequences; larger ones walk every tile of max_len)
  int tprefix[257];
  int ntiles;
};
constexpr int kMaxCompact = 256;
constexpr size_t kSmemTC = sizeof(SmemTC) + 128;  // + base alignment slack
static_assert(kSmemTC <= 232448, "shared memory of one thread block");

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

// The same wait for a thread that can afford to react late (the copy thread, a tile ahead):
// plain polls with a sleep between them, so that it takes few issue slots from the compute
// warps of its SM sub-partition; false after kWaitNs.
__device__ __forceinline__ bool bar_wait_sleepy(unsigned long long* b, uint32_t parity) {
  const uint32_t addr = s_u32(b);
  const unsigned long long t0 = global_ns();
  for (int it = 0; it < (1 << 24); ++it) {
    uint32_t done;
    asm volatile(
        "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
        " selp.u32 %0, 1, 0, p;\n}\n"
        : "=r"(done)
        : "r"(addr), "r"(parity)
        : "memory");
    if (done) return true;
    if (global_ns() - t0 > kWaitNs) break;
    __nanosleep(256);
  }
  return false;
}

__device__ __forceinline__ void bar_arrive(unsigned long long* b) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(s_u32(b)) : "memory");
}

__device__ __forceinline__ void tma_load_tile(void* dst, const CUtensorMap* map, int row0,
                                              unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], "
      "[%5];" ::"r"(s_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(row0), "r"(0), "r"(s_u32(bar))
      : "memory");
}

// Untiled bulk copy global -> shared (16-byte aligned addresses, size a multiple of 16)
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes, unsigned long long* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                   s_u32(dst)),
               "l"(reinterpret_cast<uint64_t>(src)), "r"(bytes), "r"(s_u32(bar))
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

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
          taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]),
      "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
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

// sum of squares of 32 values, two lanes of packed fp32 at a time
__device__ __forceinline__ float sumsq32(const float (&v)[32]) {
  f2_t acc0 = 0, acc1 = 0;
#pragma unroll
  for (int i = 0; i < 32; i += 4) {
    const f2_t p = f2(v[i], v[i + 1]), q = f2(v[i + 2], v[i + 3]);
    acc0 = fma2(p, p, acc0);
    acc1 = fma2(q, q, acc1);
  }
  float a, b, c, d;
  uf2(acc0, a, b);
  uf2(acc1, c, d);
  return (a + b) + (c + d);
}

// Magnitude ranks are assembled in the mantissa of a power of two plus the rank (exact
// for small integers) and shifted into place with an integer multiply-add; the exponent
// bits each coordinate drags along are subtracted up front (mod 2^32).  With 2^23 the rank
// sits at mantissa bit 0; with 2^21 (ulp 1/4) at bit 2, which is directly the byte offset
// of its entry in a table of fp32 centroids.
constexpr float kMagic23 = 8388608.f, kMagic21 = 2097152.f;
__host__ __device__ constexpr uint32_t magic_bits(int ms) { return ms == 2 ? 0x4A000000u : 0x4B000000u; }
// x << k for k >= 0, x >> -k otherwise
__host__ __device__ constexpr uint32_t shl(uint32_t x, int k) { return k >= 0 ? x << k : x >> -k; }

// Bit of coordinate e (0..31) of a 32-coordinate group in the sign plane of 3-bit codes
// (the permutation of sign_plane_pos, which the decode's byte tables read).
__host__ __device__ constexpr int plane_bit(int e) { return 4 * (e >> 3) + (e & 3) + 16 * ((e >> 2) & 1); }

// Where coordinate i (0..31 of one 32-coordinate chunk) of a b-bit code lands in the
// chunk's four words.  Field = r | s << (b - 1) with r the magnitude rank and s = [y' > 0]:
//   b = 2: 2-bit fields (words 0, 1);  b = 3: 2-bit r (words 0, 1) and s in word 2 at the
//   permuted sign-plane bit;  b = 4: nibbles (words 0..3);  merged 3-bit key: nibbles
//   r | s << 2 | sigma << 3 (words 0..3), or for other keys sigma in a word of its own.
// Sign bits are placed two at a time (coordinates i and i + pair, which land in different
// bytes of the same word).
template <int B, bool MERGED>
struct Fields {
  static constexpr bool nib = MERGED || B == 4;
  static constexpr bool plane = !MERGED && B == 3;
  __host__ __device__ static constexpr int word(int i) { return nib ? (i >> 3) : (i >> 4); }
  __host__ __device__ static constexpr int shift(int i) { return nib ? 4 * (i & 7) : 2 * (i & 15); }
  __host__ __device__ static constexpr int sword(int i) { return plane ? 2 : word(i); }
  __host__ __device__ static constexpr int spos(int i) {
    return plane ? plane_bit(i) : shift(i) + (MERGED ? 2 : (B == 2 ? 1 : 3));
  }
  __host__ __device__ static constexpr int spair() { return nib ? 2 : 4; }
  __host__ __device__ static constexpr int sigpos(int i) { return MERGED ? shift(i) + 3 : i; }
  __host__ __device__ static constexpr int sigpair() { return MERGED ? 2 : 8; }
  // minus the magic bits the ranks (at mantissa bit ms) add to word w
  __host__ __device__ static constexpr uint32_t init(int w, int ms) {
    uint32_t c = 0;
    for (int i = 0; i < 32; ++i)
      if (word(i) == w) c += shl(magic_bits(ms), shift(i) - ms);
    return 0u - c;
  }
};

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}
// The sign bits of a and b at bits pa and pb (in different bytes), all other bits 0: prmt
// with the sign-replicating selector (8 | byte) copies the top byte's sign over a whole
// byte, and the mask keeps one bit of each.
__device__ __forceinline__ uint32_t sign_bits(float a, float b, int pa, int pb) {
  const uint32_t sel = (0xBu << (4 * (pa >> 3))) | (0xFu << (4 * (pb >> 3)));
  return prmt(__float_as_uint(a), __float_as_uint(b), sel) & ((1u << pa) | (1u << pb));
}

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
// relative band.
struct TokScale {
  int e;
  float bs;
  __device__ __forceinline__ explicit TokScale(float ny) {
    e = min(max((int)((__float_as_uint(ny) >> 23) & 0xff) - 127, -40), 40);
    bs = __uint_as_float((uint32_t)(127 + 40 - e) << 23);
  }
};

// Per-token constants of the quantiser: the scaled positive boundaries tb[k] = -bs beta_k
// ||y'|| (and for three of them tb[2] - tb[0], which selects the last step's boundary from
// the middle one's outcome), and with QJL the residual scale a = 2^(8 - e) and
// a sqrt(d) fp16(||x||).
template <int NB>
struct QuantConst {
  TokScale ts;
  float tb[NB > 0 ? NB : 1];
  float d20;
  float alpha, inv_alpha, csa;
  __device__ __forceinline__ QuantConst(float ny, const float* pos, float cnorm) : ts(ny) {
#pragma unroll
    for (int k = 0; k < NB; ++k) tb[k] = -(pos[k] * ny) * ts.bs;
    d20 = NB == 3 ? tb[NB == 3 ? 2 : 0] - tb[0] : 0.f;
    alpha = __uint_as_float((uint32_t)(127 + 8 - ts.e) << 23);
    inv_alpha = __uint_as_float((uint32_t)(127 - 8 + ts.e) << 23);
    csa = alpha * kSqrtD * cnorm;
  }
};

// Codes of one 32-coordinate chunk of y' into the chunk's words w.  The magnitude rank is
// the number of positive boundaries below |y'|: with three boundaries a binary search (is
// it above the middle one; then above the upper or the lower one), otherwise a sum of unit
// steps.  s = [y' > 0] is the sign bit of tiny - y' (exact at +-0).  With KQ also the scaled
// residual a y' - a sqrt(d) fp16(||x||) c[idx] (|c| read from a table by the rank, signed
// by s) split into fp16 hi / lo pairs for the sketch MMAs, and its sum of squares (into rr2).
// SH (dithered or corrected formats): the quantiser's input is y' + shift (shift = -xi ||y'||
// for an offset xi) and the residual a (y' - sqrt(d) n (c + xi)) is formed as
// a (y' + shift) + delta - csa c with delta = a xi (||y'|| - sqrt(d) n).  CK: also the sums of
// |c| squared and of the signed c over the chunk (into cs2, cs1), for the corrected norm.
constexpr float kTiny = 1.40129846e-45f;  // 2^-149
template <int NB, class F, bool KQ, bool SH = false, bool CK = false>
__device__ __forceinline__ void quantise32(const float (&y)[32], const QuantConst<NB>& qc, const float* cmag,
                                           uint32_t (&w)[4], uint32_t (&hi)[16], uint32_t (&lo)[16], f2_t& rr2,
                                           float shift = 0.f, float delta = 0.f, f2_t* cs1 = nullptr,
                                           f2_t* cs2 = nullptr) {
  static_assert(!(KQ && CK), "the centroid sums are taken in a pass of their own");
  constexpr int MS = KQ ? 2 : 0;
  const f2_t magic = f2s(KQ ? kMagic21 : kMagic23);
  float u[32];
#pragma unroll
  for (int i = 0; i < 32; i += 2) {
    float y0 = y[i], y1 = y[i + 1];
    if constexpr (SH) uf2(add2(f2(y0, y1), f2s(shift)), y0, y1);
    f2_t sum;
    if constexpr (NB == 3) {
      const f2_t s2 = f2(fma_sat(fabsf(y0), qc.ts.bs, qc.tb[1]), fma_sat(fabsf(y1), qc.ts.bs, qc.tb[1]));
      float t0, t1;
      uf2(fma2(s2, f2s(qc.d20), f2s(qc.tb[0])), t0, t1);
      const f2_t b0 = f2(fma_sat(fabsf(y0), qc.ts.bs, t0), fma_sat(fabsf(y1), qc.ts.bs, t1));
      sum = add2(fma2(s2, f2s(2.f), magic), b0);
    } else {
      sum = magic;
#pragma unroll
      for (int k = 0; k < NB; ++k)
        sum = add2(sum, f2(fma_sat(fabsf(y0), qc.ts.bs, qc.tb[k]), fma_sat(fabsf(y1), qc.ts.bs, qc.tb[k])));
    }
    float c0, c1;
    uf2(sum, c0, c1);
    const uint32_t code0 = __float_as_uint(c0), code1 = __float_as_uint(c1);
    w[F::word(i)] += shl(code0, F::shift(i) - MS);
    w[F::word(i + 1)] += shl(code1, F::shift(i + 1) - MS);
    uf2(fma2(f2(y0, y1), f2s(-1.f), f2s(kTiny)), u[i], u[i + 1]);
    if constexpr (CK) {
      // the rank sits at mantissa bit 0: |c| at byte offset 4 rank of the table
      const uint32_t m0 = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const char*>(cmag) + ((code0 & NB) << 2));
      const uint32_t m1 = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const char*>(cmag) + ((code1 & NB) << 2));
      const f2_t M = f2(__uint_as_float(m0), __uint_as_float(m1));
      *cs2 = fma2(M, M, *cs2);
      *cs1 = add2(*cs1, f2(__uint_as_float(m0 | (~__float_as_uint(u[i]) & 0x80000000u)),
                           __uint_as_float(m1 | (~__float_as_uint(u[i + 1]) & 0x80000000u))));
    }
    if constexpr (KQ) {
      const uint32_t m0 = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const char*>(cmag) + (code0 & 0xCu));
      const uint32_t m1 = *reinterpret_cast<const uint32_t*>(reinterpret_cast<const char*>(cmag) + (code1 & 0xCu));
      const f2_t C = f2(__uint_as_float(m0 | (~__float_as_uint(u[i]) & 0x80000000u)),
                        __uint_as_float(m1 | (~__float_as_uint(u[i + 1]) & 0x80000000u)));
      const f2_t ay = SH ? fma2(f2(y0, y1), f2s(qc.alpha), f2s(delta)) : mul2(f2(y0, y1), f2s(qc.alpha));
      const f2_t R = fma2(C, f2s(-qc.csa), ay);
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
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (i & F::spair()) continue;
    const int j = i + F::spair();
    w[F::sword(i)] |= sign_bits(u[i], u[j], F::spos(i), F::spos(j));
  }
}

// QJL signs sigma = [p >= 0] (the complement of p's sign bit) of one 32-entry chunk of the
// sketch: into bit 3 of the chunk's key nibbles, or into a sign-plane word of their own.
template <bool MERGED, class F>
__device__ __forceinline__ void sigma32(const float (&p)[32], uint4& w, uint32_t& sgw) {
  uint32_t wa[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    if (i & F::sigpair()) continue;
    const int j = i + F::sigpair();
    const int pa = F::sigpos(i), pb = F::sigpos(j);
    const uint32_t sel = (0xBu << (4 * (pa >> 3))) | (0xFu << (4 * (pb >> 3)));
    const uint32_t m = ~prmt(__float_as_uint(p[i]), __float_as_uint(p[j]), sel) & ((1u << pa) | (1u << pb));
    if constexpr (MERGED) wa[F::word(i)] |= m;
    else sgw |= m;
  }
  w = make_uint4(wa[0], wa[1], wa[2], wa[3]);
}

// The cache block and slot of the token this thread owns in tile j (blk null when the
// token is past its sequence or its page is invalid).
struct TokRef {
  uint8_t* blk;
  int slot;
};

// MODE bit 0: the dithered (offsets read per token, stored in KD / VD) and corrected-norm
// (keys: a first pass over the key chunks collects |c| sums for the stored norm) formats.
// MODE bit 1: a batch of several sequences, whose tiles past each sequence's length are
// skipped (the tile list is built from the lengths at the start).
// MODE bit 2: the value sketch of values with QJL, a second launch after the first one has
// stored every code: the value tiles go through the key path (KB = VB, KQ = 1, the value
// codebook in the key tables), which recomputes their codes, forms the residual against the
// stored norm and sketches it; only the signs (VS) and the residual norm (VR) are stored.
template <int KB, int KQ, int VB, int MODE_>
__global__ void __launch_bounds__(kThreadsTC, 1)
    compress_tc_kernel(CompressArgs a, const __grid_constant__ CUtensorMap tmk,
                       const __grid_constant__ CUtensorMap tmv) {
  extern __shared__ __align__(128) unsigned char smem_raw[];
  const uint32_t pad = (128u - (s_u32(smem_raw) & 127u)) & 127u;
  SmemTC& sm = *reinterpret_cast<SmemTC*>(smem_raw + pad);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool producer = warp >= kComputeWarps;  // the producer warpgroup
  const int qd = warp & 3;           // tensor-memory lane quadrant
  const int row = 32 * qd + lane;    // token within the tile
  const Layout& L = a.cache.L;
  constexpr int MODE = MODE_ & 1;
  constexpr bool compact = (MODE_ & 2) != 0;
  constexpr bool VSP = (MODE_ & 4) != 0;
  static_assert(!VSP || (KB == VB && KQ && MODE == 0), "the value-sketch pass runs the key path");
  constexpr int HK = 1 << (KB - 1), HV = 1 << (VB - 1);
  constexpr bool kMerged = KQ && KB == 3 && !VSP;
  constexpr int kComputeThreads = kComputeWarps * 32;

  // Tiles: for a batch of 2 .. kMaxCompact sequences only those that hold tokens (a ragged
  // batch skips the tails of its shorter sequences; the list costs a read of the lengths
  // before the first copy); otherwise every tile of max_len.  The CTAs take the tiles round
  // robin.
  const int tiles_per_head = (a.max_len + TT - 1) / TT;
  const int all_tiles = a.cache.batch * a.cache.kv_heads * tiles_per_head;
  int my_tiles = compact ? 0 : ((int)blockIdx.x < all_tiles ? (all_tiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0);
  // cursor: the caller's sequence index from its previous tile (its tiles only move forward)
  auto tile_coords = [&](int j, int& b, int& h, int& t0, int& cursor) {
    const int t = blockIdx.x + j * gridDim.x;
    if (compact) {
      // the sequence: tprefix[b] <= t < tprefix[b + 1] (a sequence without tiles has
      // tprefix[b] == tprefix[b + 1] and is stepped over)
      while (sm.tprefix[cursor + 1] <= t) ++cursor;
      b = cursor;
      const int nt = (sm.tprefix[b + 1] - sm.tprefix[b]) / a.cache.kv_heads;
      const int local = t - sm.tprefix[b];
      h = local / nt;
      t0 = (local - h * nt) * TT;
    } else {
      t0 = (t % tiles_per_head) * TT;
      h = (t / tiles_per_head) % a.cache.kv_heads;
      b = t / (tiles_per_head * a.cache.kv_heads);
    }
  };
  int load_cursor = 0;
  auto issue_load = [&](int j) {
    int b, h, t0;
    tile_coords(j, b, h, t0, load_cursor);
    const int row0 = (int)(((size_t)b * a.cache.kv_heads + h) * a.max_len + t0);
    unsigned long long* bar = &sm.bar_load[j & 1];
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(s_u32(bar)),
                 "r"((VSP ? 1 : 2) * kTileBytes)
                 : "memory");
    tma_load_tile(sm.x[j & 1][0], &tmk, row0, bar);
    if (!VSP) tma_load_tile(sm.x[j & 1][1], &tmv, row0, bar);
  };

  // ---------------- set-up ----------------
  // Launched as a programmatic dependent: the next kernel on the stream may be scheduled as
  // SMs free up, and this one touches no global memory before its predecessor has finished.
  asm volatile("griddepcontrol.launch_dependents;");
  if (warp == 0) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(s_u32(&sm.tmem_base)),
                 "r"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  if (tid == 0) {
    for (int g = 0; g < 2; ++g) {
      bar_init(&sm.bar_load[g], 1);
      bar_init(&sm.stage_free[g], 1);
      bar_init(&sm.fwd_done[g], 1);
      for (int c = 0; c < 4; ++c) bar_init(&sm.a_chunk[g][c], kGroupWarps);
      bar_init(&sm.sig_done[g], 1);
      bar_init(&sm.tm_free[g], kGroupWarps);
      bar_init(&sm.bar_drain[g], 1);
    }
    bar_init(&sm.ops_ready, 1);
    bar_init(&sm.hd_ready, kComputeWarps);
    bar_init(&sm.s_ready, kComputeWarps);
    bar_init(&sm.bar_setup, 1);
    bar_init(&sm.setup_read, kGroupWarps);
    sm.bad_s = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  asm volatile("griddepcontrol.wait;" ::: "memory");
  // With prepared operands B = H D and S D H hi / lo are copied in (one 96 KB bulk copy);
  // otherwise each CTA builds them (stage 1 is then set-up scratch for S).  Tile 0 streams
  // in meanwhile.  (The copy thread issues tile 1 right after; group 1 starts its first tile
  // that much later, and the two groups stay out of phase, which their ping-pong relies on.)
  // (The dense rotation always comes prepared: sqrt(d) Pi hi / lo, two tiles.)
  const bool prep = a.operands != nullptr;
  const bool dense = a.dense != 0;
  if (warp == kLoaderWarp) {
    if (prep && lane == 0) {
      const uint32_t nops = dense ? 2 : 3;
      asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(s_u32(&sm.ops_ready)),
                   "r"(nops * kTileBytes)
                   : "memory");
      const unsigned char* ops = static_cast<const unsigned char*>(a.operands);
      bulk_load(sm.bhd, ops, kTileBytes, &sm.ops_ready);
      bulk_load(sm.bshi, ops + kTileBytes, kTileBytes, &sm.ops_ready);
      if (!dense) bulk_load(sm.bslo, ops + 2 * kTileBytes, kTileBytes, &sm.ops_ready);
    }
    // the tile list: H ceil(len / TT) tiles per sequence (one per head for a length out of
    // range, whose first tile reports it), by a warp-wide scan
    if (compact) {
      int carry = 0;
      for (int b0 = 0; b0 < a.cache.batch; b0 += 32) {
        const int b = b0 + lane;
        int n = 0;
        if (b < a.cache.batch) {
          const int len = a.seq_lens[b];
          const bool bad = len < 0 || len > a.max_len || len > a.cache.max_pages * PT;
          n = a.cache.kv_heads * (bad ? 1 : (len + TT - 1) / TT);
        }
        int x = n;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int y = __shfl_up_sync(0xffffffffu, x, o);
          if (lane >= o) x += y;
        }
        if (b < a.cache.batch) sm.tprefix[b + 1] = carry + x;
        carry += __shfl_sync(0xffffffffu, x, 31);
      }
      if (lane == 0) {
        sm.tprefix[0] = 0;
        sm.ntiles = carry;
      }
      __syncwarp();
      my_tiles = (int)blockIdx.x < sm.ntiles ? (sm.ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
    }
    if (lane == 0 && my_tiles > 0) issue_load(0);
  }
  __syncwarp();
  if (!producer) {
    // The small tables (the rotation's D, the codebooks) are requested first, then S (fp16-
    // exact by contract): lanes read consecutive 16-byte pieces of a row (coalesced), and
    // each CTA starts at a different row, so that the CTAs' requests for the same 64 KB
    // spread over the L2.  Nothing waits for S but the S D H operands: the forward MMAs of
    // group 0's first tile need only B = H D (hd_ready).
    const float sgn = !prep && tid < D ? a.signs[tid] : 0.f;
    float tkc = 0.f, tkb = 0.f, tvc = 0.f, tvb = 0.f;
    if (tid < 16) {
      tkc = tid < 2 * HK ? (VSP ? a.v_centroids : a.k_centroids)[tid] : 0.f;
      tkb = tid < 2 * HK - 1 ? (VSP ? a.v_boundaries : a.k_boundaries)[tid] : 0.f;
      tvc = tid < 2 * HV ? a.v_centroids[tid] : 0.f;
      tvb = tid < 2 * HV - 1 ? a.v_boundaries[tid] : 0.f;
    }
    constexpr int kSIter = QM * 16 / kComputeThreads;
    float4 sraw[KQ ? 2 * kSIter : 1];
    auto s_row = [&](int c) { return ((c >> 4) + 8 * (int)blockIdx.x) & (QM - 1); };
    if (KQ && !prep) {
#pragma unroll
      for (int it = 0; it < kSIter; ++it) {
        const int c = tid + it * kComputeThreads;
        const float4* src = reinterpret_cast<const float4*>(a.s + (size_t)s_row(c) * D + 8 * (c & 15));
        sraw[2 * it] = src[0];
        sraw[2 * it + 1] = src[1];
      }
    }
    // D of the rotation, for the set-up only (in the space of the S D H operand, filled later)
    float* signs = reinterpret_cast<float*>(sm.bshi);
    if (!prep && tid < D) signs[tid] = sgn;
    if (tid < 16) {
      sm.kc[tid] = tkc;
      sm.kb[tid] = tkb;
      sm.vc[tid] = tvc;
      sm.vb[tid] = tvb;
    }
    asm volatile("bar.sync 5, %0;" ::"n"(kComputeThreads) : "memory");
    if (tid < 8) sm.kmag[tid] = tid < HK ? sm.kc[HK + tid] : 0.f;
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
      if (prep) break;
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
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
    __syncwarp();
    if (lane == 0) bar_arrive(&sm.hd_ready);
    if (KQ && !prep) {
      // S as an fp16 A operand in stage 1; S D H = S (H D)^T is then one MMA against the
      // B = H D operand above.  The D values in bshi are no longer read once every warp has
      // passed hd_ready's arrival (the S D H readout, which overwrites them, waits for the MMA).
      unsigned char* sa = sm.x[1][0];
      int bad = 0;
#pragma unroll
      for (int it = 0; it < kSIter; ++it) {
        const int c = tid + it * kComputeThreads;
        const int m = s_row(c), ch = c & 15;
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
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) bar_arrive(&sm.s_ready);
    }
  }
  if (compact) {
    // the tile list is in shared memory for every role (compact is the same in every thread)
    asm volatile("bar.sync 6, %0;" ::"n"(kThreadsTC) : "memory");
    my_tiles = (int)blockIdx.x < sm.ntiles ? (sm.ntiles - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  }
  const uint32_t tmem = sm.tmem_base;

  if (producer) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegsProducer));
    // ---------------- producer: one MMA issuer per group, one copy issuer ----------------
    // Group g owns tiles j = g, g + 2, ... and the tensor-memory columns K[g], V[g].  For its
    // n-th tile its issuer waits until the group has released K[g] / V[g] (tile n - 1 read
    // out) and the tile has landed in stage g, issues the forward MMAs (y'_K -> K[g],
    // y'_V -> V[g]), and with QJL waits for the group's A (in place in K[g]) before issuing
    // the sketch into V[g].  The copy issuer refills stage s with the next tile of that
    // stage once both forward MMAs of the previous one have read it.  Each wait's phase is
    // one the other side cannot run two phases past.
    if ((warp == kIssuerWarp0 || warp == kIssuerWarp1) && lane == 0) {
      const int g = warp == kIssuerWarp0 ? 0 : 1;
      const uint32_t colK = tmem + kColGroup * g, colV = colK + kColV;
      // B = H D in shared memory (and for the S D H MMA, S as an A operand), or the
      // prepared operands copied in
      bool ok = bar_wait(prep ? &sm.ops_ready : &sm.hd_ready, 0);
      if (ok && KQ && g == 1 && !prep) ok = bar_wait(&sm.s_ready, 0);
      if (ok && KQ && g == 1 && !prep) {
        // S D H into K[1] (free until tile 1): read out by group 1 before its first tile
        tc_fence_after();
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) mma_ss(colK, smem_desc(sm.x[1][0], ks), smem_desc(sm.bhd, ks), ks > 0);
        mma_commit(&sm.bar_setup);
      }
      // S D H read out of K[1]: group 1's first tile may land there
      if (ok && KQ && g == 1 && my_tiles > 1 && !prep) ok = bar_wait(&sm.setup_read, 0);
      // MMA issue is not on any critical path: the loops stay rolled to keep the producer's
      // registers few
      auto fwd = [&](int kv, uint32_t dcol) {
#pragma unroll 1
        for (int ks = 0; ks < 8; ++ks) mma_ss(dcol, smem_desc(sm.x[g][kv], ks), smem_desc(sm.bhd, ks), ks > 0);
        if (dense) {
#pragma unroll 1
          for (int ks = 0; ks < 8; ++ks) mma_ss(dcol, smem_desc(sm.x[g][kv], ks), smem_desc(sm.bshi, ks), 1);
        }
      };
      bool k_issued = false;  // y'_K of the group's next tile already requested
      for (int n = 0, j = g; ok && j < my_tiles; ++n, j += 2) {
        if (!k_issued) {
          if (n > 0 && !(ok = bar_wait(&sm.tm_free[g], (n - 1) & 1))) break;
          if (!(ok = bar_wait(&sm.bar_load[g], n & 1))) break;
          tc_fence_after();
          fwd(0, colK);
        } else {
          // y'_V of the previous tile, then the sketch output, read out of V[g]
          if (!(ok = bar_wait(&sm.tm_free[g], (n - 1) & 1))) break;
          tc_fence_after();
        }
        if (!VSP) fwd(1, colV);
        mma_commit(&sm.fwd_done[g]);
        mma_commit(&sm.stage_free[g]);  // both forward MMAs of tile j have read stage g
        k_issued = false;
        if (KQ) {
          // The sketch goes into V[g] (y'_V is read before the first key chunk is released),
          // chunk by chunk as the group writes A into K[g]; its B operands (S D H hi / lo) are
          // in shared memory once group 1 has read them out
          if (g == 0 && n == 0 && !prep && !(ok = bar_wait(&sm.setup_read, 0))) break;
#pragma unroll 1
          for (int c = 0; c < 4 && ok; ++c) {
            if (!(ok = bar_wait(&sm.a_chunk[g][c], n & 1))) break;
            tc_fence_after();
#pragma unroll 1
            for (int h = 0; h < 2; ++h) {
              // coordinates 16 ks ..: chunk c, half h (hi at +0, lo at +16)
              const int ks = 2 * c + h;
              const uint32_t ahi = colK + 32 * c + 8 * h;
              mma_ts(colV, ahi, smem_desc(sm.bshi, ks), ks > 0);
              mma_ts(colV, ahi, smem_desc(sm.bslo, ks), 1);
              mma_ts(colV, ahi + 16, smem_desc(sm.bshi, ks), 1);
            }
          }
          if (!ok) break;
          mma_commit(&sm.sig_done[g]);
          // once the sketch is done with A, K[g] takes y'_K of the group's next tile
          if (j + 2 < my_tiles) {
            if (!(ok = bar_wait(&sm.sig_done[g], n & 1))) break;
            if (!(ok = bar_wait(&sm.bar_load[g], (n + 1) & 1))) break;
            tc_fence_after();
            fwd(0, colK);
            k_issued = true;
          }
        }
      }
      if (!ok) {
        report(a.status, TQ_ERR_TIMEOUT);
        // let the MMAs already issued finish (bounded) before tensor memory is freed
        mma_commit(&sm.bar_drain[g]);
        bar_wait(&sm.bar_drain[g], 0);
      }
    } else if (warp == kLoaderWarp && lane == 0 && my_tiles > 0) {
      int issued = 1;  // tile 0 went out before the set-up
      bool ok = true;
      // stage 1 holds S until the S D H MMA has read it (operands built in the CTA)
      if (KQ && !prep && !(ok = bar_wait(&sm.bar_setup, 0))) report(a.status, TQ_ERR_TIMEOUT);
      if (ok && my_tiles > 1) {
        issue_load(1);
        issued = 2;
      }
      for (int i = 0; ok && i + 2 < my_tiles; ++i) {
        // phase i >> 1 of stage_free[i & 1]: the forward MMAs of tile i are done with it
        if (!(ok = bar_wait_sleepy(&sm.stage_free[i & 1], (i >> 1) & 1))) break;
        issue_load(i + 2);
        issued = i + 3;
      }
      if (!ok) report(a.status, TQ_ERR_TIMEOUT);
      // the last copy into each stage is that stage's final phase: wait (bounded) for both to
      // land so that no copy is still in flight when the shared memory goes away
      for (int i = (issued > 2 ? issued - 2 : 0); i < issued; ++i) bar_wait(&sm.bar_load[i & 1], (i >> 1) & 1);
      if (prep) bar_wait(&sm.ops_ready, 0);
    }
    __syncwarp();
  } else {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegsCompute));
    // ---------------- compute groups ----------------
    typedef Fields<KB, kMerged> FK;
    typedef Fields<VB, false> FV;
    const int g = warp / kGroupWarps;  // tiles g, g + 2, ...
    const uint32_t lane_base = (uint32_t)(32 * qd) << 16;
    const uint32_t colK = tmem + lane_base + kColGroup * g, colV = colK + kColV;
    // The sequence length and the page entry of the token this thread owns in tile j: two
    // independent loads, issued one group tile ahead and checked when the tile starts.
    struct TokLoad {
      int len, phys, t0, h;
      float ko, vo;  // dithered: the token's key and value offsets
    };
    const bool dith = MODE != 0 && L.dither != 0;
    int tok_cursor = 0;
    auto token_load = [&](int j) -> TokLoad {
      int b, h, t0;
      tile_coords(j, b, h, t0, tok_cursor);
      const int page = (t0 + row) / PT;
      TokLoad l{a.seq_lens[b],
                page < a.cache.max_pages ? a.cache.block_table[(size_t)b * a.cache.max_pages + page] : -1, t0, h,
                0.f, 0.f};
      if (dith && t0 + row < a.max_len) {
        const size_t o = ((size_t)b * a.cache.kv_heads + h) * a.max_len + t0 + row;
        l.ko = a.k_off[o];
        l.vo = a.v_off[o];
      }
      return l;
    };
    float cur_ko = 0.f, cur_vo = 0.f;
    auto token_ref = [&](const TokLoad& l) -> TokRef {
      cur_ko = l.ko;
      cur_vo = l.vo;
      const int tok = l.t0 + row;
      const bool bad_len = l.len < 0 || l.len > a.max_len || l.len > a.cache.max_pages * PT;
      if (bad_len && row == 0 && l.t0 == 0) report(a.status, TQ_ERR_BOUNDS);
      TokRef r{nullptr, tok % PT};
      if (!bad_len && tok < l.len) {
        TQ_DCHECK(a.status, tok < a.max_len && tok / PT < a.cache.max_pages && l.h < a.cache.kv_heads);
        if (l.phys < 0 || l.phys >= a.cache.num_pages) {
          report(a.status, TQ_ERR_BOUNDS);
        } else {
          r.blk = a.cache.block(l.phys, l.h);
        }
      }
      return r;
    };
    bool failed = false;
    if (KQ && g == 1 && !prep) {
      // S D H (fp32 in K[1], row = sketch index) split into the fp16 hi / lo B operands
      if (!bar_wait(&sm.bar_setup, 0) || !bar_wait(&sm.s_ready, 0)) failed = true;
      if (tid == kGroupWarps * 32 && sm.bad_s) report(a.status, TQ_ERR_INVALID_ARG);
      __syncwarp();
      tc_fence_after();
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float v[32];
        tmem_ld32(colK + 32 * c, v);
        tmem_wait_ld();
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          uint32_t hi[4], lo[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = v[8 * q + 2 * e], x1 = v[8 * q + 2 * e + 1];
            const __half2 h2 = __floats2half2_rn(x0, x1);
            const float2 hf = __half22float2(h2);
            const __half2 l2 = __floats2half2_rn(x0 - hf.x, x1 - hf.y);
            hi[e] = *reinterpret_cast<const uint32_t*>(&h2);
            lo[e] = *reinterpret_cast<const uint32_t*>(&l2);
          }
          const int k = 32 * c + 8 * q;
          *reinterpret_cast<uint4*>(sm.bshi + canon(row, k)) = make_uint4(hi[0], hi[1], hi[2], hi[3]);
          *reinterpret_cast<uint4*>(sm.bslo + canon(row, k)) = make_uint4(lo[0], lo[1], lo[2], lo[3]);
        }
      }
      // visible to the sketch MMAs, which wait for setup_read after these writes
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) bar_arrive(&sm.setup_read);
    }
    TokLoad next = g < my_tiles ? token_load(g) : TokLoad{0, -1, 0, 0};
    for (int n = 0, j = g; j < my_tiles; ++n, j += 2) {
      const TokRef cur = token_ref(next);
      if (j + 2 < my_tiles) next = token_load(j + 2);

      // ---- norms of y'_K and y'_V ----
      if (!failed && !bar_wait(&sm.fwd_done[g], n & 1)) failed = true;
      __syncwarp();
      tc_fence_after();
      float ssk = 0.f, ssv = 0.f;
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        float y[32], z[32];
        tmem_ld32(colK + 32 * c, y);
        if (!VSP) tmem_ld32(colV + 32 * c, z);
        tmem_wait_ld();
        ssk += sumsq32(y);
        if (!VSP) ssv += sumsq32(z);
      }
      const float nyk = sqrtf(ssk);  // ||y'_K|| = sqrt(d) ||k||
      const float nyv = sqrtf(ssv);
      __half nk16 = __float2half_rn(nyk * (1.0f / kSqrtD));
      const __half nv16 = __float2half_rn(nyv * (1.0f / kSqrtD));
      // dithered: the offsets as used and stored (fp16); the quantiser's input is
      // y' - xi ||y'|| (y - xi in unit-vector coordinates)
      const __half kxi16 = __float2half_rn(cur_ko), vxi16 = __float2half_rn(cur_vo);
      const float kxi = dith ? __half2float(kxi16) : 0.f, vxi = dith ? __half2float(vxi16) : 0.f;

      // ---- values, then keys chunk by chunk; the keys' residual goes to TMEM in place and each
      // chunk is released to the sketch MMAs while the next chunk's load is in flight ----
      QuantConst<HK - 1> qk(nyk, sm.kb + HK, __half2float(nk16));
      const QuantConst<HV - 1> qv(nyv, sm.vb + HV, 0.f);
      // Value chunks are quantised from one register buffer while the next chunk's load into
      // the other is in flight (two chunks per iteration, the buffers alternating).
      auto quant_v = [&](const float (&z)[32], int c) {
        constexpr uint32_t vw0 = FV::init(0, 0), vw1 = FV::init(1, 0), vw2 = FV::init(2, 0), vw3 = FV::init(3, 0);
        uint32_t vw[4] = {vw0, vw1, vw2, vw3}, dh[16], dl[16];
        f2_t drr = 0;
        quantise32<HV - 1, FV, false, MODE != 0>(z, qv, sm.kmag, vw, dh, dl, drr, -vxi * nyv);
        if (cur.blk && !failed)
          store_chunk<VB, false>(cur.blk + L.vc, c >> 1, c & 1, cur.slot, make_uint4(vw[0], vw[1], vw[2], vw[3]));
      };
      if (!VSP) {
        float za[32], zb[32];
        tmem_ld32(colV, za);
        tmem_wait_ld();
#pragma unroll 1
        for (int c = 0; c < 4; c += 2) {
          tmem_ld32(colV + 32 * (c + 1), zb);
          quant_v(za, c);
          tmem_wait_ld();
          if (c + 2 < 4) tmem_ld32(colV + 32 * (c + 2), za);
          quant_v(zb, c + 1);
          if (c + 2 < 4) tmem_wait_ld();
        }
      }
      // corrected norm: a first pass over the key chunks collects sum |c|^2 and sum c for
      // ||y_hat||^2 = sum (c + xi)^2; without QJL its words are the stored ones
      const bool corr = MODE != 0 && a.key_corr != 0;
      if (corr) {
        f2_t cs1 = 0, cs2 = 0;
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          float y[32];
          tmem_ld32(colK + 32 * c, y);
          tmem_wait_ld();
          constexpr uint32_t pw0 = FK::init(0, 0), pw1 = FK::init(1, 0), pw2 = FK::init(2, 0), pw3 = FK::init(3, 0);
          uint32_t pw[4] = {pw0, pw1, pw2, pw3}, dh[16], dl[16];
          f2_t drr = 0;
          quantise32<HK - 1, FK, false, true, true>(y, qk, sm.kmag, pw, dh, dl, drr, -kxi * nyk, 0.f, &cs1, &cs2);
          if (!KQ && cur.blk && !failed)
            store_chunk<KB, false>(cur.blk + L.kc, c >> 1, c & 1, cur.slot, make_uint4(pw[0], pw[1], pw[2], pw[3]));
        }
        float p0, p1, q0, q1;
        uf2(cs1, p0, p1);
        uf2(cs2, q0, q1);
        const float yy = (q0 + q1) + kxi * (2.f * (p0 + p1) + (float)D * kxi);
        const float yn = sqrtf(fmaxf(yy, 0.f));
        nk16 = __float2half_rn(yn > 0.f ? (nyk * (1.0f / kSqrtD)) / yn : 0.f);
        qk.csa = qk.alpha * kSqrtD * __half2float(nk16);
      }
      if (cur.blk && (__hisinf(nk16) || __hisinf(nv16))) report(a.status, TQ_ERR_OVERFLOW);
      // residual offset of the dithered keys: a xi (||y'|| - sqrt(d) n)
      const float kdelta = qk.alpha * kxi * (nyk - kSqrtD * __half2float(nk16));
      if (MODE != 0 && dith && cur.blk && !failed) {
        reinterpret_cast<__half*>(cur.blk + L.kd)[cur.slot] = kxi16;
        reinterpret_cast<__half*>(cur.blk + L.vd)[cur.slot] = vxi16;
      }
      f2_t rr2 = 0;
      // key words of the four chunks (completed by the signs)
      uint4 kw0 = make_uint4(0, 0, 0, 0), kw1 = kw0, kw2 = kw0, kw3 = kw0;
      auto release = [&](int c) {
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(&sm.a_chunk[g][c]);
      };
#pragma unroll 1
      for (int c = 0; c < 4 && !(corr && !KQ); ++c) {
        float y[32];
        tmem_ld32(colK + 32 * c, y);
        if (KQ && c > 0) release(c - 1);
        tmem_wait_ld();
        constexpr int kMS = KQ ? 2 : 0;  // key ranks at mantissa bit 2 (table offsets)
        constexpr uint32_t kwi0 = FK::init(0, kMS), kwi1 = FK::init(1, kMS), kwi2 = FK::init(2, kMS),
                           kwi3 = FK::init(3, kMS);
        uint32_t kw[4] = {kwi0, kwi1, kwi2, kwi3}, hi[16], lo[16];
        quantise32<HK - 1, FK, KQ != 0, MODE != 0>(y, qk, sm.kmag, kw, hi, lo, rr2, -kxi * nyk, kdelta);
        const uint4 kq = make_uint4(kw[0], kw[1], kw[2], kw[3]);
        if constexpr (KQ) {
          tmem_st16(colK + 32 * c, hi);
          tmem_st16(colK + 32 * c + 16, lo);
          kw0 = c == 0 ? kq : kw0;
          kw1 = c == 1 ? kq : kw1;
          kw2 = c == 2 ? kq : kw2;
          kw3 = c == 3 ? kq : kw3;
        } else if (cur.blk && !failed && !VSP) {
          store_chunk<KB, false>(cur.blk + L.kc, c >> 1, c & 1, cur.slot, kq);
        }
      }
      if constexpr (KQ) {
        release(3);
        float ra, rb;
        uf2(rr2, ra, rb);
        const float rho = sqrtf(ra + rb) * qk.inv_alpha * (1.0f / kSqrtD);
        if (cur.blk && !failed) {
          if (VSP) {
            reinterpret_cast<__half*>(cur.blk + L.vr)[cur.slot] = __float2half_rn(rho);
          } else {
            reinterpret_cast<__half*>(cur.blk + L.vn)[cur.slot] = nv16;
            reinterpret_cast<__half*>(cur.blk + L.kn)[cur.slot] = nk16;
            reinterpret_cast<__half*>(cur.blk + L.kr)[cur.slot] = __float2half_rn(rho);
          }
        }
        // the sketch's signs complete the key words
        if (!failed && !bar_wait(&sm.sig_done[g], n & 1)) failed = true;
        __syncwarp();
        tc_fence_after();
        float sk0[32], sk1[32], sk2[32], sk3[32];
        tmem_ld32(colV, sk0);
        tmem_ld32(colV + 32, sk1);
        tmem_ld32(colV + 64, sk2);
        tmem_ld32(colV + 96, sk3);
        tmem_wait_ld();
        // K[g] and V[g] are read out: the group's next tile may land in them
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(&sm.tm_free[g]);
        auto finish = [&](const float (&sk)[32], uint4 w, int c) {
          uint32_t sgw = 0;
          sigma32<kMerged, FK>(sk, w, sgw);
          if (cur.blk && !failed) {
            if (VSP) {
              *reinterpret_cast<uint32_t*>(cur.blk + L.vs + (size_t)cur.slot * 16 + 4 * c) = sgw;
            } else {
              store_chunk<KB, kMerged>(cur.blk + L.kc, c >> 1, c & 1, cur.slot, w);
              if (!kMerged) *reinterpret_cast<uint32_t*>(cur.blk + L.ks + (size_t)cur.slot * 16 + 4 * c) = sgw;
            }
          }
        };
        finish(sk0, kw0, 0);
        finish(sk1, kw1, 1);
        finish(sk2, kw2, 2);
        finish(sk3, kw3, 3);
      } else {
        tc_fence_before();
        __syncwarp();
        if (lane == 0) bar_arrive(&sm.tm_free[g]);
        if (cur.blk && !failed) {
          reinterpret_cast<__half*>(cur.blk + L.vn)[cur.slot] = nv16;
          reinterpret_cast<__half*>(cur.blk + L.kn)[cur.slot] = nk16;
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
// prepared operands: B = H D, then S D H split into fp16 hi and lo, each a canonical tile
// ---------------------------------------------------------------------------
// The last CTA builds B = H D.  With QJL, CTA m < QM forms row m of S D H = (S D) H by a
// Walsh-Hadamard transform of S_m . D (fp32, H symmetric and unnormalised) and splits it
// into fp16 hi + lo (the same operands the compress kernel otherwise forms in every CTA).
__global__ void __launch_bounds__(128) prepare_operands_kernel(const float* signs, const float* s,
                                                               unsigned char* ops) {
  const int t = threadIdx.x;
  if ((int)blockIdx.x == (int)gridDim.x - 1) {
    for (int c = t; c < D * 16; c += 128) {
      const int i = c & 127, ch = c >> 7;
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int k0 = ch * 8 + 2 * e;
        const float s0 = signs[k0], s1 = signs[k0 + 1];
        const __half2 h = __floats2half2_rn((__popc(i & k0) & 1) ? -s0 : s0, (__popc(i & (k0 + 1)) & 1) ? -s1 : s1);
        w[e] = *reinterpret_cast<const uint32_t*>(&h);
      }
      *reinterpret_cast<uint4*>(ops + canon(i, ch * 8)) = make_uint4(w[0], w[1], w[2], w[3]);
    }
    return;
  }
  __shared__ float v[D];
  const int m = blockIdx.x;
  v[t] = s[(size_t)m * D + t] * signs[t];
  __syncthreads();
#pragma unroll
  for (int h = 1; h < D; h <<= 1) {
    const float x = v[t], y = v[t ^ h];
    __syncthreads();
    v[t] = (t & h) ? y - x : x + y;
    __syncthreads();
  }
  const float x = v[t];
  const __half hi = __float2half_rn(x);
  const __half lo = __float2half_rn(x - __half2float(hi));
  *reinterpret_cast<__half*>(ops + kTileBytes + canon(m, t)) = hi;
  *reinterpret_cast<__half*>(ops + 2 * kTileBytes + canon(m, t)) = lo;
}

// Dense rotation: B = sqrt(d) Pi (row i = output coordinate, column k = input coordinate,
// y = Pi u) as an fp16 hi tile and the fp16 rounding of the fp32 remainder; one CTA per row.
__global__ void __launch_bounds__(128) prepare_dense_kernel(const float* pi, unsigned char* ops) {
  const int i = blockIdx.x, k = threadIdx.x;
  const float x = pi[(size_t)i * D + k] * kSqrtD;
  const __half hi = __float2half_rn(x);
  const __half lo = __float2half_rn(x - __half2float(hi));
  *reinterpret_cast<__half*>(ops + canon(i, k)) = hi;
  *reinterpret_cast<__half*>(ops + kTileBytes + canon(i, k)) = lo;
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
cudaError_t launch_tc(const CompressArgs& a, const CUtensorMap& mk, const CUtensorMap& mv, cudaStream_t stream,
                      bool value_sketch = false) {
  const bool cmp = a.cache.batch > 1 && a.cache.batch <= kMaxCompact;
  const int mode = ((a.cache.L.dither || a.key_corr) ? 1 : 0) | (cmp ? 2 : 0);
  void (*k)(CompressArgs, const CUtensorMap, const CUtensorMap);
  if constexpr (KB == VB && KQ == 1) {
    if (value_sketch) k = cmp ? compress_tc_kernel<VB, 1, VB, 6> : compress_tc_kernel<VB, 1, VB, 4>;
  }
  if (!value_sketch)
    k = mode == 0 ? compress_tc_kernel<KB, KQ, VB, 0>
        : mode == 1 ? compress_tc_kernel<KB, KQ, VB, 1>
        : mode == 2 ? compress_tc_kernel<KB, KQ, VB, 2>
                    : compress_tc_kernel<KB, KQ, VB, 3>;
  else if (!(KB == VB && KQ == 1))
    return cudaErrorInvalidValue;
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
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreadsTC);
  cfg.dynamicSmemBytes = kSmemTC;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, k, a, mk, mv);
}

}  // namespace

bool compress_tc_supported(const CompressArgs& a) {
  const Layout& L = a.cache.L;
  if (a.in_dtype != TQ_F16) return false;
  if (a.dense && (L.qjl || a.operands == nullptr)) return false;
  // values with QJL: a second launch sketches them through the key path (2- or 3-bit
  // values, the randomized Hadamard rotation, not dithered)
  if (L.vqjl && (a.dense || L.dither || !(L.vbits == 2 || L.vbits == 3))) return false;
  if ((size_t)a.cache.batch * a.cache.kv_heads * a.max_len >= (1ull << 31)) return false;
  if (L.qjl && !(L.kbits == 2 || L.kbits == 3)) return false;
  if (!L.qjl && !(L.kbits >= 2 && L.kbits <= 4)) return false;
  if (!(L.vbits >= 2 && L.vbits <= 4)) return false;
  if ((reinterpret_cast<uintptr_t>(a.k) & 15) || (reinterpret_cast<uintptr_t>(a.v) & 15)) return false;
  if (reinterpret_cast<uintptr_t>(a.operands) & 15) return false;
  return encode_fn() != nullptr;
}

size_t operand_bytes(bool dense) { return (dense ? 2 : 3) * (size_t)kTileBytes; }

cudaError_t launch_prepare_operands(const float* signs, const float* s, int qjl, void* ops, cudaStream_t stream) {
  prepare_operands_kernel<<<qjl ? QM + 1 : 1, 128, 0, stream>>>(signs, s, static_cast<unsigned char*>(ops));
  return cudaGetLastError();
}

cudaError_t launch_prepare_dense(const float* pi, void* ops, cudaStream_t stream) {
  prepare_dense_kernel<<<D, D, 0, stream>>>(pi, static_cast<unsigned char*>(ops));
  return cudaGetLastError();
}

cudaError_t launch_compress_tc(const CompressArgs& a, cudaStream_t stream) {
  const Layout& L = a.cache.L;
  const size_t rows = (size_t)a.cache.batch * a.cache.kv_heads * a.max_len;
  if (rows == 0) return cudaSuccess;
  CUtensorMap mk, mv;
  if (!make_tile_map(&mk, a.k, rows) || !make_tile_map(&mv, a.v, rows)) return cudaErrorInvalidValue;
  cudaError_t e = cudaErrorInvalidValue;
#define TQ_TC(KB, KQ, VB) \
  if (L.kbits == KB && L.qjl == KQ && L.vbits == VB) e = launch_tc<KB, KQ, VB>(a, mk, mv, stream);
#define TQ_TC_V(KB, KQ) TQ_TC(KB, KQ, 2) TQ_TC(KB, KQ, 3) TQ_TC(KB, KQ, 4)
  TQ_TC_V(3, 1)
  TQ_TC_V(2, 1)
  TQ_TC_V(2, 0)
  TQ_TC_V(3, 0)
  TQ_TC_V(4, 0)
#undef TQ_TC_V
#undef TQ_TC
  if (e != cudaSuccess || !L.vqjl) return e;
  // the value sketch, once every code is stored (a programmatic dependent of the first launch)
  if (L.vbits == 2) return launch_tc<2, 1, 2>(a, mv, mv, stream, true);
  if (L.vbits == 3) return launch_tc<3, 1, 3>(a, mv, mv, stream, true);
  return cudaErrorInvalidValue;
}

}  // namespace tqk
