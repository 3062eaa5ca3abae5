// Tensor-core split-KV decode over the packed cache.
//
// Same computation as the generic split kernel in decode.cu ("turboquant_cutile" function
// list: asymmetric estimator + online softmax + on-chip V; "TurboQuant explained",
// section "How is this different from PolarQuant's reconstruction?": pre-rotated
// query), organised for B200:
//
//  * one producer warp streams the split's half pages (128 tokens; the splits are dealt
//    contiguous runs of half pages, so they stay balanced) into a 3-stage shared-memory
//    ring with bulk asynchronous copies (cp.async.bulk, completion on mbarriers);
//  * four consumer warps each take 16-token steps.  A lane dequantises codes straight
//    into fp16 mma fragments with byte permutes against a centroid table held in
//    registers; the key term  sum_j (R q)_j c[idx_j]  is an fp16 m16n8k16 mma (query in
//    hi+lo fp16 halves, fp32 accumulation), the QJL term  sum_i (S q)_i sigma_i  an int8
//    m16n8k32 mma on 16-bit fixed-point (S q) digits, and  sum_t p_t ||v_t|| c[idx]  an
//    fp16 mma after an in-register 8x8 transpose (movmatrix) of the dequantised values;
//  * online softmax per warp, then a log-sum-exp merge of the four warps; the partial
//    (m, l, acc) per query row goes to the workspace, and the last split of each
//    (sequence, kv head) to finish (a counter the prologue zeroes) merges all partials
//    and applies R^T.
//
// The R = G * seq_q query rows of a KV head are taken four or eight at a time (eight when R
// exceeds four): one run of rows per CTA along the grid's z, each run with its own merge
// counter.
//
// Supported here: keys 3-bit + QJL (merged nibbles), 2-bit + QJL, or 4-bit without QJL
// (sign-magnitude nibbles, the signs applied by byte masks), values 3-bit or 2-bit, any R;
// the randomized Hadamard rotation or a dense Pi (R^T applied in the merge); dithered codes
// (DT: a key's offset adds xi_k sum_i (R q)_i to its dot product, a value's adds xi_v to
// every coordinate, carried as one running sum per row next to the accumulator); values
// with QJL for up to four rows (VQ: the value product's four spare columns accumulate the
// sign-space sums sum_t p_t ||r_v||_t (2 sigma_t - 1) through a second mma per step, and the
// merge adds sqrt(pi/2)/m S^T of them).
// Everything else uses decode.cu.
#include <climits>
#include <cuda_fp16.h>
#include <math_constants.h>

#include "tq_device.cuh"
#include "tq_kernels.h"

namespace tqk {

namespace {

constexpr int kConsumerWarps = 4;
constexpr int kThreads = (kConsumerWarps + 1) * 32;
constexpr int kStages = 3;
constexpr int kUnit = PT / 2;                  // tokens per copy unit: half a page
constexpr int kUnitsPerPage = PT / kUnit;
constexpr int kChunkStride = kUnit * 16 + 32;  // padded so the 4 lanes of a token group hit distinct banks
constexpr int kNormBytes = 6 * kUnit * 2;      // KN | KR | VN | KD | VD | VR of the unit
constexpr int kMaxKChunks = 4;
constexpr int kMaxVChunks = 4;  // 3-bit values: 2 crumb chunks + the sign plane; + VS
constexpr int kStageBytes = kNormBytes + (kMaxKChunks + kMaxVChunks) * kChunkStride;
constexpr unsigned long long kWaitLimitNs = 1000000000ull;  // every mbarrier wait gives up after 1 s
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kInvSqrtD = 0.08838834764831845f;
constexpr float kQjlScale = 1.2533141373155003f / QM;  // sqrt(pi/2)/m

enum KPol { K3Q = 0, K2Q = 1, K4 = 2 };
enum VPol { V3 = 0, V2 = 1 };

// Query rows per CTA: 4 or 8 (the key and QJL products take one n-tile of the mma per four
// rows; the value product's eight columns hold eight rows).
constexpr int kMaxRows = 8;
// the merging CTA copies the partials of up to 160 / rows splits into shared memory at once
constexpr int kMergeFloats = 160 * D;
struct SmemFast {
  union {
    struct {
      unsigned char stage[kStages][kStageBytes];
      float wacc[kConsumerWarps][kMaxRows][D];
      float wsig[kConsumerWarps][4][QM];  // values with QJL: the sign-space sums of each warp
    } ring;
    // at the end: the partial accumulators of every split of the (sequence, kv head) being
    // merged, [row][split][D] (the ring and the warp partials are no longer used then)
    float merge[kMergeFloats];
  };
  unsigned long long full[kStages];
  unsigned long long empty[kStages];
  unsigned long long mbar;  // the merge copies landed
  unsigned long long never;  // completed by nothing: the target of the bounded-wait test
  float wm[kConsumerWarps][kMaxRows], wl[kConsumerWarps][kMaxRows], wf[kConsumerWarps][kMaxRows];
  float wx[kConsumerWarps][kMaxRows];  // dithered values: sum_t p_t ||v_t|| xi_t of each warp and row
  float xsig[4][QM];  // values with QJL, at the merge: each row's sign-space sum / l
  int cu;  // units per split
  int last;
};

// ---------------------------------------------------------------------------
// PTX helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(unsigned long long* bar, int count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_expect_tx(unsigned long long* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(unsigned long long* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ unsigned long long global_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ bool mbar_try(uint32_t addr, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n .reg .pred p;\n mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      " selp.u32 %0, 1, 0, p;\n}\n"
      : "=r"(done)
      : "r"(addr), "r"(parity)
      : "memory");
  return done != 0;
}

// Wait on the given phase parity for at most limit_ns nanoseconds of the global timer
// (read once every 256 polls, so that a wait that succeeds soon costs no timer reads);
// false if it gave up.
__device__ __forceinline__ bool mbar_wait(unsigned long long* bar, uint32_t parity,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_try(addr, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    for (int it = 0; it < 256; ++it)
      if (mbar_try(addr, parity)) return true;
    if (global_ns() - t0 > limit_ns) return false;
  }
}

// The same wait for a thread that can afford to react late (the copy producer, three stages
// ahead): between polls it sleeps, so that it takes few issue slots from the consumer warps
// of its SM sub-partition.
__device__ __forceinline__ bool mbar_wait_sleepy(unsigned long long* bar, uint32_t parity) {
  const uint32_t addr = smem_u32(bar);
  if (mbar_try(addr, parity)) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    __nanosleep(128);
    if (mbar_try(addr, parity)) return true;
    if (global_ns() - t0 > kWaitLimitNs) return false;
  }
}

// Wait (bounded by the global timer) until a ready word of the prologue is set.  It is read
// with acquire semantics, so that what the prologue wrote before setting it is visible to
// this thread's later reads.  false (and TQ_ERR_TIMEOUT) if it gave up.
__device__ __forceinline__ bool acquire_ready(const unsigned int* rw, int32_t* status) {
  unsigned int v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(rw) : "memory");
  if (v) return true;
  const unsigned long long t0 = global_ns();
  for (;;) {
    __nanosleep(32);
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(rw) : "memory");
    if (v) return true;
    if (global_ns() - t0 > kWaitLimitNs) {
      report(status, TQ_ERR_TIMEOUT);
      return false;
    }
  }
}

__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes, unsigned long long* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t s) {
  uint32_t r;
  asm("prmt.b32 %0, %1, %2, %3;" : "=r"(r) : "r"(a), "r"(b), "r"(s));
  return r;
}

__device__ __forceinline__ uint32_t movm_t(uint32_t x) {
  uint32_t r;
  asm volatile("movmatrix.sync.aligned.m8n8.trans.b16 %0, %1;" : "=r"(r) : "r"(x));
  return r;
}

__device__ __forceinline__ void hmma(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                     uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void imma(int (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                     uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k32.row.col.s32.s8.s8.s32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+r"(d[0]), "+r"(d[1]), "+r"(d[2]), "+r"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ uint16_t h_bits(float v) {
  const __half h = __float2half_rn(v);
  return *reinterpret_cast<const uint16_t*>(&h);
}

__device__ __forceinline__ float ld_h(const unsigned char* p) {
  return __half2float(*reinterpret_cast<const __half*>(p));
}

// Byte tables for fp16 values: lo bytes of 4 entries in one word, hi bytes in another.
__device__ __forceinline__ void table4(const float (&v)[4], uint32_t& lo, uint32_t& hi) {
  lo = hi = 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint16_t b = h_bits(v[i]);
    lo |= (uint32_t)(b & 0xff) << (8 * i);
    hi |= (uint32_t)(b >> 8) << (8 * i);
  }
}

// Coordinates (within the lane's quarter of 32) of crumb pair cb: (base, base + 4).
__device__ __forceinline__ int pair_base(int cb) { return 8 * (cb >> 2) + (cb & 3); }

// The two 2-bit fields of crumb pair cb of a quarter, from its crumb words c0 (coords 0..15)
// and c1 (16..31), placed at bits 0-1 and 8-9, turned into a byte-permute selector that
// picks [lo, hi] of entry f from a (lo-bytes, hi-bytes) table pair.
__device__ __forceinline__ uint32_t crumb_t(uint32_t c0, uint32_t c1, int cb) {
  const uint32_t w = (cb < 8) ? c0 : c1;
  const int s = 2 * (cb & 3) + 16 * ((cb >> 2) & 1);
  return (s == 0 ? w : __umulhi(w, 1u << (32 - s))) & 0x0303u;
}

__device__ __forceinline__ uint32_t crumb_sel(uint32_t c0, uint32_t c1, int cb) {
  return crumb_t(c0, c1, cb) * 0x11u + 0x4040u;
}

// The selectors of crumb pairs cb = 8 h + k and 8 h + 4 + k (k < 4) at once, from crumb word
// w = c0 (h = 0) or c1 (h = 1): one mask keeps both pairs' fields (bits 2k, 2k + 8 and
// 2k + 16, 2k + 24), one multiply-add turns both into selectors (the low one's product stays
// below bit 16), and the high one is shifted down.
__device__ __forceinline__ void crumb_sel2(uint32_t w, int k, uint32_t& lo, uint32_t& hi) {
  const uint32_t f = ((w >> (2 * k)) & 0x03030303u) * 0x11u + 0x40404040u;
  lo = f;
  hi = f >> 16;
}

// Selector of the int8 residual codes of crumb pairs n and n+1: bytes (a_n, a_n+1, b_n, b_n+1).
__device__ __forceinline__ uint32_t crumb_pair_sel(uint32_t c0, uint32_t c1, int n) {
  const uint32_t t1 = crumb_t(c0, c1, n), t2 = crumb_t(c0, c1, n + 1);
  return (t1 & 0x3u) | ((t2 & 0x3u) << 4) | (t1 & 0x300u) | ((t2 & 0x300u) << 4);
}

template <int KP, int VP, int NR, bool DT, bool VQ>
__global__ void __launch_bounds__(kThreads, 2) fast_split_kernel(DecodeArgs a) {
  static_assert(!VQ || (NR == 4 && !DT), "values with QJL: four rows, not dithered");
  static_assert(NR == 4 || NR == 8, "four or eight rows per CTA");
  constexpr int NT = NR / 4;  // n-tiles of the key and QJL products
  // the next kernel on the stream may be scheduled now; a programmatic dependent waits for
  // this grid to finish before it touches what it writes
  asm volatile("griddepcontrol.launch_dependents;");
  extern __shared__ __align__(128) unsigned char smem_raw[];
  SmemFast& sm = *reinterpret_cast<SmemFast*>(smem_raw);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // The query rows of one (sequence, kv head) (its G heads times seq_q positions, consecutive)
  // are taken in runs of up to NR, one run per CTA along the grid's z with the sequence.
  const int nchunk = (a.rows + NR - 1) / NR;
  const int split = blockIdx.x, gh = blockIdx.y, b = blockIdx.z / nchunk, chunk = blockIdx.z % nchunk;
  const Layout& L = a.cache.L;
  const int R = min(NR, a.rows - NR * chunk);
  const size_t row0 = ((size_t)b * a.q_heads + (size_t)gh * a.group) * a.seq_q + NR * chunk;
  TQ_DCHECK(a.status, R >= 1 && R <= NR && row0 + R <= (size_t)a.cache.batch * a.q_heads * a.seq_q);

  const int len = a.seq_lens[b];
  const bool bad_len = len < 0 || len > a.cache.max_pages * PT;
  if (bad_len && tid == 0 && split == 0) report(a.status, TQ_ERR_BOUNDS);
  const int n_eff = bad_len ? 0 : len;
  // the sequence in half-page units, dealt to the splits in contiguous runs of sm.cu units
  // (formed below, before the first barrier)
  const int units_all = (n_eff + kUnit - 1) / kUnit;

  constexpr int kKChunks = (KP == K2Q) ? 3 : 4;  // K2Q: 2 code chunks + the KS chunk
  constexpr int kVChunks = (VP == V3) ? 3 : 2;
  constexpr bool kQjl = KP != K4;
  // without QJL there is no KR region: its norm slots stay unused
  const uint32_t unit_bytes = 2u * kUnit * (2 + (kQjl ? 1 : 0) + (DT ? 2 : 0) + (VQ ? 1 : 0)) +
                              16u * kUnit * (kKChunks + kVChunks + (VQ ? 1 : 0));

  if (tid == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&sm.full[s], 1);
      mbar_init(&sm.empty[s], kConsumerWarps);
    }
    mbar_init(&sm.mbar, 1);
    mbar_init(&sm.never, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0) {
    // Units per split.  Sequences of one length: the longest's units over the n_splits splits
    // (every sequence takes all of them).  Sequences of different lengths: no longer than the
    // batch's mean share of one wave of target_ctas thread blocks, so that the longest
    // sequence is cut into more splits and the shorter ones into fewer (each stream of u
    // units takes ceil(u / cu) of the n_splits), instead of every sequence taking n_splits
    // splits and the longest ones' setting the pace.
    const int cap = a.cache.max_pages * PT;
    int maxu = 0, minu = INT_MAX;
    long long total = 0;
    for (int bb = lane; bb < a.cache.batch; bb += 32) {
      const int l = a.seq_lens[bb];
      const int u = (l < 0 || l > cap) ? 0 : (l + kUnit - 1) / kUnit;
      maxu = max(maxu, u);
      minu = min(minu, u);
      total += u;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      maxu = max(maxu, __shfl_xor_sync(FULL, maxu, o));
      minu = min(minu, __shfl_xor_sync(FULL, minu, o));
      total += __shfl_xor_sync(FULL, total, o);
    }
    int c = (maxu + a.n_splits - 1) / a.n_splits;
    const long long streams = (long long)a.cache.batch * a.cache.kv_heads * nchunk;
    if (minu != maxu && a.target_ctas > streams) {
      const long long work = total * a.cache.kv_heads * nchunk;
      c = max(c, (int)((work + (a.target_ctas - streams) - 1) / (a.target_ctas - streams)));
    }
    if (lane == 0) sm.cu = max(1, c);
  }
  __syncthreads();
  const int cu = sm.cu;
  // this stream's splits (at most n_splits: cu is at least the longest's share); thread
  // blocks past them have nothing to do (uniform per block)
  const int n_split_b = max(1, (units_all + cu - 1) / cu);
  if (split >= n_split_b) return;
  const int u_begin = min(units_all, split * cu);
  const int u_end = min(units_all, (split + 1) * cu);
  const int nunits = u_end - u_begin;
  const int t_end = min(n_eff, u_end * kUnit);

  if (warp == kConsumerWarps) {
    // ---------------- producer ----------------
    if (lane == 0) {
      // tokens from t_new on are appended by the prologue of this call: a unit that holds
      // one is copied only after the prologue has finished
      const int t_new = n_eff - a.n_new;
      bool prologue_done = false;
      int issued = 0;
      for (int i = 0; i < nunits; ++i) {
        const int s = i % kStages;
        if (i >= kStages && !mbar_wait_sleepy(&sm.empty[s], ((i / kStages) - 1) & 1)) {
          report(a.status, TQ_ERR_TIMEOUT);
          break;
        }
        issued = i + 1;
        const int u = u_begin + i, half = u % kUnitsPerPage;
        TQ_DCHECK(a.status, u >= 0 && u < units_all && u / kUnitsPerPage < a.cache.max_pages);
        TQ_DCHECK(a.status, unit_bytes <= (uint32_t)kStageBytes);
        if (a.n_new > 0 && !prologue_done && (u + 1) * kUnit > t_new) {
          asm volatile("griddepcontrol.wait;" ::: "memory");
          asm volatile("fence.proxy.async.global;" ::: "memory");
          prologue_done = true;
        }
        int phys = a.cache.block_table[(size_t)b * a.cache.max_pages + u / kUnitsPerPage];
        if (phys < 0 || phys >= a.cache.num_pages) {
          report(a.status, TQ_ERR_BOUNDS);
          phys = 0;
        }
        const unsigned char* blk = a.cache.block(phys, gh);
        unsigned char* st = sm.ring.stage[s];
        const uint32_t hb2 = half * kUnit * 2, hb16 = half * kUnit * 16;
        mbar_expect_tx(&sm.full[s], unit_bytes);
        bulk_g2s(st, blk + L.kn + hb2, kUnit * 2, &sm.full[s]);
        if (kQjl) bulk_g2s(st + kUnit * 2, blk + L.kr + hb2, kUnit * 2, &sm.full[s]);
        bulk_g2s(st + kUnit * 4, blk + L.vn + hb2, kUnit * 2, &sm.full[s]);
        if (DT) {
          bulk_g2s(st + kUnit * 6, blk + L.kd + hb2, kUnit * 2, &sm.full[s]);
          bulk_g2s(st + kUnit * 8, blk + L.vd + hb2, kUnit * 2, &sm.full[s]);
        }
        unsigned char* kc = st + kNormBytes;
        const int kcode_chunks = (KP == K2Q) ? 2 : 4;
        for (int c = 0; c < kcode_chunks; ++c)
          bulk_g2s(kc + c * kChunkStride, blk + L.kc + c * PT * 16 + hb16, kUnit * 16, &sm.full[s]);
        if (KP == K2Q) bulk_g2s(kc + 2 * kChunkStride, blk + L.ks + hb16, kUnit * 16, &sm.full[s]);
        unsigned char* vc = kc + kMaxKChunks * kChunkStride;
        for (int c = 0; c < kVChunks; ++c)
          bulk_g2s(vc + c * kChunkStride, blk + L.vc + c * PT * 16 + hb16, kUnit * 16, &sm.full[s]);
        if (VQ) {
          bulk_g2s(st + kUnit * 10, blk + L.vr + hb2, kUnit * 2, &sm.full[s]);
          bulk_g2s(vc + kVChunks * kChunkStride, blk + L.vs + hb16, kUnit * 16, &sm.full[s]);
        }
      }
      // the last copy into each stage has landed (consumers that gave up early did not wait
      // for it) before the ring's space is reused or released; bounded
      for (int i = issued > kStages ? issued - kStages : 0; i < issued; ++i)
        mbar_wait(&sm.full[i % kStages], (i / kStages) & 1);
    }
  } else {
    // ---------------- consumers ----------------
    const int g = lane >> 2, t4 = lane & 3;
    // centroid tables
    uint32_t kt_lo0 = 0, kt_lo1 = 0, kt_hi0 = 0, kt_hi1 = 0, vt_lo = 0, vt_hi = 0;
    {
      const int hk = 1 << (L.kbits - 1), hv = 1 << (L.vbits - 1);
      if (KP == K3Q) {
        // stored code (r0, r1, s) -> index r + 4 s; value s ? +a[r] : -a[r]
        float neg[4], pos[4];
        for (int r = 0; r < 4; ++r) {
          pos[r] = a.k_centroids[hk + r];
          neg[r] = -pos[r];
        }
        table4(neg, kt_lo0, kt_hi0);
        table4(pos, kt_lo1, kt_hi1);
      } else if (KP == K4) {
        // stored code (r0, r1, r2, s) -> magnitude a[r] (the sign is applied by a byte mask)
        float m0[4], m1[4];
        for (int r = 0; r < 4; ++r) {
          m0[r] = a.k_centroids[hk + r];
          m1[r] = a.k_centroids[hk + 4 + r];
        }
        table4(m0, kt_lo0, kt_hi0);
        table4(m1, kt_lo1, kt_hi1);
      } else {
        // stored code (r0, s) -> f = r0 + 2 s; value s ? +a[r0] : -a[r0]
        float t[4] = {-a.k_centroids[hk], -a.k_centroids[hk + 1], a.k_centroids[hk], a.k_centroids[hk + 1]};
        table4(t, kt_lo0, kt_hi0);
      }
      if (VP == V3) {
        // negative magnitudes: a set sign bit (s = 1, the positive half) flips them to +a[r]
        float t[4] = {-a.v_centroids[hv], -a.v_centroids[hv + 1], -a.v_centroids[hv + 2], -a.v_centroids[hv + 3]};
        table4(t, vt_lo, vt_hi);
      } else {
        float t[4] = {-a.v_centroids[hv], -a.v_centroids[hv + 1], a.v_centroids[hv], a.v_centroids[hv + 1]};
        table4(t, vt_lo, vt_hi);
      }
    }
    // fp16 rounding residual of the key centroids, eps = c - fp16(c), as int8 codes scaled by
    // eps_up (a power of two); the correction term sum_j q_j eps_j restores fp32 centroids
    uint32_t et0 = 0, et1 = 0;
    float eps_up = 1.f;
    {
      const int hk = 1 << (L.kbits - 1);
      float e8[8];
      int n = 0;
      if (KP == K3Q) {
        for (int i = 0; i < 8; ++i) {
          const float c = (i >= 4) ? a.k_centroids[hk + (i & 3)] : -a.k_centroids[hk + (i & 3)];
          e8[i] = c - __half2float(__float2half_rn(c));
        }
        n = 8;
      } else if (KP == K4) {
        // magnitudes; a negative centroid's residual is the negated code (its bitwise
        // complement, -e - 1: one LSB of the scaled residual, 2^-7 of its largest entry)
        for (int i = 0; i < 8; ++i) {
          const float c = a.k_centroids[hk + i];
          e8[i] = c - __half2float(__float2half_rn(c));
        }
        n = 8;
      } else {
        const float c4[4] = {-a.k_centroids[hk], -a.k_centroids[hk + 1], a.k_centroids[hk], a.k_centroids[hk + 1]};
        for (int i = 0; i < 4; ++i) e8[i] = c4[i] - __half2float(__float2half_rn(c4[i]));
        for (int i = 4; i < 8; ++i) e8[i] = 0.f;
        n = 4;
      }
      float emax = 0.f;
      for (int i = 0; i < n; ++i) emax = fmaxf(emax, fabsf(e8[i]));
      int ex = 0;
      if (emax > 0.f) {
        frexpf(127.f / emax, &ex);
        ex -= 1;
      }
      eps_up = ldexpf(1.f, ex);
      for (int i = 0; i < 8; ++i) {
        const uint32_t v = (uint32_t)(__float2int_rn(e8[i] * eps_up) & 255);
        if (i < 4) et0 |= v << (8 * i);
        else et1 |= v << (8 * (i - 4));
      }
    }
    // The prologue (our programmatic predecessor) publishes the query terms of each row in
    // kQueryParts parts, each with a ready word: acquire those of this CTA's rows (bounded;
    // the acquires, ordered before the other warps' reads by the barrier, make the terms and
    // the zeroed merge counter visible), instead of waiting for the whole prologue grid.
    if (warp == 0 && lane < R * kQueryParts) acquire_ready(a.ready + row0 * kQueryParts + lane, a.status);
    asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
    // B fragments, one n-tile per four rows (tile nt: rows 4 nt .. 4 nt + 3)
    uint32_t bq[NT][8][2], bc[NT][4][2], bs[NT][4][2];
    int sq_sum_nt[NT];        // of row 4 nt + g/2: the sum of its fixed-point S q
    float sq_scale_nt[NT];    // and the power of two that scales it
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      // this lane's 32-coordinate slices of row 4 nt + g/2: rotated query, its int8 copy,
      // 16-bit S q
      const int fr = 4 * nt + (g >> 1);
      const bool frow = fr < R;
      float qv[32];
      int q8v[32], sqv[32];
      {
        const size_t rr = row0 + (frow ? fr : 0);
        const float4* qp = reinterpret_cast<const float4*>(a.qrot + rr * D + 32 * t4);
        const int4* q8p = reinterpret_cast<const int4*>(a.q8 + rr * D + 32 * t4);
        const float4* sqp = reinterpret_cast<const float4*>(a.sq + rr * QM + 32 * t4);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 f = frow ? qp[k] : make_float4(0.f, 0.f, 0.f, 0.f);
          qv[4 * k] = f.x; qv[4 * k + 1] = f.y; qv[4 * k + 2] = f.z; qv[4 * k + 3] = f.w;
        }
#pragma unroll
        for (int k = 0; k < 2; ++k) {
          const int4 v = frow ? q8p[k] : make_int4(0, 0, 0, 0);
          const int w4[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int bb = 0; bb < 4; ++bb) q8v[16 * k + 4 * u + bb] = (int)(int8_t)((w4[u] >> (8 * bb)) & 255);
        }
        // S q of the row in 16-bit fixed point: scale 2^ex with 2^ex <= 32000 / max |S q| over
        // the row (its 128 entries are spread over the four lanes t4 of this group), the sum
        // of the fixed-point entries with it
        float mx = 0.f;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const float4 f = (frow && kQjl) ? sqp[k] : make_float4(0.f, 0.f, 0.f, 0.f);
          mx = fmaxf(mx, fmaxf(fmaxf(fabsf(f.x), fabsf(f.y)), fmaxf(fabsf(f.z), fabsf(f.w))));
          sqv[4 * k] = __float_as_int(f.x);
          sqv[4 * k + 1] = __float_as_int(f.y);
          sqv[4 * k + 2] = __float_as_int(f.z);
          sqv[4 * k + 3] = __float_as_int(f.w);
        }
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 1));
        mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 2));
        int ex = 0;
        if (mx > 0.f) {
          frexpf(32000.f / mx, &ex);
          ex -= 1;
        }
        const float up = ldexpf(1.f, ex);
        int rs = 0;
#pragma unroll
        for (int c = 0; c < 32; ++c) {
          sqv[c] = __float2int_rn(__int_as_float(sqv[c]) * up);
          rs += sqv[c];
        }
        rs += __shfl_xor_sync(FULL, rs, 1);
        rs += __shfl_xor_sync(FULL, rs, 2);
        sq_sum_nt[nt] = rs;
        sq_scale_nt[nt] = ldexpf(1.f, -ex);
      }
      // the key term: column g = (row 4 nt + g/2, hi or lo half)
#pragma unroll
      for (int ks = 0; ks < 8; ++ks) {
        float v[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          int c;  // quarter-local coordinate of B row (ks, e)
          if (KP != K2Q) {
            c = 4 * ks + e;
          } else {
            const int n = 2 * ks + (e >> 1);  // half2 index: word n/8, pair n%8
            c = 16 * (n >> 3) + pair_base(n & 7) + 4 * (e & 1);
          }
          const float x = qv[c];
          const float hi = __half2float(__float2half_rn(x));
          v[e] = (g & 1) ? (x - hi) : hi;
        }
        bq[nt][ks][0] = pack_h2(v[0], v[1]);
        bq[nt][ks][1] = pack_h2(v[2], v[3]);
      }
      // the centroid correction: int8 R q in column 2r (odd columns zero)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t word = 0;
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            int c;  // quarter-local coordinate of byte i of correction register (w, h)
            if (KP != K2Q) {
              c = 8 * w + 4 * h + i;
            } else {
              // register (w, h) holds pairs n = 4w + 2h and 4w + 2h + 1: bytes (a1, a2, b1, b2)
              const int n = 4 * w + 2 * h + (i & 1);
              c = 16 * (n >> 3) + pair_base(n & 7) + 4 * (i >> 1);
            }
            const int v = (g & 1) ? 0 : q8v[c];
            word |= (uint32_t)(v & 255) << (8 * i);
          }
          bc[nt][w][h] = word;
        }
      }
      // the QJL term: column g = (row 4 nt + g/2, digit g%2) of 16-bit (S q)
#pragma unroll
      for (int w = 0; w < 4; ++w) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t word = 0;
#pragma unroll
          for (int i = 0; i < 4 && kQjl; ++i) {
            int c;  // quarter-local QJL index of byte i of register (w, h)
            if (KP == K3Q)
              c = 8 * w + 2 * i + h;
            else
              c = 8 * i + 7 - (2 * w + h);
            const int v = sqv[c];
            const int d0 = ((v + 128) & 255) - 128;
            const int d1 = (v - d0) >> 8;
            word |= (uint32_t)(((g & 1) ? d1 : d0) & 255) << (8 * i);
          }
          bs[nt][w][h] = word;
        }
      }
    }
    // With eight rows (two n-tiles) the B fragments (64 registers per lane) live in shared
    // memory during the page loop, over the warp partials' space (written only after every
    // consumer warp has left the loop), and are read back per n-tile at each step; every warp
    // formed the same fragments, warp 0 stores them: [n-tile][8 slots][lane] of 16 bytes
    constexpr bool kBSmem = NT == 2;
    uint4* const bfrag = reinterpret_cast<uint4*>(&sm.ring.wacc[0][0][0]);
    if constexpr (kBSmem) {
      if (warp == 0) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
          for (int j = 0; j < 4; ++j)
            bfrag[(nt * 8 + j) * 32 + lane] = make_uint4(bq[nt][2 * j][0], bq[nt][2 * j][1], bq[nt][2 * j + 1][0],
                                                         bq[nt][2 * j + 1][1]);
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            bfrag[(nt * 8 + 4 + j) * 32 + lane] = make_uint4(bc[nt][2 * j][0], bc[nt][2 * j][1],
                                                             bc[nt][2 * j + 1][0], bc[nt][2 * j + 1][1]);
            bfrag[(nt * 8 + 6 + j) * 32 + lane] = make_uint4(bs[nt][2 * j][0], bs[nt][2 * j][1],
                                                             bs[nt][2 * j + 1][0], bs[nt][2 * j + 1][1]);
          }
        }
      }
      asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
    }
    // per-row constants of the lane's own score rows t4 + 4 nt
    int T_row[NT];
    float c_row_q[NT], corr_down[NT];
    const float c_row_k = kInvSqrtD * kLog2e;
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int rr = t4 + 4 * nt;
      // row rr's fixed-point sum and scale sit with the lanes g = 2 t4, 2 t4 + 1
      const int rsum = __shfl_sync(FULL, sq_sum_nt[nt], 8 * t4);
      const float rscale = __shfl_sync(FULL, sq_scale_nt[nt], 8 * t4);
      T_row[nt] = 0;
      c_row_q[nt] = 0.f;
      corr_down[nt] = 0.f;
      if (rr < R) {
        T_row[nt] = kQjl ? rsum : 0;
        c_row_q[nt] = kQjl ? kQjlScale * rscale * kInvSqrtD * kLog2e : 0.f;
        const float lam = a.q8_scale[row0 + rr];
        corr_down[nt] = lam > 0.f ? 1.f / (lam * eps_up) : 0.f;
      }
    }

    // dithered keys: sum_i (R q)_i of the lane's score rows (the 8 lanes of a row add 16
    // coordinates each)
    float qs[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      qs[nt] = 0.f;
      if (DT) {
        const int rr = t4 + 4 * nt;
        float t = 0.f;
        if (rr < R) {
          const float4* qp = reinterpret_cast<const float4*>(a.qrot + (row0 + rr) * D + 16 * g);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float4 f = qp[k];
            t += (f.x + f.y) + (f.z + f.w);
          }
        }
        t += __shfl_xor_sync(FULL, t, 4);
        t += __shfl_xor_sync(FULL, t, 8);
        t += __shfl_xor_sync(FULL, t, 16);
        qs[nt] = t;
      }
    }

    if (a.debug_wait_ns > 0 && warp == 0 && split == 0 && gh == 0 && blockIdx.z == 0 &&
        !mbar_wait(&sm.never, 0, (unsigned long long)a.debug_wait_ns) && lane == 0)
      report(a.status, TQ_ERR_TIMEOUT);

    float m_run[NT], l_run[NT], x_run[NT];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      m_run[nt] = -CUDART_INF_F;
      l_run[nt] = 0.f;
      x_run[nt] = 0.f;
    }
    float acc[8][4];
#pragma unroll
    for (int mt = 0; mt < 8; ++mt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][e] = 0.f;

    for (int i = 0; i < nunits; ++i) {
      const int s = i % kStages;
      if (!mbar_wait(&sm.full[s], (i / kStages) & 1)) {
        if (lane == 0) report(a.status, TQ_ERR_TIMEOUT);
        break;
      }
      const unsigned char* st = sm.ring.stage[s];
      const unsigned char* kc = st + kNormBytes;
      const unsigned char* vc = kc + kMaxKChunks * kChunkStride;
      const int tok0 = (u_begin + i) * kUnit;
      const int valid = min(kUnit, t_end - tok0);
      TQ_DCHECK(a.status, valid >= 1 && valid <= kUnit && tok0 + valid <= n_eff);
      // two 16-token steps per iteration: their key and value work interleave, and one
      // joint running maximum (one rescale) serves both
      for (int pr = warp; pr * 32 < valid; pr += kConsumerWarps) {
        float sc[2][NT][2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int step = 2 * pr + u;
            const int ta = step * 16 + g, tb = ta + 8;
            // ---- keys: dequantise into fp16 A fragments and int8 sign fragments
            uint32_t ha[16], hb[16], sa[8], sb[8], ea[8], eb[8];
            if (KP == K3Q) {
              const uint4 wa = *reinterpret_cast<const uint4*>(kc + t4 * kChunkStride + ta * 16);
              const uint4 wb = *reinterpret_cast<const uint4*>(kc + t4 * kChunkStride + tb * 16);
              const uint32_t A4[4] = {wa.x, wa.y, wa.z, wa.w}, B4[4] = {wb.x, wb.y, wb.z, wb.w};
    #pragma unroll
              for (int w = 0; w < 4; ++w) {
    #pragma unroll
                for (int side = 0; side < 2; ++side) {
                  const uint32_t W = side ? B4[w] : A4[w];
                  uint32_t* h = side ? hb : ha;
                  uint32_t* sg = side ? sb : sa;
                  uint32_t* ep = side ? eb : ea;
                  const uint32_t s0 = W & 0x7777u;
                  const uint32_t s1 = __umulhi(W, 1u << 16) & 0x7777u;
                  ep[2 * w + 0] = prmt(et0, et1, s0);
                  ep[2 * w + 1] = prmt(et0, et1, s1);
                  const uint32_t l0 = prmt(kt_lo0, kt_lo1, s0), h0 = prmt(kt_hi0, kt_hi1, s0);
                  const uint32_t l1 = prmt(kt_lo0, kt_lo1, s1), h1 = prmt(kt_hi0, kt_hi1, s1);
                  h[4 * w + 0] = prmt(l0, h0, 0x5140);
                  h[4 * w + 1] = prmt(l0, h0, 0x7362);
                  h[4 * w + 2] = prmt(l1, h1, 0x5140);
                  h[4 * w + 3] = prmt(l1, h1, 0x7362);
                  sg[2 * w + 0] = (W << 4) & 0x80808080u;
                  sg[2 * w + 1] = W & 0x80808080u;
                }
              }
            } else if (KP == K4) {
              const uint4 wa = *reinterpret_cast<const uint4*>(kc + t4 * kChunkStride + ta * 16);
              const uint4 wb = *reinterpret_cast<const uint4*>(kc + t4 * kChunkStride + tb * 16);
              const uint32_t A4[4] = {wa.x, wa.y, wa.z, wa.w}, B4[4] = {wb.x, wb.y, wb.z, wb.w};
    #pragma unroll
              for (int w = 0; w < 4; ++w) {
    #pragma unroll
                for (int side = 0; side < 2; ++side) {
                  const uint32_t W = side ? B4[w] : A4[w];
                  uint32_t* h = side ? hb : ha;
                  uint32_t* ep = side ? eb : ea;
                  const uint32_t s0 = W & 0x7777u;
                  const uint32_t s1 = __umulhi(W, 1u << 16) & 0x7777u;
                  // 0xFF in the byte of each coordinate whose s bit (nibble bit 3) is set:
                  // the sign bits of nibbles 1, 3, ... are byte tops already, those of
                  // nibbles 0, 2, ... become byte tops four bits up
                  const uint32_t W4 = W << 4;
                  const uint32_t m0 = prmt(W4, W, 0xD9C8u), m1 = prmt(W4, W, 0xFBEAu);
                  ep[2 * w + 0] = prmt(et0, et1, s0) ^ ~m0;
                  ep[2 * w + 1] = prmt(et0, et1, s1) ^ ~m1;
                  const uint32_t l0 = prmt(kt_lo0, kt_lo1, s0), l1 = prmt(kt_lo0, kt_lo1, s1);
                  const uint32_t h0 = prmt(kt_hi0, kt_hi1, s0) ^ (~m0 & 0x80808080u);
                  const uint32_t h1 = prmt(kt_hi0, kt_hi1, s1) ^ (~m1 & 0x80808080u);
                  h[4 * w + 0] = prmt(l0, h0, 0x5140);
                  h[4 * w + 1] = prmt(l0, h0, 0x7362);
                  h[4 * w + 2] = prmt(l1, h1, 0x5140);
                  h[4 * w + 3] = prmt(l1, h1, 0x7362);
                }
              }
            } else {
              const unsigned char* kq = kc + (t4 >> 1) * kChunkStride + (t4 & 1) * 8;
              const uint2 ca = *reinterpret_cast<const uint2*>(kq + ta * 16);
              const uint2 cbv = *reinterpret_cast<const uint2*>(kq + tb * 16);
              const uint32_t sA = *reinterpret_cast<const uint32_t*>(kc + 2 * kChunkStride + ta * 16 + 4 * t4);
              const uint32_t sB = *reinterpret_cast<const uint32_t*>(kc + 2 * kChunkStride + tb * 16 + 4 * t4);
    #pragma unroll
              for (int hk = 0; hk < 8; ++hk) {
                const int h = hk >> 2, k = hk & 3;
                uint32_t sla, sha, slb, shb;
                crumb_sel2(h ? ca.y : ca.x, k, sla, sha);
                crumb_sel2(h ? cbv.y : cbv.x, k, slb, shb);
                ha[8 * h + k] = prmt(kt_lo0, kt_hi0, sla);
                ha[8 * h + 4 + k] = prmt(kt_lo0, kt_hi0, sha);
                hb[8 * h + k] = prmt(kt_lo0, kt_hi0, slb);
                hb[8 * h + 4 + k] = prmt(kt_lo0, kt_hi0, shb);
              }
    #pragma unroll
              for (int n = 0; n < 16; n += 2) {
                // pairs n, n+1 -> int8 residual codes (a_n, a_n+1, b_n, b_n+1)
                ea[n >> 1] = prmt(et0, et1, crumb_pair_sel(ca.x, ca.y, n));
                eb[n >> 1] = prmt(et0, et1, crumb_pair_sel(cbv.x, cbv.y, n));
              }
    #pragma unroll
              for (int k = 0; k < 8; ++k) {
                sa[k] = (sA << k) & 0x80808080u;
                sb[k] = (sB << k) & 0x80808080u;
              }
            }
#pragma unroll
          for (int nt = 0; nt < NT; ++nt) {
            // this n-tile's B fragments: from shared memory (two n-tiles) or registers
            uint32_t fq[8][2], fc[4][2], fs[4][2];
            if constexpr (kBSmem) {
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const uint4 v = bfrag[(nt * 8 + j) * 32 + lane];
                fq[2 * j][0] = v.x; fq[2 * j][1] = v.y; fq[2 * j + 1][0] = v.z; fq[2 * j + 1][1] = v.w;
              }
#pragma unroll
              for (int j = 0; j < 2; ++j) {
                const uint4 c = bfrag[(nt * 8 + 4 + j) * 32 + lane], q = bfrag[(nt * 8 + 6 + j) * 32 + lane];
                fc[2 * j][0] = c.x; fc[2 * j][1] = c.y; fc[2 * j + 1][0] = c.z; fc[2 * j + 1][1] = c.w;
                fs[2 * j][0] = q.x; fs[2 * j][1] = q.y; fs[2 * j + 1][0] = q.z; fs[2 * j + 1][1] = q.w;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 8; ++j) {
                fq[j][0] = bq[nt][j][0];
                fq[j][1] = bq[nt][j][1];
              }
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                fc[j][0] = bc[nt][j][0];
                fc[j][1] = bc[nt][j][1];
                fs[j][0] = bs[nt][j][0];
                fs[j][1] = bs[nt][j][1];
              }
            }
            // two accumulators per term halve the dependent mma chains
            float dk[4] = {0.f, 0.f, 0.f, 0.f}, dk2[4] = {0.f, 0.f, 0.f, 0.f};
    #pragma unroll
            for (int ks = 0; ks < 8; ks += 2) {
              hmma(dk, ha[2 * ks], hb[2 * ks], ha[2 * ks + 1], hb[2 * ks + 1], fq[ks][0], fq[ks][1]);
              hmma(dk2, ha[2 * ks + 2], hb[2 * ks + 2], ha[2 * ks + 3], hb[2 * ks + 3], fq[ks + 1][0],
                   fq[ks + 1][1]);
            }
            int dsum[4] = {0, 0, 0, 0}, dsum2[4] = {0, 0, 0, 0};
            int dcor[4] = {0, 0, 0, 0}, dcor2[4] = {0, 0, 0, 0};
    #pragma unroll
            for (int w = 0; w < 4; w += 2) {
              if (kQjl) {
                imma(dsum, sa[2 * w], sb[2 * w], sa[2 * w + 1], sb[2 * w + 1], fs[w][0], fs[w][1]);
                imma(dsum2, sa[2 * w + 2], sb[2 * w + 2], sa[2 * w + 3], sb[2 * w + 3], fs[w + 1][0],
                     fs[w + 1][1]);
              }
              imma(dcor, ea[2 * w], eb[2 * w], ea[2 * w + 1], eb[2 * w + 1], fc[w][0], fc[w][1]);
              imma(dcor2, ea[2 * w + 2], eb[2 * w + 2], ea[2 * w + 3], eb[2 * w + 3], fc[w + 1][0],
                   fc[w + 1][1]);
            }
    #pragma unroll
            for (int e = 0; e < 4; ++e) {
              dk[e] += dk2[e];
              dsum[e] += dsum2[e];
              dcor[e] += dcor2[e];
            }
            // ---- scores of row t4 + 4 nt for tokens ta, tb (log2 domain)
            const float nA = ld_h(st + 2 * ta), nB = ld_h(st + 2 * tb);
            const float rA = kQjl ? ld_h(st + 2 * kUnit + 2 * ta) : 0.f;
            const float rB = kQjl ? ld_h(st + 2 * kUnit + 2 * tb) : 0.f;
            // every product of the QJL mma is -128 sigma d: the sums are exact multiples of 128
            const int s1a = -((dsum[0] + 256 * dsum[1]) >> 7), s1b = -((dsum[2] + 256 * dsum[3]) >> 7);
            float dotA = dk[0] + dk[1] + (float)dcor[0] * corr_down[nt];
            float dotB = dk[2] + dk[3] + (float)dcor[2] * corr_down[nt];
            if (DT) {
              dotA = fmaf(ld_h(st + 6 * kUnit + 2 * ta), qs[nt], dotA);
              dotB = fmaf(ld_h(st + 6 * kUnit + 2 * tb), qs[nt], dotB);
            }
            float sca = nA * dotA * c_row_k + rA * (float)(2 * s1a - T_row[nt]) * c_row_q[nt];
            float scb = nB * dotB * c_row_k + rB * (float)(2 * s1b - T_row[nt]) * c_row_q[nt];
            if (t4 + 4 * nt >= R || ta >= valid) sca = -CUDART_INF_F;
            if (t4 + 4 * nt >= R || tb >= valid) scb = -CUDART_INF_F;
            sc[u][nt][0] = sca;
            sc[u][nt][1] = scb;
          }
        }
        float m_new[NT];
        bool up = false;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          float mx = fmaxf(fmaxf(sc[0][nt][0], sc[0][nt][1]), fmaxf(sc[1][nt][0], sc[1][nt][1]));
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 4));
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 8));
          mx = fmaxf(mx, __shfl_xor_sync(FULL, mx, 16));
          m_new[nt] = fmaxf(m_run[nt], mx);
          up |= m_new[nt] > m_run[nt];
        }
        // the running sums are rescaled only when some row maximum grew
        const bool grow = __any_sync(FULL, up);
        float alpha[NT], p[2][NT][2];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
          alpha[nt] = 1.f;
          p[0][nt][0] = p[0][nt][1] = p[1][nt][0] = p[1][nt][1] = 0.f;
          if (m_new[nt] != -CUDART_INF_F) {
            if (grow) alpha[nt] = exp2f(m_run[nt] - m_new[nt]);
#pragma unroll
            for (int u = 0; u < 2; ++u) {
              p[u][nt][0] = exp2f(sc[u][nt][0] - m_new[nt]);
              p[u][nt][1] = exp2f(sc[u][nt][1] - m_new[nt]);
            }
          }
          l_run[nt] = l_run[nt] * alpha[nt] + (p[0][nt][0] + p[0][nt][1]) + (p[1][nt][0] + p[1][nt][1]);
          if (DT) x_run[nt] *= alpha[nt];
          m_run[nt] = m_new[nt];
        }
        if (grow) {
          // the accumulator columns are rows 2 t4 and 2 t4 + 1: their factors come from the
          // lanes holding those rows' scores (row r: lane r % 4, tile r / 4)
          const int r0 = 2 * t4, r1 = 2 * t4 + 1;
          float al0 = __shfl_sync(FULL, alpha[0], r0 & 3);
          float al1 = __shfl_sync(FULL, alpha[0], r1 & 3);
          if (NT == 2) {
            const float b0 = __shfl_sync(FULL, alpha[NT - 1], r0 & 3);
            const float b1 = __shfl_sync(FULL, alpha[NT - 1], r1 & 3);
            if (r0 >= 4) al0 = b0;
            if (r1 >= 4) al1 = b1;
          }
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) {
            acc[mt][0] *= al0;
            acc[mt][1] *= al1;
            acc[mt][2] *= al0;
            acc[mt][3] *= al1;
          }
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int step = 2 * pr + u;
          const int ta = step * 16 + g, tb = ta + 8;
          const float vnA = ld_h(st + 4 * kUnit + 2 * ta), vnB = ld_h(st + 4 * kUnit + 2 * tb);
          if (DT) {
            // the values' offsets: xi_v to every coordinate, one running sum per row
            const float xa = ta < valid ? vnA * ld_h(st + 8 * kUnit + 2 * ta) : 0.f;
            const float xb = tb < valid ? vnB * ld_h(st + 8 * kUnit + 2 * tb) : 0.f;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) x_run[nt] = fmaf(p[u][nt][0], xa, fmaf(p[u][nt][1], xb, x_run[nt]));
          }
          // B = weights: column g is row g, from the lane holding row g's scores for the
          // tokens of B rows 2 t4 (+ 1, + 8, + 9); slots past the end may hold stale bytes:
          // their weight is forced to exactly 0
          const int src1 = 4 * (2 * t4) + (g & 3), src2 = 4 * (2 * t4 + 1) + (g & 3);
          uint32_t pk = pack_h2(ta < valid ? p[u][0][0] * vnA : 0.f, tb < valid ? p[u][0][1] * vnB : 0.f);
          uint32_t x1 = __shfl_sync(FULL, pk, src1);
          uint32_t x2 = __shfl_sync(FULL, pk, src2);
          if (NT == 2) {
            pk = pack_h2(ta < valid ? p[u][NT - 1][0] * vnA : 0.f, tb < valid ? p[u][NT - 1][1] * vnB : 0.f);
            const uint32_t y1 = __shfl_sync(FULL, pk, src1);
            const uint32_t y2 = __shfl_sync(FULL, pk, src2);
            if (g >= 4) {
              x1 = y1;
              x2 = y2;
            }
          }
          uint32_t b0 = prmt(x1, x2, 0x5410), b1 = prmt(x1, x2, 0x7632);
          uint32_t b0r = 0, b1r = 0;
          if (VQ) {
            // the value product keeps columns 0..3 (rows); columns 4..7 take the sign-space
            // weights p_t ||r_v||_t of rows 0..3 in a second mma
            const float rvA = ld_h(st + 10 * kUnit + 2 * ta), rvB = ld_h(st + 10 * kUnit + 2 * tb);
            const uint32_t pr2 = pack_h2(ta < valid ? p[u][0][0] * rvA : 0.f, tb < valid ? p[u][0][1] * rvB : 0.f);
            const uint32_t r1 = __shfl_sync(FULL, pr2, src1), r2 = __shfl_sync(FULL, pr2, src2);
            if (g >= 4) {
              b0r = prmt(r1, r2, 0x5410);
              b1r = prmt(r1, r2, 0x7632);
              b0 = b1 = 0u;
            }
          }
            // ---- values: dequantise (pairs of coordinates of one token), transpose, mma
            uint32_t va[16], vb[16];
            {
              const unsigned char* vq = vc + (t4 >> 1) * kChunkStride + (t4 & 1) * 8;
              const uint2 ca = *reinterpret_cast<const uint2*>(vq + ta * 16);
              const uint2 cbv = *reinterpret_cast<const uint2*>(vq + tb * 16);
              uint32_t sgA = 0, sgB = 0;
              if (VP == V3) {
                sgA = *reinterpret_cast<const uint32_t*>(vc + 2 * kChunkStride + ta * 16 + 4 * t4);
                sgB = *reinterpret_cast<const uint32_t*>(vc + 2 * kChunkStride + tb * 16 + 4 * t4);
              }
    #pragma unroll
              for (int hk = 0; hk < 8; ++hk) {
                const int h = hk >> 2, k = hk & 3;
                uint32_t sa[2], sb[2];
                crumb_sel2(h ? ca.y : ca.x, k, sa[0], sa[1]);
                crumb_sel2(h ? cbv.y : cbv.x, k, sb[0], sb[1]);
    #pragma unroll
                for (int q = 0; q < 2; ++q) {
                  const int cb = 8 * h + 4 * q + k;
                  uint32_t xa = prmt(vt_lo, vt_hi, sa[q]);
                  uint32_t xb = prmt(vt_lo, vt_hi, sb[q]);
                  if (VP == V3) {
                    xa ^= (sgA << (15 - cb)) & 0x80008000u;
                    xb ^= (sgB << (15 - cb)) & 0x80008000u;
                  }
                  va[cb] = movm_t(xa);
                  vb[cb] = movm_t(xb);
                }
              }
            }
#pragma unroll
          for (int mt = 0; mt < 8; ++mt) hmma(acc[mt], va[2 * mt], va[2 * mt + 1], vb[2 * mt], vb[2 * mt + 1], b0, b1);
          if (VQ) {
            // the signs as fp16 +-1 for the same coordinate pairs, transposed like the values
            const unsigned char* vsq = vc + kVChunks * kChunkStride;
            const uint32_t wA = ~*reinterpret_cast<const uint32_t*>(vsq + ta * 16 + 4 * t4);
            const uint32_t wB = ~*reinterpret_cast<const uint32_t*>(vsq + tb * 16 + 4 * t4);
            uint32_t qa[16], qb[16];
#pragma unroll
            for (int cb = 0; cb < 16; ++cb) {
              const int pb = pair_base(cb);
              // bits pb and pb + 4 (a clear sigma means -1) to the two halves' sign bits
              const uint32_t xa = (((wA >> pb) & 0x11u) * 0x08008000u & 0x80008000u) | 0x3C003C00u;
              const uint32_t xb = (((wB >> pb) & 0x11u) * 0x08008000u & 0x80008000u) | 0x3C003C00u;
              qa[cb] = movm_t(xa);
              qb[cb] = movm_t(xb);
            }
#pragma unroll
            for (int mt = 0; mt < 8; ++mt)
              hmma(acc[mt], qa[2 * mt], qa[2 * mt + 1], qb[2 * mt], qb[2 * mt + 1], b0r, b1r);
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&sm.empty[s]);
    }
    // the B fragments in shared memory are read until every consumer warp has left the loop
    if constexpr (kBSmem) asm volatile("bar.sync 1, %0;" ::"n"(kConsumerWarps * 32) : "memory");
    // ---- warp partial: l summed over the 8 lanes of a row, acc scattered by coordinate
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      float lr = l_run[nt], xr = x_run[nt];
      lr += __shfl_xor_sync(FULL, lr, 4);
      lr += __shfl_xor_sync(FULL, lr, 8);
      lr += __shfl_xor_sync(FULL, lr, 16);
      if (DT) {
        xr += __shfl_xor_sync(FULL, xr, 4);
        xr += __shfl_xor_sync(FULL, xr, 8);
        xr += __shfl_xor_sync(FULL, xr, 16);
      }
      if (g == 0 && t4 + 4 * nt < R) {
        sm.wm[warp][t4 + 4 * nt] = m_run[nt];
        sm.wl[warp][t4 + 4 * nt] = lr;
        sm.wx[warp][t4 + 4 * nt] = xr;
      }
    }
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int row = 2 * t4 + (e & 1);
        const int cb = 2 * mt + (e >> 1);
        const int coord = 32 * (g >> 1) + pair_base(cb) + 4 * (g & 1);
        if (VQ && row >= 4) {
          if (row - 4 < R) sm.ring.wsig[warp][row - 4][coord] = acc[mt][e];
        } else if (row < R) {
          sm.ring.wacc[warp][row][coord] = acc[mt][e];
        }
      }
    }
  }
  __syncthreads();
  // ---- merge the consumer warps and write this split's partial
  // per row: the maximum over the warps, each warp's factor, the sum (natural-log domain
  // for the merge across splits)
  if (tid < R) {
    float M = -CUDART_INF_F;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) M = fmaxf(M, sm.wm[w][tid]);
    float l = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w) {
      const float f = (M == -CUDART_INF_F || sm.wm[w][tid] == -CUDART_INF_F) ? 0.f : exp2f(sm.wm[w][tid] - M);
      sm.wf[w][tid] = f;
      l = fmaf(f, sm.wl[w][tid], l);
    }
    const size_t pr = (row0 + tid) * a.n_splits + split;
    TQ_DCHECK(a.status, split < a.n_splits);
    a.part_ml[pr * 2] = (M == -CUDART_INF_F) ? M : M / kLog2e;
    a.part_ml[pr * 2 + 1] = l;
  }
  __syncthreads();
  for (int idx = tid; idx < R * D; idx += blockDim.x) {
    const int r = idx / D, j = idx % D;
    float o = 0.f;
#pragma unroll
    for (int w = 0; w < kConsumerWarps; ++w)
      o = fmaf(sm.wf[w][r], DT ? sm.ring.wacc[w][r][j] + sm.wx[w][r] : sm.ring.wacc[w][r][j], o);
    a.part_acc[((row0 + r) * a.n_splits + split) * D + j] = o;
    if (VQ) {
      float os = 0.f;
#pragma unroll
      for (int w = 0; w < kConsumerWarps; ++w) os = fmaf(sm.wf[w][r], sm.ring.wsig[w][r][j], os);
      a.part_sig[((row0 + r) * a.n_splits + split) * QM + j] = os;
    }
  }
  // ---- the last split of this (sequence, kv head) to finish merges all of them ----
  __syncthreads();
  if (tid == 0) {
    // release: the CTA's partial writes (ordered before this by the barrier) are visible to
    // whoever reads the count after it; acquire: the last one sees all the others' partials
    unsigned int done;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;"
                 : "=r"(done)
                 : "l"(&a.counter[((size_t)b * a.cache.kv_heads + gh) * nchunk + chunk])
                 : "memory");
    sm.last = done == (unsigned int)n_split_b - 1;
  }
  __syncthreads();
  if (!sm.last) return;
  const int ns = n_split_b;      // the partials to merge
  const size_t nst = a.n_splits;  // their row stride in the workspace
  // every split's accumulators of every row in one round trip when they fit: a bulk copy per
  // row (the rows' partials are contiguous), landing while the maxima are formed from the
  // (m, l) pairs; otherwise register batches from L2
  constexpr int kCap = kMergeFloats / (NR * D);
  const bool in_smem = ns <= kCap;
  TQ_DCHECK(a.status, ns >= 1 && (size_t)R * kCap * D <= (size_t)kMergeFloats);
  if (in_smem && tid == 0) {
    // the other splits' partials were made visible to this thread by the acquire above;
    // order them before this thread's async-proxy reads
    asm volatile("fence.proxy.async.global;" ::: "memory");
    mbar_expect_tx(&sm.mbar, (uint32_t)(R * ns * D * sizeof(float)));
    for (int rr = 0; rr < R; ++rr)
      bulk_g2s(&sm.merge[rr * kCap * D], a.part_acc + (row0 + rr) * nst * D, (uint32_t)(ns * D * sizeof(float)),
               &sm.mbar);
  }
  // warp w merges rows w, w + 5, ...; lane c4 owns coordinates 4 c4 .. 4 c4 + 3
  for (int r = warp; r < R; r += kThreads / 32) {
    const int c4 = lane;
    const size_t rowq = row0 + r;
    const float2* ml2 = reinterpret_cast<const float2*>(a.part_ml + rowq * nst * 2);
    float* rs = &sm.merge[r * kCap * D];  // row r's region (its partials when in_smem)
    float M = -CUDART_INF_F, l = 0.f;
    float4 o = make_float4(0.f, 0.f, 0.f, 0.f);
    float4 osg = make_float4(0.f, 0.f, 0.f, 0.f);  // values with QJL: the sign-space sums
    const float4* ps4 = reinterpret_cast<const float4*>(a.part_sig + (VQ ? rowq * nst * QM : 0)) + c4;
    if (in_smem) {
      for (int sp = c4; sp < ns; sp += 32) M = fmaxf(M, ml2[sp].x);
#pragma unroll
      for (int h = 16; h > 0; h >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, h));
      const bool live = M != -CUDART_INF_F;
      if (!mbar_wait(&sm.mbar, 0)) {
        report(a.status, TQ_ERR_TIMEOUT);
        mbar_wait(&sm.mbar, 0);  // the copies in flight land before the CTA ends (bounded)
      }
      const float4* pa4 = reinterpret_cast<const float4*>(rs) + c4;
#pragma unroll 8
      for (int sp = 0; sp < ns; ++sp) {
        const float2 m2 = ml2[sp];
        const float4 v = pa4[sp * (D / 4)];
        const float wgt = live ? __expf(m2.x - M) : 0.f;
        l = fmaf(wgt, m2.y, l);
        o.x = fmaf(wgt, v.x, o.x);
        o.y = fmaf(wgt, v.y, o.y);
        o.z = fmaf(wgt, v.z, o.z);
        o.w = fmaf(wgt, v.w, o.w);
        if (VQ) {
          const float4 q = ps4[sp * (QM / 4)];
          osg.x = fmaf(wgt, q.x, osg.x);
          osg.y = fmaf(wgt, q.y, osg.y);
          osg.z = fmaf(wgt, q.z, osg.z);
          osg.w = fmaf(wgt, q.w, osg.w);
        }
      }
    } else {
      // many splits: the partials in register batches of kMB, the first batch before the
      // maximum is formed (about ns / kMB round trips to L2)
      constexpr int kMB = 20;
      const float4* pa4 = reinterpret_cast<const float4*>(a.part_acc + rowq * nst * D) + c4;
      for (int s0 = 0; s0 < ns; s0 += kMB) {
        float4 v[kMB];
        float2 m2[kMB];
#pragma unroll
        for (int k = 0; k < kMB; ++k) {
          if (s0 + k < ns) {
            v[k] = pa4[(size_t)(s0 + k) * (D / 4)];
            m2[k] = ml2[s0 + k];
          }
        }
        if (s0 == 0) {
          for (int sp = c4; sp < ns; sp += 32) M = fmaxf(M, ml2[sp].x);
#pragma unroll
          for (int h = 16; h > 0; h >>= 1) M = fmaxf(M, __shfl_xor_sync(FULL, M, h));
        }
        const bool live = M != -CUDART_INF_F;
#pragma unroll
        for (int k = 0; k < kMB; ++k) {
          if (s0 + k < ns) {
            const float wgt = live ? __expf(m2[k].x - M) : 0.f;
            l = fmaf(wgt, m2[k].y, l);
            o.x = fmaf(wgt, v[k].x, o.x);
            o.y = fmaf(wgt, v[k].y, o.y);
            o.z = fmaf(wgt, v[k].z, o.z);
            o.w = fmaf(wgt, v[k].w, o.w);
            if (VQ) {
              const float4 q = ps4[(size_t)(s0 + k) * (QM / 4)];
              osg.x = fmaf(wgt, q.x, osg.x);
              osg.y = fmaf(wgt, q.y, osg.y);
              osg.z = fmaf(wgt, q.z, osg.z);
              osg.w = fmaf(wgt, q.w, osg.w);
            }
          }
        }
      }
    }
    const float inv = l > 0.f ? 1.f / l : 0.f;
    float x[4] = {o.x * inv, o.y * inv, o.z * inv, o.w * inv};
    // values with QJL: + sqrt(pi/2)/m S^T (sign-space sums / l), lane c4 forming outputs
    // 4 c4 .. 4 c4 + 3 from rows of S (coalesced across c4)
    float sg[4] = {0.f, 0.f, 0.f, 0.f};
    if (VQ) {
      float* xs = sm.xsig[r];
      *reinterpret_cast<float4*>(xs + 4 * c4) = make_float4(osg.x * inv, osg.y * inv, osg.z * inv, osg.w * inv);
      __syncwarp();
      const float4* s4 = reinterpret_cast<const float4*>(a.s) + c4;
#pragma unroll 8
      for (int i = 0; i < QM; ++i) {
        const float4 p = s4[(size_t)i * (D / 4)];
        const float xi = xs[i];
        sg[0] = fmaf(p.x, xi, sg[0]);
        sg[1] = fmaf(p.y, xi, sg[1]);
        sg[2] = fmaf(p.z, xi, sg[2]);
        sg[3] = fmaf(p.w, xi, sg[3]);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) sg[e] *= kQjlScale;
    }
    if (a.dense) {
      // out = Pi^T (o / l): the row's 128 values through its own region of shared memory
      // (every lane of this warp is past reading it), then lane c4 forms outputs
      // 4 c4 .. 4 c4 + 3 from rows of Pi (coalesced across c4)
      __syncwarp();
      *reinterpret_cast<float4*>(rs + 4 * c4) = make_float4(x[0], x[1], x[2], x[3]);
      __syncwarp();
      float4 y = make_float4(0.f, 0.f, 0.f, 0.f);
      const float4* pi4 = reinterpret_cast<const float4*>(a.pi) + c4;
#pragma unroll 8
      for (int i = 0; i < D; ++i) {
        const float4 p = pi4[(size_t)i * (D / 4)];
        const float xi = rs[i];
        y.x = fmaf(p.x, xi, y.x);
        y.y = fmaf(p.y, xi, y.y);
        y.z = fmaf(p.z, xi, y.z);
        y.w = fmaf(p.w, xi, y.w);
      }
      *reinterpret_cast<float4*>(a.out + rowq * D + 4 * c4) = make_float4(y.x + sg[0], y.y + sg[1], y.z + sg[2], y.w + sg[3]);
      continue;
    }
    // out = D H (o / l) / sqrt(d): H over coordinates 4 c4 + e, spans 1 and 2 in the
    // thread, spans 4..64 across the row's 32 lanes
    {
      const float a0 = x[0] + x[1], a1 = x[0] - x[1], a2 = x[2] + x[3], a3 = x[2] - x[3];
      x[0] = a0 + a2;
      x[1] = a1 + a3;
      x[2] = a0 - a2;
      x[3] = a1 - a3;
    }
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float y = __shfl_xor_sync(FULL, x[e], h);
        x[e] = (c4 & h) ? (y - x[e]) : (x[e] + y);
      }
    }
#pragma unroll
    for (int e = 0; e < 4; ++e) a.out[rowq * D + 4 * c4 + e] = fmaf(x[e] * kInvSqrtD, a.signs[4 * c4 + e], sg[e]);
  }
}

}  // namespace

bool fast_decode_supported(const DecodeArgs& a) {
  const Layout& L = a.cache.L;
  // the merge reads Pi as float4
  if (a.dense && (reinterpret_cast<uintptr_t>(a.pi) & 15)) return false;
  const bool kok = (L.kbits == 3 && L.qjl) || (L.kbits == 2 && L.qjl) || (L.kbits == 4 && !L.qjl);
  // values with QJL: up to four query rows per KV head, not dithered, S read as float4
  const bool vqok = !L.vqjl || (a.rows <= 4 && !L.dither && !(reinterpret_cast<uintptr_t>(a.s) & 15));
  const bool vok = (L.vbits == 3 || L.vbits == 2) && vqok;
  return kok && vok;
}

size_t fast_decode_smem_bytes() { return sizeof(SmemFast); }

cudaError_t launch_fast_split(const DecodeArgs& a, cudaStream_t stream) {
  const Layout& L = a.cache.L;
  const size_t smem = sizeof(SmemFast);
  // eight rows per CTA when a KV head has more than four query rows
  const int nr = a.rows > 4 ? 8 : 4;
  dim3 grid(a.n_splits, a.cache.kv_heads, a.cache.batch * ((a.rows + nr - 1) / nr));
  void (*k)(DecodeArgs) = nullptr;
#define TQ_FAST(KB, KPOL, VB, VPOL)                                                                   \
  if (L.kbits == KB && L.vbits == VB) {                                                                \
    if (L.vqjl)                                                                                        \
      k = fast_split_kernel<KPOL, VPOL, 4, false, true>;                                               \
    else if (L.dither)                                                                                 \
      k = nr == 8 ? fast_split_kernel<KPOL, VPOL, 8, true, false> : fast_split_kernel<KPOL, VPOL, 4, true, false>; \
    else                                                                                               \
      k = nr == 8 ? fast_split_kernel<KPOL, VPOL, 8, false, false> : fast_split_kernel<KPOL, VPOL, 4, false, false>; \
  }
  TQ_FAST(3, K3Q, 3, V3)
  TQ_FAST(3, K3Q, 2, V2)
  TQ_FAST(2, K2Q, 3, V3)
  TQ_FAST(2, K2Q, 2, V2)
  TQ_FAST(4, K4, 3, V3)
  TQ_FAST(4, K4, 2, V2)
#undef TQ_FAST
  if (!k) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  // programmatic launch: page streaming starts while the prologue is still running
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  e = cudaLaunchKernelEx(&cfg, k, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace tqk
