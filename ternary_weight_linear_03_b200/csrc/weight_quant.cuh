// Absmean ternary weight quantization (BitNet b1.58; dmarx anthology record LIT-380, Key
// takeaways bullet 1: weights constrained to {-1, 0, +1} by an absmean quantization
// function; searcharxiv.com abstract page, Abstract: every weight is ternary).
//
// One cooperative kernel, two lean passes over W. The second pass reads the stages still
// held in shared memory when a block's whole range fits its ring, and is otherwise served
// from L2 whenever W fits there. Every block owns a contiguous range of 16-weight words
// and streams it through a ring of 16 KB bulk copies (cp.async.bulk into shared memory, 4
// in flight per block); thread t handles the 16-byte chunks t + 256 i of each stage.
//   A  exact sum of |w| (below) into exponent buckets, folded into column sums;
//   -- grid barrier (bounded wait) --
//      every block turns the column sums into gamma = fl32(fl64(S) / n) and the
//      threshold T;
//   B  code = (w >= T) - (-w >= T), stored as u = code + 1; the 4 (fp32) or 2 (bf16) lanes
//      holding the chunks of one packed word merge their bits with shuffles.
//
// Threshold. RoundClip(fl(w/d), -1, 1) is +1 exactly when fl(w/d) > 0.5 (0.5 itself
// rounds to the even 0, and every quotient >= 1.5 clips to 1). Correctly rounded
// division is monotone in w, so there is one smallest float T with fl(T/d) > 0.5, and
// c = +1 iff w >= T, c = -1 iff -w >= T.
//
// Exact sum. Each warp fixes an exponent window [base, base + 20] from the largest
// exponent in its first stage (base = that exponent - 17, at least 1). A float |w| in the
// window is an integer multiple of u = 2^(base - 150) below 2^44 u, so up to 256 of them
// add up exactly in a double; a thread keeps two such doubles (alternate weights, so the
// additions do not form one long dependency chain) and every 16 stages the warp converts
// them to integers, sums those with shuffles and adds the result into 64-bit exponent
// buckets (low 32 bits at exponent base, the rest at base + 32). Values outside the
// window (subnormals, far larger or smaller ones) go straight into the buckets as
// (exponent, 24-bit mantissa). Each block then folds its buckets into the 14 column sums
// of a 448-bit integer (bucket e adds B[e] << ((e - 1) % 32) at 32-bit limb (e - 1) / 32)
// and adds the non-zero ones into one of kWqCopies copies in the workspace (spreading the
// same-address atomics); after the grid barrier every block adds the copies, propagates
// the carries and rounds once. All of it is integer arithmetic, so gamma depends neither
// on the grid nor on the order of the atomic adds.
#pragma once

#include "act_quant.cuh"
#include "common.cuh"

namespace bl {

constexpr int kWqBuckets = 320;  // exponent buckets: e in [0, 254] plus spill-over
constexpr int kWqThreads = 256;
constexpr int kWqLimbs = 14;     // 32-bit limbs of the exact sum (S * 2^149 < 2^448)
constexpr int kWqWindow = 21;    // exponents covered by the fp64 window
constexpr int kWqFlushWords = 16;  // words a thread sums in fp64 between bucket flushes
constexpr int kWqCopies = 8;       // copies of the column sums and arrival counters

// The quantize_weights workspace (zeroed by the host before each launch). Block b adds
// into copy b % kWqCopies.
struct WqWorkspace {
  unsigned long long cols[kWqCopies][kWqLimbs];  // column sums (below 2^39 per block)
  unsigned int arrived[kWqCopies];               // grid-barrier arrivals
  double est_sum;                                // single-read mode: sampled sum of |w|
  unsigned long long est_cnt;                    //   and the number of sampled weights
  unsigned int arrived_est[kWqCopies];           //   arrivals at the estimate barrier
};

// Single-read mode (large matrices): band entries per block, and the band's half width
// relative to the estimated threshold.
constexpr int kWqListCap = 4096;
constexpr int kWqMaxBlocks = 1024;
constexpr float kWqBand = 1.0f / 256.0f;

// Bounded grid barrier on spread arrival counters (thread 0 of each block calls it).
__device__ __forceinline__ bool wq_grid_barrier(unsigned int* arrived, unsigned int nblocks,
                                                unsigned long long limit_ns) {
  __threadfence();
  atomicAdd(&arrived[blockIdx.x % kWqCopies], 1u);
  const uint64_t t0 = global_ns();
  while (true) {
    unsigned int total = 0u;
#pragma unroll
    for (int c = 0; c < kWqCopies; ++c) {
      unsigned v;
      asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(arrived + c) : "memory");
      total += v;
    }
    if (total >= nblocks) return true;
    if (global_ns() - t0 > limit_ns) {
      record_status(kStatusTimeout);
      return false;
    }
    __nanosleep(64);
  }
}

// |w| outside the fp64 window: added as (exponent, mantissa) into the shared buckets.
__device__ __forceinline__ void wq_fallback(uint32_t bits, unsigned long long* sb,
                                            bool& nonfinite) {
  const uint32_t e = bits >> 23;
  if (e == 255u) {
    nonfinite = true;
  } else if (e == 0u) {
    atomicAdd(&sb[1], static_cast<unsigned long long>(bits));  // subnormal: unit 2^-149
  } else {
    atomicAdd(&sb[e], static_cast<unsigned long long>((bits & 0x7fffffu) | 0x800000u));
  }
}

// Moves a warp's fp64 window sums into the buckets. Called by all 32 lanes together (the
// window base is the same for the whole warp). Each lane's a0 + a1 is an integer multiple
// of 2^(base-150) below 2^52 of those units, so the scaled conversion is exact; the warp
// adds the 32 integers with shuffles (below 2^57) and one lane adds the low 32 bits at
// exponent base and the rest at base + 32, so the shared buckets see 2 atomics per warp.
__device__ __forceinline__ void wq_flush(double& a0, double& a1, int base,
                                         unsigned long long* sb) {
  const double scale = __longlong_as_double(static_cast<long long>(1023 + 150 - base) << 52);
  unsigned long long u = __double2ull_rz(__dmul_rn(__dadd_rn(a0, a1), scale));
  a0 = 0.0;
  a1 = 0.0;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) u += __shfl_xor_sync(0xffffffffu, u, off);
  if ((threadIdx.x & 31) == 0 && u != 0ull) {
    atomicAdd(&sb[base], u & 0xffffffffull);
    if (u >> 32) atomicAdd(&sb[base + 32], u >> 32);
  }
}

__device__ __forceinline__ int wq_shift(int k) { return 8 * (k & 3) + 2 * (k >> 2); }

// Rounds the non-negative integer sum_j L[j] 2^(32 j) times 2^-149 once to double (ties
// to even). L has kWqLimbs little-endian 32-bit limbs.
__device__ double wq_limbs_to_double(const uint32_t* L) {
  int top = kWqLimbs - 1;
  while (top >= 0 && L[top] == 0u) --top;
  if (top < 0) return 0.0;
  const int lz = __clz(L[top]);
  const int topbit = top * 32 + (31 - lz);  // position of the leading one
  const uint32_t w2 = L[top];
  const uint32_t w1 = (top >= 1) ? L[top - 1] : 0u;
  const uint32_t w0 = (top >= 2) ? L[top - 2] : 0u;
  bool sticky = false;
  for (int i = 0; i < top - 2; ++i) sticky |= (L[i] != 0u);
  // X = (w2:w1:w0) << lz has the leading one in bit 95; limbs below only feed sticky.
  const uint32_t x2 = __funnelshift_l(w1, w2, lz);
  const uint32_t x1 = __funnelshift_l(w0, w1, lz);
  const uint32_t x0 = w0 << lz;
  const uint64_t hi64 = (static_cast<uint64_t>(x2) << 32) | x1;  // X bits 95..32
  uint64_t mant = hi64 >> 11;                                       // X bits 95..43
  const bool half = (hi64 >> 10) & 1ull;                            // X bit 42
  sticky |= ((hi64 & 0x3ffull) != 0ull) || (x0 != 0u);
  if (half && (sticky || (mant & 1ull))) mant += 1ull;
  return ldexp(static_cast<double>(mant), topbit - 52 - 149);
}

// Smallest float t with fl(t / d) > 0.5, +inf when no finite t qualifies (d == 0 or inf).
// For d > 0, correctly rounded division gives fl(t / d) > 0.5 exactly when t / d lies
// above the midpoint 0.5 + 2^-25 between 0.5 and the next float (at the midpoint itself
// the tie goes to the even 0.5), i.e. when t > m = d * (0.5 + 2^-25). m has at most
// 24 + 26 significant bits, so the double product is exact, and t is the smallest float
// strictly above m: m rounded up, stepped once more if m is itself a float.
__device__ float wq_threshold(float d) {
  if (!(d > 0.0f) || isinf(d)) return __int_as_float(0x7f800000);
  const double m = __dmul_rn(static_cast<double>(d), 0.5 + 0x1p-25);
  float t = __double2float_ru(m);
  if (static_cast<double>(t) == m) t = __int_as_float(__float_as_int(t) + 1);  // m > 0
  return t;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// 1-D bulk copy global -> shared, completing on an mbarrier (no tensor map, no multicast).
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

constexpr int kWqStageBytes = 16384;  // one bulk copy
constexpr int kWqStages = 4;          // ring depth per block
constexpr int kWqChunks = kWqStageBytes / 16 / kWqThreads;  // 16-byte chunks per thread

// The weights of one 16-byte chunk as floats: 4 fp32 or 8 bf16 (widened exactly).
template <bool kBf16>
__device__ __forceinline__ void wq_chunk_floats(const uint4 c, float (&w)[kBf16 ? 8 : 4]) {
  if (kBf16) {
    const uint32_t h[4] = {c.x, c.y, c.z, c.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      w[2 * q] = __uint_as_float(h[q] << 16);
      w[2 * q + 1] = __uint_as_float(h[q] & 0xffff0000u);
    }
  } else {
    w[0] = __uint_as_float(c.x);
    w[1] = __uint_as_float(c.y);
    w[2] = __uint_as_float(c.z);
    w[3] = __uint_as_float(c.w);
  }
}

// Position in its packed word of element e of a chunk: a word holds 16 weights = 4 fp32
// chunks (chunk part p = 0..3) or 2 bf16 chunks (p = 0..1); relative index k = E*p + e.
template <bool kBf16>
__device__ __forceinline__ int wq_k(int part, int e) {
  return (kBf16 ? 8 : 4) * part + e;
}

// OR of a value over the lanes that hold the parts of one packed word.
template <bool kBf16>
__device__ __forceinline__ uint32_t wq_or_parts(uint32_t v) {
  v |= __shfl_xor_sync(0xffffffffu, v, 1);
  if (!kBf16) v |= __shfl_xor_sync(0xffffffffu, v, 2);
  return v;
}

// Streams the block's byte range [src, src + bytes) through the stage ring; `g` counts
// the stages this block has consumed so far (slot and phase parity follow from it).
struct WqRing {
  unsigned char* stage;  // kWqStages x kWqStageBytes
  uint64_t* full;        // kWqStages mbarriers
  const char* src;
  long long bytes;
  int nst;               // stages of one pass over the range
};

// Issues stage st of a pass (bytes st * 16 KB ..) as the block's g-th stage overall.
__device__ __forceinline__ void wq_issue(const WqRing& r, int st, int g) {
  const uint32_t nb = static_cast<uint32_t>(
      min(static_cast<long long>(kWqStageBytes), r.bytes - 1ll * st * kWqStageBytes));
  const int slot = g % kWqStages;
  mbar_arrive_expect_tx(&r.full[slot], nb);
  bulk_load(r.stage + slot * kWqStageBytes, r.src + 1ll * st * kWqStageBytes, nb, &r.full[slot]);
}

// What one launch does. A matrix split over several GPUs (tensor parallelism) still has
// one gamma, the mean over the whole matrix: every shard computes its part of the exact
// sum (kWqPartial), the parts are added across the GPUs (the kWqLimbs 64-bit column sums
// add exactly, like any integers below 2^64), and every shard then codes its weights
// against that total (kWqFinish).
enum WqMode : int {
  kWqFull = 0,     // exact sum, gamma, codes: the whole matrix in one launch
  kWqPartial = 1,  // exact sum only: writes the kWqLimbs column sums to sums_io
  kWqFinish = 2,   // gamma and codes from the column sums in sums_io, over n_total values
};

// The kWqLimbs column sums of the block copies in the workspace, added (below 2^64: each
// is below 2^39 times the grid size).
__device__ __forceinline__ unsigned long long wq_column_total(const WqWorkspace* ws, int j) {
  unsigned long long t = 0ull;
#pragma unroll
  for (int c = 0; c < kWqCopies; ++c) t += __ldcg(&ws->cols[c][j]);
  return t;
}

// W holds n values (fp32, or bf16 if kBf16), n % 16 == 0, 16-byte aligned. Launched
// cooperatively (all blocks resident) with kWqStages * kWqStageBytes of dynamic shared
// memory. ws is zeroed by the host (kWqFull, kWqPartial). gamma is the exact sum over
// n_total values (n_total = n except for kWqFinish on a shard).
template <bool kBf16, int MODE>
__global__ void __launch_bounds__(kWqThreads) weight_quant_kernel(
    const void* __restrict__ W, long long n, long long n_total, float eps,
    WqWorkspace* __restrict__ ws, unsigned long long* __restrict__ sums_io,
    float* __restrict__ gamma_out, uint32_t* __restrict__ packed, unsigned long long limit_ns,
    uint2* __restrict__ list) {
  extern __shared__ __align__(128) unsigned char wq_stage[];  // kWqStages x 16 KB
  __shared__ unsigned long long sb[kWqBuckets];
  __shared__ unsigned long long col[kWqLimbs];
  __shared__ uint64_t full[kWqStages];
  __shared__ float s_T;
  __shared__ int s_ok;
  __shared__ float s_that;          // single-read mode: estimated threshold
  __shared__ unsigned int s_cnt;    //   band entries of this block
  __shared__ double s_red[kWqThreads / 32];
  constexpr int E = kBf16 ? 8 : 4;   // weights per 16-byte chunk
  constexpr int PARTS = 16 / E;      // chunks per packed word
  constexpr int WORD_BYTES = kBf16 ? 32 : 64;

  const int tid = threadIdx.x;
  for (int i = tid; i < kWqBuckets; i += blockDim.x) sb[i] = 0ull;
  if (tid < kWqLimbs) col[tid] = 0ull;
  const long long nwords = n / 16;
  const long long per_block = (nwords + gridDim.x - 1) / gridDim.x;
  const long long wb0 = min(nwords, static_cast<long long>(blockIdx.x) * per_block);
  const long long wb1 = min(nwords, wb0 + per_block);
  WqRing ring;
  ring.stage = wq_stage;
  ring.full = full;
  ring.src = static_cast<const char*>(W) + wb0 * WORD_BYTES;
  ring.bytes = (wb1 - wb0) * WORD_BYTES;
  ring.nst = static_cast<int>((ring.bytes + kWqStageBytes - 1) / kWqStageBytes);
  if (tid == 0) {
    s_ok = 1;
    for (int i = 0; i < kWqStages; ++i) mbar_init(&full[i], 1);
    fence_mbar_init();
    for (int st = 0; st < min(ring.nst, kWqStages); ++st) wq_issue(ring, st, st);
  }
  __syncthreads();

  // Single-read mode (MODE kWqFull with a band list, chosen by the host when the blocks'
  // ranges do not fit their rings): pass A also codes every weight against an estimated
  // threshold T^ (from the mean |w| of every block's first stage, after a first grid
  // barrier) and lists the weights with |w| within kWqBand * T^ of it. Once the exact T is
  // known, a code can differ from the provisional one only for |w| between T^ and T, so
  // when T lies inside the band each block patches its listed weights; otherwise (or when
  // its list overflowed) it streams its range again as in the two-pass mode.
  const bool single = (MODE == kWqFull) && (list != nullptr);
  float t_hat = 0.0f, band_lo = 1.0f, band_hi = 0.0f;  // empty band
  const int mypart = tid & (PARTS - 1);
  uint32_t mulA[E];
#pragma unroll
  for (int e = 0; e < E; ++e) mulA[e] = 1u << wq_shift(wq_k<kBf16>(mypart, e));
  if (single) {
    double part = 0.0;
    const int n0c = static_cast<int>(min(static_cast<long long>(kWqStageBytes), ring.bytes) / 16);
    if (ring.nst > 0) {
      if (!mbar_wait(&full[0], 0u, limit_ns)) s_ok = 0;
      const uint4* stage = reinterpret_cast<const uint4*>(wq_stage);
#pragma unroll
      for (int i = 0; i < kWqChunks; ++i) {
        const int c = tid + i * kWqThreads;
        if (c < n0c) {
          float w[E];
          wq_chunk_floats<kBf16>(stage[c], w);
#pragma unroll
          for (int e = 0; e < E; ++e) part += static_cast<double>(abs_bits(w[e]));
        }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) part += __shfl_xor_sync(0xffffffffu, part, off);
    if ((tid & 31) == 0) s_red[tid >> 5] = part;
    __syncthreads();
    if (tid == 0) {
      double b = 0.0;
      for (int w = 0; w < kWqThreads / 32; ++w) b += s_red[w];
      atomicAdd(&ws->est_sum, b);
      atomicAdd(&ws->est_cnt, static_cast<unsigned long long>(n0c) * E);
      if (!wq_grid_barrier(ws->arrived_est, gridDim.x, limit_ns)) s_ok = 0;
      const unsigned long long cnt = __ldcg(&ws->est_cnt);
      const double est = __ldcg(&ws->est_sum) / static_cast<double>(cnt > 0ull ? cnt : 1ull);
      s_that = wq_threshold(__fadd_rn(__double2float_rn(est), eps));
      s_cnt = 0u;
    }
    __syncthreads();
    t_hat = s_that;
    band_lo = t_hat * (1.0f - kWqBand);
    band_hi = t_hat * (1.0f + kWqBand);
  }

  // ---------------------------------------------------------------- pass A: exact sum
  bool resident = false;  // pass B reads pass A's stages from shared memory
  if (MODE != kWqFinish) {
  double acc0 = 0.0, acc1 = 0.0;
  bool nonfinite = false;
  int base = 1;
  float lo_f = 0.0f, hi_f = 0.0f;
  for (int st = 0; st < ring.nst; ++st) {
    const int slot = st % kWqStages;
    if (!mbar_wait(&full[slot], static_cast<uint32_t>((st / kWqStages) & 1), limit_ns)) s_ok = 0;
    const uint4* stage = reinterpret_cast<const uint4*>(wq_stage + slot * kWqStageBytes);
    const int nchunks = static_cast<int>(
        min(static_cast<long long>(kWqStageBytes), ring.bytes - 1ll * st * kWqStageBytes) / 16);
    uint4 ch[kWqChunks];
#pragma unroll
    for (int i = 0; i < kWqChunks; ++i) {
      const int c = tid + i * kWqThreads;
      ch[i] = (c < nchunks) ? stage[c] : make_uint4(0u, 0u, 0u, 0u);  // zeros add nothing
    }
    if (st == 0) {  // exponent window of this warp
      int emax = 0;
#pragma unroll
      for (int i = 0; i < kWqChunks; ++i) {
        float w[E];
        wq_chunk_floats<kBf16>(ch[i], w);
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const int ex = static_cast<int>((__float_as_uint(w[e]) >> 23) & 0xffu);
          if (ex != 255) emax = max(emax, ex);
        }
      }
      emax = __reduce_max_sync(0xffffffffu, emax);
      base = max(1, emax + 4 - kWqWindow);
      lo_f = __uint_as_float(static_cast<uint32_t>(base) << 23);
      hi_f = (base + kWqWindow <= 254)
                 ? __uint_as_float(static_cast<uint32_t>(base + kWqWindow) << 23)
                 : __int_as_float(0x7f800000);
    }
    // Non-negative floats order like their bit patterns: the window test and (single-read
    // mode) the threshold and band tests are single unsigned compares of |w|'s bits.
    const uint32_t lo_b = __float_as_uint(lo_f), span_b = __float_as_uint(hi_f) - lo_b;
    const uint32_t t_b = __float_as_uint(t_hat);
    const uint32_t band_b = __float_as_uint(band_lo);
    const uint32_t bspan_b = __float_as_uint(band_hi) - band_b;
#pragma unroll
    for (int i = 0; i < kWqChunks; ++i) {
      float w[E];
      wq_chunk_floats<kBf16>(ch[i], w);
      bool out_any = false;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const uint32_t ab = __float_as_uint(w[e]) & 0x7fffffffu;
        const bool in = (ab - lo_b) < span_b;  // lo_f <= |w| < hi_f
        out_any |= !in;
        const float a = __uint_as_float(in ? ab : 0u);
        if (e & 1) acc1 += static_cast<double>(a);  // exact: see the header
        else acc0 += static_cast<double>(a);
      }
      if (out_any) {  // rare: zeros and values outside the window
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const float a = abs_bits(w[e]);
          if (!((a >= lo_f) & (a < hi_f)) && a != 0.0f)
            wq_fallback(__float_as_uint(a), sb, nonfinite);
        }
      }
      if (single) {  // provisional codes against T^, and the band entries
        const int c = tid + i * kWqThreads;
        uint32_t bits = 0u;
        uint32_t in_band = 0u;  // bit e: |w[e]| within the band
#pragma unroll
        for (int e = 0; e < E; ++e) {
          const uint32_t wb = __float_as_uint(w[e]);
          const uint32_t ab = wb & 0x7fffffffu;
          bits += ((ab >= t_b) ? 2u - ((wb >> 30) & 2u) : 1u) * mulA[e];  // |w| >= T^
          in_band |= ((ab - band_b) <= bspan_b ? 1u : 0u) << e;
        }
        // Rare: list the band entries. Kept out of the loop above, where a branch holding
        // the atomic would make every weight's work wait for the one before.
        if (c < nchunks && in_band != 0u) {
#pragma unroll
          for (int e = 0; e < E; ++e) {
            if ((in_band >> e) & 1u) {
              const unsigned idx = atomicAdd(&s_cnt, 1u);
              if (idx < static_cast<unsigned>(kWqListCap))
                list[static_cast<long long>(blockIdx.x) * kWqListCap + idx] = make_uint2(
                    static_cast<uint32_t>((1ll * st * kWqStageBytes + 16ll * c) / (16 / E) + e),
                    __float_as_uint(w[e]));
            }
          }
        }
        bits = wq_or_parts<kBf16>(bits);
        if (c < nchunks && mypart == 0)
          packed[wb0 + (1ll * st * kWqStageBytes + 16ll * c) / WORD_BYTES] = bits;
      }
    }
    if ((st & 15) == 15) wq_flush(acc0, acc1, base, sb);
    __syncthreads();  // every thread is done with this slot
    if (tid == 0 && st + kWqStages < ring.nst) wq_issue(ring, st + kWqStages, st + kWqStages);
  }
  wq_flush(acc0, acc1, base, sb);
  if (nonfinite) record_status(kStatusNonfinite);
  __syncthreads();
  // Column sums of this block: bucket e contributes B[e] << ((e-1) % 32) to limbs
  // (e-1)/32 .. +2, each part below 2^32, so a column of one block stays below 2^39.
  for (int e = 1 + tid; e < kWqBuckets; e += blockDim.x) {
    const unsigned long long b = sb[e];
    if (b == 0ull) continue;
    const int pos = e - 1, wd = pos >> 5, sh = pos & 31;
    const uint32_t lo = static_cast<uint32_t>(b), hi = static_cast<uint32_t>(b >> 32);
    atomicAdd(&col[wd], static_cast<unsigned long long>(lo << sh));
    atomicAdd(&col[wd + 1], static_cast<unsigned long long>(__funnelshift_l(lo, hi, sh)));
    const uint32_t p2 = __funnelshift_l(hi, 0u, sh);
    if (p2) atomicAdd(&col[wd + 2], static_cast<unsigned long long>(p2));
  }
  __syncthreads();
  const int copy = static_cast<int>(blockIdx.x % kWqCopies);
  if (tid < kWqLimbs && col[tid] != 0ull) atomicAdd(&ws->cols[copy][tid], col[tid]);
  // When the block's whole range fits the ring, pass A left every stage in its slot
  // (stage st in slot st) and pass B reads them there; otherwise pass B streams the range
  // again, starting now (its stages do not depend on gamma).
  resident = ring.nst <= kWqStages;
  if (MODE == kWqFull && !single && tid == 0 && !resident)
    for (int st = 0; st < kWqStages; ++st) wq_issue(ring, st, ring.nst + st);

  // ---------------------------------------------------------------- grid barrier
  __syncthreads();  // this block's column adds are issued; thread 0 fences for all
  if (tid == 0) {
    __threadfence();
    atomicAdd(&ws->arrived[copy], 1u);
    const uint64_t t0 = global_ns();
    while (true) {
      unsigned int total = 0u;
#pragma unroll
      for (int c = 0; c < kWqCopies; ++c) total += ld_acquire_u32(&ws->arrived[c]);
      if (total >= gridDim.x) break;
      if (global_ns() - t0 > limit_ns) {
        record_status(kStatusTimeout);
        s_ok = 0;
        break;
      }
      __nanosleep(64);
    }
  }
  __syncthreads();
  if (MODE == kWqPartial) {  // this shard's column sums are the result
    if (blockIdx.x == 0 && tid < kWqLimbs) sums_io[tid] = wq_column_total(ws, tid);
    return;
  }
  if (tid < kWqLimbs) col[tid] = wq_column_total(ws, tid);
  }  // pass A
  if (MODE == kWqFinish && tid < kWqLimbs) col[tid] = sums_io[tid];  // added over all shards

  // ---------------------------------------------------------------- gamma and T
  __syncthreads();
  if (tid == 0) {
    uint32_t L[kWqLimbs];
    unsigned long long carry = 0ull;
#pragma unroll
    for (int j = 0; j < kWqLimbs; ++j) {
      // no overflow: a column is below 2^39 per block (2^57 for 2^18 blocks over all
      // shards) and a carry below 2^32
      const unsigned long long t = col[j] + carry;
      L[j] = static_cast<uint32_t>(t);
      carry = t >> 32;
    }
    const double S = wq_limbs_to_double(L);
    const float gamma = __double2float_rn(__ddiv_rn(S, static_cast<double>(n_total)));
    if (blockIdx.x == 0) *gamma_out = gamma;
    s_T = wq_threshold(__fadd_rn(gamma, eps));
  }
  __syncthreads();

  // ---------------------------------------------------------------- pass B: codes
  const float T = s_T;
  if (single) {
    const unsigned cnt = s_cnt;
    const bool patch = (T >= band_lo) && (T <= band_hi) && cnt <= static_cast<unsigned>(kWqListCap);
    if (patch) {
      for (unsigned i = tid; i < cnt; i += kWqThreads) {
        const uint2 en = list[static_cast<long long>(blockIdx.x) * kWqListCap + i];
        const float w = __uint_as_float(en.y);
        const float a = abs_bits(w);
        const uint32_t neg = (en.y >> 30) & 2u;
        const uint32_t u_old = (a >= t_hat) ? 2u - neg : 1u;
        const uint32_t u_new = (a >= T) ? 2u - neg : 1u;
        if (u_old != u_new)
          atomicXor(&packed[wb0 + en.x / 16], (u_old ^ u_new) << wq_shift(static_cast<int>(en.x % 16)));
      }
      return;
    }
    if (tid == 0 && !resident)  // T outside the band, or the list overflowed: stream again
      for (int st = 0; st < min(ring.nst, kWqStages); ++st) wq_issue(ring, st, ring.nst + st);
  }
  const int part = tid & (PARTS - 1);  // which part of its packed word this thread holds
  uint32_t mul[E];                     // 1 << bit position of element e of this part
#pragma unroll
  for (int e = 0; e < E; ++e) mul[e] = 1u << wq_shift(wq_k<kBf16>(part, e));
  const int g0 = (MODE == kWqFinish) ? 0 : ring.nst;  // stages pass A consumed
  for (int st = 0; st < ring.nst; ++st) {
    const int g = g0 + st;  // stages consumed by this block so far
    const int slot = resident ? st : g % kWqStages;
    if (!resident && !mbar_wait(&full[slot], static_cast<uint32_t>((g / kWqStages) & 1), limit_ns))
      s_ok = 0;
    const uint4* stage = reinterpret_cast<const uint4*>(wq_stage + slot * kWqStageBytes);
    const int nchunks = static_cast<int>(
        min(static_cast<long long>(kWqStageBytes), ring.bytes - 1ll * st * kWqStageBytes) / 16);
#pragma unroll
    for (int i = 0; i < kWqChunks; ++i) {
      const int c = tid + i * kWqThreads;
      float w[E];
      wq_chunk_floats<kBf16>((c < nchunks) ? stage[c] : make_uint4(0u, 0u, 0u, 0u), w);
      uint32_t bits = 0u;
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const uint32_t u = (abs_bits(w[e]) >= T) ? 2u - ((__float_as_uint(w[e]) >> 30) & 2u) : 1u;
        bits += u * mul[e];
      }
      bits = wq_or_parts<kBf16>(bits);
      if (c < nchunks && part == 0)
        packed[wb0 + (1ll * st * kWqStageBytes + 16ll * c) / WORD_BYTES] = bits;
    }
    if (resident) continue;
    __syncthreads();
    if (tid == 0 && st + kWqStages < ring.nst)
      wq_issue(ring, st + kWqStages, g0 + st + kWqStages);
  }
  (void)s_ok;
}

}  // namespace bl
