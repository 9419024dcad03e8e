// Absmean ternary weight quantization (BitNet b1.58; dmarx anthology record LIT-380, Key
// takeaways bullet 1: weights constrained to {-1, 0, +1} by an absmean quantization
// function; searcharxiv.com abstract page, Abstract: every weight is ternary).
//
// One cooperative kernel that reads W from HBM once:
//   1  every block streams its own contiguous range of 16-weight words and
//      a) adds every |w| into an exact sum (below),
//      b) ternarizes provisionally against a bracket [T_lo, T_hi] of the final threshold,
//         estimated from the block's first 4096 weights: |w| >= T_hi is +-1, |w| < T_lo is 0,
//         anything in between is written as 0 and appended (index, value) to the block's
//         list of ambiguous weights (a few percent),
//      and writes its packed words.
//   -- grid barrier (bounded wait) --
//   2  every block turns the exact sum into gamma = fl32(fl64(S) / n) and the threshold T
//   3  if T lies inside the block's bracket and its list did not overflow, only the listed
//      weights are re-decided (atomicXor of their 2-bit fields); otherwise the block
//      re-reads its range and ternarizes it again with T. Either way every code equals
//      RoundClip(fl(w / (gamma + eps)), -1, 1).
//
// Threshold. RoundClip(fl(w/d), -1, 1) is +1 exactly when fl(w/d) > 0.5 (0.5 itself
// rounds to the even 0, and every quotient >= 1.5 clips to 1). Correctly rounded
// division is monotone in w, so there is one smallest float T with fl(T/d) > 0.5, and
// c = +1 iff w >= T, c = -1 iff -w >= T.
//
// Exact sum. Each warp fixes an exponent window [base, base + 20] from the largest
// exponent in its first loads (base = that exponent - 17, at least 1). A float |w| in the
// window is an integer multiple of u = 2^(base - 150) below 2^44 u, so up to 256 of them
// add up exactly in a double; a thread keeps two such doubles (weights k % 2 of each
// word, so the additions do not form one long dependency chain) and every 16 words
// converts them to integers and adds those into 64-bit exponent buckets (low 32 bits at
// exponent base, the rest at base + 32). Values outside the window (subnormals, far larger or smaller ones)
// go straight into the buckets as (exponent, 24-bit mantissa). The buckets are summed
// exactly, so gamma depends neither on the grid nor on the order of the atomic adds.
#pragma once

#include "act_quant.cuh"
#include "common.cuh"

namespace bl {

constexpr int kWqBuckets = 320;  // exponent buckets: e in [0, 254] plus spill-over
constexpr int kWqThreads = 256;
constexpr int kWqLimbs = 14;     // 32-bit limbs of the exact sum (S * 2^149 < 2^448)
constexpr int kWqWindow = 21;    // exponents covered by the fp64 window
constexpr int kWqFlushWords = 16;  // words a thread sums in fp64 between bucket flushes
constexpr float kWqBand = 0.03f;   // relative half-width of the per-block gamma bracket

// Header of the quantize_weights workspace (zeroed by the host before each launch). It is
// followed by gridDim.x lists of `cap` ambiguous-weight entries (uint64 each).
struct WqWorkspace {
  unsigned long long buckets[kWqBuckets];
  unsigned int arrived;  // grid-barrier arrivals
  unsigned int pad[3];
};

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

// Moves a thread's fp64 window sum into the buckets: acc is an integer multiple of
// 2^(base-150) below 2^53 of those units, so the scaled conversion is exact.
__device__ __forceinline__ void wq_flush(double& acc, int base, unsigned long long* sb) {
  if (acc != 0.0) {
    const double scale = __longlong_as_double(static_cast<long long>(1023 + 150 - base) << 52);
    const unsigned long long u = __double2ull_rz(__dmul_rn(acc, scale));
    atomicAdd(&sb[base], u & 0xffffffffull);
    if (u >> 32) atomicAdd(&sb[base + 32], u >> 32);
    acc = 0.0;
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
__device__ float wq_threshold(float d) {
  if (!(d > 0.0f) || isinf(d)) return __int_as_float(0x7f800000);
  float t = __fmul_rn(0.5f, d);
  for (int i = 0; i < 64 && t > 0.0f; ++i) {  // step down while the predecessor qualifies
    const float prev = __int_as_float(__float_as_int(t) - 1);
    if (__fdiv_rn(prev, d) > 0.5f) t = prev; else break;
  }
  for (int i = 0; i < 64; ++i) {  // step up until t qualifies
    if (__fdiv_rn(t, d) > 0.5f) break;
    t = __int_as_float(__float_as_int(t) + 1);
  }
  return t;
}

__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// The 16 weights of word wi as floats (fp32, or bf16 widened exactly).
template <bool kBf16>
__device__ __forceinline__ void wq_load_word(const uint4* v, long long wi, uint4 (&raw)[4]) {
  if (kBf16) {
    raw[0] = ld_stream_v4(v + 2 * wi);
    raw[1] = ld_stream_v4(v + 2 * wi + 1);
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) raw[q] = ld_stream_v4(v + 4 * wi + q);
  }
}
template <bool kBf16>
__device__ __forceinline__ void wq_unpack_word(const uint4 (&raw)[4], float (&w)[16]) {
  if (kBf16) {
    const uint32_t h[8] = {raw[0].x, raw[0].y, raw[0].z, raw[0].w,
                           raw[1].x, raw[1].y, raw[1].z, raw[1].w};
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      w[2 * q] = __uint_as_float(h[q] << 16);
      w[2 * q + 1] = __uint_as_float(h[q] & 0xffff0000u);
    }
  } else {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      w[4 * q + 0] = __uint_as_float(raw[q].x);
      w[4 * q + 1] = __uint_as_float(raw[q].y);
      w[4 * q + 2] = __uint_as_float(raw[q].z);
      w[4 * q + 3] = __uint_as_float(raw[q].w);
    }
  }
}

// Exact codes of one word against the final threshold T.
__device__ __forceinline__ uint32_t wq_pack16(const float (&w)[16], float T) {
  uint32_t word = 0u;
#pragma unroll
  for (int k = 0; k < 16; ++k) {
    const uint32_t u = 1u + (w[k] >= T ? 1u : 0u) - (-w[k] >= T ? 1u : 0u);
    word |= u << wq_shift(k);
  }
  return word;
}

// W holds n values (fp32, or bf16 if kBf16), n % 16 == 0, 16-byte aligned. Launched
// cooperatively (all blocks resident). ws: header zeroed by the host, then gridDim.x
// ambiguous lists of cap entries.
template <bool kBf16>
__global__ void __launch_bounds__(kWqThreads) weight_quant_kernel(
    const void* __restrict__ W, long long n, float eps, WqWorkspace* __restrict__ ws,
    unsigned long long* __restrict__ lists, int cap, float* __restrict__ gamma_out,
    uint32_t* __restrict__ packed, unsigned long long limit_ns) {
  __shared__ unsigned long long sb[kWqBuckets];
  __shared__ unsigned long long col[kWqLimbs];
  __shared__ float s_red[2][kWqThreads / 32];
  __shared__ float s_Tlo, s_Thi, s_T;
  __shared__ unsigned int s_cnt;
  __shared__ int s_ok;
  for (int i = threadIdx.x; i < kWqBuckets; i += blockDim.x) sb[i] = 0ull;
  if (threadIdx.x < kWqLimbs) col[threadIdx.x] = 0ull;
  if (threadIdx.x == 0) s_cnt = 0u;

  const uint4* __restrict__ v = static_cast<const uint4*>(W);
  const long long nwords = n / 16;
  const long long per_block = (nwords + gridDim.x - 1) / gridDim.x;
  const long long wb0 = min(nwords, static_cast<long long>(blockIdx.x) * per_block);
  const long long wb1 = min(nwords, wb0 + per_block);
  unsigned long long* list = lists + static_cast<long long>(blockIdx.x) * cap;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;

  // ---------------------------------------------------------------- first words
  long long wi = wb0 + threadIdx.x;
  uint4 cur[4] = {}, nxt[4] = {};
  if (wi < wb1) wq_load_word<kBf16>(v, wi, cur);
  float w[16];
  wq_unpack_word<kBf16>(cur, w);
  int emax = 0;
  float asum = 0.0f, acnt = 0.0f;
  if (wi < wb1) {
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t b = __float_as_uint(w[k]) & 0x7fffffffu;
      const int e = static_cast<int>(b >> 23);
      if (e != 255) {
        emax = max(emax, e);
        asum += __uint_as_float(b);
        acnt += 1.0f;
      }
    }
  }
  emax = __reduce_max_sync(0xffffffffu, emax);
  const int base = max(1, emax + 4 - kWqWindow);
  const float lo_f = __uint_as_float(static_cast<uint32_t>(base) << 23);
  const float hi_f = (base + kWqWindow <= 254)
                         ? __uint_as_float(static_cast<uint32_t>(base + kWqWindow) << 23)
                         : __int_as_float(0x7f800000);
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    asum += __shfl_xor_sync(0xffffffffu, asum, off);
    acnt += __shfl_xor_sync(0xffffffffu, acnt, off);
  }
  if (lane == 0) {
    s_red[0][warp] = asum;
    s_red[1][warp] = acnt;
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    float sum = 0.0f, cnt = 0.0f;
    for (int i = 0; i < kWqThreads / 32; ++i) {
      sum += s_red[0][i];
      cnt += s_red[1][i];
    }
    const float ghat = (cnt > 0.0f) ? sum / cnt : 0.0f;
    s_Tlo = 0.5f * (ghat * (1.0f - kWqBand) + eps) * (1.0f - 1e-6f);
    s_Thi = 0.5f * (ghat * (1.0f + kWqBand) + eps) * (1.0f + 1e-6f);
  }
  __syncthreads();
  const float Tlo = s_Tlo, Thi = s_Thi;

  // ---------------------------------------------------------------- phase 1: one pass
  double acc[2] = {0.0, 0.0};  // two independent chains (k % 2)
  bool nonfinite = false;
  int since_flush = 0;
  for (; wi < wb1; wi += kWqThreads) {
    const long long wn = wi + kWqThreads;
    if (wn < wb1) wq_load_word<kBf16>(v, wn, nxt);
    // Common path, branch-free: fp64 window sum, provisional code, two any-flags.
    uint32_t word = 0u;
    bool out_any = false, amb_any = false;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const float x = w[k];
      const float a = abs_bits(x);
      const bool in = (a >= lo_f) & (a < hi_f);
      out_any |= !in;
      acc[k & 1] += static_cast<double>(in ? a : 0.0f);  // exact: see the header
      const bool big = a >= Thi;
      const uint32_t neg = __float_as_uint(x) >> 31;
      word += (big ? 2u - 2u * neg : 1u) << wq_shift(k);
      amb_any |= (!big) & (a >= Tlo);
    }
    // Rare paths: weights outside the window (zeros included) and ambiguous weights.
    if (out_any) {
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float a = abs_bits(w[k]);
        if (!((a >= lo_f) & (a < hi_f)) && a != 0.0f)
          wq_fallback(__float_as_uint(a), sb, nonfinite);
      }
    }
    if (amb_any) {
      uint32_t m16 = 0u;
#pragma unroll
      for (int k = 0; k < 16; ++k) {
        const float a = abs_bits(w[k]);
        m16 |= ((a < Thi) & (a >= Tlo) ? 1u : 0u) << k;
      }
      unsigned int slot = atomicAdd(&s_cnt, static_cast<unsigned int>(__popc(m16)));
#pragma unroll
      for (int k = 0; k < 16; ++k) {  // constant indices keep w[] in registers
        if ((m16 >> k) & 1u) {
          if (slot < static_cast<unsigned int>(cap))
            list[slot] = (static_cast<unsigned long long>(__float_as_uint(w[k])) << 32) |
                         (static_cast<unsigned long long>(wi) << 4) | static_cast<unsigned>(k);
          ++slot;
        }
      }
    }
    packed[wi] = word;
    if (++since_flush == kWqFlushWords) {
#pragma unroll
      for (int j = 0; j < 2; ++j) wq_flush(acc[j], base, sb);
      since_flush = 0;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) cur[q] = nxt[q];
    wq_unpack_word<kBf16>(cur, w);
  }
#pragma unroll
  for (int j = 0; j < 2; ++j) wq_flush(acc[j], base, sb);
  if (nonfinite) record_status(kStatusNonfinite);
  __syncthreads();
  for (int i = threadIdx.x; i < kWqBuckets; i += blockDim.x)
    if (sb[i]) atomicAdd(&ws->buckets[i], sb[i]);

  // ---------------------------------------------------------------- grid barrier
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    atomicAdd(&ws->arrived, 1u);
    int ok = 1;
    const uint64_t t0 = global_ns();
    while (ld_acquire_u32(&ws->arrived) < gridDim.x) {
      if (global_ns() - t0 > limit_ns) {
        record_status(kStatusTimeout);
        ok = 0;
        break;
      }
      __nanosleep(64);
    }
    s_ok = ok;
  }
  __syncthreads();
  if (!s_ok) return;

  // ---------------------------------------------------------------- phase 2: gamma, T
  // Column sums: bucket e contributes B[e] << ((e-1) % 32) to limbs (e-1)/32 .. +2.
  for (int e = 1 + threadIdx.x; e < kWqBuckets; e += blockDim.x) {
    const unsigned long long b = __ldcg(&ws->buckets[e]);
    if (b == 0ull) continue;
    const int pos = e - 1, wd = pos >> 5, sh = pos & 31;
    const uint32_t lo = static_cast<uint32_t>(b), hi = static_cast<uint32_t>(b >> 32);
    atomicAdd(&col[wd], static_cast<unsigned long long>(lo << sh));
    atomicAdd(&col[wd + 1], static_cast<unsigned long long>(__funnelshift_l(lo, hi, sh)));
    const uint32_t p2 = __funnelshift_l(hi, 0u, sh);
    if (p2) atomicAdd(&col[wd + 2], static_cast<unsigned long long>(p2));
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t L[kWqLimbs];
    unsigned long long carry = 0ull;
#pragma unroll
    for (int j = 0; j < kWqLimbs; ++j) {
      const unsigned long long t = col[j] + carry;
      L[j] = static_cast<uint32_t>(t);
      carry = t >> 32;
    }
    const double S = wq_limbs_to_double(L);
    const float gamma = __double2float_rn(__ddiv_rn(S, static_cast<double>(n)));
    if (blockIdx.x == 0) *gamma_out = gamma;
    s_T = wq_threshold(__fadd_rn(gamma, eps));
  }
  __syncthreads();

  // ---------------------------------------------------------------- phase 3: settle
  const float T = s_T;
  const unsigned int cnt = s_cnt;
  if (T >= Tlo && T <= Thi && cnt <= static_cast<unsigned int>(cap)) {
    for (unsigned int i = threadIdx.x; i < cnt; i += blockDim.x) {
      const unsigned long long e = list[i];
      const float x = __uint_as_float(static_cast<uint32_t>(e >> 32));
      const long long widx = static_cast<long long>((e & 0xffffffffull) >> 4);
      const int k = static_cast<int>(e & 15ull);
      const uint32_t u = 1u + (x >= T ? 1u : 0u) - (-x >= T ? 1u : 0u);
      if (u != 1u) atomicXor(&packed[widx], (1u ^ u) << wq_shift(k));
    }
  } else {
    for (long long wj = wb0 + threadIdx.x; wj < wb1; wj += kWqThreads) {
      uint4 raw[4] = {};
      float ww[16];
      wq_load_word<kBf16>(v, wj, raw);
      wq_unpack_word<kBf16>(raw, ww);
      packed[wj] = wq_pack16(ww, T);
    }
  }
}

}  // namespace bl
