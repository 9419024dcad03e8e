// Absmean ternary weight quantization (BitNet b1.58; dmarx anthology record LIT-380, Key
// takeaways bullet 1: weights constrained to {-1, 0, +1} by an absmean quantization
// function; searcharxiv.com abstract page, Abstract: every weight is ternary).
//
//   pass 1  absmean_partial_kernel   exact sum of |w| (order-independent integer sum)
//           -> the last block to finish rounds it once, gamma = fl32(fl64(S) / n), and
//              derives the ternarization threshold T from d = gamma + eps
//   pass 2  ternarize_pack_kernel    code = (w >= T) - (w <= -T), 2-bit packed
//
// Exact sum. Every |w| is m * 2^(max(e,1) - 150) with 8-bit biased exponent e and 24-bit
// integer mantissa m. Each warp fixes a 32-exponent window [base, base+31] from the
// largest exponent in its first loads (base = that exponent - 27, at least 1). Inside the
// window a thread adds m << (e - base) into a 96-bit integer (three 32-bit limbs, exact
// for 2^31 terms). Anything outside it (zeros excluded, subnormals, far larger or far
// smaller values) goes to a shared-memory array of 320 exponent buckets with 64-bit
// atomics. A warp's 96-bit total is deposited as three bucket entries (limb i has the
// unit of exponent base + 32i), so every partial sum is an exact integer combination of
// powers of two and the final value does not depend on the grid or on the order of the
// atomic adds.
//
// Threshold. RoundClip(fl(w/d), -1, 1) is +1 exactly when fl(w/d) > 0.5 (0.5 itself
// rounds to the even 0, and every quotient >= 1.5 clips to 1). Correctly rounded
// division is monotone in w, so there is one smallest float T with fl(T/d) > 0.5, and
// c = +1 iff w >= T, c = -1 iff -w >= T. T is found once per matrix with a handful of
// divisions; the per-element work is two compares.
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kWqBuckets = 320;  // exponent buckets: e in [0, 254] plus limb spill-over
constexpr int kWqThreads = 256;

// Layout of the quantize_weights workspace (bytes).
struct WqWorkspace {
  unsigned long long buckets[kWqBuckets];
  unsigned int blocks_done;
  unsigned int pad0;
  float threshold;  // T: c = +1 iff w >= T
  float d;          // gamma + eps
};

__device__ __forceinline__ void wq_add_window(uint32_t m, int s, uint32_t& a0, uint32_t& a1,
                                              uint32_t& a2) {
  // (m << s) as a 56-bit value in two limbs, added into the 96-bit accumulator
  const uint32_t lo = m << s;
  const uint32_t hi = __funnelshift_l(m, 0u, s);  // upper bits of m << s, 0 when s == 0
  asm("add.cc.u32 %0, %0, %3;\n\t"
      "addc.cc.u32 %1, %1, %4;\n\t"
      "addc.u32 %2, %2, 0;"
      : "+r"(a0), "+r"(a1), "+r"(a2)
      : "r"(lo), "r"(hi));
}

// One element: bits = |w| as an fp32 bit pattern (sign already cleared).
__device__ __forceinline__ void wq_accumulate(uint32_t bits, int base, uint32_t& a0,
                                              uint32_t& a1, uint32_t& a2,
                                              unsigned long long* sb, bool& nonfinite) {
  const int e = static_cast<int>(bits >> 23);
  const uint32_t m = (bits & 0x7fffffu) | 0x800000u;
  const int s = e - base;
  if (static_cast<unsigned>(s) < 32u) {
    wq_add_window(m, s, a0, a1, a2);
  } else if (bits != 0u) {
    if (e == 255) {
      nonfinite = true;
    } else if (e == 0) {
      atomicAdd(&sb[1], static_cast<unsigned long long>(bits));  // subnormal: unit 2^-149
    } else {
      atomicAdd(&sb[e], static_cast<unsigned long long>(m));
    }
  }
}

// 96-bit sum of the accumulators of all 32 lanes (result valid in every lane).
__device__ __forceinline__ void warp_sum96(uint32_t& a0, uint32_t& a1, uint32_t& a2) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const uint32_t b0 = __shfl_xor_sync(0xffffffffu, a0, off);
    const uint32_t b1 = __shfl_xor_sync(0xffffffffu, a1, off);
    const uint32_t b2 = __shfl_xor_sync(0xffffffffu, a2, off);
    asm("add.cc.u32 %0, %0, %3;\n\t"
        "addc.cc.u32 %1, %1, %4;\n\t"
        "addc.u32 %2, %2, %5;"
        : "+r"(a0), "+r"(a1), "+r"(a2)
        : "r"(b0), "r"(b1), "r"(b2));
  }
}

// Exact sum  sum_e B[e] * 2^(max(e,1) - 150)  rounded once to double (ties to even).
// Runs on one thread. B has kWqBuckets entries; entries >= 255 come from limb spill-over
// and follow the same rule.
__device__ double wq_exact_sum_to_double(const unsigned long long* B) {
  // Integer S * 2^149 in 32-bit limbs: term e sits at bit e - 1; e <= 319, value < 2^64
  // -> bits < 383; 13 limbs with headroom for carries.
  constexpr int kL = 14;
  uint32_t L[kL];
#pragma unroll
  for (int i = 0; i < kL; ++i) L[i] = 0u;
  for (int e = 1; e < kWqBuckets; ++e) {
    const unsigned long long v = B[e];
    if (v == 0ull) continue;
    const int pos = e - 1;
    const int w = pos >> 5;
    const int b = pos & 31;
    const uint32_t p0 = static_cast<uint32_t>(v) << b;
    const uint32_t p1 = __funnelshift_l(static_cast<uint32_t>(v),
                                        static_cast<uint32_t>(v >> 32), b);
    const uint32_t p2 = __funnelshift_l(static_cast<uint32_t>(v >> 32), 0u, b);
    uint64_t carry = 0;
    for (int i = w; i < kL; ++i) {
      const uint32_t add = (i == w) ? p0 : (i == w + 1) ? p1 : (i == w + 2) ? p2 : 0u;
      if (i > w + 2 && carry == 0) break;
      const uint64_t s = static_cast<uint64_t>(L[i]) + add + carry;
      L[i] = static_cast<uint32_t>(s);
      carry = s >> 32;
    }
  }
  int top = kL - 1;
  while (top >= 0 && L[top] == 0u) --top;
  if (top < 0) return 0.0;
  // Gather the leading 64 bits below and including the top set bit, plus a sticky flag.
  const int lz = __clz(L[top]);
  const int topbit = top * 32 + (31 - lz);  // position of the leading one
  // 96-bit window of limbs top, top-1, top-2
  const uint32_t w2 = L[top];
  const uint32_t w1 = (top >= 1) ? L[top - 1] : 0u;
  const uint32_t w0 = (top >= 2) ? L[top - 2] : 0u;
  bool sticky = false;
  for (int i = 0; i < top - 2; ++i) sticky |= (L[i] != 0u);
  // Left-align: X = window << lz holds the leading one in bit 95 (bits 95..0 of 96).
  const uint32_t x2 = __funnelshift_l(w1, w2, lz);
  const uint32_t x1 = __funnelshift_l(w0, w1, lz);
  const uint32_t x0 = w0 << lz;  // limbs below the window only feed the sticky flag
  // significand = top 53 bits of X: bits 95..43
  const uint64_t hi64 = (static_cast<uint64_t>(x2) << 32) | x1;  // X bits 95..32
  uint64_t mant = hi64 >> 11;                                       // 53 bits
  const uint64_t rest = hi64 & 0x7ffull;                            // X bits 42..32
  const bool half = (rest >> 10) & 1ull;
  sticky |= ((rest & 0x3ffull) != 0ull) || (x0 != 0u);
  if (half && (sticky || (mant & 1ull))) mant += 1ull;
  // value = mant * 2^(topbit - 52) * 2^-149
  return ldexp(static_cast<double>(mant), topbit - 52 - 149);
}

// Smallest float t with fl(t / d) > 0.5, +inf when no finite t qualifies (d == 0 or inf).
__device__ float wq_threshold(float d) {
  if (!(d > 0.0f) || isinf(d)) return __int_as_float(0x7f800000);
  float t = __fmul_rn(0.5f, d);
  // step down while the next smaller float still qualifies
  for (int i = 0; i < 64 && t > 0.0f; ++i) {
    const float prev = __int_as_float(__float_as_int(t) - 1);
    if (__fdiv_rn(prev, d) > 0.5f) t = prev; else break;
  }
  // step up until t qualifies
  for (int i = 0; i < 64; ++i) {
    if (__fdiv_rn(t, d) > 0.5f) break;
    t = __int_as_float(__float_as_int(t) + 1);
  }
  return t;
}

// Pass 1. W holds n values (fp32 if !is_bf16, else bf16), n % 8 == 0, 16-byte aligned.
// ws->buckets and ws->blocks_done must be zero on entry (the host clears them).
template <bool kBf16>
__global__ void __launch_bounds__(kWqThreads) absmean_partial_kernel(
    const void* __restrict__ W, long long n, float eps, WqWorkspace* __restrict__ ws,
    float* __restrict__ gamma_out) {
  __shared__ unsigned long long sb[kWqBuckets];
  __shared__ bool s_last;
  for (int i = threadIdx.x; i < kWqBuckets; i += blockDim.x) sb[i] = 0ull;
  __syncthreads();

  constexpr int kPerVec = kBf16 ? 8 : 4;  // elements per 16-byte vector
  constexpr int kUnroll = 4;
  const long long nvec = n / kPerVec;
  const uint4* __restrict__ v = static_cast<const uint4*>(W);
  const long long tid = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;

  uint32_t a0 = 0u, a1 = 0u, a2 = 0u;
  bool nonfinite = false;

  // First batch: fixes the warp's exponent window.
  uint4 buf[kUnroll];
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const long long i = tid + u * stride;
    buf[u] = (i < nvec) ? ld_stream_v4(v + i) : make_uint4(0u, 0u, 0u, 0u);
  }
  int emax = 0;
#pragma unroll
  for (int u = 0; u < kUnroll; ++u) {
    const uint32_t words[4] = {buf[u].x, buf[u].y, buf[u].z, buf[u].w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (kBf16) {
        const int e0 = static_cast<int>((words[q] >> 7) & 0xffu);
        const int e1 = static_cast<int>((words[q] >> 23) & 0xffu);
        if (e0 != 255) emax = max(emax, e0);
        if (e1 != 255) emax = max(emax, e1);
      } else {
        const int e = static_cast<int>((words[q] >> 23) & 0xffu);
        if (e != 255) emax = max(emax, e);
      }
    }
  }
  emax = __reduce_max_sync(0xffffffffu, emax);
  const int base = max(1, emax - 27);

  long long i0 = tid;
  while (true) {
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      if (i0 + u * stride < nvec) {
        const uint32_t words[4] = {buf[u].x, buf[u].y, buf[u].z, buf[u].w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          if (kBf16) {
            wq_accumulate((words[q] << 16) & 0x7fffffffu, base, a0, a1, a2, sb, nonfinite);
            wq_accumulate(words[q] & 0x7fff0000u, base, a0, a1, a2, sb, nonfinite);
          } else {
            wq_accumulate(words[q] & 0x7fffffffu, base, a0, a1, a2, sb, nonfinite);
          }
        }
      }
    }
    i0 += kUnroll * stride;
    if (i0 >= nvec) break;
#pragma unroll
    for (int u = 0; u < kUnroll; ++u) {
      const long long i = i0 + u * stride;
      buf[u] = (i < nvec) ? ld_stream_v4(v + i) : make_uint4(0u, 0u, 0u, 0u);
    }
  }

  if (nonfinite) record_status(kStatusNonfinite);
  warp_sum96(a0, a1, a2);
  if ((threadIdx.x & 31) == 0) {
    if (a0) atomicAdd(&sb[base], static_cast<unsigned long long>(a0));
    if (a1) atomicAdd(&sb[base + 32], static_cast<unsigned long long>(a1));
    if (a2) atomicAdd(&sb[base + 64], static_cast<unsigned long long>(a2));
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kWqBuckets; i += blockDim.x)
    if (sb[i]) atomicAdd(&ws->buckets[i], sb[i]);

  // The last block to finish turns the buckets into gamma and the threshold.
  __threadfence();
  __syncthreads();
  if (threadIdx.x == 0) {
    const unsigned int done = atomicAdd(&ws->blocks_done, 1u);
    s_last = (done == gridDim.x - 1);
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int i = threadIdx.x; i < kWqBuckets; i += blockDim.x)
    sb[i] = __ldcg(&ws->buckets[i]);
  __syncthreads();
  if (threadIdx.x == 0) {
    const double S = wq_exact_sum_to_double(sb);
    const float gamma = __double2float_rn(__ddiv_rn(S, static_cast<double>(n)));
    const float d = __fadd_rn(gamma, eps);
    *gamma_out = gamma;
    ws->d = d;
    ws->threshold = wq_threshold(d);
  }
}

// Pass 2. One 32-bit output word (16 consecutive weights of a row) per thread iteration.
// Trit k = 4j + i of the word (relative index) goes to bits 8i + 2j as u = c + 1.
template <bool kBf16>
__global__ void __launch_bounds__(256) ternarize_pack_kernel(
    const void* __restrict__ W, long long nwords, const WqWorkspace* __restrict__ ws,
    uint32_t* __restrict__ packed) {
  const float T = ws->threshold;
  const long long stride = static_cast<long long>(gridDim.x) * blockDim.x;
  for (long long wi = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x;
       wi < nwords; wi += stride) {
    float w[16];
    if (kBf16) {
      const uint4* src = static_cast<const uint4*>(W) + 2 * wi;
      const uint4 p0 = ld_stream_v4(src), p1 = ld_stream_v4(src + 1);
      const uint32_t h[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        w[2 * q] = __uint_as_float(h[q] << 16);
        w[2 * q + 1] = __uint_as_float(h[q] & 0xffff0000u);
      }
    } else {
      const uint4* src = static_cast<const uint4*>(W) + 4 * wi;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint4 p = ld_stream_v4(src + q);
        w[4 * q + 0] = __uint_as_float(p.x);
        w[4 * q + 1] = __uint_as_float(p.y);
        w[4 * q + 2] = __uint_as_float(p.z);
        w[4 * q + 3] = __uint_as_float(p.w);
      }
    }
    uint32_t word = 0u;
#pragma unroll
    for (int k = 0; k < 16; ++k) {
      const uint32_t u = 1u + (w[k] >= T ? 1u : 0u) - (-w[k] >= T ? 1u : 0u);
      word |= u << (8 * (k & 3) + 2 * (k >> 2));
    }
    packed[wi] = word;
  }
}

}  // namespace bl
