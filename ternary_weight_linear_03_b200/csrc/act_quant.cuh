// Per-token absmax int8 activation quantization (8-bit activations, dmarx anthology
// record LIT-380, Key takeaways bullet 1):
//   a_t = max_k |x[t,k]|,  r_t = fl(127 / a_t),  s_t = fl(a_t / 127),
//   q[t,k] = clip(rne(fl(x[t,k] * r_t)), -127, 127)   (0 when a_t == 0 or x == 0).
// One block per token row; the row is read once from HBM (the second pass hits L1/L2).
// Optionally also writes rowsum_t = sum_k q[t,k], which the tensor-core GEMM subtracts
// from its accumulators (trit c is stored as u = c + 1, so sum_k u q = acc + sum_k q).
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kAqThreads = 256;

// Loads 8 consecutive elements (one 16-byte bf16 vector or two fp32 vectors) as floats.
template <bool kBf16>
__device__ __forceinline__ void load8(const void* row, int c, float (&v)[8]) {
  if (kBf16) {
    const uint4 p = reinterpret_cast<const uint4*>(row)[c];
    const uint32_t h[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      v[2 * q] = __uint_as_float(h[q] << 16);
      v[2 * q + 1] = __uint_as_float(h[q] & 0xffff0000u);
    }
  } else {
    const float4 a = reinterpret_cast<const float4*>(row)[2 * c];
    const float4 b = reinterpret_cast<const float4*>(row)[2 * c + 1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = (lane < static_cast<int>(blockDim.x >> 5)) ? red[lane] : 0.0f;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
  return v;
}

__device__ __forceinline__ int block_sum(int v, int* red) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();
  if (lane == 0) red[warp] = v;
  __syncthreads();
  v = (lane < static_cast<int>(blockDim.x >> 5)) ? red[lane] : 0;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
  return v;
}

// Absolute value as a plain sign-bit clear (exact); NaN stays NaN and is caught by the
// finiteness test on the row maximum.
__device__ __forceinline__ float abs_bits(float x) {
  return __uint_as_float(__float_as_uint(x) & 0x7fffffffu);
}

// Per-halfword unsigned maximum.
__device__ __forceinline__ uint32_t max_u16x2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("max.u16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Largest |x| of 16 bf16 values (two 16-byte vectors at p), kept as two halfword bit
// patterns: with the sign cleared, bf16 patterns order like their values, and the NaN
// patterns lie above infinity (0x7f80), so a maximum at or above 0x7f80 flags a
// non-finite value.
__device__ __forceinline__ uint32_t absmax16_bf16(const uint4 a, const uint4 b, uint32_t m2) {
  const uint32_t h[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
  for (int q = 0; q < 8; ++q) m2 = max_u16x2(m2, h[q] & 0x7fff7fffu);
  return m2;
}
__device__ __forceinline__ uint32_t absmax16_bf16(const void* p, uint32_t m2) {
  return absmax16_bf16(reinterpret_cast<const uint4*>(p)[0], reinterpret_cast<const uint4*>(p)[1], m2);
}

// Quantizes 16 bf16 values with a finite r (the same rounding and clamping as quant_i8;
// its zero test only matters for an infinite r) into four words of int8, byte i & 3 of
// word i >> 2 holding element i, and adds their sum into *sum.
__device__ __forceinline__ uint4 quant16_bf16(const uint4 a, const uint4 b, float r, int* sum) {
  const uint32_t h[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
  uint32_t w[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    int q[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t hw = h[2 * j + (e >> 1)];
      const float v = __uint_as_float((e & 1) ? (hw & 0xffff0000u) : (hw << 16));
      q[e] = max(-127, min(127, __float2int_rn(__fmul_rn(v, r))));
    }
    w[j] = __byte_perm(__byte_perm(q[0], q[1], 0x0040), __byte_perm(q[2], q[3], 0x0040), 0x5410);
    *sum = __dp4a(static_cast<int>(w[j]), 0x01010101, *sum);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}
__device__ __forceinline__ uint4 quant16_bf16(const void* p, float r, int* sum) {
  return quant16_bf16(reinterpret_cast<const uint4*>(p)[0], reinterpret_cast<const uint4*>(p)[1], r, sum);
}

// Zeroes n16 16-byte words at z with the whole grid (the split-K sums and counters of the
// tensor-core kernel that follows, so that no separate memset sits between the two).
__device__ __forceinline__ void grid_zero(uint4* __restrict__ z, long long n16) {
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < n16;
       i += static_cast<long long>(gridDim.x) * blockDim.x)
    z[i] = make_uint4(0u, 0u, 0u, 0u);
}

// Where a token's absmax a_t comes from.
enum AqMode : int {
  kAqRow = 0,     // from the row itself (the whole row is in x)
  kAqGiven = 1,   // from amax[t], computed elsewhere: over the whole row when x holds only
                  // a K-shard of it (tensor parallelism), or by the kernel that produced x
  kAqAbsmax = 2,  // only compute a_t = max_k |x[t,k]| into amax[t]; no codes
};

// grid = M blocks, K % 8 == 0. rowsum may be null; zero/zero_n16 name an extra region to
// clear (may be null/0). Lets the dependent kernel launch at once (it waits for this
// grid's completion before reading any of these outputs).
template <bool kBf16, int AMODE = kAqRow, int NT = kAqThreads>
__global__ void __launch_bounds__(NT) act_quant_kernel(
    const void* __restrict__ x, int K, int8_t* __restrict__ xq, float* __restrict__ scale,
    int* __restrict__ rowsum, uint4* __restrict__ zero, long long zero_n16,
    float* __restrict__ amax = nullptr) {
  __shared__ float redf[32];
  __shared__ int redi[32];
  // The tensor-core kernel after this one may launch at once: it only loads its weights
  // and sets up until this grid has finished.
  allow_dependent_launch();
  grid_dependency_wait();  // x (and amax) may come from the kernel before; no-op otherwise
  grid_zero(zero, zero_n16);
  const int t = blockIdx.x;
  const char* row = static_cast<const char*>(x) + static_cast<size_t>(t) * K * (kBf16 ? 2 : 4);
  const int nc = K / 8;
  float a = 0.0f;
  if (AMODE == kAqGiven) {
    a = amax[t];
    if (!(a <= 3.4028234663852886e38f)) record_status(kStatusNonfinite);
  } else {
    bool bad = false;
    // the float pass (fp32 x, or a bf16 thread that saw a non-finite value: NaN is skipped
    // by fmaxf and flagged)
    auto float_pass = [&]() {
      float m = 0.0f;
      for (int c = threadIdx.x; c < nc; c += blockDim.x) {
        float v[8];
        load8<kBf16>(row, c, v);
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float e = abs_bits(v[i]);
          bad |= !(e <= 3.4028234663852886e38f);
          m = fmaxf(m, e);
        }
      }
      return m;
    };
    if (kBf16) {  // K % 16 == 0: one max.u16x2 per two values
      // two groups' loads in flight per thread before either is reduced
      uint32_t m2 = 0u;
      const int ng = K / 16;
      for (int c0 = threadIdx.x; c0 < ng; c0 += 2 * blockDim.x) {
        uint4 v[2][2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int c = c0 + u * blockDim.x;
          const uint4* p = reinterpret_cast<const uint4*>(row + 32 * static_cast<size_t>(c));
          v[u][0] = (c < ng) ? p[0] : make_uint4(0u, 0u, 0u, 0u);
          v[u][1] = (c < ng) ? p[1] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < 2; ++u) m2 = absmax16_bf16(v[u][0], v[u][1], m2);
      }
      const uint32_t m = max(m2 & 0xffffu, m2 >> 16);
      a = (m < 0x7f80u) ? __uint_as_float(m << 16) : float_pass();
    } else {
      a = float_pass();
    }
    if (bad) record_status(kStatusNonfinite);
    a = block_max(a, redf);
    if (AMODE == kAqAbsmax) {
      if (threadIdx.x == 0) amax[t] = a;
      return;
    }
  }
  const float r = (a > 0.0f) ? __fdiv_rn(127.0f, a) : 0.0f;
  int8_t* qrow = xq + static_cast<size_t>(t) * K;
  int sum = 0;
  if (kBf16 && r <= 3.4028234663852886e38f) {  // finite r; 16 values a step (K % 16 == 0)
    for (int c = threadIdx.x; c < K / 16; c += blockDim.x)
      reinterpret_cast<uint4*>(qrow)[c] = quant16_bf16(row + 32 * static_cast<size_t>(c), r, &sum);
  } else for (int c = threadIdx.x; c < nc; c += blockDim.x) {
    float v[8];
    load8<kBf16>(row, c, v);
    uint32_t lo = 0u, hi = 0u;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int q = (a > 0.0f) ? quant_i8(v[i], r) : 0;
      sum += q;
      const uint32_t b = static_cast<uint32_t>(q) & 0xffu;
      if (i < 4) lo |= b << (8 * i); else hi |= b << (8 * (i - 4));
    }
    reinterpret_cast<uint2*>(qrow)[c] = make_uint2(lo, hi);
  }
  if (threadIdx.x == 0) scale[t] = (a > 0.0f) ? __fdiv_rn(a, 127.0f) : 0.0f;
  if (rowsum != nullptr) {
    sum = block_sum(sum, redi);
    if (threadIdx.x == 0) rowsum[t] = sum;
  }
}

// rowsum_t = sum_k xq[t,k] for int8 input given directly (the integer test hook).
// zero/zero_n16 as for act_quant_kernel.
__global__ void __launch_bounds__(kAqThreads) rowsum_i8_kernel(const int8_t* __restrict__ xq,
                                                              int K, int* __restrict__ rowsum,
                                                              uint4* __restrict__ zero,
                                                              long long zero_n16) {
  __shared__ int redi[32];
  allow_dependent_launch();
  grid_zero(zero, zero_n16);
  const int t = blockIdx.x;
  const int4* row = reinterpret_cast<const int4*>(xq + static_cast<size_t>(t) * K);
  int sum = 0;
  for (int c = threadIdx.x; c < K / 16; c += blockDim.x) {
    const int4 p = row[c];
    const int w[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) sum = __dp4a(w[i], 0x01010101, sum);
  }
  sum = block_sum(sum, redi);
  if (threadIdx.x == 0) rowsum[t] = sum;
}

}  // namespace bl
