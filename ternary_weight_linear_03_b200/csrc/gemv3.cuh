// Decode BitLinear on the base-3 weight format: five trits per byte, 1.6 bits per weight
// (hackerpaper HN page, thread 3: 3^5 = 243 fits in a byte), 0.8 of the bytes the 2-bit
// format streams from HBM.
//
// Format (16-byte chunks of 80 trits; a row is ceil(K/80) chunks): byte i of chunk j
// holds trits k = 80 j + 16 p + i (p = 0..4) as B = ceil(256 v / 243), v the base-3 number
// with digits u_p = c_p + 1 (u_0 leading). Multiplying B by 3 carries the leading digit
// into bits 8..9 and leaves the rest as a fixed-point fraction in the low byte, so the
// digits come out one per multiply (exact for every v: the rounding error of B, below
// 1/256 of a unit, stays under the gap to the next digit through all five steps).
//
// In a 32-bit word of four packed bytes the even bytes (0, 2) and the odd bytes (1, 3)
// sit in two registers as 16-bit lanes; x 3 never carries across a lane (765 < 2^16).
// After each multiply the four digits are bytes 1 and 3 of the two registers, and one
// byte permute assembles them as four bytes in the order of bytes 0..3 of the word, i.e.
// u of four consecutive k (trits 80 j + 16 p + 4 w .. +3 for word w): exactly the int8x4
// of activations at those positions, which a dp4a multiplies. The contraction is the
// same u = c + 1 form as the 2-bit kernels: acc = sum_k u q - rowsum_t.
//
// Structure as the 2-bit GEMV: the M (<= 4) tokens are quantized in the prologue into
// shared memory in natural order (zero beyond K up to the chunk boundary); LPR lanes share
// a weight row, each streaming its 16-byte chunks with no-allocate loads, and the lanes of
// a row reduce with shuffles. Warps take rows in turns, numbered across the grid as the
// 2-bit GEMV numbers them (warp w of block b is w * grid + b).
#pragma once

#include "act_quant.cuh"
#include "common.cuh"
#include "gemv.cuh"

namespace bl {

constexpr int kGemv3Threads = 512;
constexpr int kGemv3Warps = kGemv3Threads / 32;
constexpr int kGemv3Unroll = 2;  // chunks a lane has in flight

// The five digit words (p = 0..4) of one packed word w, each dp4a'ed with the activation
// word of its position: xw[p] holds activations k = 80 j + 16 p + 4 w .. +3.
template <int MT>
__device__ __forceinline__ void gemv3_word(uint32_t w, const uint32_t (&xw)[MT][5],
                                           int (&acc)[MT]) {
  uint32_t e = w & 0x00FF00FFu;         // bytes 0 and 2, one per 16-bit lane
  uint32_t o = (w >> 8) & 0x00FF00FFu;  // bytes 1 and 3
#pragma unroll
  for (int p = 0; p < 5; ++p) {
    e *= 3u;
    o *= 3u;
    const uint32_t d = __byte_perm(e, o, 0x7351);  // digits of bytes 0, 1, 2, 3
    e &= 0x00FF00FFu;
    o &= 0x00FF00FFu;
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[t] = __dp4a(static_cast<int>(d), static_cast<int>(xw[t][p]), acc[t]);
  }
}

// M = MT tokens (1..4), x fp32 or bf16 (XM), y fp32 or bf16 (OM); smem = MT * 80 * CH
// bytes (CH = chunks per row).
template <int MT, int XM, int OM>
__global__ void __launch_bounds__(kGemv3Threads) gemv3_kernel(
    const void* __restrict__ x, const uint8_t* __restrict__ packed3,
    const float* __restrict__ gamma_ptr, void* __restrict__ y, int N, int K, int lpr_log2) {
  extern __shared__ __align__(16) unsigned char xs3[];  // [MT][80 * CH] int8
  __shared__ GemvShared<MT> sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int CH = (K + 79) / 80;
  const int KP = 80 * CH;  // padded row of activations
  const int KB = K >> 4;

  // ---------------------------------------------------------------- prologue: x -> int8
  float amax[MT];
  bool bad = false;
#pragma unroll
  for (int t = 0; t < MT; ++t) amax[t] = 0.0f;
  // the float pass (fp32 x, or a bf16 thread that saw a non-finite value: NaN is skipped by
  // fmaxf and flagged)
  auto amax_pass = [&](int t) {
    float a = 0.0f;
    for (int kb = tid; kb < KB; kb += kGemv3Threads) {
      float v[16];
      load16<XM>(x, static_cast<long long>(t) * K + 16 * kb, v);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float m = abs_bits(v[i]);
        bad |= !(m <= 3.4028234663852886e38f);
        a = fmaxf(a, m);
      }
    }
    return a;
  };
  if (XM == kXbf16) {  // one max.u16x2 per two values on the sign-cleared bit patterns
    uint32_t m2[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) m2[t] = 0u;
    for (int kb = tid; kb < KB; kb += kGemv3Threads) {
#pragma unroll
      for (int t = 0; t < MT; ++t)
        m2[t] = absmax16_bf16(static_cast<const uint16_t*>(x) + static_cast<long long>(t) * K + 16 * kb,
                              m2[t]);
    }
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      const uint32_t m = max(m2[t] & 0xffffu, m2[t] >> 16);
      amax[t] = (m < 0x7f80u) ? __uint_as_float(m << 16) : amax_pass(t);
    }
  } else {
#pragma unroll
    for (int t = 0; t < MT; ++t) amax[t] = amax_pass(t);
  }
  if (bad) record_status(kStatusNonfinite);
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    float v = amax[t];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, off));
    if (lane == 0) sh.red_f[t][warp] = v;
  }
  __syncthreads();
  float r[MT];
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    float a = 0.0f;
    for (int w = 0; w < kGemv3Warps; ++w) a = fmaxf(a, sh.red_f[t][w]);
    amax[t] = a;
    r[t] = (a > 0.0f) ? __fdiv_rn(127.0f, a) : 0.0f;
  }
  int sum[MT];
#pragma unroll
  for (int t = 0; t < MT; ++t) sum[t] = 0;
  for (int kb = tid; kb < KP / 16; kb += kGemv3Threads) {
#pragma unroll
    for (int t = 0; t < MT; ++t) {
      uint4 q4 = make_uint4(0u, 0u, 0u, 0u);
      if (kb < KB) {
        if (XM == kXbf16 && r[t] <= 3.4028234663852886e38f) {  // finite r (0 when amax is 0)
          q4 = quant16_bf16(static_cast<const uint16_t*>(x) + static_cast<long long>(t) * K + 16 * kb,
                            r[t], &sum[t]);
        } else {
          float v[16];
          load16<XM>(x, static_cast<long long>(t) * K + 16 * kb, v);
          uint32_t w4[4] = {0u, 0u, 0u, 0u};
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const int q = (amax[t] > 0.0f) ? quant_i8(v[i], r[t]) : 0;
            sum[t] += q;
            w4[i >> 2] |= (static_cast<uint32_t>(q) & 0xffu) << (8 * (i & 3));
          }
          q4 = make_uint4(w4[0], w4[1], w4[2], w4[3]);
        }
      }
      reinterpret_cast<uint4*>(xs3 + t * KP)[kb] = q4;
    }
  }
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    int v = sum[t];
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
    if (lane == 0) sh.red_i[t][warp] = v;
  }
  __syncthreads();
  if (tid < MT) {
    int v = 0;
    for (int w = 0; w < kGemv3Warps; ++w) v += sh.red_i[tid][w];
    sh.rowsum[tid] = v;
    const float s = (amax[tid] > 0.0f) ? __fdiv_rn(amax[tid], 127.0f) : 0.0f;
    sh.f[tid] = __fmul_rn(s, *gamma_ptr);
  }
  __syncthreads();

  // ---------------------------------------------------------------- stream the weights
  const int LPR = 1 << lpr_log2;
  const int RPW = 32 >> lpr_log2;
  const int sub = lane & (LPR - 1);
  const int rsel = lane >> lpr_log2;
  const long long warps_total = static_cast<long long>(gridDim.x) * kGemv3Warps;
  const long long row_bytes = 16ll * CH;
  for (long long rg = static_cast<long long>(warp) * gridDim.x + blockIdx.x; rg * RPW < N;
       rg += warps_total) {
    const long long n = rg * RPW + rsel;
    const bool valid = n < N;
    const uint4* prow = reinterpret_cast<const uint4*>(packed3 + (valid ? n : 0) * row_bytes);
    int acc[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) acc[t] = 0;
    for (int c0 = sub; c0 < CH; c0 += LPR * kGemv3Unroll) {
      uint4 wv[kGemv3Unroll];
#pragma unroll
      for (int u = 0; u < kGemv3Unroll; ++u) {
        const int c = c0 + u * LPR;
        wv[u] = (valid && c < CH) ? ld_stream_v4(prow + c) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int u = 0; u < kGemv3Unroll; ++u) {
        const int c = c0 + u * LPR;
        if (c >= CH) continue;
        uint32_t xw[4][MT][5];  // [word w][token][digit p]
#pragma unroll
        for (int t = 0; t < MT; ++t)
#pragma unroll
          for (int p = 0; p < 5; ++p) {
            const uint4 xv = *reinterpret_cast<const uint4*>(xs3 + t * KP + 80 * c + 16 * p);
            xw[0][t][p] = xv.x;
            xw[1][t][p] = xv.y;
            xw[2][t][p] = xv.z;
            xw[3][t][p] = xv.w;
          }
        gemv3_word<MT>(wv[u].x, xw[0], acc);
        gemv3_word<MT>(wv[u].y, xw[1], acc);
        gemv3_word<MT>(wv[u].z, xw[2], acc);
        gemv3_word<MT>(wv[u].w, xw[3], acc);
      }
    }
    for (int off = LPR >> 1; off > 0; off >>= 1) {
#pragma unroll
      for (int t = 0; t < MT; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
    }
    if (valid && sub == 0) {
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int a = acc[t] - sh.rowsum[t];
        const long long o = static_cast<long long>(t) * N + n;
        const float v = __fmul_rn(__int2float_rn(a), sh.f[t]);
        if (OM == kOf32) static_cast<float*>(y)[o] = v;
        else static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(v);
      }
    }
  }
}

// 2-bit format -> base-3 format, one thread per 16-byte output chunk (80 trits). The
// 2-bit word g of a row holds trits 16 g .. 16 g + 15, trit 16 g + 4 jj + ii in bits
// 8 ii + 2 jj as u = c + 1; chunk j draws on words 5 j .. 5 j + 4 (u = 1, a zero weight,
// past the row's end).
__global__ void __launch_bounds__(256) pack_base3_kernel(const uint32_t* __restrict__ packed,
                                                         uint4* __restrict__ packed3, int N,
                                                         int K) {
  const int CH = (K + 79) / 80;
  const int words = K / 16;
  const long long total = static_cast<long long>(N) * CH;
  for (long long id = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; id < total;
       id += static_cast<long long>(gridDim.x) * blockDim.x) {
    const long long n = id / CH;
    const int j = static_cast<int>(id % CH);
    uint32_t wd[5];
#pragma unroll
    for (int p = 0; p < 5; ++p) {
      const int g = 5 * j + p;
      wd[p] = (g < words) ? packed[n * words + g] : 0x55555555u;  // u = 1 everywhere
    }
    uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      uint32_t v = 0u;
#pragma unroll
      for (int p = 0; p < 5; ++p)
        v = 3u * v + ((wd[p] >> (8 * (i & 3) + 2 * (i >> 2))) & 3u);  // trit 80 j + 16 p + i
      const uint32_t b = (256u * v + 242u) / 243u;  // ceil(256 v / 243)
      out[i >> 2] |= b << (8 * (i & 3));
    }
    packed3[id] = make_uint4(out[0], out[1], out[2], out[3]);
  }
}

}  // namespace bl
