// Decode BitLinear (small M): one CUDA-core kernel that quantizes the M tokens in its
// prologue and then streams the packed ternary weights once from HBM.
//
// The contraction is the addition-only integer product of BitNet b1.58 (dmarx anthology record
// LIT-380, Key takeaways bullet 4). Weights are stored as u = c + 1 in {0, 1, 2}, so
//   acc[t,n] = sum_k c[n,k] q[t,k] = sum_k u[n,k] q[t,k] - rowsum_t,
// and one packed 32-bit word (16 trits) unpacks to four int8x4 registers with one shift
// and one mask each (the packed layout puts trits 16g+4j .. 16g+4j+3 in bits 2j of the
// four bytes). The shift is not even needed: w & (3 << 2j) holds 4^j u per byte, so the
// dp4a of group j accumulates 4^j times the wanted sum in its own register, and the four
// chains are recombined with exact arithmetic shifts. rowsum_t = sum_k q[t,k] comes from
// the prologue.
//
// When a lane's activation chunks fit in registers (one token, at most kGemvRegChunks
// chunks), they are loaded once and every weight row reuses them (no shared-memory
// traffic in the inner loop), and the next row's weights are loaded while the current
// row is being summed. Otherwise the activations are read from shared memory, and when
// one warp covers a whole row and rows are plentiful a warp sums two rows at once, so
// each activation load feeds both.
//
// Layout. Each lane owns 16-byte chunks (64 trits) of a weight row; LPR lanes share a row
// and reduce with warp shuffles. The quantized activations live in shared memory with
// chunk-major order inside each 16-trit group (unit g * CPR + c holds k = 64c + 16g ..
// 64c + 16g + 15), so the lanes of a row read consecutive 16-byte units (no bank
// conflicts) and lanes of different rows read the same unit (broadcast). Rows go to warps
// in turns. On the shared-memory path warps are numbered w * grid + b (warp w of block b):
// when the rows do not divide evenly, the warps that take one turn more are spread over
// every SM instead of filling the first blocks (70B down at one token: 55 or 56 rows on
// every SM, not 64 on some and 48 on the rest; 18.6 -> 18.3 us). The register path keeps
// block-major numbering (warp-major measured 2-3 % slower on the 700M and 3B shapes).
#pragma once

#include "act_quant.cuh"
#include "common.cuh"

namespace bl {

constexpr int kGemvThreads = 512;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvUnroll = 4;
constexpr int kGemvRegChunks = 4;  // chunks per lane whose activations stay in registers

// dp4a with the first operand's bytes unsigned (weights masked in place reach 128).
__device__ __forceinline__ int dp4a_us(uint32_t a, int b, int c) {
  int d;
  asm("dp4a.u32.s32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}

// Adds one packed word's 16 trits times 16 int8 activations into the four chains
// (chain j holds 4^j times its part of the sum).
__device__ __forceinline__ void gemv_word(uint32_t w, const uint4& xv, int (&a)[4]) {
  a[0] = __dp4a(static_cast<int>(w & 0x03030303u), static_cast<int>(xv.x), a[0]);
  a[1] = __dp4a(static_cast<int>(w & 0x0C0C0C0Cu), static_cast<int>(xv.y), a[1]);
  a[2] = __dp4a(static_cast<int>(w & 0x30303030u), static_cast<int>(xv.z), a[2]);
  a[3] = dp4a_us(w & 0xC0C0C0C0u, static_cast<int>(xv.w), a[3]);
}
// The exact sum of the four chains.
__device__ __forceinline__ int gemv_combine(const int (&a)[4]) {
  return a[0] + (a[1] >> 2) + (a[2] >> 4) + (a[3] >> 6);
}

enum XMode { kXf32 = 0, kXbf16 = 1, kXi8 = 2 };
enum OMode { kOf32 = 0, kObf16 = 1, kOi32 = 2 };

template <int MT>
struct GemvShared {
  float red_f[MT][32];
  int red_i[MT][32];
  float f[MT];      // s_t * gamma
  int rowsum[MT];
  float ymax[MT][32];  // per-warp max |y| of each token (layer chains)
};

// Largest |y| of the outputs this thread stored, per token, merged over the block and added
// into amax_out[t] with one atomic max per block and token: the absmax the next layer of a
// chain quantizes its input (this layer's output) with. Non-negative floats order like
// their bit patterns, so the maximum is taken on the bits. Called by every thread.
template <int MT>
__device__ __forceinline__ void block_amax_out(const float (&ymax)[MT], GemvShared<MT>& sh,
                                               float* __restrict__ amax_out) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int t = 0; t < MT; ++t) {
    const unsigned m = __reduce_max_sync(0xffffffffu, __float_as_uint(ymax[t]));
    if (lane == 0) sh.ymax[t][warp] = __uint_as_float(m);
  }
  __syncthreads();
  if (threadIdx.x < MT) {
    float m = 0.0f;
    for (int w = 0; w < static_cast<int>(blockDim.x >> 5); ++w) m = fmaxf(m, sh.ymax[threadIdx.x][w]);
    if (m > 0.0f) atomicMax(reinterpret_cast<unsigned*>(amax_out) + threadIdx.x, __float_as_uint(m));
  }
}

// |value| of an output as stored (the bf16 rounding is monotone, so the largest stored
// magnitude is the rounding of the largest fp32 one; taken per value here for clarity).
template <int OM>
__device__ __forceinline__ float stored_mag(float v) {
  if (OM == 1) return fabsf(__bfloat162float(__float2bfloat16_rn(v)));
  return fabsf(v);
}

// Loads 16 consecutive x values of row t starting at element k (k % 16 == 0).
template <int XM>
__device__ __forceinline__ void load16(const void* x, long long off, float (&v)[16]) {
  if (XM == kXbf16) {
    const uint4* p = reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(x) + off);
    const uint4 a = p[0], b = p[1];
    const uint32_t h[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      v[2 * q] = __uint_as_float(h[q] << 16);
      v[2 * q + 1] = __uint_as_float(h[q] & 0xffff0000u);
    }
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(x) + off);
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 a = p[q];
      v[4 * q] = a.x; v[4 * q + 1] = a.y; v[4 * q + 2] = a.z; v[4 * q + 3] = a.w;
    }
  }
}

// XR: activations in registers (one token). R: rows a warp sums at once on the shared-
// memory path (2 lets every activation load feed two rows; worth it only with many rows).
// Layer chains (optional, null when unused): amax_in[t] is the absmax of token t's row of
// x, formed by the kernel that wrote x, so the prologue skips its max pass; amax_out
// receives the absmax of this kernel's outputs per token (atomic max; zeroed beforehand).
// Launched with programmatic dependent launch, the kernel starts the L2 prefetch of its own
// weights before it waits for the kernel that wrote x, and lets the next kernel launch once
// that wait is over.
template <int MT, int XM, int OM, bool XR, int R>
__global__ void __launch_bounds__(kGemvThreads) gemv_kernel(
    const void* __restrict__ x, const uint8_t* __restrict__ packed,
    const float* __restrict__ gamma_ptr, void* __restrict__ y, int N, int K, int lpr_log2,
    const float* __restrict__ amax_in = nullptr, float* __restrict__ amax_out = nullptr,
    int chain = 0) {
  extern __shared__ __align__(16) unsigned char xs_raw[];  // [MT][K] int8, permuted
  __shared__ GemvShared<MT> sh;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int CPR = K >> 6;   // 16-byte packed chunks per weight row
  const int KB = K >> 4;    // 16-element groups per token row
  if (chain) {
    // L2 prefetch of this block's share of the packed weights (it does not depend on the
    // kernel before), in 4 KB pieces, then wait for that kernel's outputs
    const long long wbytes = static_cast<long long>(N) * (K >> 2);
    const long long per = (wbytes + gridDim.x - 1) / gridDim.x;
    const long long b0 = min(wbytes, per * blockIdx.x), b1 = min(wbytes, b0 + per);
    for (long long o = (b0 & ~4095ll) + 4096ll * tid; o < b1; o += 4096ll * kGemvThreads) {
      const long long len = min(4096ll, wbytes - o);
      asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(packed + o),
                   "r"(static_cast<unsigned>(len & ~15ll))
                   : "memory");
    }
  }
  grid_dependency_wait();
  // Only now (this kernel's input is complete) may the next kernel start and prefetch its
  // own weights: one layer ahead, not a cascade of every later layer into L2.
  allow_dependent_launch();

  // ---------------------------------------------------------------- prologue: x -> int8
  if (XM == kXi8) {
    int sum[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) sum[t] = 0;
    for (int kb = tid; kb < KB; kb += kGemvThreads) {
      const int unit = (kb & 3) * CPR + (kb >> 2);
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        const int4 q = reinterpret_cast<const int4*>(
            static_cast<const int8_t*>(x) + static_cast<long long>(t) * K)[kb];
        reinterpret_cast<int4*>(xs_raw + t * K)[unit] = q;
        sum[t] = __dp4a(q.x, 0x01010101, sum[t]);
        sum[t] = __dp4a(q.y, 0x01010101, sum[t]);
        sum[t] = __dp4a(q.z, 0x01010101, sum[t]);
        sum[t] = __dp4a(q.w, 0x01010101, sum[t]);
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
      for (int w = 0; w < kGemvWarps; ++w) v += sh.red_i[tid][w];
      sh.rowsum[tid] = v;
      sh.f[tid] = 0.0f;
    }
  } else {
    float amax[MT];
    bool bad = false;
#pragma unroll
    for (int t = 0; t < MT; ++t) amax[t] = 0.0f;
    // The float form of the max pass (fp32 x, or a bf16 thread that saw a non-finite value:
    // NaN is skipped by fmaxf and flagged).
    auto amax_pass = [&](int t) {
      float a = 0.0f;
      for (int kb = tid; kb < KB; kb += kGemvThreads) {
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
    if (amax_in == nullptr) {
      if (XM == kXbf16) {
        // one max.u16x2 per two values on the sign-cleared bit patterns
        uint32_t m2[MT];
#pragma unroll
        for (int t = 0; t < MT; ++t) m2[t] = 0u;
        for (int kb = tid; kb < KB; kb += kGemvThreads) {
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
    } else if (tid == 0) {
#pragma unroll
      for (int t = 0; t < MT; ++t) amax[t] = amax_in[t];  // reduced below like the others
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
      for (int w = 0; w < kGemvWarps; ++w) a = fmaxf(a, sh.red_f[t][w]);
      amax[t] = a;
      r[t] = (a > 0.0f) ? __fdiv_rn(127.0f, a) : 0.0f;
    }
    int sum[MT];
#pragma unroll
    for (int t = 0; t < MT; ++t) sum[t] = 0;
    bool fast = (XM == kXbf16);  // bf16 with every r finite (0 when amax is 0)
#pragma unroll
    for (int t = 0; t < MT; ++t) fast &= r[t] <= 3.4028234663852886e38f;
    if (fast) {
      for (int kb = tid; kb < KB; kb += kGemvThreads) {
        const int unit = (kb & 3) * CPR + (kb >> 2);
#pragma unroll
        for (int t = 0; t < MT; ++t)
          reinterpret_cast<uint4*>(xs_raw + t * K)[unit] = quant16_bf16(
              static_cast<const uint16_t*>(x) + static_cast<long long>(t) * K + 16 * kb, r[t], &sum[t]);
      }
    } else for (int kb = tid; kb < KB; kb += kGemvThreads) {
      const int unit = (kb & 3) * CPR + (kb >> 2);
#pragma unroll
      for (int t = 0; t < MT; ++t) {
        uint4 q4;
        if (XM == kXbf16 && r[t] <= 3.4028234663852886e38f) {
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
        reinterpret_cast<uint4*>(xs_raw + t * K)[unit] = q4;
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
      for (int w = 0; w < kGemvWarps; ++w) v += sh.red_i[tid][w];
      sh.rowsum[tid] = v;
      const float s = (amax[tid] > 0.0f) ? __fdiv_rn(amax[tid], 127.0f) : 0.0f;
      sh.f[tid] = __fmul_rn(s, *gamma_ptr);
    }
  }
  __syncthreads();

  // ---------------------------------------------------------------- stream the weights
  float ymax[MT];  // largest |y| this thread stored, per token
#pragma unroll
  for (int t = 0; t < MT; ++t) ymax[t] = 0.0f;
  const int LPR = 1 << lpr_log2;
  const int RPW = 32 >> lpr_log2;
  const int sub = lane & (LPR - 1);
  const int rsel = lane >> lpr_log2;
  const long long warps_total = static_cast<long long>(gridDim.x) * kGemvWarps;
  const uint4* xs4 = reinterpret_cast<const uint4*>(xs_raw);
  const int xs_row_units = K >> 4;

  if constexpr (XR) {
    // ------------------------------------------------------------ activations in registers
    uint4 xr[MT][kGemvRegChunks][4];
#pragma unroll
    for (int t = 0; t < MT; ++t)
#pragma unroll
      for (int u = 0; u < kGemvRegChunks; ++u) {
        const int c = sub + u * LPR;
#pragma unroll
        for (int g = 0; g < 4; ++g)
          xr[t][u][g] = (c < CPR) ? xs4[t * xs_row_units + g * CPR + c] : make_uint4(0u, 0u, 0u, 0u);
      }
    const long long stride = warps_total * RPW;  // rows between two turns of this warp
    const long long rows_of = (static_cast<long long>(blockIdx.x) * kGemvWarps + warp) * RPW;
    uint4 wv[kGemvRegChunks];
    auto load_row = [&](long long row, uint4 (&w)[kGemvRegChunks]) {
      const uint4* prow = reinterpret_cast<const uint4*>(packed + row * (K >> 2));
#pragma unroll
      for (int u = 0; u < kGemvRegChunks; ++u) {
        const int c = sub + u * LPR;
        w[u] = (row < N && c < CPR) ? ld_stream_v4(prow + c) : make_uint4(0u, 0u, 0u, 0u);
      }
    };
    load_row(rows_of + rsel, wv);
    for (long long rbase = rows_of; rbase < N; rbase += stride) {
      const long long n = rbase + rsel;
      uint4 wn[kGemvRegChunks];
      load_row(n + stride, wn);  // next turn's row, in flight while this one is summed
      int ch[MT][4];
#pragma unroll
      for (int t = 0; t < MT; ++t)
#pragma unroll
        for (int j = 0; j < 4; ++j) ch[t][j] = 0;
#pragma unroll
      for (int u = 0; u < kGemvRegChunks; ++u) {
        const uint32_t words[4] = {wv[u].x, wv[u].y, wv[u].z, wv[u].w};
#pragma unroll
        for (int g = 0; g < 4; ++g)
#pragma unroll
          for (int t = 0; t < MT; ++t) gemv_word(words[g], xr[t][u][g], ch[t]);
      }
      int acc[MT];
#pragma unroll
      for (int t = 0; t < MT; ++t) acc[t] = gemv_combine(ch[t]);
      for (int off = LPR >> 1; off > 0; off >>= 1) {
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
      }
      if (n < N && sub == 0) {
#pragma unroll
        for (int t = 0; t < MT; ++t) {
          const int a = acc[t] - sh.rowsum[t];
          const long long o = static_cast<long long>(t) * N + n;
          if (OM == kOi32) {
            static_cast<int*>(y)[o] = a;
          } else {
            const float v = __fmul_rn(__int2float_rn(a), sh.f[t]);
            ymax[t] = fmaxf(ymax[t], stored_mag<OM>(v));
            if (OM == kOf32) static_cast<float*>(y)[o] = v;
            else static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(v);
          }
        }
      }
#pragma unroll
      for (int u = 0; u < kGemvRegChunks; ++u) wv[u] = wn[u];
    }
  } else {
    // ------------------------------------------------------------ activations in smem
    // A warp sums R rows at once (rg, rg + warps_total, ...), so every activation load from
    // shared memory feeds R rows.
    for (long long rg = static_cast<long long>(warp) * gridDim.x + blockIdx.x;
         rg * RPW < N; rg += R * warps_total) {
      long long n[R];
      bool valid[R];
      const uint4* prow[R];
#pragma unroll
      for (int q = 0; q < R; ++q) {
        n[q] = (rg + q * warps_total) * RPW + rsel;
        valid[q] = n[q] < N;
        prow[q] = reinterpret_cast<const uint4*>(packed + (valid[q] ? n[q] : 0) * (K >> 2));
      }
      int acc4[R][MT][4];  // chain j of token t (4^j times its part: see the header)
#pragma unroll
      for (int q = 0; q < R; ++q)
#pragma unroll
        for (int t = 0; t < MT; ++t)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc4[q][t][j] = 0;
      for (int c0 = sub; c0 < CPR; c0 += LPR * kGemvUnroll) {
        uint4 wv[R][kGemvUnroll];
#pragma unroll
        for (int q = 0; q < R; ++q)
#pragma unroll
          for (int u = 0; u < kGemvUnroll; ++u) {
            const int c = c0 + u * LPR;
            wv[q][u] = (valid[q] && c < CPR) ? ld_stream_v4(prow[q] + c) : make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
        for (int u = 0; u < kGemvUnroll; ++u) {
          const int c = c0 + u * LPR;
          if (c < CPR) {
#pragma unroll
            for (int g = 0; g < 4; ++g)
#pragma unroll
              for (int t = 0; t < MT; ++t) {
                const uint4 xv = xs4[t * xs_row_units + g * CPR + c];
#pragma unroll
                for (int q = 0; q < R; ++q) {
                  const uint32_t w = g == 0 ? wv[q][u].x : g == 1 ? wv[q][u].y
                                   : g == 2 ? wv[q][u].z : wv[q][u].w;
                  gemv_word(w, xv, acc4[q][t]);
                }
              }
          }
        }
      }
#pragma unroll
      for (int q = 0; q < R; ++q) {
        int acc[MT];
#pragma unroll
        for (int t = 0; t < MT; ++t) acc[t] = gemv_combine(acc4[q][t]);
        for (int off = LPR >> 1; off > 0; off >>= 1) {
#pragma unroll
          for (int t = 0; t < MT; ++t) acc[t] += __shfl_xor_sync(0xffffffffu, acc[t], off);
        }
        if (valid[q] && sub == 0) {
#pragma unroll
          for (int t = 0; t < MT; ++t) {
            const int a = acc[t] - sh.rowsum[t];
            const long long o = static_cast<long long>(t) * N + n[q];
            if (OM == kOi32) {
              static_cast<int*>(y)[o] = a;
            } else {
              const float v = __fmul_rn(__int2float_rn(a), sh.f[t]);
              ymax[t] = fmaxf(ymax[t], stored_mag<OM>(v));
              if (OM == kOf32) static_cast<float*>(y)[o] = v;
              else static_cast<__nv_bfloat16*>(y)[o] = __float2bfloat16_rn(v);
            }
          }
        }
      }
    }
  }
  if (OM != kOi32 && amax_out != nullptr) block_amax_out<MT>(ymax, sh, amax_out);
}

}  // namespace bl
