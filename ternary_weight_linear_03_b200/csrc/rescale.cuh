// The BitLinear rescale on its own, for an int32 product formed elsewhere (a sum of
// per-GPU partial products under tensor parallelism):
//   y[t,n] = fl(float(acc[t,n]) * fl(scale_t * gamma))     (fp32, or its bf16 RNE)
// the same operation order as the epilogues of the fused kernels (acc is exact below
// 2^24 in magnitude, so float(acc) is exact). Elementwise and HBM-bound: each thread
// handles 4 consecutive outputs of one row.
#pragma once

#include "common.cuh"

namespace bl {

constexpr int kRsThreads = 256;

// grid-stride over groups of 4 outputs; N % 4 == 0. OM: 0 fp32, 1 bf16.
template <int OM>
__global__ void __launch_bounds__(kRsThreads) rescale_kernel(
    const int* __restrict__ acc, const float* __restrict__ scale,
    const float* __restrict__ gamma_ptr, void* __restrict__ y, int M, int N) {
  const float gamma = *gamma_ptr;
  const long long groups = static_cast<long long>(M) * (N / 4);
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < groups;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const int t = static_cast<int>(i / (N / 4));
    const float f = __fmul_rn(scale[t], gamma);
    const int4 a = reinterpret_cast<const int4*>(acc)[i];
    const float r0 = __fmul_rn(__int2float_rn(a.x), f), r1 = __fmul_rn(__int2float_rn(a.y), f);
    const float r2 = __fmul_rn(__int2float_rn(a.z), f), r3 = __fmul_rn(__int2float_rn(a.w), f);
    if (OM == 0) {
      reinterpret_cast<float4*>(y)[i] = make_float4(r0, r1, r2, r3);
    } else {
      __nv_bfloat162 h0 = __floats2bfloat162_rn(r0, r1), h1 = __floats2bfloat162_rn(r2, r3);
      reinterpret_cast<uint2*>(y)[i] =
          make_uint2(*reinterpret_cast<uint32_t*>(&h0), *reinterpret_cast<uint32_t*>(&h1));
    }
  }
}

}  // namespace bl

namespace bl {

// The same rescale one output per thread, for rows whose length is not a multiple of 4.
template <int OM>
__global__ void __launch_bounds__(kRsThreads) rescale_scalar_kernel(
    const int* __restrict__ acc, const float* __restrict__ scale,
    const float* __restrict__ gamma_ptr, void* __restrict__ y, int M, int N) {
  const float gamma = *gamma_ptr;
  const long long total = static_cast<long long>(M) * N;
  for (long long i = static_cast<long long>(blockIdx.x) * blockDim.x + threadIdx.x; i < total;
       i += static_cast<long long>(gridDim.x) * blockDim.x) {
    const float f = __fmul_rn(scale[i / N], gamma);
    const float r = __fmul_rn(__int2float_rn(acc[i]), f);
    if (OM == 0) static_cast<float*>(y)[i] = r;
    else static_cast<__nv_bfloat16*>(y)[i] = __float2bfloat16_rn(r);
  }
}

}  // namespace bl
