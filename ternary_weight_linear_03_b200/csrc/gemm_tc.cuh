// Prefill / batched BitLinear on the 5th-generation tensor cores (tcgen05, sm_100a).
//
// At large M the BitLinear product is a dense int8 contraction, so it runs as
//   D[m][n] = sum_k xq[m][k] * u[n][k]          (tcgen05.mma kind::i8, int32 in TMEM)
//   acc     = D - rowsum_m                       (u = c + 1, so sum_k u q = acc + sum_k q)
//   y       = float(acc) * (scale_m * gamma)     (epilogue, fp32 or bf16)
// which is exactly the addition-only integer product of BitNet b1.58 (dmarx anthology record
// LIT-380, Key takeaways bullet 4) evaluated by the tensor core.
//
// One persistent CTA per SM, 10 warps, warp-specialized:
//   warp 0        TMA producer: xq tile [128 x 128] (128-byte swizzle) and the packed
//                 weight tile [256 rows x 32 bytes] into a STAGES-deep ring
//   warps 2,3,8,9 unpack: 2-bit codes -> one int8 per trit (shift + mask), written in the
//                 128-byte swizzled K-major layout the MMA reads, USTAGES-deep ring
//   warp 1        allocates 512 TMEM columns; one lane issues 4 MMAs (K = 32 each) per
//                 stage into a double-buffered 128 x 256 int32 accumulator
//   warps 4..7    epilogue: tcgen05.ld of their 32 TMEM lanes, subtract rowsum, rescale,
//                 store, while the MMA fills the other accumulator buffer
// Every mbarrier wait is bounded; on a timeout the kernel records BL_ERR_TIMEOUT, waits
// (bounded) for its own copies and MMAs in flight, frees TMEM and exits.
#pragma once

#include "common.cuh"

namespace bl {

namespace tc {
constexpr int BM = 128;              // tokens per tile (MMA M)
constexpr int BN = 256;              // weight rows per tile (MMA N)
constexpr int BK = 128;              // K per stage: one 128-byte swizzle row of int8
constexpr int MMA_K = 32;            // K per tcgen05.mma kind::i8
constexpr int STAGES = 4;            // TMA ring depth (xq tile + packed tile)
constexpr int USTAGES = 2;           // unpacked-weight ring depth
constexpr int A_BYTES = BM * BK;     // 16 KB
constexpr int BP_BYTES = BN * BK / 4;  // 8 KB
constexpr int BU_BYTES = BN * BK;    // 32 KB
constexpr int TMEM_COLS = 2 * BN;    // two accumulator buffers
constexpr int THREADS = 320;
constexpr uint32_t IDESC = idesc_i8(BM, BN);

struct Barriers {
  uint64_t full_tma[STAGES];
  uint64_t empty_tma[STAGES];
  uint64_t full_unp[USTAGES];
  uint64_t empty_unp[USTAGES];
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

constexpr int SMEM_BYTES =
    1024 /* alignment slack */ + STAGES * A_BYTES + USTAGES * BU_BYTES + STAGES * BP_BYTES +
    static_cast<int>(sizeof(Barriers));
}  // namespace tc

// Bounded wait that also gives up when another role has already aborted.
__device__ __forceinline__ bool tc_wait(uint64_t* bar, uint32_t parity, uint64_t limit_ns,
                                        volatile int* abort) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = global_ns();
  while (true) {
#pragma unroll 1
    for (int i = 0; i < 32; ++i)
      if (mbar_try_wait(bar, parity)) return true;
    if (*abort) return false;
    if (global_ns() - t0 > limit_ns) {
      record_status(kStatusTimeout);
      *abort = 1;
      return false;
    }
  }
}

// OM: 0 fp32 out, 1 bf16 out, 2 int32 out (acc only).
template <int OM>
__global__ void __launch_bounds__(tc::THREADS, 1) gemm_tc_kernel(
    const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
    const int* __restrict__ rowsum, const float* __restrict__ scale,
    const float* __restrict__ gamma_ptr, void* __restrict__ y, int M, int N, int K,
    unsigned long long limit_ns, float* __restrict__ amax_out) {
  using namespace tc;
  allow_dependent_launch();  // the next kernel may set up (it waits before using y)
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sA = smem;
  unsigned char* sBu = sA + STAGES * A_BYTES;
  unsigned char* sBp = sBu + USTAGES * BU_BYTES;
  Barriers* bar = reinterpret_cast<Barriers*>(sBp + STAGES * BP_BYTES);
  volatile int* abort_flag = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m_tiles = (M + BM - 1) / BM;
  const int n_tiles = (N + BN - 1) / BN;
  const int num_tiles = m_tiles * n_tiles;
  const int KB = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bar->full_tma[s], 1);
      mbar_init(&bar->empty_tma[s], 1);
    }
    for (int u = 0; u < USTAGES; ++u) {
      mbar_init(&bar->full_unp[u], 4);
      mbar_init(&bar->empty_unp[u], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar->tmem_full[b], 1);
      mbar_init(&bar->tmem_empty[b], 4);
    }
    mbar_init(&bar->drain, 1);
    bar->abort = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&bar->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bar->tmem_base;
  // Set-up done; the operands come from the kernel before (programmatic dependent launch:
  // returns at once when launched without it).
  grid_dependency_wait();

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&map_a);
      prefetch_tmap(&map_b);
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int m0 = (tile % m_tiles) * BM;
        const int n0 = (tile / m_tiles) * BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!tc_wait(&bar->empty_tma[s], ph ^ 1u, limit_ns, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&bar->full_tma[s], A_BYTES + BP_BYTES);
          tma_load_2d(sA + s * A_BYTES, &map_a, kb * BK, m0, &bar->full_tma[s]);
          tma_load_2d(sBp + s * BP_BYTES, &map_b, kb * (BK / 4), n0, &bar->full_tma[s]);
          ++issued;
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        // wait (bounded) for the copies this thread still has in flight
        const long long last = issued - 1;
        for (long long i = last; i >= 0 && i > last - STAGES; --i) {
          const int slot = static_cast<int>(i % STAGES);
          const uint32_t par = static_cast<uint32_t>((i / STAGES) & 1);
          mbar_wait(&bar->full_tma[slot], par, 100000000ull);
        }
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      // Descriptors are built once; a stage or K step only moves the 14-bit start-address
      // field (16-byte units), which keeps the single issuing thread's work per MMA tiny.
      const uint64_t a_desc0 = smem_desc_k128(smem_u32(sA));
      const uint64_t b_desc0 = smem_desc_k128(smem_u32(sBu));
      int s = 0, u = 0, ab = 0;
      uint32_t ph = 0, uph = 0, aph = 0;
      bool ok = true, issued_any = false;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        if (!tc_wait(&bar->tmem_empty[ab], aph ^ 1u, limit_ns, abort_flag)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(ab * BN);
        for (int kb = 0; kb < KB; ++kb) {
          if (!tc_wait(&bar->full_unp[u], uph, limit_ns, abort_flag) ||
              !tc_wait(&bar->full_tma[s], ph, limit_ns, abort_flag)) { ok = false; break; }
          tc_fence_after();
          const uint64_t a_desc = a_desc0 + static_cast<uint64_t>(s * (A_BYTES >> 4));
          const uint64_t b_desc = b_desc0 + static_cast<uint64_t>(u * (BU_BYTES >> 4));
#pragma unroll
          for (int kk = 0; kk < BK / MMA_K; ++kk) {
            mma_i8(d_tmem, a_desc + static_cast<uint64_t>(kk * (MMA_K >> 4)),
                   b_desc + static_cast<uint64_t>(kk * (MMA_K >> 4)), IDESC,
                   (kb | kk) != 0 ? 1u : 0u);
          }
          issued_any = true;
          mma_commit(&bar->empty_tma[s]);
          mma_commit(&bar->empty_unp[u]);
          if (++s == STAGES) { s = 0; ph ^= 1u; }
          if (++u == USTAGES) { u = 0; uph ^= 1u; }
        }
        if (!ok) break;
        mma_commit(&bar->tmem_full[ab]);
        if (++ab == 2) { ab = 0; aph ^= 1u; }
      }
      if (!ok && issued_any) {
        mma_commit(&bar->drain);  // completes once every MMA issued above has finished
        mbar_wait(&bar->drain, 0u, 100000000ull);
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp - 4;  // TMEM lanes 32*quarter .. 32*quarter+31
    const int row = quarter * 32 + lane;
    const float gamma = (OM == 2) ? 0.0f : *gamma_ptr;
    int ab = 0;
    uint32_t aph = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int m0 = (tile % m_tiles) * BM;
      const int n0 = (tile / m_tiles) * BN;
      // every lane waits; the decision is made warp-uniform because tcgen05.ld is .aligned
      const bool got = tc_wait(&bar->tmem_full[ab], aph, limit_ns, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int m = m0 + row;
      const bool valid = m < M;
      const int rs = valid ? rowsum[m] : 0;
      const float f = (OM != 2 && valid) ? __fmul_rn(scale[m], gamma) : 0.0f;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(ab * BN);
      float ymax = 0.0f;  // largest |y| of this row in the tile (layer chains)
#pragma unroll 1
      for (int cb = 0; cb < BN / 32; ++cb) {
        uint32_t v[32];
        tmem_ld_x32(taddr + cb * 32, v);
        tmem_ld_wait();
        const int n = n0 + cb * 32;
        if (!valid || n >= N) continue;
        const long long o = static_cast<long long>(m) * N + n;
        const bool vec = (n + 32 <= N) && ((N & 7) == 0);
        if (OM == 2) {
          int* out = static_cast<int*>(y) + o;
          if (vec) {
#pragma unroll
            for (int j = 0; j < 32; j += 4)
              *reinterpret_cast<int4*>(out + j) =
                  make_int4(static_cast<int>(v[j]) - rs, static_cast<int>(v[j + 1]) - rs,
                            static_cast<int>(v[j + 2]) - rs, static_cast<int>(v[j + 3]) - rs);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < N) out[j] = static_cast<int>(v[j]) - rs;
          }
        } else {
          float r[32];
#pragma unroll
          for (int j = 0; j < 32; ++j)
            r[j] = __fmul_rn(__int2float_rn(static_cast<int>(v[j]) - rs), f);
          if (amax_out != nullptr) {
            // the bf16 rounding is monotone: the largest stored magnitude is the rounding
            // of the largest fp32 one
#pragma unroll
            for (int j = 0; j < 32; ++j)
              if (n + j < N) ymax = fmaxf(ymax, fabsf(r[j]));
          }
          if (OM == 0) {
            float* out = static_cast<float*>(y) + o;
            if (vec) {
#pragma unroll
              for (int j = 0; j < 32; j += 4)
                *reinterpret_cast<float4*>(out + j) = make_float4(r[j], r[j + 1], r[j + 2], r[j + 3]);
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (n + j < N) out[j] = r[j];
            }
          } else {
            __nv_bfloat16* out = static_cast<__nv_bfloat16*>(y) + o;
            if (vec) {
#pragma unroll
              for (int j = 0; j < 32; j += 8) {
                uint4 pk;
                __nv_bfloat162 h0 = __floats2bfloat162_rn(r[j], r[j + 1]);
                __nv_bfloat162 h1 = __floats2bfloat162_rn(r[j + 2], r[j + 3]);
                __nv_bfloat162 h2 = __floats2bfloat162_rn(r[j + 4], r[j + 5]);
                __nv_bfloat162 h3 = __floats2bfloat162_rn(r[j + 6], r[j + 7]);
                pk.x = *reinterpret_cast<uint32_t*>(&h0);
                pk.y = *reinterpret_cast<uint32_t*>(&h1);
                pk.z = *reinterpret_cast<uint32_t*>(&h2);
                pk.w = *reinterpret_cast<uint32_t*>(&h3);
                *reinterpret_cast<uint4*>(out + j) = pk;
              }
            } else {
#pragma unroll
              for (int j = 0; j < 32; ++j)
                if (n + j < N) out[j] = __float2bfloat16_rn(r[j]);
            }
          }
        }
      }
      if (OM != 2 && amax_out != nullptr && valid && ymax > 0.0f) {
        const float m = (OM == 1) ? __bfloat162float(__float2bfloat16_rn(ymax)) : ymax;
        atomicMax(reinterpret_cast<unsigned*>(amax_out) + m0 + row, __float_as_uint(m));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->tmem_empty[ab]);
      if (++ab == 2) { ab = 0; aph ^= 1u; }
    }
  } else {
    // ------------------------------------------------------------------ unpack warps
    const int uw = (warp < 4) ? (warp - 2) : (warp - 6);  // 0..3
    const int ut = uw * 32 + lane;                          // 0..127
    int s = 0, u = 0;
    uint32_t ph = 0, uph = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb) {
        const bool got = tc_wait(&bar->full_tma[s], ph, limit_ns, abort_flag) &&
                         tc_wait(&bar->empty_unp[u], uph ^ 1u, limit_ns, abort_flag);
        if (!__all_sync(0xffffffffu, got)) { ok = false; break; }
        const unsigned char* src = sBp + s * BP_BYTES;
        unsigned char* dst = sBu + u * BU_BYTES;
#pragma unroll
        for (int it = 0; it < (BN * 2) / 128; ++it) {
          const int task = it * 128 + ut;
          const int h = task & 1;   // which 16-byte half of the 32-byte packed row
          const int r = task >> 1;  // weight row within the tile
          const uint4 p = *reinterpret_cast<const uint4*>(src + r * 32 + h * 16);
          const uint32_t words[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
          for (int mq = 0; mq < 4; ++mq) {
            const uint32_t w = words[mq];
            const int chunk = 4 * h + mq;  // 16-trit group = 16-byte chunk of the row
            const uint4 o = make_uint4(w & 0x03030303u, (w >> 2) & 0x03030303u,
                                       (w >> 4) & 0x03030303u, (w >> 6) & 0x03030303u);
            *reinterpret_cast<uint4*>(dst + r * 128 + ((chunk ^ (r & 7)) << 4)) = o;
          }
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->full_unp[u]);
        if (++s == STAGES) { s = 0; ph ^= 1u; }
        if (++u == USTAGES) { u = 0; uph ^= 1u; }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace bl
