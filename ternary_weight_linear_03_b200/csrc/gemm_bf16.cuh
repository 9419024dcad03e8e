// BitLinear backward for quantization-aware training on the 5th-generation tensor cores:
// bf16 x bf16 -> fp32 tcgen05 MMAs (kind::f16) with TMEM accumulators. With the
// straight-through estimator (hackerpaper HN page, thread 21) the two gradients are dense
// contractions:
//   grad_x [M][K] = gamma * G [M][N] . C [N][K]   (tokens x n, weights unpacked to bf16)
//   grad_w [N][K] = G^T [N][M] . X~ [M][K]        (X~ = bf16(q s), contraction over tokens)
// Both run as D[r][c] = alpha * sum_j A[r][j] B[c][j] with A and B K-major (contiguous in
// the contraction index j) in 128-byte swizzled shared memory:
//   grad_x: A = G (rows t), B = C^T (rows k) unpacked from the transposed 2-bit weights
//           (bitlinear_pack_transpose), alpha = gamma;
//   grad_w: A = G^T (rows n), B = X~^T (rows k), both written by a transposing prologue
//           kernel, alpha = 1.
// The trits are exact in bf16 (+-1, 0) and every bf16 x bf16 product is exact in fp32, so
// the only rounding is the fp32 accumulation.
//
// One persistent CTA per SM, 12 warps: warp 0 issues the TMA loads (A tile 128 x 64, B
// tile 192 x 64 bf16, or the packed B tile 192 x 16 bytes), warp 1 owns TMEM (two
// 128 x 192 fp32 accumulators) and issues 4 MMAs (K = 16) per stage (whole-warp loop, one
// elected lane issues), warps 2, 3, 8, 9 unpack the trits to bf16 (when B is packed),
// warps 4..7 drain the accumulator (tcgen05.ld), scale and store. Warps 10 and 11 are
// sentinels: they do the per-stage mbarrier tests for the MMA warp (stage landed, B
// unpacked) and for the unpack warps (stage landed, unpacked slot free), each test about
// 200 to 450 cycles on B200 even for a completed phase, and hand over once per stage at a
// named barrier (bar.red, which also ORs the failure flags so that both sides leave
// together). Every wait is bounded (status word).
#pragma once

#include "common.cuh"
#include "gemm_skinny.cuh"

namespace bl {

namespace bf {
constexpr int BM = 128;                // A rows per tile (MMA M)
constexpr int BN = 192;                // B rows per tile (MMA N); 192 rather than 256: the
                                       // 700M shapes make 256 tiles instead of 192 over 148
                                       // SMs (measured 117 against 133 us for grad_x)
constexpr int BKE = 64;                // contraction elements per stage (128 bytes of bf16)
constexpr int MMA_K = 16;              // K per tcgen05.mma kind::f16
constexpr int STAGES = 5;               // TMA ring (A and B, or A and packed B)
constexpr int USTAGES = 3;              // unpacked B ring (5 / 3 against 4 / 2:
                                        // 105 against 117 us for grad_x)
constexpr int A_BYTES = BM * 128;      // 16 KB
constexpr int BT_BYTES = BN * 128;     // 24 KB bf16 B tile
constexpr int BP_BYTES = BN * BKE / 4; // 3 KB packed B tile
constexpr int TMEM_COLS = 512;         // two accumulators of BN columns (a power of two)
constexpr int THREADS = 384;
constexpr int MMA_SENTINEL = 10, UNPACK_SENTINEL = 11;

// D fp32 (bits 4-5 = 1), A and B bf16 (bits 7-9 = 1, 10-12 = 1), both K-major, N >> 3 in
// bits 17-22, M >> 4 in bits 24-28.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | (static_cast<uint32_t>(N >> 3) << 17) |
         (static_cast<uint32_t>(M >> 4) << 24);
}
constexpr uint32_t IDESC = idesc_bf16(BM, BN);

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

// B packed: TMA ring of (A, packed B) plus a ring of unpacked B tiles; else (A, B) by TMA.
template <bool kPacked>
__host__ __device__ constexpr int smem_bytes() {
  return 1024 + STAGES * A_BYTES +
         (kPacked ? USTAGES * BT_BYTES + STAGES * BP_BYTES : STAGES * BT_BYTES) +
         static_cast<int>(sizeof(Barriers));
}
}  // namespace bf

// Warp-collective bf16 MMA: every lane calls it, one elected lane issues.
__device__ __forceinline__ void mma_bf16_elect(uint32_t d_tmem, uint64_t a_desc,
                                               uint64_t b_desc, uint32_t idesc,
                                               uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// The per-stage handoffs: MMA warp and its sentinel (named barrier 4, 64 threads); the
// four unpack warps and theirs (named barrier 5, 160 threads).
__device__ __forceinline__ bool bf_mma_bar_or(bool v) { return bar_or<4, 64>(v); }
__device__ __forceinline__ bool bf_unp_bar_or(bool v) { return bar_or<5, 160>(v); }

// Two trits of one packed word as two bf16 codes c = u - 1 (low half = the first):
// t holds u of the first trit in bits 0-1 and of the second in bits 8-9. The byte permute
// picks, per trit, the low and high byte of bf16(-1) = 0xBF80, bf16(0) = 0, bf16(1) =
// 0x3F80 from an 8-byte table indexed by u (low bytes at 0..2, high bytes at 4..6).
__device__ __forceinline__ uint32_t trit_pair_bf16(uint32_t t) {
  const uint32_t sel = t | (t << 4) | 0x4040u;
  return __byte_perm(0x00800080u, 0x003F00BFu, sel);
}

// D[r][c] = alpha * sum_j A[r][j] B[c][j], r < R, c < C, j < J (J % 64 == 0 not needed: the
// tensor maps zero-fill past the end). kPacked: B comes as 2-bit trits [C][J/4] (the
// library's packed format, rows c) and is unpacked to bf16 here. alpha: device float or
// null (1). out fp32 [R][C] row-major.
template <bool kPacked>
__global__ void __launch_bounds__(bf::THREADS, 1) gemm_bf16_kernel(
    const __grid_constant__ CUtensorMap map_a, const __grid_constant__ CUtensorMap map_b,
    const float* __restrict__ alpha_ptr, float* __restrict__ out, int R, int C, int J,
    unsigned long long limit_ns) {
  using namespace bf;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sA = smem;
  unsigned char* sB = sA + STAGES * A_BYTES;                 // bf16 B tiles (TMA or unpacked)
  unsigned char* sBp = sB + (kPacked ? USTAGES : STAGES) * BT_BYTES;  // packed B (kPacked)
  Barriers* bar = reinterpret_cast<Barriers*>(sBp + (kPacked ? STAGES * BP_BYTES : 0));
  volatile int* abort_flag = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r_tiles = (R + BM - 1) / BM;
  const int c_tiles = (C + BN - 1) / BN;
  const int num_tiles = r_tiles * c_tiles;
  const int KB = (J + BKE - 1) / BKE;

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

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&map_a);
      prefetch_tmap(&map_b);
      constexpr uint32_t kBytes = A_BYTES + (kPacked ? BP_BYTES : BT_BYTES);
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int r0 = (tile % r_tiles) * BM;
        const int c0 = (tile / r_tiles) * BN;
        for (int kb = 0; kb < KB; ++kb) {
          if (!tc_wait(&bar->empty_tma[s], ph ^ 1u, limit_ns, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&bar->full_tma[s], kBytes);
          tma_load_2d(sA + s * A_BYTES, &map_a, kb * BKE, r0, &bar->full_tma[s]);
          if (kPacked)
            tma_load_2d(sBp + s * BP_BYTES, &map_b, kb * (BKE / 4), c0, &bar->full_tma[s]);
          else
            tma_load_2d(sB + s * BT_BYTES, &map_b, kb * BKE, c0, &bar->full_tma[s]);
          ++issued;
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {
        const long long last = issued - 1;
        for (long long i = last; i >= 0 && i > last - STAGES; --i)
          mbar_wait(&bar->full_tma[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1),
                    100000000ull);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    const uint64_t a_desc0 = smem_desc_k128(smem_u32(sA));
    const uint64_t b_desc0 = smem_desc_k128(smem_u32(sB));
    int s = 0, u = 0, ab = 0;
    uint32_t aph = 0;
    bool ok = true, issued_any = false;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      bool got = true;
      if (lane == 0) got = tc_wait(&bar->tmem_empty[ab], aph ^ 1u, limit_ns, abort_flag);
      got = __shfl_sync(0xffffffffu, got, 0);
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(ab * BN);
      for (int kb = 0; kb < KB; ++kb) {
        // the sentinel has seen the stage land (and its B unpacked); a failed accumulator
        // wait leaves at the first handoff
        if (bf_mma_bar_or(!got)) { ok = false; break; }
        tc_fence_after();
        const uint64_t a_desc = a_desc0 + static_cast<uint64_t>(s * (A_BYTES >> 4));
        const uint64_t b_desc =
            b_desc0 + static_cast<uint64_t>((kPacked ? u : s) * (BT_BYTES >> 4));
#pragma unroll
        for (int kk = 0; kk < BKE / MMA_K; ++kk)  // 32 bytes of bf16 per MMA
          mma_bf16_elect(d_tmem, a_desc + static_cast<uint64_t>(kk * 2),
                         b_desc + static_cast<uint64_t>(kk * 2), IDESC, (kb | kk) != 0 ? 1u : 0u);
        issued_any = true;
        mma_commit_elect(&bar->empty_tma[s]);
        if (kPacked) mma_commit_elect(&bar->empty_unp[u]);
        if (++s == STAGES) s = 0;
        if (kPacked && ++u == USTAGES) u = 0;
      }
      if (!ok) break;
      mma_commit_elect(&bar->tmem_full[ab]);
      if (++ab == 2) { ab = 0; aph ^= 1u; }
    }
    if (!ok && issued_any) {
      mma_commit_elect(&bar->drain);
      if (lane == 0) mbar_wait(&bar->drain, 0u, 100000000ull);
      __syncwarp();
    }
  } else if (warp == MMA_SENTINEL) {
    // ------------------------------------------------------------------ MMA sentinel
    // lane 0: stage g's TMA data landed; lane 1 (packed B): its B tile unpacked
    long long g = 0;
    bool stop = false;
    for (int tile = blockIdx.x; tile < num_tiles && !stop; tile += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb, ++g) {
        bool got = true;
        if (lane == 0)
          got = tc_wait(&bar->full_tma[g % STAGES], static_cast<uint32_t>((g / STAGES) & 1),
                        limit_ns, abort_flag);
        else if (kPacked && lane == 1)
          got = tc_wait(&bar->full_unp[g % USTAGES], static_cast<uint32_t>((g / USTAGES) & 1),
                        limit_ns, abort_flag);
        if (bf_mma_bar_or(!__all_sync(0xffffffffu, got))) { stop = true; break; }
      }
    }
  } else if (warp == UNPACK_SENTINEL) {
    // ------------------------------------------------------------------ unpack sentinel
    // lane 0: stage g's TMA data landed; lane 1: its unpacked slot is free
    if (kPacked) {
      long long g = 0;
      bool stop = false;
      for (int tile = blockIdx.x; tile < num_tiles && !stop; tile += gridDim.x) {
        for (int kb = 0; kb < KB; ++kb, ++g) {
          bool got = true;
          if (lane == 0)
            got = tc_wait(&bar->full_tma[g % STAGES], static_cast<uint32_t>((g / STAGES) & 1),
                          limit_ns, abort_flag);
          else if (lane == 1)
            got = tc_wait(&bar->empty_unp[g % USTAGES],
                          static_cast<uint32_t>(((g / USTAGES) & 1) ^ 1), limit_ns, abort_flag);
          if (bf_unp_bar_or(!__all_sync(0xffffffffu, got))) { stop = true; break; }
        }
      }
    }
  } else if (warp >= 4 && warp < 8) {
    // ------------------------------------------------------------------ epilogue
    const int quarter = warp - 4;
    const int row = quarter * 32 + lane;
    const float alpha = (alpha_ptr != nullptr) ? *alpha_ptr : 1.0f;
    int ab = 0;
    uint32_t aph = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int r0 = (tile % r_tiles) * BM;
      const int c0 = (tile / r_tiles) * BN;
      const bool got = tc_wait(&bar->tmem_full[ab], aph, limit_ns, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int r = r0 + row;
      const bool valid = r < R;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) +
                             static_cast<uint32_t>(ab * BN);
#pragma unroll 1
      for (int cb = 0; cb < BN / 32; ++cb) {
        uint32_t v[32];
        tmem_ld_x32(taddr + cb * 32, v);
        tmem_ld_wait();
        const int c = c0 + cb * 32;
        if (!valid || c >= C) continue;
        float* o = out + static_cast<long long>(r) * C + c;
        float f[32];
#pragma unroll
        for (int j = 0; j < 32; ++j) f[j] = __fmul_rn(__uint_as_float(v[j]), alpha);
        if (c + 32 <= C && (C & 3) == 0) {
#pragma unroll
          for (int j = 0; j < 32; j += 4)
            *reinterpret_cast<float4*>(o + j) = make_float4(f[j], f[j + 1], f[j + 2], f[j + 3]);
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (c + j < C) o[j] = f[j];
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->tmem_empty[ab]);
      if (++ab == 2) { ab = 0; aph ^= 1u; }
    }
  } else if (kPacked) {
    // ------------------------------------------------------------------ unpack warps
    // Task (row, word): one packed 32-bit word = 16 trits of a B row -> 16 bf16 codes = two
    // 16-byte chunks of the swizzled row (row r's chunk ch at (ch ^ (r & 7)) * 16).
    const int uw = (warp < 4) ? (warp - 2) : (warp - 6);
    const int ut = uw * 32 + lane;
    int s = 0, u = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb) {
        // the sentinel has seen the stage land and the unpacked slot freed
        if (bf_unp_bar_or(false)) { ok = false; break; }
        const uint32_t* src = reinterpret_cast<const uint32_t*>(sBp + s * BP_BYTES);
        unsigned char* dst = sB + u * BT_BYTES;
#pragma unroll 2
        for (int it = 0; it < (BN * 4) / 128; ++it) {
          const int task = it * 128 + ut;
          const int r = task >> 2;  // B row within the tile
          const int w = task & 3;   // word of the row's 64 trits
          const uint32_t word = src[r * 4 + w];
          uint32_t o[8];
#pragma unroll
          for (int q = 0; q < 8; ++q) {
            // trits m = 2q, 2q + 1 of the word: group j = m >> 2, bytes i = m & 3, i + 1
            const int m = 2 * q;
            const uint32_t t = (word >> (2 * (m >> 2) + 8 * (m & 3))) & 0x0303u;
            o[q] = trit_pair_bf16(t);
          }
          const int ch = 2 * w;
          *reinterpret_cast<uint4*>(dst + r * 128 + ((ch ^ (r & 7)) << 4)) =
              make_uint4(o[0], o[1], o[2], o[3]);
          *reinterpret_cast<uint4*>(dst + r * 128 + (((ch + 1) ^ (r & 7)) << 4)) =
              make_uint4(o[4], o[5], o[6], o[7]);
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->full_unp[u]);
        if (++s == STAGES) s = 0;
        if (++u == USTAGES) u = 0;
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

// Tile transpose into bf16, for the grad_w operands: out[c][r] for r < R (columns R..Rp-1
// of out are written as zero; Rp = the padded row length of out, a multiple of 8). MODE 0:
// in is bf16 [R][C] (G -> G^T). MODE 1: in is int8 codes q [R][C] with per-row scale s
// (X~ = bf16(q s), round half to even, transposed). C % 64 == 0. 64 x 64 tiles through
// shared memory, every global access 8 elements wide (16 bytes of bf16, 8 of int8); the
// shared rows are 66 elements apart, so that both the row writes and the column gathers
// meet at most two threads per bank.
template <int MODE>
__global__ void __launch_bounds__(256) transpose_bf16_kernel(
    const void* __restrict__ in, const float* __restrict__ scale,
    __nv_bfloat16* __restrict__ out, int R, int C, int Rp) {
  constexpr int TS = 66;  // shared row stride in elements
  __shared__ __align__(16) uint16_t tile[64 * TS];
  const int tiles_r = (Rp + 63) / 64, tiles_c = C / 64;
  for (long long tl = blockIdx.x; tl < static_cast<long long>(tiles_r) * tiles_c; tl += gridDim.x) {
    const int r0 = static_cast<int>(tl % tiles_r) * 64, c0 = static_cast<int>(tl / tiles_r) * 64;
    // rows r0 .. r0 + 63 in: piece p = 8 elements of row p / 8
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int p = threadIdx.x + 256 * h;
      const int rr = p >> 3, c8 = p & 7;
      const int r = r0 + rr, c = c0 + 8 * c8;
      uint32_t w[4] = {0u, 0u, 0u, 0u};
      if (r < R) {
        if (MODE == 0) {
          const uint4 v = *reinterpret_cast<const uint4*>(
              static_cast<const uint16_t*>(in) + static_cast<long long>(r) * C + c);
          w[0] = v.x; w[1] = v.y; w[2] = v.z; w[3] = v.w;
        } else {
          const uint2 q = *reinterpret_cast<const uint2*>(
              static_cast<const int8_t*>(in) + static_cast<long long>(r) * C + c);
          const float sr = scale[r];
          const uint32_t qq[2] = {q.x, q.y};
#pragma unroll
          for (int e = 0; e < 8; e += 2) {
            const int b0 = static_cast<int8_t>((qq[e >> 2] >> (8 * (e & 3))) & 0xffu);
            const int b1 = static_cast<int8_t>((qq[e >> 2] >> (8 * ((e + 1) & 3))) & 0xffu);
            const __nv_bfloat16 h0 = __float2bfloat16_rn(__fmul_rn(static_cast<float>(b0), sr));
            const __nv_bfloat16 h1 = __float2bfloat16_rn(__fmul_rn(static_cast<float>(b1), sr));
            w[e >> 1] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                        (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
          }
        }
      }
      uint32_t* dst = reinterpret_cast<uint32_t*>(tile + rr * TS + 8 * c8);
#pragma unroll
      for (int k = 0; k < 4; ++k) dst[k] = w[k];
    }
    __syncthreads();
    // columns c0 .. c0 + 63 out: piece p = 8 rows of output row p / 8
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int p = threadIdx.x + 256 * h;
      const int cc = p >> 3, r8 = p & 7;
      const int r = r0 + 8 * r8;
      if (r < Rp) {  // Rp % 8 == 0: a piece is all in or all out
        uint32_t w[4];
#pragma unroll
        for (int k = 0; k < 4; ++k)
          w[k] = static_cast<uint32_t>(tile[(8 * r8 + 2 * k) * TS + cc]) |
                 (static_cast<uint32_t>(tile[(8 * r8 + 2 * k + 1) * TS + cc]) << 16);
        *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) +
                                  static_cast<long long>(c0 + cc) * Rp + r) =
            make_uint4(w[0], w[1], w[2], w[3]);
      }
    }
    __syncthreads();
  }
}

// 2-bit weights [N][K/4] -> their transpose [K][N/4] in the same format (row k holds the
// trits of column k along n). N % 64 == 0. One block per 64 x 64 tile: 64 rows x 16 bytes
// in, 64 rows x 16 bytes out; thread (k, g) assembles output word g of row k.
__global__ void __launch_bounds__(256) pack_transpose_kernel(const uint32_t* __restrict__ packed,
                                                             uint32_t* __restrict__ packedT,
                                                             int N, int K) {
  __shared__ uint32_t tin[64][5];  // [n][word of the tile's 64 k] (padded)
  const int wk = K / 16, wn = N / 16;  // words per input row, per output row
  const int tn = N / 64, tk = K / 64;
  for (long long tl = blockIdx.x; tl < static_cast<long long>(tn) * tk; tl += gridDim.x) {
    const int n0 = static_cast<int>(tl % tn) * 64, k0 = static_cast<int>(tl / tn) * 64;
    {
      const int n = threadIdx.x >> 2, w = threadIdx.x & 3;
      tin[n][w] = packed[static_cast<long long>(n0 + n) * wk + k0 / 16 + w];
    }
    __syncthreads();
    const int kk = threadIdx.x >> 2, g = threadIdx.x & 3;  // output row k0 + kk, word g
    const int src_w = kk >> 4, p = kk & 15;
    const int src_shift = 8 * (p & 3) + 2 * (p >> 2);
    uint32_t word = 0u;
#pragma unroll
    for (int m = 0; m < 16; ++m) {
      const uint32_t u = (tin[16 * g + m][src_w] >> src_shift) & 3u;
      word |= u << (8 * (m & 3) + 2 * (m >> 2));
    }
    packedT[static_cast<long long>(k0 + kk) * wn + n0 / 16 + g] = word;
    __syncthreads();
  }
}

}  // namespace bl
