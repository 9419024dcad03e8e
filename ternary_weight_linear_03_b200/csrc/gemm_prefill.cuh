// Prefill BitLinear (many tokens) on the 5th-generation tensor cores, operands swapped so
// that the ternary weights never pass through shared memory unpacked:
//   D[n][t] = sum_k u[n][k] * xq[t][k]        (tcgen05.mma kind::i8, A from TMEM)
//   y[t][n] = float(D - rowsum_t) * (scale_t * gamma)
// the addition-only integer product of BitNet b1.58 (dmarx anthology record LIT-380, Key
// takeaways bullet 4) in the u = c + 1 form of the other kernels.
//
// Why swapped: with the weights as the B operand in shared memory, every K block moves the
// packed tile in, the unpacked int8 tile out and back in to the tensor core, next to the
// token tile: about 112 KB of shared-memory traffic per 128 x 256 x 128 block of MMA work,
// more than shared memory sustains while the tensor core works. Here the four unpack warps
// turn each thread's weight row (32 packed bytes = 128 trits of a K block) into 32
// registers and write them with one tcgen05.st into that row's TMEM lane; the MMA reads A
// from TMEM. Shared memory carries only the token tile (written by TMA, read by the MMA)
// and the 4 KB packed tile: 56 KB per 128 x 192 x 128 block.
//
// Tiles: 128 weight rows (MMA M, TMEM lanes) x bnt <= 192 tokens (MMA N). TMEM (512
// columns): two accumulators of 192 columns (the epilogue drains one while the MMAs fill
// the other) and ASLOTS unpacked K blocks of 32 columns. Shared memory holds STAGES > ASLOTS
// TMA stages, deeper than TMEM allows A slots, so that the L2 latency of the token tiles
// stays covered; stage g's weights go to slot g % ASLOTS once the MMAs of stage
// g - ASLOTS, its last readers, have completed (their commit arrives on a_empty).
//
// Warps: 0-7 unpack in two sets of four that take alternate stages (each set's chain of
// barrier waits, shared-memory load, tcgen05.st, wait::st and arrival per stage is longer
// than the MMAs of one stage; thread r of a set owns weight row r, TMEM lane r), 8-11
// epilogue (tcgen05.ld of their 32 lanes, rowsum, rescale, store), 12 TMA producer, 13
// TMEM owner and MMA issuer (whole-warp loop, one elected lane issues), 14-16 sentinels.
// Three sets over five slots of 176 columns measured slower on B200 (0.89 ms against
// 0.77 ms at M = 4096).
//
// Sentinels take every per-stage mbarrier test off the MMA and unpack warps. Measured with
// clock64 stamps on B200, a test costs 150 to 450 cycles even for a phase completed long
// before: the MMA warp's (is the stage's A slot written?) cost it about 190 cycles per
// stage against about 250 for the four MMAs and two commits, and an unpack set's two
// (stage landed, A slot free) about 335 of its 765 cycles per stage. Warp 14 tests for
// the MMA warp, warps 15 and 16 for unpack sets 0 and 1. Each pair meets once per stage at
// a named barrier (bar.red, which also ORs the failure flags so that both sides leave
// together), and the sentinel tests the next stage while its partner works on the
// current one (0.68 against 0.70 ms per step at M = 4096).
//
// Persistent: one CTA per SM walks the tiles, consecutive CTAs taking consecutive token
// tiles of one weight tile (L2 reuse of both).
// Every mbarrier wait is bounded; on a timeout the kernel records BL_ERR_TIMEOUT, waits
// (bounded) for its own copies and MMAs, frees TMEM and exits.
#pragma once

#include "common.cuh"
#include "gemm_skinny.cuh"

namespace bl {

namespace pf {
constexpr int BW = 128;                   // weight rows per tile (MMA M)
constexpr int BK = 128;                   // K per stage (one 128-byte swizzle row of int8)
constexpr int MMA_K = 32;                 // K per tcgen05.mma kind::i8
constexpr int STAGES = 7;                 // TMA stages (token tile + packed weights)
constexpr int ASLOTS = 4;                 // unpacked A slots in TMEM
constexpr int MAX_BNT = 192;              // tokens per tile, at most (MMA N)
constexpr int X_BYTES = MAX_BNT * BK;     // 24 KB token tile (128-byte swizzle)
constexpr int WP_BYTES = BW * BK / 4;     // 4 KB packed weight tile
constexpr int A_COLS = BK / 4;            // TMEM columns of one unpacked K block
constexpr int A_COL0 = 2 * MAX_BNT;       // first A slot column, after two accumulators
constexpr int TMEM_COLS = 512;
constexpr int UNPACK_SETS = 2;
constexpr int UNPACK_WARPS = 4 * UNPACK_SETS;
constexpr int EPI_WARP0 = UNPACK_WARPS;        // 4 epilogue warps
constexpr int TMA_WARP = EPI_WARP0 + 4;
constexpr int MMA_WARP = TMA_WARP + 1;
constexpr int SENTINEL_WARP = MMA_WARP + 1;        // tests for the MMA warp
constexpr int SET_SENTINEL0 = SENTINEL_WARP + 1;    // tests for unpack set 0, then set 1
constexpr int THREADS = 32 * (SET_SENTINEL0 + UNPACK_SETS);
static_assert(A_COL0 + ASLOTS * A_COLS <= TMEM_COLS, "TMEM budget");
static_assert(X_BYTES % 1024 == 0, "swizzle atoms of the token stages stay aligned");
static_assert(EPI_WARP0 % 4 == 0, "epilogue warp q reads TMEM lanes 32 q");
static_assert(ASLOTS % UNPACK_SETS == 0, "each set keeps to its own A slots");

struct Barriers {
  uint64_t full[STAGES];     // token tile + packed weights of a stage landed
  uint64_t empty[STAGES];    // the stage's MMAs are done (its shared memory is free)
  uint64_t a_full[ASLOTS];   // a stage's weights are in this TMEM slot
  uint64_t a_empty[ASLOTS];  // the MMAs that read this slot are done
  uint64_t tmem_full[2];
  uint64_t tmem_empty[2];
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
};

struct Shared {
  int rowsum[2][MAX_BNT];
  float f[2][MAX_BNT];  // scale_t * gamma
  Barriers bar;
};

constexpr int SMEM_BYTES = 1024 /* alignment slack */ + STAGES * (X_BYTES + WP_BYTES) +
                           static_cast<int>(sizeof(Shared));

// Token tile for M tokens: as even as the tile count allows, a multiple of 16, <= 192.
__host__ __device__ constexpr int token_tile(int M) {
  const int tiles = (M + MAX_BNT - 1) / MAX_BNT;
  const int per = (M + tiles - 1) / tiles;
  return (per + 15) / 16 * 16;
}
}  // namespace pf

__device__ __forceinline__ void epi4_bar_sync() {  // the 4 epilogue warps only
  asm volatile("bar.sync 3, 128;" ::: "memory");
}
// The per-stage handoff of the sentinel and MMA warps (named barrier 4): returns the OR of
// both warps' flags.
__device__ __forceinline__ bool stage_bar_or(bool v) { return bar_or<4, 64>(v); }
// The per-stage handoff of unpack set `set` and its sentinel (named barriers 5 and 6, the
// set's four warps and the sentinel warp).
__device__ __forceinline__ bool set_bar_or(int set, bool v) {
  return set == 0 ? bar_or<5, 160>(v) : bar_or<6, 160>(v);
}

// OM: 0 fp32 out, 1 bf16 out, 2 int32 out (acc only). bnt = token tile (multiple of 16,
// <= MAX_BNT; the token tensor map's box has bnt rows). amax_out (layer chains, may be
// null): receives the absmax of each token's outputs.
template <int OM>
__global__ void __launch_bounds__(pf::THREADS, 1) gemm_prefill_kernel(
    const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
    const int* __restrict__ rowsum, const float* __restrict__ scale,
    const float* __restrict__ gamma_ptr, void* __restrict__ y, int M, int N, int K, int bnt,
    unsigned long long limit_ns, float* __restrict__ amax_out) {
  using namespace pf;
  allow_dependent_launch();  // the next kernel may set up (it waits before using y)
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  unsigned char* sX = smem;                          // STAGES x [bnt][128] swizzled
  unsigned char* sW = sX + STAGES * X_BYTES;         // STAGES x [128][32] packed
  Shared* sh = reinterpret_cast<Shared*>(sW + STAGES * WP_BYTES);
  Barriers* bar = &sh->bar;
  volatile int* abort_flag = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t_tiles = (M + bnt - 1) / bnt;
  const int w_tiles = (N + BW - 1) / BW;
  const int num_tiles = t_tiles * w_tiles;
  const int KB = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&bar->full[s], 1);
      mbar_init(&bar->empty[s], 1);
    }
    for (int a = 0; a < ASLOTS; ++a) {
      mbar_init(&bar->a_full[a], 4);
      mbar_init(&bar->a_empty[a], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&bar->tmem_full[b], 1);
      mbar_init(&bar->tmem_empty[b], 4);
    }
    mbar_init(&bar->drain, 1);
    bar->abort = 0;
    fence_mbar_init();
  }
  if (warp == MMA_WARP) {
    tmem_alloc(&bar->tmem_base, TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bar->tmem_base;
  grid_dependency_wait();  // operands from the kernel before (no-op without the attribute)

  if (warp == TMA_WARP) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      prefetch_tmap(&map_x);
      prefetch_tmap(&map_w);
      const uint32_t bytes = static_cast<uint32_t>(bnt * BK + WP_BYTES);
      int s = 0;
      uint32_t ph = 0;
      long long issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int t0 = (tile % t_tiles) * bnt;
        const int n0 = (tile / t_tiles) * BW;
        for (int kb = 0; kb < KB; ++kb) {
          if (!tc_wait(&bar->empty[s], ph ^ 1u, limit_ns, abort_flag)) { ok = false; break; }
          mbar_arrive_expect_tx(&bar->full[s], bytes);
          tma_load_2d(sX + s * X_BYTES, &map_x, kb * BK, t0, &bar->full[s]);
          tma_load_2d(sW + s * WP_BYTES, &map_w, kb * (BK / 4), n0, &bar->full[s]);
          ++issued;
          if (++s == STAGES) { s = 0; ph ^= 1u; }
        }
      }
      if (!ok) {  // wait (bounded) for the copies still in flight
        const long long last = issued - 1;
        for (long long i = last; i >= 0 && i > last - STAGES; --i)
          mbar_wait(&bar->full[i % STAGES], static_cast<uint32_t>((i / STAGES) & 1),
                    100000000ull);
      }
    }
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_i8(BW, bnt);
    const uint64_t x_desc0 = smem_desc_k128(smem_u32(sX));
    int s = 0, a = 0, ab = 0;
    uint32_t sph = 0, abph = 0;
    bool ok = true, issued_any = false;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      bool got = true;
      if (lane == 0) got = tc_wait(&bar->tmem_empty[ab], abph ^ 1u, limit_ns, abort_flag);
      got = __shfl_sync(0xffffffffu, got, 0);
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + static_cast<uint32_t>(ab * MAX_BNT);
      for (int kb = 0; kb < KB; ++kb) {
        // The sentinel has seen a_full of slot a, which implies the stage's TMA data landed
        // (the unpack waited for it). A failed accumulator wait leaves at the first handoff.
        if (stage_bar_or(!got)) { ok = false; break; }
        tc_fence_after();
        const uint32_t a_tmem = tmem_base + static_cast<uint32_t>(A_COL0 + a * A_COLS);
        const uint64_t b_desc = x_desc0 + static_cast<uint64_t>(s * (X_BYTES >> 4));
#pragma unroll
        for (int kk = 0; kk < BK / MMA_K; ++kk)
          mma_i8_ts_elect(d_tmem, a_tmem + static_cast<uint32_t>(kk * (MMA_K / 4)),
                          b_desc + static_cast<uint64_t>(kk * (MMA_K >> 4)), idesc,
                          (kb | kk) != 0 ? 1u : 0u);
        issued_any = true;
        mma_commit_elect(&bar->empty[s]);
        mma_commit_elect(&bar->a_empty[a]);
        if (++s == STAGES) { s = 0; sph ^= 1u; }
        if (++a == ASLOTS) a = 0;
      }
      if (!ok) break;
      mma_commit_elect(&bar->tmem_full[ab]);
      if (++ab == 2) { ab = 0; abph ^= 1u; }
    }
    (void)sph;
    if (!ok && issued_any) {
      mma_commit_elect(&bar->drain);  // completes once every MMA issued above has finished
      if (lane == 0) mbar_wait(&bar->drain, 0u, 100000000ull);
      __syncwarp();
    }
  } else if (warp == SENTINEL_WARP) {
    // ------------------------------------------------------------------ sentinel
    int a = 0;
    uint32_t aph = 0;
    bool stop = false;
    for (int tile = blockIdx.x; tile < num_tiles && !stop; tile += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb) {
        bool got = true;
        if (lane == 0) got = tc_wait(&bar->a_full[a], aph, limit_ns, abort_flag);
        if (stage_bar_or(!__shfl_sync(0xffffffffu, got, 0))) { stop = true; break; }
        if (++a == ASLOTS) { a = 0; aph ^= 1u; }
      }
    }
  } else if (warp >= SET_SENTINEL0) {
    // ------------------------------------------------------------------ set sentinels
    const int set = warp - SET_SENTINEL0;
    long long g = 0;
    bool stop = false;
    for (int tile = blockIdx.x; tile < num_tiles && !stop; tile += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb, ++g) {
        if (static_cast<int>(g % UNPACK_SETS) != set) continue;
        bool got = true;
        if (lane == 0)
          got = tc_wait(&bar->full[g % STAGES], static_cast<uint32_t>((g / STAGES) & 1),
                        limit_ns, abort_flag);
        else if (lane == 1)
          got = tc_wait(&bar->a_empty[g % ASLOTS], static_cast<uint32_t>(((g / ASLOTS) & 1) ^ 1),
                        limit_ns, abort_flag);
        if (set_bar_or(set, !__all_sync(0xffffffffu, got))) { stop = true; break; }
      }
    }
  } else if (warp < UNPACK_WARPS) {
    // ------------------------------------------------------------------ unpack warps
    const int set = warp >> 2;   // stages g with g % UNPACK_SETS == set
    const int wq = warp & 3;     // TMEM lane quarter
    const int r = wq * 32 + lane;  // weight row of the tile = TMEM lane
    const uint32_t a_lane = tmem_base + (static_cast<uint32_t>(wq * 32) << 16) + A_COL0;
    // Rows are 32 bytes apart: lanes 0-3 of each quarter-warp read their first 16-byte
    // half first and lanes 4-7 their second, so the 8 rows of a 128-byte wavefront fall
    // in 8 distinct bank groups.
    const int h0 = (lane >> 2) & 1;
    long long g = 0;  // stages of this CTA so far
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
      for (int kb = 0; kb < KB; ++kb, ++g) {
        if (static_cast<int>(g % UNPACK_SETS) != set) continue;
        const int s = static_cast<int>(g % STAGES);
        const int a = static_cast<int>(g % ASLOTS);
        // the set's sentinel has seen the stage land and the slot freed
        if (set_bar_or(set, false)) { ok = false; break; }
        tc_fence_after();
        const uint4* src = reinterpret_cast<const uint4*>(sW + s * WP_BYTES + r * 32);
        const uint4 first = src[h0], second = src[h0 ^ 1];
        const uint4 halves[2] = {h0 ? second : first, h0 ? first : second};
        uint32_t codes[32];  // the row's 128 codes of this K block, 4 per register
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint4 p = halves[h];
          const uint32_t words[4] = {p.x, p.y, p.z, p.w};
#pragma unroll
          for (int mq = 0; mq < 4; ++mq) {
            const int c = 16 * h + 4 * mq;  // column of trits 4c .. 4c + 15
            codes[c + 0] = words[mq] & 0x03030303u;
            codes[c + 1] = (words[mq] >> 2) & 0x03030303u;
            codes[c + 2] = (words[mq] >> 4) & 0x03030303u;
            codes[c + 3] = (words[mq] >> 6) & 0x03030303u;
          }
        }
        tmem_st_x32(a_lane + static_cast<uint32_t>(a * A_COLS), codes);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&bar->a_full[a]);
      }
    }
  } else {
    // ------------------------------------------------------------------ epilogue
    const int q = warp - EPI_WARP0;  // TMEM lanes 32q .. 32q + 31
    const int et = threadIdx.x - 32 * EPI_WARP0;  // 0..127
    const float gamma = (OM == 2) ? 0.0f : *gamma_ptr;
    int ab = 0;
    uint32_t aph = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
      const int t0 = (tile % t_tiles) * bnt;
      const int n0 = (tile / t_tiles) * BW;
      // the tile's per-token factors (the buffer of this accumulator was last read two
      // tiles ago, before the barrier of the previous tile)
      for (int j = et; j < bnt; j += 128) {
        const int t = t0 + j;
        sh->rowsum[ab][j] = (t < M) ? rowsum[t] : 0;
        sh->f[ab][j] = (OM != 2 && t < M) ? __fmul_rn(scale[t], gamma) : 0.0f;
      }
      epi4_bar_sync();
      const bool got = tc_wait(&bar->tmem_full[ab], aph, limit_ns, abort_flag);
      if (!__all_sync(0xffffffffu, got)) break;
      tc_fence_after();
      const int n = n0 + q * 32 + lane;
      const bool nvalid = n < N;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) +
                             static_cast<uint32_t>(ab * MAX_BNT);
      for (int c0 = 0; c0 < bnt; c0 += 32) {
        uint32_t v[32];
        if (c0 + 32 <= bnt) {
          tmem_ld_x32(taddr + c0, v);
        } else {  // bnt % 32 == 16: the last 16 columns
          uint32_t w16[16];
          tmem_ld_x16(taddr + c0, w16);
#pragma unroll
          for (int j = 0; j < 16; ++j) { v[j] = w16[j]; v[j + 16] = 0u; }
        }
        tmem_ld_wait();
        // Per half (bnt is a multiple of 16, so a 16-column half is all in or all out): the
        // factors, then the values, the stores and the chain's absmax, each in its own loop.
        // A branch inside the value loop would make every value's convert-multiply-convert
        // chain wait for the one before.
#pragma unroll
        for (int hh = 0; hh < 32; hh += 16) {  // halves of 16 columns (fewer live registers)
          if (c0 + hh >= bnt) break;  // the same for the whole warp
          int rs[16];
          float fs[16];
#pragma unroll
          for (int j = 0; j < 16; j += 4) {
            const int4 r4 = *reinterpret_cast<const int4*>(&sh->rowsum[ab][c0 + hh + j]);
            const float4 f4 = *reinterpret_cast<const float4*>(&sh->f[ab][c0 + hh + j]);
            rs[j] = r4.x; rs[j + 1] = r4.y; rs[j + 2] = r4.z; rs[j + 3] = r4.w;
            fs[j] = f4.x; fs[j + 1] = f4.y; fs[j + 2] = f4.z; fs[j + 3] = f4.w;
          }
          uint32_t bits[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int a = static_cast<int>(v[hh + j]) - rs[j];
            if (OM == 2) {
              bits[j] = static_cast<uint32_t>(a);
            } else {
              const float val = __fmul_rn(__int2float_rn(a), fs[j]);
              bits[j] = (OM == 0) ? __float_as_uint(val)
                                  : static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(val)));
            }
          }
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = t0 + c0 + hh + j;
            if (t < M && nvalid) {
              const long long o = static_cast<long long>(t) * N + n;
              if (OM == 1) static_cast<uint16_t*>(y)[o] = static_cast<uint16_t>(bits[j]);
              else static_cast<uint32_t*>(y)[o] = bits[j];
            }
          }
          if (OM != 2 && amax_out != nullptr) {
            const unsigned m = warp_amax16<OM>(bits, nvalid);
            const int t = t0 + c0 + hh + lane;
            if (lane < 16 && t < M && m != 0u) red_max_u32(amax_out + t, m);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&bar->tmem_empty[ab]);
      if (++ab == 2) { ab = 0; aph ^= 1u; }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == MMA_WARP) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace bl
