// Skinny BitLinear (up to 256 tokens, above the GEMV range) on the tcgen05 tensor cores,
// operands swapped:
//   D[n][t] = sum_k u[n][k] * xq[t][k]     (A = 128 unpacked weight rows, B = the M tokens)
// so the weights fill the MMA's 128-row slot and the few tokens its N slot (16..256), and
// every weight tile is unpacked once no matter how many tokens there are. This is the
// addition-only integer product of BitNet b1.58 (dmarx anthology record LIT-380, Key takeaways
// bullet 4) in the same u = c + 1 form as the other kernels (acc = D - rowsum_t).
//
// Data path:
//   W  packed weight super-tiles (128 rows x 128 bytes = 512 K, four K blocks) arrive by
//      TMA with the 128-byte swizzle, so every row is one 128-byte burst;
//   A  thread r of warps 0-3 unpacks its row's 128 trits of a K block in registers and
//      writes them with one tcgen05.st into TMEM lane r (4 int8 per column): the MMA takes
//      its A operand straight from tensor memory, so unpacked weights never touch shared
//      memory (no shared-memory write/read traffic and no proxy fence for them);
//   X  int8 token tiles (bnt rows x 128 per K block, 128-byte swizzle), one ring slot per
//      group of K blocks.
//
// Work unit = (128-row weight tile, K range of whole super-tiles). When there are too few
// weight tiles to fill the GPU, K is split across CTAs: each split adds its exact int32
// partial tile into a zeroed int32 buffer with fire-and-forget atomic adds, and the last
// split to finish (per-tile arrival counter) rescales the sums and writes y. Integer
// adds, so the split does not change a single bit.
//
// The loop moves in groups of KG = 2 K blocks. Per group the four unpack warps write
// their rows' codes to TMEM and meet the MMA and sentinel warps at a hardware named
// barrier (bar.red of 192 threads, far cheaper than an mbarrier arrive/poll round trip;
// the reduction also makes every abort decision uniform, so no participant can be left
// waiting). The MMA warp then issues the group's 8 MMAs and one commit while the unpack
// warps go on to the next group; the commit's barrier (done ring) frees the A slot and
// the token tile.
//
// At small M these per-group handoffs, not bandwidth, set the pace. Measured on B200 with
// clock64 stamps (70B up projection, M = 16): issuing the 8 MMAs and the commit takes
// about 400 cycles, unpacking a group about 430 (plus 50 for the stores to land), and
// every mbarrier test 200 to 450 cycles even for a phase completed long before. So
// neither the MMA warp nor the unpack warps test anything: a sentinel warp joins every
// handoff, and each handoff also certifies what the next steps need. Before the handoff
// of group g the sentinel has seen, with three lanes testing at once,
//   lane 0: group g's token tile land (the MMAs of g read it),
//   lane 1: group g + 1's W super-tile land, when g + 1 starts one,
//   lane 2: the MMAs of group g + 1 - SU complete (the last readers of the A slot that
//           group g + 1 is unpacked into),
// while the unpack warps work on group g.
//
// 7 warps: warps 0-3 unpack (thread t owns weight row t, TMEM lane t) and run the
// epilogue at the end; warp 4 issues the TMA loads; warp 5 owns the TMEM allocation and
// issues the MMAs (whole-warp loop, one elected lane issues, operands precomputed);
// warp 6 is the sentinel.
#pragma once

#include <cstddef>

#include "common.cuh"

namespace bl {

namespace sk {
constexpr int BW = 128;                 // weight rows per tile (MMA M)
constexpr int BK = 128;                 // K per K block (one 128-byte swizzle row of int8)
constexpr int KPS = 4;                  // K blocks per packed super-tile
constexpr int KG = 2;                   // K blocks per group (one synchronisation round)
constexpr int MMA_K = 32;
constexpr int WP_BYTES = BW * BK * KPS / 4;  // 16 KB packed super-tile
constexpr int A_COLS = BK / 4;               // TMEM columns of one unpacked K block
constexpr int G_COLS = KG * A_COLS;          // TMEM columns of one unpacked group
constexpr int MAX_SU = 8;                    // unpacked groups in flight (TMEM slots), at most
constexpr int THREADS = 224;
constexpr int MAX_SW = 4, MAX_SX = 16;
constexpr int MAX_M = 256;  // tokens, at most

static_assert(KPS % KG == 0, "groups tile a super-tile");
// Ring of per-group completion barriers. Group g's MMAs arrive on done[g % SD]; the MMA
// warp waits for group g - SU before group g may be unpacked into A slot g % SU, the
// producer for group g - SX before reusing token slot g % SX. SD >= SU and SD >= SX make a
// waited-for phase unable to be overtaken by the next phase of the same barrier (that one
// needs the waiter's own later work first), and every waiter waits on every index in
// order.
constexpr int SD = 16;
static_assert(SD >= MAX_SU && SD >= MAX_SX && (SD & (SD - 1)) == 0, "done ring");

struct Barriers {
  uint64_t w_full[MAX_SW], w_empty[MAX_SW];
  uint64_t x_full[MAX_SX];
  uint64_t done[SD];
  uint64_t acc_full;
  uint64_t drain;
  uint32_t tmem_base;
  int abort;
  int last;
  int rowsum[MAX_M];  // per token, staged once for the epilogue
  float f[MAX_M];     // per token s_t * gamma
  unsigned tmax[MAX_M];  // per token, this CTA's largest |y| (bits), for a chain's next layer
};

// The mbarriers above, w_full through drain, are consecutive 8-byte words.
constexpr int kNumMbar = 2 * MAX_SW + MAX_SX + SD + 2;
static_assert(offsetof(Barriers, drain) - offsetof(Barriers, w_full) == (kNumMbar - 1) * 8,
              "mbarriers are contiguous");

struct Plan {
  int sw, sx;
};

// One token tile of a K block: bnt rows x 128 bytes; a group holds KG of them.
__host__ __device__ constexpr int x_tile_bytes(int bnt) { return bnt * BK; }
__host__ __device__ constexpr int x_group_bytes(int bnt) { return KG * x_tile_bytes(bnt); }
// Shared memory per CTA: small token tiles keep two CTAs per SM, large ones use one.
__host__ __device__ constexpr int smem_budget(int bnt) {
  return bnt <= 64 ? 110 * 1024 : 200 * 1024;
}
__host__ __device__ constexpr Plan plan_for(int bnt) {
  const int sw = bnt <= 64 ? 4 : 2;
  const int room = smem_budget(bnt) - 1024 - static_cast<int>(sizeof(Barriers)) - sw * WP_BYTES;
  const int sx = room / x_group_bytes(bnt);
  return Plan{sw, sx > MAX_SX ? MAX_SX : sx};
}
__host__ __device__ constexpr int smem_bytes(int bnt) {
  return 1024 + plan_for(bnt).sw * WP_BYTES + plan_for(bnt).sx * x_group_bytes(bnt) +
         static_cast<int>(sizeof(Barriers));
}
// Columns of the accumulator (bnt rounded up to a power of two, at least 32).
__host__ __device__ constexpr uint32_t acc_cols(int bnt) {
  return bnt <= 32 ? 32u : bnt <= 64 ? 64u : bnt <= 128 ? 128u : 256u;
}
// TMEM allocation: 256 columns for small token tiles (two CTAs per SM), else 512.
__host__ __device__ constexpr uint32_t tmem_cols(int bnt) { return bnt <= 64 ? 256u : 512u; }
// Unpacked A slots in flight: the rest of the allocation after the accumulator.
__host__ __device__ constexpr int n_slots(int bnt) {
  return (static_cast<int>(tmem_cols(bnt)) - static_cast<int>(acc_cols(bnt))) / G_COLS > MAX_SU
             ? MAX_SU
             : (static_cast<int>(tmem_cols(bnt)) - static_cast<int>(acc_cols(bnt))) / G_COLS;
}
static_assert(n_slots(16) >= 3 && n_slots(64) >= 3 && n_slots(128) >= 4 && n_slots(256) >= 4,
              "TMEM slot budget");
}  // namespace sk

__device__ __forceinline__ void tmem_ld_x16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// Each thread of the warp writes 32 consecutive 32-bit columns of its own TMEM lane.
__device__ __forceinline__ void tmem_st_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]),
      "r"(r[22]), "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]),
      "r"(r[29]), "r"(r[30]), "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}
// D[tmem] (+)= A[tmem] * B[smem]^T, int8 x int8 -> int32, one CTA; warp-collective like
// mma_i8_elect (one elected lane issues).
__device__ __forceinline__ void mma_i8_ts_elect(uint32_t d_tmem, uint32_t a_tmem,
                                                uint64_t b_desc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p, e;\n\t"
      "elect.sync _|e, 0xffffffff;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "@e tcgen05.mma.cta_group::1.kind::i8 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
      "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// 16 consecutive accumulator columns of this thread's TMEM lane.
__device__ __forceinline__ void ld_acc16(uint32_t taddr, uint32_t (&v)[16]) {
  tmem_ld_x16(taddr, v);
  tmem_ld_wait();
}

// Fire-and-forget atomic add (the result is not returned, so the issuer does not wait).
__device__ __forceinline__ void red_add_s32(int* p, int v) {
  asm volatile("red.relaxed.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

__device__ __forceinline__ void epi_bar_sync() {  // the 4 unpack/epilogue warps only
  asm volatile("bar.sync 1, 128;" ::: "memory");
}
// Named barriers that also return the OR of every participant's flag, so that all of them
// take the same branch afterwards: id 1 = the 4 unpack/epilogue warps, id 2 = those, the
// MMA warp and the sentinel warp (the per-group handoff).
template <int ID, int COUNT>
__device__ __forceinline__ bool bar_or(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\t"
      "selp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(ID), "n"(COUNT)
      : "memory");
  return r != 0;
}
__device__ __forceinline__ bool epi_bar_or(bool v) { return bar_or<1, 128>(v); }
__device__ __forceinline__ bool group_bar_or(bool v) { return bar_or<2, 192>(v); }

// Atomic max of a non-negative float given by its bits (fire and forget).
__device__ __forceinline__ void red_max_u32(float* p, unsigned bits) {
  asm volatile("red.relaxed.gpu.global.max.u32 [%0], %1;" ::"l"(p), "r"(bits) : "memory");
}

// The warp's largest |y| of each of 16 tokens, for a layer chain's next quantization.
// bits[j] is this lane's stored value of token j (fp32 or bf16 bits), valid whether the
// lane's row exists. Sixteen reductions with no branch between them (a branch holding an
// atomic inside this loop made every reduction wait for the atomic before it, about 3.5 us
// per 3B-sized layer at 64 tokens); lane j < 16 returns the maximum of token j as float
// bits, the other lanes 0. The caller adds it with one atomic per lane.
template <int OM>
__device__ __forceinline__ unsigned warp_amax16(const uint32_t (&bits)[16], bool valid) {
  const int lane = threadIdx.x & 31;
  unsigned mine = 0u;
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const uint32_t mag = (OM == 0) ? (bits[j] & 0x7fffffffu) : ((bits[j] << 16) & 0x7fffffffu);
    const unsigned r = __reduce_max_sync(0xffffffffu, valid ? mag : 0u);
    mine = (lane == j) ? r : mine;
  }
  return mine;
}

// Rescales and writes the 16 values of tokens c0 .. c0 + 15 of this thread's weight row
// (a[j] = accumulator - rowsum) to y. With vec (rows of y 16-byte aligned: N a multiple of
// 16 / element size) they go through a 16 x 128 tile in shared memory and leave as 16-byte
// row pieces, else one store per value. Called by all 128 epilogue threads.
template <int OM>
__device__ __forceinline__ void epi_store_chunk(const int (&a)[16], const float (&fs)[16], int c0,
                                                int M, int N, int n0, bool nvalid, bool vec,
                                                unsigned char* stage, void* y, unsigned* tmax) {
  constexpr int ES = (OM == 1) ? 2 : 4;  // bytes per element of y
  const int nl = threadIdx.x;            // row within the tile
  const int n = n0 + nl;
  // Values first, stores next, the chain's absmax last: a branch inside the value loop
  // would make each value's convert-multiply-convert chain wait for the one before.
  uint32_t bits[16];
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    if (OM == 2) {
      bits[j] = static_cast<uint32_t>(a[j]);
    } else {
      const float val = __fmul_rn(__int2float_rn(a[j]), fs[j]);
      bits[j] = (OM == 0) ? __float_as_uint(val)
                          : static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(val)));
    }
  }
  if (vec) {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      if (ES == 2) reinterpret_cast<uint16_t*>(stage)[j * 128 + nl] = static_cast<uint16_t>(bits[j]);
      else reinterpret_cast<uint32_t*>(stage)[j * 128 + nl] = bits[j];
    }
  } else {
#pragma unroll
    for (int j = 0; j < 16; ++j) {
      const long long o = static_cast<long long>(c0 + j) * N + n;
      if (c0 + j < M && nvalid) {
        if (ES == 2) static_cast<uint16_t*>(y)[o] = static_cast<uint16_t>(bits[j]);
        else static_cast<uint32_t*>(y)[o] = bits[j];
      }
    }
  }
  if (OM != 2 && tmax != nullptr) {  // into the CTA's per-token maxima in shared memory
    const unsigned m = warp_amax16<OM>(bits, nvalid);
    const int lane = threadIdx.x & 31;
    if (lane < 16 && c0 + lane < M && m != 0u) atomicMax(tmax + c0 + lane, m);
  }
  if (vec) {
    epi_bar_sync();
    constexpr int PPR = 128 * ES / 16;  // 16-byte pieces per tile row
    for (int p = threadIdx.x; p < 16 * PPR; p += 128) {
      const int j = p / PPR, q = p % PPR;
      const int t = c0 + j, col = n0 + q * (16 / ES);
      if (t < M && col < N)
        *reinterpret_cast<uint4*>(static_cast<unsigned char*>(y) +
                                  (static_cast<long long>(t) * N + col) * ES) =
            *reinterpret_cast<const uint4*>(stage + (j * 128 + q * (16 / ES)) * ES);
    }
    epi_bar_sync();  // the tile is rewritten by the next chunk
  }
}

// bnt = token tile (multiple of 16, >= M). grid = n_tiles * splits; CTA u handles weight
// tile u / splits and the K blocks [split * kbps, min(KB, (split + 1) * kbps)), kbps a
// multiple of KPS. A trailing partial group reads K blocks past KB, which the tensor maps
// fill with zeros (their products vanish).
// Two CTAs per SM for token tiles up to 64 (the 110 KB shared-memory plan): the bound keeps
// the registers within 128 per thread, the most that 2 x 7 warps leave on one SM quarter.
template <int OM>
__global__ void __launch_bounds__(sk::THREADS, 2) gemm_skinny_kernel(
    const __grid_constant__ CUtensorMap map_x, const __grid_constant__ CUtensorMap map_w,
    const int* __restrict__ rowsum, const float* __restrict__ scale,
    const float* __restrict__ gamma_ptr, void* __restrict__ y, int* __restrict__ partial,
    unsigned int* __restrict__ counters, int M, int N, int K, int bnt, int splits,
    int kb_per_split, unsigned long long limit_ns, float* __restrict__ amax_out) {
  using namespace sk;
  allow_dependent_launch();  // the next kernel may set up (it waits before using y)
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = reinterpret_cast<unsigned char*>(
      (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
  const Plan pl = plan_for(bnt);
  const int XB = x_tile_bytes(bnt);
  const int XG = x_group_bytes(bnt);
  unsigned char* sWp = smem;                    // SW x [128][128 B] swizzled
  unsigned char* sX = sWp + pl.sw * WP_BYTES;   // SX x KG x [bnt][128] swizzled
  Barriers* bar = reinterpret_cast<Barriers*>(sX + pl.sx * XG);
  volatile int* abort_flag = &bar->abort;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tile = blockIdx.x / splits;
  const int split = blockIdx.x % splits;
  const int n0 = tile * BW;
  const int KB = (K + BK - 1) / BK;
  const int kb0 = split * kb_per_split;
  const int kb1 = min(KB, kb0 + kb_per_split);
  const int ng = (kb1 - kb0 + KG - 1) / KG;  // groups of this CTA
  const uint32_t ncols = tmem_cols(bnt);
  const uint32_t a_col0 = acc_cols(bnt);  // first TMEM column of the unpacked A slots
  const int SU = n_slots(bnt);

  // The first W super-tiles (at most the ring) do not depend on the kernel before, nor on
  // the TMEM allocation: the producer warp initialises the mbarriers (every one has one
  // arrival per phase; a lane each) and issues those loads before the block-wide sync.
  const int pre = min(pl.sw, (kb1 - kb0 + KPS - 1) / KPS);
  if (warp == 4) {
    if (lane == 0) {
      prefetch_tmap(&map_x);
      prefetch_tmap(&map_w);
    }
    uint64_t* first = &bar->w_full[0];
    for (int i = lane; i < kNumMbar; i += 32) mbar_init(first + i, 1);
    if (lane == 0) {
      bar->abort = 0;
      bar->last = 0;
    }
    fence_mbar_init();
    __syncwarp();
    if (lane == 0) {
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&bar->w_full[i], WP_BYTES);
        tma_load_2d(sWp + i * WP_BYTES, &map_w, (kb0 + i * KPS) * (BK / 4), n0, &bar->w_full[i]);
      }
    }
  }
  if (warp == 5) {
    tmem_alloc(&bar->tmem_base, ncols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bar->tmem_base;

  if (warp == 4) {
    // ------------------------------------------------------------------ TMA producer
    bool ok = true;  // lane 0's verdict on its loads
    if (lane == 0) {
      int sw = 0, sx = 0;
      uint32_t wph = 0;
      long long w_issued = pre, x_issued = 0;  // the first W loads went out before the sync
      grid_dependency_wait();  // the token tiles come from the kernel before
      for (int g = 0; g < ng; ++g) {
        const int kb = kb0 + g * KG;
        if (((g * KG) & (KPS - 1)) == 0) {
          if ((g * KG) / KPS >= pre) {  // not one of the super-tiles issued above
            if (!tc_wait(&bar->w_empty[sw], wph ^ 1u, limit_ns, abort_flag)) { ok = false; break; }
            mbar_arrive_expect_tx(&bar->w_full[sw], WP_BYTES);
            tma_load_2d(sWp + sw * WP_BYTES, &map_w, kb * (BK / 4), n0, &bar->w_full[sw]);
            ++w_issued;
          }
          if (++sw == pl.sw) { sw = 0; wph ^= 1u; }
        }
        if (g >= pl.sx) {  // token slot sx is free once group g - SX has been consumed
          const int i = g - pl.sx;
          if (!tc_wait(&bar->done[i & (SD - 1)], static_cast<uint32_t>((i / SD) & 1), limit_ns,
                       abort_flag)) { ok = false; break; }
        }
        mbar_arrive_expect_tx(&bar->x_full[sx], XG);
#pragma unroll
        for (int kq = 0; kq < KG; ++kq)
          tma_load_2d(sX + sx * XG + kq * XB, &map_x, (kb + kq) * BK, 0, &bar->x_full[sx]);
        ++x_issued;
        if (++sx == pl.sx) sx = 0;
      }
      if (!ok) {  // wait (bounded) for the copies still in flight
        for (long long i = w_issued - 1; i >= 0 && i > w_issued - 1 - pl.sw; --i)
          mbar_wait(&bar->w_full[i % pl.sw], static_cast<uint32_t>((i / pl.sw) & 1),
                    100000000ull);
        for (long long i = x_issued - 1; i >= 0 && i > x_issued - 1 - pl.sx; --i)
          mbar_wait(&bar->x_full[i % pl.sx], static_cast<uint32_t>((i / pl.sx) & 1),
                    100000000ull);
      }
    }
    // The last commits' arrivals land on done[] asynchronously: see each barrier's final
    // phase before the CTA can exit, so no arrival reaches a later CTA's shared memory.
    // One barrier per lane (a test costs a few hundred cycles; in series they would
    // outlast the epilogue).
    if (__shfl_sync(0xffffffffu, ok, 0)) {
      const int i = ng - 1 - lane;
      if (lane < SD && i >= 0)
        tc_wait(&bar->done[i & (SD - 1)], static_cast<uint32_t>((i / SD) & 1), limit_ns, abort_flag);
    }
    __syncwarp();
  } else if (warp == 5) {
    // ------------------------------------------------------------------ MMA issuer
    const uint32_t idesc = idesc_i8(BW, bnt);
    // built once; a stage or K step only moves the 14-bit start-address field
    const uint64_t x_desc0 = smem_desc_k128(smem_u32(sX));
    const uint32_t a_tmem0 = tmem_base + a_col0;
    int su = 0, sx = 0, sw = 0;
    bool stop = group_bar_or(false);  // the sentinel has seen group 0's W land
    int g = 0;
    for (; !stop && g < ng; ++g) {
      tc_fence_before();
      // group g's rows are in TMEM, its token tile has landed, its W reads are over
      if (group_bar_or(false)) break;
      tc_fence_after();
      const int q0 = (g * KG) & (KPS - 1);
      const bool last_of_tile = (q0 + KG == KPS) || (g == ng - 1);
      if (lane == 0 && last_of_tile) mbar_arrive(&bar->w_empty[sw]);  // every row has read it
      const uint32_t a_tmem = a_tmem0 + static_cast<uint32_t>(su * G_COLS);
      const uint64_t b_desc = x_desc0 + static_cast<uint64_t>(sx * (XG >> 4));
#pragma unroll
      for (int kq = 0; kq < KG; ++kq)
#pragma unroll
        for (int kk = 0; kk < BK / MMA_K; ++kk)
          mma_i8_ts_elect(tmem_base,
                          a_tmem + static_cast<uint32_t>(kq * A_COLS + kk * (MMA_K / 4)),
                          b_desc + static_cast<uint64_t>(kq * (XB >> 4) + kk * (MMA_K >> 4)),
                          idesc, (g | kq | kk) != 0 ? 1u : 0u);
      mma_commit_elect(&bar->done[g & (SD - 1)]);
      if (++su == SU) su = 0;
      if (++sx == pl.sx) sx = 0;
      if (last_of_tile && ++sw == pl.sw) sw = 0;
    }
    if (g == ng) {
      mma_commit_elect(&bar->acc_full);
    } else if (g > 0) {
      mma_commit_elect(&bar->drain);  // completes once every MMA issued above has finished
      if (lane == 0) mbar_wait(&bar->drain, 0u, 100000000ull);
      __syncwarp();
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------------ sentinel
    // Lane i tests barrier b_i for phase p_i (lanes without one pass); the warp's verdict
    // is the AND over its lanes.
    auto test_lanes = [&](uint64_t* b, uint32_t parity, bool active) -> bool {
      bool ok = true;
      if (active) ok = tc_wait(b, parity, limit_ns, abort_flag);
      return __all_sync(0xffffffffu, ok);
    };
    int sx = 0;
    uint32_t xph = 0;
    bool stop = group_bar_or(ng > 0 && !test_lanes(&bar->w_full[0], 0u, lane == 0));
    int g = 0;
    for (; !stop && g < ng; ++g) {
      const int gn = g + 1;
      uint64_t* b = &bar->x_full[sx];
      uint32_t parity = xph;
      bool active = (lane == 0);
      if (lane == 1 && gn < ng && ((gn * KG) & (KPS - 1)) == 0) {
        const int st = (gn * KG) / KPS;  // super-tiles before group gn's
        b = &bar->w_full[st % pl.sw];
        parity = static_cast<uint32_t>((st / pl.sw) & 1);
        active = true;
      }
      if (lane == 2 && gn < ng && gn >= SU) {
        const int i = gn - SU;
        b = &bar->done[i & (SD - 1)];
        parity = static_cast<uint32_t>((i / SD) & 1);
        active = true;
      }
      const bool ok = test_lanes(b, parity, active);
      if (group_bar_or(!ok)) break;  // the handoff of group g
      if (++sx == pl.sx) { sx = 0; xph ^= 1u; }
    }
  } else {
    // ------------------------------------------------------------------ warps 0-3
    // Passing the handoff before group g means group g's W super-tile has landed and its
    // A slot is free (tested by the sentinel before the previous handoff).
    const int r = threadIdx.x;  // weight row of the tile owned by this thread (0..127)
    const int rs = r & 7;       // its 128-byte swizzle phase
    const uint32_t a_lane = tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + a_col0;
    int sw = 0, su = 0;
    bool stop = group_bar_or(false);  // group 0 may start
    int g = 0;
    for (; !stop && g < ng; ++g) {
      const int q0 = (g * KG) & (KPS - 1);  // first K block of the group in its super-tile
      tc_fence_after();
      const unsigned char* src = sWp + sw * WP_BYTES + r * 128;
      // The group's packed chunks (logical 16-byte chunk 2q+h of the row = K block q,
      // words 4h .. 4h+3), all loaded before any is unpacked.
      uint4 pk[KG][2];
#pragma unroll
      for (int kq = 0; kq < KG; ++kq)
#pragma unroll
        for (int h = 0; h < 2; ++h)
          pk[kq][h] = *reinterpret_cast<const uint4*>(src + (((2 * (q0 + kq) + h) ^ rs) << 4));
#pragma unroll
      for (int kq = 0; kq < KG; ++kq) {
        uint32_t a[32];  // the row's 128 unpacked codes of K block q0 + kq, 4 per register
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const uint32_t words[4] = {pk[kq][h].x, pk[kq][h].y, pk[kq][h].z, pk[kq][h].w};
#pragma unroll
          for (int mq = 0; mq < 4; ++mq) {
            const uint32_t w = words[mq];
            const int c = 16 * h + 4 * mq;  // first column of this 16-trit group
            a[c + 0] = w & 0x03030303u;
            a[c + 1] = (w >> 2) & 0x03030303u;
            a[c + 2] = (w >> 4) & 0x03030303u;
            a[c + 3] = (w >> 6) & 0x03030303u;
          }
        }
        tmem_st_x32(a_lane + static_cast<uint32_t>(su * G_COLS + kq * A_COLS), a);
      }
      tmem_st_wait();
      tc_fence_before();
      if (group_bar_or(*abort_flag != 0)) break;  // hand group g to the MMA warp
      const bool last_of_tile = (q0 + KG == KPS) || (g == ng - 1);
      if (++su == SU) su = 0;
      if (last_of_tile && ++sw == pl.sw) sw = 0;
    }
    const bool ok = (g == ng);
    // ---------------------------------------------------------------- epilogue
    grid_dependency_wait();  // rowsum, scale and the zeroed split-K sums come from it
    const bool got = ok && tc_wait(&bar->acc_full, 0u, limit_ns, abort_flag);
    if (!epi_bar_or(!got)) {  // the same decision in all four warps
      // Per-token rowsum and s_t * gamma, staged once: read in the store loops below, global
      // loads would wait behind the stores (up to one memory round trip per token).
      {
        const float gamma = (OM == 2) ? 0.0f : *gamma_ptr;
        for (int t = threadIdx.x; t < M; t += 128) {
          bar->rowsum[t] = rowsum[t];
          bar->f[t] = (OM == 2) ? 0.0f : __fmul_rn(scale[t], gamma);
          bar->tmax[t] = 0u;
        }
      }
      epi_bar_sync();
      unsigned* tmax = (OM != 2 && amax_out != nullptr) ? bar->tmax : nullptr;
      tc_fence_after();
      const int n = n0 + warp * 32 + lane;  // this thread's TMEM lane = weight row
      const bool nvalid = n < N;
      // output tiles leave through the token ring, free once the last MMA is done
      const bool vec = (N % (OM == 1 ? 8 : 4)) == 0;
      unsigned char* stage = sX;
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(warp * 32) << 16);
      if (splits == 1) {
        for (int c0 = 0; c0 < bnt; c0 += 16) {
          uint32_t v[16];
          ld_acc16(taddr + c0, v);
          // the chunk's factors into registers first: a shared-memory read after a global
          // store would wait for it (the compiler cannot tell the two apart)
          int rs[16];
          float fs[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            rs[j] = bar->rowsum[c0 + j];
            fs[j] = bar->f[c0 + j];
          }
          int a[16];
#pragma unroll
          for (int j = 0; j < 16; ++j) a[j] = static_cast<int>(v[j]) - rs[j];
          epi_store_chunk<OM>(a, fs, c0, M, N, n0, nvalid, vec, stage, y, tmax);
        }
      } else {
        // exact int32 partial of this split, added into acc32[t][n] (zeroed by the host)
        for (int c0 = 0; c0 < bnt; c0 += 16) {
          uint32_t v[16];
          ld_acc16(taddr + c0, v);
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = c0 + j;
            if (t < M && nvalid)
              red_add_s32(partial + static_cast<long long>(t) * N + n, static_cast<int>(v[j]));
          }
        }
        __threadfence();
        epi_bar_sync();
        if (threadIdx.x == 0) {
          const unsigned int prev = atomicAdd(&counters[tile], 1u);
          bar->last = (prev == static_cast<unsigned int>(splits - 1)) ? 1 : 0;
        }
        epi_bar_sync();
        if (bar->last) {  // the same for the whole CTA
          __threadfence();
          for (int t0 = 0; t0 < M; t0 += 16) {
            int a[16];
            // all 16 loads first (a store between them would order each behind the last)
#pragma unroll
            for (int j = 0; j < 16; ++j)
              a[j] = (t0 + j < M && nvalid) ? __ldcg(partial + static_cast<long long>(t0 + j) * N + n)
                                            : 0;
            // leave the sums zeroed for the next launch that shares them (layer chains)
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (t0 + j < M && nvalid) __stcg(partial + static_cast<long long>(t0 + j) * N + n, 0);
            int rs[16];
            float fs[16];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              rs[j] = bar->rowsum[t0 + j];
              fs[j] = bar->f[t0 + j];
            }
#pragma unroll
            for (int j = 0; j < 16; ++j) a[j] -= rs[j];
            epi_store_chunk<OM>(a, fs, t0, M, N, n0, nvalid, vec, stage, y, tmax);
          }
          if (threadIdx.x == 0) counters[tile] = 0u;  // every split has arrived
        }
      }
      if (tmax != nullptr) {  // this CTA's per-token maxima into the chain's absmax
        epi_bar_sync();
        for (int t = threadIdx.x; t < M; t += 128)
          if (tmax[t] != 0u) red_max_u32(amax_out + t, tmax[t]);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, ncols);
  }
}

}  // namespace bl
