// gemm_tc_kernel: C = A B in bf16 with fp32 accumulation on the sm_100a
// tensor cores -- the projections of the full multi-head layer (Eq. 5:
// [Q | K | V] = X [W_Q | W_K | W_V]; Eq. 11: Y = [A_1 ... A_H] W_O).
//
// All three matrices are row-major: A [M, K] (its rows are the MMA's M index,
// K contiguous: a K-major operand), B [K, N] (N contiguous: an MN-major
// operand, like V in the attention kernel), C [M, N].  Output tiles of
// 128 x 256 are distributed over a persistent grid (one CTA per SM); K runs in
// blocks of 64 through a 4-stage ring of TMA loads (128-byte swizzle).  The
// fp32 accumulator of a tile lives in tensor memory, double buffered (2 x 256
// columns), so the epilogue of one tile overlaps the products of the next.
//
// Warps: 0 loads (TMA), 1 issues the MMAs and owns TMEM, 2-5 are the
// epilogue (thread = tile row = TMEM lane; warp w reads lanes 32 (w % 4) ..).
// Tails: TMA reads zeros past M, N and K, and the epilogue stores only rows
// < M and 8-column groups < N (N % 8 == 0).
#pragma once

#include "sm100_common.cuh"

namespace infini {
namespace tc {

constexpr int kGemmBM = 128, kGemmBN = 256, kGemmBK = 64;
constexpr int kGemmStages = 4;
constexpr int kGemmGroupM = 8;  // tile raster: groups of 8 row blocks sweep the column blocks together
constexpr uint32_t kGemmA = 16384;  // 128 rows x 64 bf16
constexpr uint32_t kGemmBBox = 8192;  // 64 K rows x 64 bf16 columns
constexpr uint32_t kGemmStage = kGemmA + 4 * kGemmBBox;  // 48 KB
constexpr uint32_t kGemmBar = kGemmStages * kGemmStage;
enum : int { G_FULL0 = 0, G_EMPTY0 = kGemmStages, G_ACCF0 = 2 * kGemmStages, G_ACCE0 = 2 * kGemmStages + 2,
             G_DONE = 2 * kGemmStages + 4, G_COUNT = 2 * kGemmStages + 5 };
constexpr uint32_t kGemmSlot = kGemmBar + 8 * G_COUNT;
constexpr uint32_t kGemmSmem = kGemmSlot + 16 + 1024;  // + alignment slack
constexpr int kGemmThreads = 192;
static_assert(kGemmSmem <= 232448, "GEMM kernel exceeds 227 KB of shared memory");

struct GemmArgs {
  __nv_bfloat16* C;
  long long ldc;  // elements
  int M, N, K;
  int tiles_m, tiles_n;
};

__global__ void __launch_bounds__(kGemmThreads, 1)
    gemm_tc_kernel(const __grid_constant__ CUtensorMap tm_a, const __grid_constant__ CUtensorMap tm_b,
                   const GemmArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto bar = [&](int i) { return base + kGemmBar + 8u * (uint32_t)i; };
  auto sA = [&](int s) { return base + (uint32_t)s * kGemmStage; };
  auto sB = [&](int s) { return base + (uint32_t)s * kGemmStage + kGemmA; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kGemmSlot);
  const int tiles = g.tiles_m * g.tiles_n;
  const int kblocks = (g.K + kGemmBK - 1) / kGemmBK;
  // tile t of the grouped raster -> (row block, column block)
  auto tile_mn = [&](int t, int& tm, int& tn) {
    const int per_group = kGemmGroupM * g.tiles_n;
    const int grp = t / per_group;
    const int gm = min(kGemmGroupM, g.tiles_m - grp * kGemmGroupM);
    const int r = t - grp * per_group;
    tm = grp * kGemmGroupM + r % gm;
    tn = r / gm;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < kGemmStages; ++i) {
      mbar_init(bar(G_FULL0 + i), 1);
      mbar_init(bar(G_EMPTY0 + i), 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(G_ACCF0 + i), 1);
      mbar_init(bar(G_ACCE0 + i), 128);
    }
    mbar_init(bar(G_DONE), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      prefetch_tensormap(&tm_a);
      prefetch_tensormap(&tm_b);
      uint32_t it = 0;  // k-blocks issued over all tiles of this CTA
      uint32_t inflight = 0;
      for (int t = blockIdx.x; t < tiles && !device_aborted(); t += gridDim.x) {
        int tm, tn;
        tile_mn(t, tm, tn);
        for (int kb = 0; kb < kblocks; ++kb, ++it) {
          const int s = (int)(it % kGemmStages);
          if (!mbar_wait(bar(G_EMPTY0 + s), ((it / kGemmStages) & 1u) ^ 1u)) goto done;
          mbar_expect_tx(bar(G_FULL0 + s), kGemmStage);
          tma_load_2d(sA(s), &tm_a, bar(G_FULL0 + s), kb * kGemmBK, tm * kGemmBM);
#pragma unroll
          for (int b = 0; b < 4; ++b)
            tma_load_2d(sB(s) + (uint32_t)b * kGemmBBox, &tm_b, bar(G_FULL0 + s), tn * kGemmBN + 64 * b, kb * kGemmBK);
          inflight = min(inflight + 1u, (uint32_t)kGemmStages);
        }
      }
    done:
      if (device_aborted()) {
        // a wait gave up: let the copies still in flight land before the CTA exits
        for (uint32_t i = 1; i <= inflight; ++i) {
          const uint32_t j = it - i;
          mbar_drain(bar(G_FULL0 + (int)(j % kGemmStages)), (j / kGemmStages) & 1u);
        }
      }
    }
  } else if (warp == 1) {
    // -------------------------------------------------------------- MMA issuer
    // the whole warp runs the loop (uniform control flow), one elected lane issues
    constexpr uint32_t idesc = idesc_bf16(kGemmBM, kGemmBN, 0, 1);
    uint32_t it = 0, local = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
      const uint32_t buf = local & 1u, use = local >> 1;
      if (!mbar_wait(bar(G_ACCE0 + (int)buf), (use & 1u) ^ 1u)) break;
      tc_fence_after();
      const uint32_t acc = tmem + buf * (uint32_t)kGemmBN;
      bool ok = true;
      for (int kb = 0; kb < kblocks; ++kb, ++it) {
        const int s = (int)(it % kGemmStages);
        if (!mbar_wait(bar(G_FULL0 + s), (it / kGemmStages) & 1u)) {
          ok = false;
          break;
        }
        tc_fence_after();
        // A: K-major, 16-element K steps 32 bytes apart inside the 128-byte
        // rows; B: MN-major, four 64-column blocks kGemmBBox apart, K steps of
        // 16 rows (2 KB)
        const uint64_t da = kmajor_base(sA(s)), db = smem_desc_sw128(sB(s), kGemmBBox, 1024u);
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < kGemmBK / 16; ++kk)
            mma_ss(acc, da + kmajor_step(kk), db + mnmajor_step(kk), idesc, (kb > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(G_EMPTY0 + s));
        }
        __syncwarp();
      }
      if (!ok) break;
      if (elect_one()) mma_commit(bar(G_ACCF0 + (int)buf));
      __syncwarp();
    }
    // every product issued has completed before TMEM is released
    if (elect_one()) {
      mma_commit(bar(G_DONE));
      mbar_drain(bar(G_DONE), 0);
    }
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- epilogue
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const uint32_t lrow = (uint32_t)(quarter * 32) << 16;
    uint32_t local = 0;
    for (int t = blockIdx.x; t < tiles; t += gridDim.x, ++local) {
      const uint32_t buf = local & 1u, use = local >> 1;
      if (!mbar_wait(bar(G_ACCF0 + (int)buf), use & 1u)) break;
      tc_fence_after();
      int tm, tn;
      tile_mn(t, tm, tn);
      const int grow = tm * kGemmBM + row;
      const int col0 = tn * kGemmBN;
      __nv_bfloat16* crow = g.C + (long long)grow * g.ldc + col0;
      const uint32_t tacc = tmem + lrow + buf * (uint32_t)kGemmBN;
#pragma unroll 1
      for (int c = 0; c < kGemmBN / 32; c += 2) {
        uint32_t r0[32], r1[32];
        tmem_ld32(tacc + 32u * (uint32_t)c, r0);
        tmem_ld32(tacc + 32u * (uint32_t)(c + 1), r1);
        tmem_ld_wait();
        if (c + 2 == kGemmBN / 32) {
          // the last columns of this buffer are in registers: the MMA warp may reuse it
          tc_fence_before();
          mbar_arrive(bar(G_ACCE0 + (int)buf));
        }
        if (grow < g.M) {
#pragma unroll
          for (int h = 0; h < 2; ++h) {
            const uint32_t* r = h ? r1 : r0;
            const int cb = col0 + 32 * (c + h);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              if (cb + 8 * e + 8 <= g.N) {
                const uint4 v = make_uint4(pack_bf16x2(__uint_as_float(r[8 * e]), __uint_as_float(r[8 * e + 1])),
                                           pack_bf16x2(__uint_as_float(r[8 * e + 2]), __uint_as_float(r[8 * e + 3])),
                                           pack_bf16x2(__uint_as_float(r[8 * e + 4]), __uint_as_float(r[8 * e + 5])),
                                           pack_bf16x2(__uint_as_float(r[8 * e + 6]), __uint_as_float(r[8 * e + 7])));
                *reinterpret_cast<uint4*>(crow + 32 * (c + h) + 8 * e) = v;
              }
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace infini
