// mem_update_tc_kernel: the segment's share of sigma(K)^T U and
// sum_t sigma(K_t) for the linear (Eq. 8, U = V) or delta (Eq. 9,
// U = V - sigma(K) M_{s-1} / (sigma(K) z_{s-1})) rule, on the sm_100a tensor
// cores.
#pragma once

#include "sm100_common.cuh"

namespace infini {
namespace tc {

// ------------------------------------------------------------------------
// Memory update.  Grid: BH * nseg * G CTAs of 160 threads; CTA (bh, segment
// seg0 + sl, group grp) covers tokens [grp*cpb*128, min((grp+1)*cpb*128, n_s))
// of the segment in 128-token chunks.  Warp 0 lane 0 loads (TMA) and issues
// MMAs; warps 1-4 (thread = token row of the chunk = TMEM lane) apply sigma,
// split it into bf16 hi + lo parts and, for the delta rule, form
// U = V - R / den with R = sigma(K)_hi M_{s-1} from the tensor cores and
// den = sigma(K) . z_{s-1} in fp32, again split into hi + lo.  The products
//   dM += sK_hi^T U_hi + sK_lo^T U_hi (+ sK_hi^T U_lo)       (fp32 in TMEM)
//   dz += sK_hi^T 1 + sK_lo^T 1                            (N = 16 ones block)
// keep the update within ~2^-16 relative of fp32 arithmetic.
struct UpdArgs {
  const float* snapz;  // [BH][S][128]
  float* partial;      // [BH][nseg][G][128*128 + 128]
  int B, H, S, N;
  long long L;
  int seg0, nseg, G, cpb, delta;
};

constexpr uint32_t kU_K = 0;         // sigma(K) hi (in place over K)
constexpr uint32_t kU_KLO = 32768;   // sigma(K) lo
constexpr uint32_t kU_V = 65536;     // U hi (in place over V)
constexpr uint32_t kU_ULO = 98304;   // U lo
constexpr uint32_t kU_MT = 131072;   // M_{s-1}^T
constexpr uint32_t kU_ONES = 163840; // 4 KB of bf16 ones
constexpr uint32_t kU_Z = 167936;
constexpr uint32_t kU_BAR = kU_Z + 512;
constexpr uint32_t kU_TMEMSLOT = kU_BAR + 128;
constexpr uint32_t kUpdSmem = kU_TMEMSLOT + 16 + 1024;

enum : int { U_LD = 0, U_MT = 1, U_SK = 2, U_R = 3, U_U = 4, U_MMA = 5, U_COUNT = 6 };

__global__ void __launch_bounds__(160, 1)
    mem_update_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const __grid_constant__ CUtensorMap tm_mt, const UpdArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  int idx = blockIdx.x;
  const int grp = idx % a.G;
  idx /= a.G;
  const int sl = idx % a.nseg;
  const int bh = idx / a.nseg;
  const int s = a.seg0 + sl;
  const int b = bh / a.H, h = bh % a.H;
  const long long seg_start = (long long)s * a.N;
  const int n_s = (int)min((long long)a.N, a.L - seg_start);
  const int t_begin = grp * a.cpb * kTile;
  const int t_end = min(n_s, t_begin + a.cpb * kTile);
  float* part = a.partial + (((long long)bh * a.nseg + sl) * a.G + grp) * (long long)(128 * 128 + 128);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (t_begin >= t_end) {  // group past the end of a short segment: contributes nothing
    for (int e = threadIdx.x; e < 128 * 128 + 128; e += blockDim.x) part[e] = 0.f;
    return;
  }
  const int nchunks = (t_end - t_begin + kTile - 1) / kTile;
  const bool delta = a.delta != 0;

  auto bar = [&](int i) { return base + kU_BAR + 8u * (uint32_t)i; };
  float* zs = reinterpret_cast<float*>(gbase + kU_Z);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kU_TMEMSLOT);
  if (threadIdx.x == 0) {
    mbar_init(bar(U_LD), 1);
    mbar_init(bar(U_MT), 1);
    mbar_init(bar(U_SK), 128);
    mbar_init(bar(U_R), 1);
    mbar_init(bar(U_U), 128);
    mbar_init(bar(U_MMA), 1);
    fence_barrier_init();
  }
  {
    uint32_t* ones = reinterpret_cast<uint32_t*>(gbase + kU_ONES);
    for (int e = threadIdx.x; e < 1024; e += blockDim.x) ones[e] = 0x3f803f80u;  // bf16 1.0 pairs
  }
  if (warp >= 1) zs[threadIdx.x - 32] = delta ? a.snapz[((long long)bh * a.S + s) * 128 + (threadIdx.x - 32)] : 0.f;
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tR = tmem, tM = tmem + 128, tZ = tmem + 256;
  const uint32_t sKt = base + kU_K, sKlo = base + kU_KLO, sVt = base + kU_V, sUlo = base + kU_ULO,
                 sMt = base + kU_MT, sOnes = base + kU_ONES;

  if (warp == 0) {
    if (lane == 0) {
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      if (delta) {
        prefetch_tensormap(&tm_mt);
        const int row = (bh * a.S + s) * 128;
        mbar_expect_tx(bar(U_MT), kTileBytes);
        tma_load_2d(sMt, &tm_mt, bar(U_MT), 0, row);
        tma_load_2d(sMt + kBox, &tm_mt, bar(U_MT), 64, row);
      }
      constexpr uint32_t idesc_r = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_m = idesc_bf16(128, 128, 1, 1);
      constexpr uint32_t idesc_z = idesc_bf16(128, 16, 1, 0);
      for (int c = 0; c < nchunks; ++c) {
        if (c > 0) mbar_wait(bar(U_MMA), (c - 1) & 1);
        const int lt = (int)(seg_start + t_begin + (long long)c * kTile);
        mbar_expect_tx(bar(U_LD), 2 * kTileBytes);
        tma_load_4d(sKt, &tm_k, bar(U_LD), 0, lt, h, b);
        tma_load_4d(sKt + kBox, &tm_k, bar(U_LD), 64, lt, h, b);
        tma_load_4d(sVt, &tm_v, bar(U_LD), 0, lt, h, b);
        tma_load_4d(sVt + kBox, &tm_v, bar(U_LD), 64, lt, h, b);
        if (delta) {
          mbar_wait(bar(U_SK), c & 1);
          if (c == 0) mbar_wait(bar(U_MT), 0);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tR, kmajor_desc(sKt, kk), kmajor_desc(sMt, kk), idesc_r, kk > 0 ? 1u : 0u);
          mma_commit(bar(U_R));
        }
        mbar_wait(bar(U_U), c & 1);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
          const uint64_t aH = mnmajor_desc(sKt, kk), aL = mnmajor_desc(sKlo, kk);
          const uint64_t bH = mnmajor_desc(sVt, kk);
          mma_ss(tM, aH, bH, idesc_m, acc);
          mma_ss(tM, aL, bH, idesc_m, 1u);
          if (delta) mma_ss(tM, aH, mnmajor_desc(sUlo, kk), idesc_m, 1u);
          const uint64_t bO = ones_desc(sOnes, kk);
          mma_ss(tZ, aH, bO, idesc_z, acc);
          mma_ss(tZ, aL, bO, idesc_z, 1u);
        }
        mma_commit(bar(U_MMA));
      }
    }
  } else {
    const int wq = warp & 3;
    const int row = wq * 32 + lane;
    const uint32_t lrow = (uint32_t)(wq * 32) << 16;
    for (int c = 0; c < nchunks; ++c) {
      mbar_wait(bar(U_LD), c & 1);
      const bool valid = t_begin + c * kTile + row < t_end;
      float den = 0.f;
#pragma unroll
      for (int ch = 0; ch < 16; ++ch) {
        const uint32_t off = swz_chunk(row, ch);
        uint4 w = lds128(sKt + off);
        uint4 wl;
        uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
        uint32_t* lp = reinterpret_cast<uint32_t*>(&wl);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          float s0 = valid ? elu1(bf16_lo(wp[e])) : 0.f;
          float s1 = valid ? elu1(bf16_hi(wp[e])) : 0.f;
          den = fmaf(s0, zs[8 * ch + 2 * e], den);
          den = fmaf(s1, zs[8 * ch + 2 * e + 1], den);
          const uint32_t hi = pack_bf16x2(s0, s1);
          wp[e] = hi;
          lp[e] = pack_bf16x2(s0 - bf16_lo(hi), s1 - bf16_hi(hi));
        }
        sts128(sKt + off, w);
        sts128(sKlo + off, wl);
      }
      fence_proxy_async_smem();
      if (delta) {
        mbar_arrive(bar(U_SK));
        mbar_wait(bar(U_R), c & 1);
        tc_fence_after();
        const float rinv = den != 0.f ? 1.f / den : 0.f;
#pragma unroll
        for (int q4 = 0; q4 < 4; ++q4) {
          uint32_t r[32];
          tmem_ld32(tR + lrow + 32u * q4, r);
          tmem_ld_wait();
#pragma unroll
          for (int cc = 0; cc < 4; ++cc) {
            const int ch = q4 * 4 + cc;  // 16-byte chunk = 8 value columns
            const uint32_t off = swz_chunk(row, ch);
            uint4 w = lds128(sVt + off);
            uint4 wl;
            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
            uint32_t* lp = reinterpret_cast<uint32_t*>(&wl);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float u0 = bf16_lo(wp[e]) - __uint_as_float(r[8 * cc + 2 * e]) * rinv;
              const float u1 = bf16_hi(wp[e]) - __uint_as_float(r[8 * cc + 2 * e + 1]) * rinv;
              const uint32_t hi = pack_bf16x2(u0, u1);
              wp[e] = hi;
              lp[e] = pack_bf16x2(u0 - bf16_lo(hi), u1 - bf16_hi(hi));
            }
            sts128(sVt + off, w);
            sts128(sUlo + off, wl);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
      }
      mbar_arrive(bar(U_U));
    }
    mbar_wait(bar(U_MMA), (nchunks - 1) & 1);
    tc_fence_after();
    float* prow = part + (long long)row * 128;
#pragma unroll
    for (int q4 = 0; q4 < 4; ++q4) {
      uint32_t r[32];
      tmem_ld32(tM + lrow + 32u * q4, r);
      tmem_ld_wait();
      float4* dst = reinterpret_cast<float4*>(prow + 32 * q4);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        dst[e] = make_float4(__uint_as_float(r[4 * e]), __uint_as_float(r[4 * e + 1]), __uint_as_float(r[4 * e + 2]),
                             __uint_as_float(r[4 * e + 3]));
    }
    uint32_t zr;
    tmem_ld1(tZ + lrow, zr);
    tmem_ld_wait();
    part[128 * 128 + row] = __uint_as_float(zr);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace infini
