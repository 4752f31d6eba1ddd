// mem_update_tc_kernel: the linear-rule memory update (Eq. 8): each CTA's
// share of sigma(K)^T V and sum_t sigma(K_t) over a segment, on the sm_100a
// tensor cores; the scan over segments (state_kernel) adds the partials.
// The delta rule's update is delta_update_tc_kernel (sm100_delta.cuh).
#pragma once

#include "sm100_common.cuh"

namespace infini {
namespace tc {

// Per-chunk timestamps of one update CTA (block INFINI_UPD_TRACE) for tuning
// builds; shares the attention kernel's trace array (slots 3200 and up).
#if defined(INFINI_UPD_TRACE) && defined(INFINI_ATTN_TRACE)
#define UPD_TRACE(cond, slot)                                                                          \
  do {                                                                                                 \
    if ((cond) && blockIdx.x == INFINI_UPD_TRACE && (slot) < 4096) g_attn_trace[(slot)] = clock64();  \
  } while (0)
#else
#define UPD_TRACE(cond, slot) \
  do {                        \
  } while (0)
#endif

// ------------------------------------------------------------------------
// Memory update.  Grid: BH * nseg * G CTAs; CTA (bh, segment seg0 + sl,
// group grp) covers tokens [grp*cpb*128, min((grp+1)*cpb*128, n_s)) of the
// segment in 128-token chunks.
//
// Compute warps: thread (row r of the chunk = TMEM lane, part hh = warp / 4)
// handles 16-byte chunks [CH hh, CH hh + CH) of its token's key row: sigma(K)
// split into bf16 hi + lo parts.  A TMA warp loads (K ring of 3 stages, V
// ring of 2), an MMA warp issues
//   dM += sK_hi^T V + sK_lo^T V          (fp32 in TMEM)
//   dz += sK_hi^T 1 + sK_lo^T 1          (N = 16 block of ones)
// which keeps the update within ~2^-16 relative of fp32 arithmetic.  The lo
// parts of the next chunk wait in registers until the MMAs of the previous
// chunk have released the lo buffer, so the CUDA-core pass overlaps them.
//
// UpdArgs is shared with the delta-rule kernel, which reads M, z and writes
// the per-segment snapshots.
struct UpdArgs {
  float* partial;               // [BH][nseg][G][128*128 + 128] (linear)
  float* M;                     // running state (delta)
  float* z;
  __nv_bfloat16* snapM;         // [BH][S][128][128] bf16 [dk][dv] (delta: M_{s-1} for segment s); nullptr: not written
  float* snapzw;                // [BH][S][128] (delta: z_{s-1} for segment s); nullptr: not written
  float* snapM32;               // delta, optional: fp32 copy of the snapshot (the backward's recomputation)
  int B, H, S, N;
  long long L;
  int seg0, nseg, G, cpb;
};
constexpr int kMaxDeltaCluster = 8;

struct UpdSmem {
  static constexpr int KST = 3;                 // K ring depth
  static constexpr int VST = 2;                 // V ring depth
  static constexpr uint32_t K0 = 0;             // K ring (KST x 32 KB); sigma(K)_hi in place
  static constexpr uint32_t V0 = KST * 32768u;  // V ring
  static constexpr uint32_t KLO = V0 + VST * 32768u;
  static constexpr uint32_t ONES = KLO + 32768u;  // 16-row K-major block of ones (4 KB)
  static constexpr uint32_t BAR = ONES + 4096u;
  static constexpr uint32_t SLOT = BAR + 256u;
  static constexpr uint32_t BYTES = SLOT + 16u + 1024u;
  static_assert(BYTES <= 232448, "update kernel exceeds 227 KB of shared memory");
};

enum : int { U_KF0 = 0, U_KE0 = 3, U_VF0 = 6, U_VE0 = 8, U_SK = 10, U_MMA = 11, U_COUNT = 12 };
// Compute warps: 16 (four threads per token row, 32 columns each), so that
// enough warps hide the latency of the sigma pass.  Plus a TMA and an MMA warp.
struct UpdWarps {
  static constexpr int NCW = 16;
  static constexpr int PARTS = NCW / 4;  // threads per token row
  static constexpr int CH = 16 / PARTS;  // 16-byte chunks (8 columns) per thread
  static constexpr int THREADS = 32 * (NCW + 2);
};

__global__ void __launch_bounds__(UpdWarps::THREADS, 1)
    mem_update_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const UpdArgs a) {
  using SL = UpdSmem;
  using WR = UpdWarps;
  constexpr int KST = SL::KST, VST = SL::VST;
  constexpr int NCW = WR::NCW, PARTS = WR::PARTS, CH = WR::CH;
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
  const int nchunks = t_begin < t_end ? (t_end - t_begin + kTile - 1) / kTile : 0;

  if (nchunks == 0) {  // group past the end of a short segment: contributes nothing
    for (int e = threadIdx.x; e < 128 * 128 + 128; e += blockDim.x) part[e] = 0.f;
  } else {
    auto bar = [&](int i) { return base + SL::BAR + 8u * (uint32_t)i; };
    auto sK = [&](int st) { return base + SL::K0 + (uint32_t)st * kTileBytes; };
    auto sV = [&](int st) { return base + SL::V0 + (uint32_t)st * kTileBytes; };
    const uint32_t sKlo = base + SL::KLO, sOnes = base + SL::ONES;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + SL::SLOT);
    if (threadIdx.x == 0) {
      for (int i = 0; i < 3; ++i) {
        mbar_init(bar(U_KF0 + i), 1);
        mbar_init(bar(U_KE0 + i), 1);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(bar(U_VF0 + i), 1);
        mbar_init(bar(U_VE0 + i), 1);
      }
      mbar_init(bar(U_SK), 32 * NCW);
      mbar_init(bar(U_MMA), 1);
      fence_barrier_init();
    }
    {
      uint32_t* ones = reinterpret_cast<uint32_t*>(gbase + SL::ONES);
      for (int e = threadIdx.x; e < 1024; e += blockDim.x) ones[e] = 0x3f803f80u;  // bf16 1.0 pairs
    }
    if (warp == NCW + 1) {
      tmem_alloc(smem_u32(tmem_slot), 512);
      tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tM = tmem + 128, tZ = tmem + 256;

    if (warp == NCW) {
      if (lane == 0) {
        // ---------------------------------------------------------- producer
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        for (int c = 0; c < nchunks; ++c) {
          const int lt = (int)(seg_start + t_begin + (long long)c * kTile);
          const int kst = c % KST;
          if (c >= KST) mbar_wait(bar(U_KE0 + kst), ((c - KST) / KST) & 1);
          mbar_expect_tx(bar(U_KF0 + kst), kTileBytes);
          tma_load_4d(sK(kst), &tm_k, bar(U_KF0 + kst), 0, lt, h, b);
          tma_load_4d(sK(kst) + kBox, &tm_k, bar(U_KF0 + kst), 64, lt, h, b);
          const int vst = c % VST;
          if (c >= VST) mbar_wait(bar(U_VE0 + vst), ((c - VST) / VST) & 1);
          mbar_expect_tx(bar(U_VF0 + vst), kTileBytes);
          tma_load_4d(sV(vst), &tm_v, bar(U_VF0 + vst), 0, lt, h, b);
          tma_load_4d(sV(vst) + kBox, &tm_v, bar(U_VF0 + vst), 64, lt, h, b);
        }
      }
    } else if (warp == NCW + 1) {
      if (lane == 0) {
        // ---------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc_m = idesc_bf16(128, 128, 1, 1);
        constexpr uint32_t idesc_z = idesc_bf16(128, 16, 1, 0);
        for (int c = 0; c < nchunks; ++c) {
          const int kst = c % KST, vst = c % VST;
          mbar_wait(bar(U_SK), c & 1);
          mbar_wait(bar(U_VF0 + vst), (c / VST) & 1);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
            const uint64_t aH = mnmajor_desc(sK(kst), kk), aL = mnmajor_desc(sKlo, kk);
            const uint64_t bH = mnmajor_desc(sV(vst), kk);
            mma_ss(tM, aH, bH, idesc_m, acc);
            mma_ss(tM, aL, bH, idesc_m, 1u);
            const uint64_t bO = ones_desc(sOnes, kk);
            mma_ss(tZ, aH, bO, idesc_z, acc);
            mma_ss(tZ, aL, bO, idesc_z, 1u);
          }
          mma_commit(bar(U_MMA));
          UPD_TRACE(c < 64, 3200 + 8 * c + 6);
          mma_commit(bar(U_KE0 + kst));
          mma_commit(bar(U_VE0 + vst));
        }
      }
    } else {
      // ------------------------------------------------------------ compute warps
      const int row = (warp & 3) * 32 + lane;
      const int hh = warp >> 2;  // which PARTS-th of the row: chunks [CH * hh, CH * hh + CH)
      const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
      for (int c = 0; c < nchunks; ++c) {
        const int kst = c % KST;
        [[maybe_unused]] const bool tr = threadIdx.x == 0 && c < 64;
        mbar_wait(bar(U_KF0 + kst), (c / KST) & 1);
        UPD_TRACE(tr, 3200 + 8 * c + 0);
        const bool valid = t_begin + c * kTile + row < t_end;
        uint32_t lo[4 * CH];
        uint4 w[CH];
#pragma unroll
        for (int i = 0; i < CH; ++i) w[i] = lds128(sK(kst) + swz_chunk(row, CH * hh + i));
#pragma unroll
        for (int i = 0; i < CH; ++i) {
          uint32_t* wp = reinterpret_cast<uint32_t*>(&w[i]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float s0 = valid ? elu1(bf16_lo(wp[e])) : 0.f;
            const float s1 = valid ? elu1(bf16_hi(wp[e])) : 0.f;
            const uint32_t hi = pack_bf16x2(s0, s1);
            wp[e] = hi;
            lo[4 * i + e] = pack_bf16x2(s0 - bf16_lo(hi), s1 - bf16_hi(hi));
          }
        }
#pragma unroll
        for (int i = 0; i < CH; ++i) sts128(sK(kst) + swz_chunk(row, CH * hh + i), w[i]);
        UPD_TRACE(tr, 3200 + 8 * c + 1);
        if (c > 0) mbar_wait(bar(U_MMA), (c - 1) & 1);  // MMAs of chunk c-1 released the lo buffer
        UPD_TRACE(tr, 3200 + 8 * c + 2);
#pragma unroll
        for (int i = 0; i < CH; ++i)
          sts128(sKlo + swz_chunk(row, CH * hh + i), make_uint4(lo[4 * i], lo[4 * i + 1], lo[4 * i + 2], lo[4 * i + 3]));
        fence_proxy_async_smem();
        mbar_arrive(bar(U_SK));
        UPD_TRACE(tr, 3200 + 8 * c + 3);
      }
      mbar_wait(bar(U_MMA), (nchunks - 1) & 1);
      tc_fence_after();
      // every load and MMA of this CTA is complete: the K/V rings can hold the partial
      constexpr int CPT = 128 / PARTS;  // value columns per thread
      float* prow = part + (long long)row * 128 + CPT * hh;
#pragma unroll
      for (int q2 = 0; q2 < CPT / 32; ++q2) {
        uint32_t rr[32];
        tmem_ld32(tM + lrow + (uint32_t)(CPT * hh) + 32u * q2, rr);
        tmem_ld_wait();
        float4* dst = reinterpret_cast<float4*>(prow + 32 * q2);
#pragma unroll
        for (int e = 0; e < 8; ++e)
          dst[e] = make_float4(__uint_as_float(rr[4 * e]), __uint_as_float(rr[4 * e + 1]),
                               __uint_as_float(rr[4 * e + 2]), __uint_as_float(rr[4 * e + 3]));
      }
      uint32_t zr;
      tmem_ld1(tZ + lrow, zr);
      tmem_ld_wait();
      if (hh == 0) part[128 * 128 + row] = __uint_as_float(zr);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == NCW + 1) {
      __syncwarp();
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  }
}

}  // namespace tc
}  // namespace infini
