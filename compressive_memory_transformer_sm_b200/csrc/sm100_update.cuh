// mem_update_tc_kernel: the segment's share of sigma(K)^T U and
// sum_t sigma(K_t) for the linear (Eq. 8, U = V) or delta (Eq. 9,
// U = V - sigma(K) M_{s-1} / (sigma(K) z_{s-1})) rule, on the sm_100a tensor
// cores.
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
// Warps 0-7: thread (row r of the chunk = TMEM lane, half hh = warp / 4)
// handles value columns [64 hh, 64 hh + 64) of its token: sigma(K) split into
// bf16 hi + lo parts, and for the delta rule U = V - R / den with
// R = sigma(K)_hi M_{s-1} from the tensor cores and den = sigma(K) . z_{s-1}
// in fp32, again split into hi + lo.  Warp 8 loads (TMA: K ring of 3 stages
// (linear) or 2 (delta), V ring of 2 stages (linear) or 1 (delta, where U
// overwrites V in place)),
// warp 9 issues the MMAs:
//   dM += sK_hi^T U_hi + sK_lo^T U_hi (+ sK_hi^T U_lo)   (fp32 in TMEM)
//   dz += sK_hi^T 1 + sK_lo^T 1                        (N = 16 block of ones; delta:
//                                                       16 extra columns of the first
//                                                       two products, B = [U_hi | 1])
// which keeps the update within ~2^-16 relative of fp32 arithmetic.  The lo
// parts of the next chunk wait in registers until the MMAs of the previous
// chunk have released the lo buffers, so the CUDA-core pass overlaps them.
//
// Delta rule: the G CTAs of a head form one thread-block cluster (G <= 8).
// Each stages its partial [dM | dz] in its own shared memory; after a cluster
// barrier, CTA g adds slice g of every partial, read from the peers' shared
// memory in rank order (deterministic), to the running M, z and writes the
// snapshot of M_s for the next segment.  A second cluster barrier keeps every
// CTA's shared memory alive until its peers have read it.
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

template <bool DELTA>
struct UpdSmem {
  static constexpr int KST = DELTA ? 2 : 3;   // K ring depth
  static constexpr int VST = DELTA ? 1 : 2;   // V ring depth
  static constexpr uint32_t K0 = 0;           // K ring (KST x 32 KB); sigma(K)_hi in place
  static constexpr uint32_t V0 = KST * 32768u;  // V ring; U_hi in place (delta)
  // delta: 16 KB of ones right after the single V stage, the third 64-column
  // block of the B operand [U_hi | 1] (N = 144) whose extra columns gather dz
  static constexpr uint32_t ONESB = V0 + VST * 32768u;
  static constexpr uint32_t KLO = ONESB + (DELTA ? 16384u : 0u);
  static constexpr uint32_t ULO = KLO + 32768u;                 // delta
  static constexpr uint32_t MT = ULO + 32768u;                  // delta: M_{s-1} [dk][dv]
  static constexpr uint32_t ONES = KLO + 32768u;                // linear: 16-row K-major block of ones (4 KB)
  static constexpr uint32_t Z = DELTA ? MT + 32768u : ONES + 4096u;
  static constexpr uint32_t DENP = Z + 512u;  // [2 buffers][4 parts of a row][128]
  static constexpr uint32_t BAR = DENP + 4096u;
  static constexpr uint32_t SLOT = BAR + 256u;
  static constexpr uint32_t BYTES = SLOT + 16u + 1024u;
  static_assert(BYTES <= 232448, "update kernel exceeds 227 KB of shared memory");
  // delta: [dM (128 x 128) | dz (128)] fp32 staged for the cluster reduction,
  // over the K and V rings once every chunk has been consumed
  static constexpr uint32_t RED = 0;
};

enum : int {
  U_KF0 = 0, U_KE0 = 3, U_VF0 = 6, U_VE0 = 8, U_MT = 10, U_SK = 11, U_R = 12, U_U = 13, U_MMA = 14,
  U_SKH = 15,  // delta: sigma(K)_hi of the chunk written (the R product may start)
  U_COUNT = 16
};
// Compute warps: 16 (four threads per token row, 32 columns each), so that
// enough warps hide the latency of the sigma and U passes.  Plus a TMA and an
// MMA warp.
template <bool DELTA> struct UpdWarps {
  static constexpr int NCW = 16;
  static constexpr int PARTS = NCW / 4;        // threads per token row
  static constexpr int CH = 16 / PARTS;        // 16-byte chunks (8 columns) per thread
  static constexpr int THREADS = 32 * (NCW + 2);
};

template <bool DELTA>
__global__ void __launch_bounds__(UpdWarps<DELTA>::THREADS, 1)
    mem_update_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                         const UpdArgs a) {
  using SL = UpdSmem<DELTA>;
  using WR = UpdWarps<DELTA>;
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

  float* red = reinterpret_cast<float*>(gbase + SL::RED);
  if (DELTA) {
    // M_{s-1}, z_{s-1} of the head: every CTA with tokens converts M to bf16
    // in its shared memory (the B operand of R, in the layout a 128-byte
    // swizzled TMA load would give); CTA grp writes slice grp of the bf16
    // snapshot of segment s that the attention kernel reads, CTA 0 the z
    // snapshot.  The running M, z change only after the cluster barrier below,
    // once every CTA of the head has passed this point.
    const float* Mh = a.M + (long long)bh * 16384;
    __nv_bfloat16* snap = a.snapM + ((long long)bh * a.S + s) * 16384;
    const int per = (2048 + a.G - 1) / a.G;  // 16-byte chunks of the snapshot per CTA
    const int c_lo = grp * per, c_hi = min(2048, c_lo + per);
    for (int ch = threadIdx.x; ch < 2048; ch += blockDim.x) {
      const bool mine = ch >= c_lo && ch < c_hi;
      if (nchunks == 0 && !mine) continue;
      const int r = ch >> 4, cc = ch & 15;
      const float4 f0 = *reinterpret_cast<const float4*>(Mh + r * 128 + 8 * cc);
      const float4 f1 = *reinterpret_cast<const float4*>(Mh + r * 128 + 8 * cc + 4);
      const uint4 v = make_uint4(pack_bf16x2(f0.x, f0.y), pack_bf16x2(f0.z, f0.w), pack_bf16x2(f1.x, f1.y),
                                 pack_bf16x2(f1.z, f1.w));
      if (nchunks > 0) sts128(base + SL::MT + swz_chunk(r, cc), v);
      if (mine && a.snapM != nullptr) *reinterpret_cast<uint4*>(snap + r * 128 + 8 * cc) = v;
      if (mine && a.snapM32 != nullptr) {
        float4* s32 = reinterpret_cast<float4*>(a.snapM32 + ((long long)bh * a.S + s) * 16384 + r * 128 + 8 * cc);
        s32[0] = f0;
        s32[1] = f1;
      }
    }
    if (grp == 0 && threadIdx.x < 128 && a.snapzw != nullptr)
      a.snapzw[((long long)bh * a.S + s) * 128 + threadIdx.x] = a.z[(long long)bh * 128 + threadIdx.x];
  }
  if (nchunks == 0) {  // group past the end of a short segment: contributes nothing
    if (DELTA) {
      for (int e = threadIdx.x; e < 128 * 128 + 128; e += blockDim.x) red[e] = 0.f;
    } else {
      for (int e = threadIdx.x; e < 128 * 128 + 128; e += blockDim.x) part[e] = 0.f;
    }
  } else {
    auto bar = [&](int i) { return base + SL::BAR + 8u * (uint32_t)i; };
    auto sK = [&](int st) { return base + SL::K0 + (uint32_t)st * kTileBytes; };
    auto sV = [&](int st) { return base + SL::V0 + (uint32_t)st * kTileBytes; };
    const uint32_t sKlo = base + SL::KLO, sUlo = base + SL::ULO, sMs = base + SL::MT, sOnes = base + SL::ONES;
    float* zs = reinterpret_cast<float*>(gbase + SL::Z);
    float* denp = reinterpret_cast<float*>(gbase + SL::DENP);
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
      mbar_init(bar(U_SKH), 32 * NCW);
      mbar_init(bar(U_R), 1);
      mbar_init(bar(U_U), 32 * NCW);
      mbar_init(bar(U_MMA), 1);
      fence_barrier_init();
    }
    {
      uint32_t* ones = reinterpret_cast<uint32_t*>(gbase + (DELTA ? SL::ONESB : SL::ONES));
      for (int e = threadIdx.x; e < (DELTA ? 4096 : 1024); e += blockDim.x) ones[e] = 0x3f803f80u;  // bf16 1.0 pairs
    }
    if (threadIdx.x < 128) zs[threadIdx.x] = DELTA ? a.z[(long long)bh * 128 + threadIdx.x] : 0.f;
    if (warp == NCW + 1) {
      tmem_alloc(smem_u32(tmem_slot), 512);
      tmem_relinquish();
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tR = tmem, tM = tmem + 128, tZ = tmem + 256;

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
        constexpr uint32_t idesc_r = idesc_bf16(128, 128, 0, 1);  // B = M_{s-1} [dk][dv], MN-major
        constexpr uint32_t idesc_m = idesc_bf16(128, 128, 1, 1);
        constexpr uint32_t idesc_m1 = idesc_bf16(128, 144, 1, 1);  // delta: B = [U_hi | 1]
        constexpr uint32_t idesc_z = idesc_bf16(128, 16, 1, 0);
        for (int c = 0; c < nchunks; ++c) {
          const int kst = c % KST, vst = c % VST;
          if (DELTA) {
            // R = sigma(K)_hi M_{s-1} needs only the hi part: it starts while
            // the compute warps store the lo part and exchange the denominators
            mbar_wait(bar(U_SKH), c & 1);
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              mma_ss(tR, kmajor_desc(sK(kst), kk), mnmajor_desc(sMs, kk), idesc_r, kk > 0 ? 1u : 0u);
            mma_commit(bar(U_R));
            mbar_wait(bar(U_U), c & 1);  // after the lo part and U: the dM products
          } else {
            mbar_wait(bar(U_SK), c & 1);
            mbar_wait(bar(U_VF0 + vst), (c / VST) & 1);
          }
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) {
            const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
            const uint64_t aH = mnmajor_desc(sK(kst), kk), aL = mnmajor_desc(sKlo, kk);
            const uint64_t bH = mnmajor_desc(sV(vst), kk);
            if (DELTA) {
              // columns 128-143 of [dM | dz] (TMEM tZ) collect sigma(K)^T 1
              mma_ss(tM, aH, bH, idesc_m1, acc);
              mma_ss(tM, aL, bH, idesc_m1, 1u);
              mma_ss(tM, aH, mnmajor_desc(sUlo, kk), idesc_m, 1u);
            } else {
              mma_ss(tM, aH, bH, idesc_m, acc);
              mma_ss(tM, aL, bH, idesc_m, 1u);
              const uint64_t bO = ones_desc(sOnes, kk);
              mma_ss(tZ, aH, bO, idesc_z, acc);
              mma_ss(tZ, aL, bO, idesc_z, 1u);
            }
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
        const int kst = c % KST, vst = c % VST;
        [[maybe_unused]] const bool tr = threadIdx.x == 0 && c < 64;
        mbar_wait(bar(U_KF0 + kst), (c / KST) & 1);
        UPD_TRACE(tr, 3200 + 8 * c + 0);
        const bool valid = t_begin + c * kTile + row < t_end;
        float dp[4] = {0.f, 0.f, 0.f, 0.f};
        uint32_t lo[4 * CH];
        uint4 w[CH];
#pragma unroll
        for (int i = 0; i < CH; ++i) w[i] = lds128(sK(kst) + swz_chunk(row, CH * hh + i));
        if (!DELTA) {
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
        } else {
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            uint32_t* wp = reinterpret_cast<uint32_t*>(&w[i]);
            float zz[8];
            {
              const float4 za = *reinterpret_cast<const float4*>(zs + 8 * (CH * hh + i));
              const float4 zb = *reinterpret_cast<const float4*>(zs + 8 * (CH * hh + i) + 4);
              zz[0] = za.x; zz[1] = za.y; zz[2] = za.z; zz[3] = za.w;
              zz[4] = zb.x; zz[5] = zb.y; zz[6] = zb.z; zz[7] = zb.w;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float s0 = elu1(bf16_lo(wp[e]));
              const float s1 = elu1(bf16_hi(wp[e]));
              dp[e] = fmaf(s0, zz[2 * e], dp[e]);
              dp[e] = fmaf(s1, zz[2 * e + 1], dp[e]);
              const uint32_t hi = pack_bf16x2(s0, s1);
              wp[e] = hi;
              lo[4 * i + e] = pack_bf16x2(s0 - bf16_lo(hi), s1 - bf16_hi(hi));
            }
          }
          if (!valid) {  // a token past the end of the segment (the TMA read zeros) contributes nothing
#pragma unroll
            for (int i = 0; i < CH; ++i) w[i] = make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
            for (int i = 0; i < 4 * CH; ++i) lo[i] = 0u;
#pragma unroll
            for (int e = 0; e < 4; ++e) dp[e] = 0.f;
          }
        }
#pragma unroll
        for (int i = 0; i < CH; ++i) sts128(sK(kst) + swz_chunk(row, CH * hh + i), w[i]);
        if (DELTA) {
          fence_proxy_async_smem();
          mbar_arrive(bar(U_SKH));
        }
        const float dpart = (dp[0] + dp[1]) + (dp[2] + dp[3]);
        UPD_TRACE(tr, 3200 + 8 * c + 1);
        if (c > 0) mbar_wait(bar(U_MMA), (c - 1) & 1);  // MMAs of chunk c-1 released the lo buffers
        UPD_TRACE(tr, 3200 + 8 * c + 2);
#pragma unroll
        for (int i = 0; i < CH; ++i)
          sts128(sKlo + swz_chunk(row, CH * hh + i), make_uint4(lo[4 * i], lo[4 * i + 1], lo[4 * i + 2], lo[4 * i + 3]));
        float den = 0.f;
        if (DELTA) {
          float* dpb = denp + (c & 1) * (PARTS * 128);
          dpb[hh * 128 + row] = dpart;
          named_bar_sync(1, 32 * NCW);
#pragma unroll
          for (int pp = 0; pp < PARTS; ++pp) den += dpb[pp * 128 + row];  // fixed order
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(U_SK));
        UPD_TRACE(tr, 3200 + 8 * c + 3);
        if (DELTA) {
          mbar_wait(bar(U_R), c & 1);
          UPD_TRACE(tr, 3200 + 8 * c + 4);
          tc_fence_after();
          const float rinv = den != 0.f ? 1.f / den : 0.f;
          constexpr int CPT = 128 / PARTS;  // value columns of this thread
          uint32_t r[CPT];
#pragma unroll
          for (int q2 = 0; q2 < CPT / 32; ++q2)
            tmem_ld32(tR + lrow + (uint32_t)(CPT * hh + 32 * q2), *reinterpret_cast<uint32_t(*)[32]>(&r[32 * q2]));
          tmem_ld_wait();
          mbar_wait(bar(U_VF0 + vst), (c / VST) & 1);
#pragma unroll
          for (int i = 0; i < CH; ++i) {
            const uint32_t off = swz_chunk(row, CH * hh + i);
            uint4 w = lds128(sV(vst) + off);
            uint4 wl;
            uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
            uint32_t* lp = reinterpret_cast<uint32_t*>(&wl);
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int col = 8 * i + 2 * e;  // within this thread's columns
              const float u0 = bf16_lo(wp[e]) - __uint_as_float(r[col]) * rinv;
              const float u1 = bf16_hi(wp[e]) - __uint_as_float(r[col + 1]) * rinv;
              const uint32_t hi = pack_bf16x2(u0, u1);
              wp[e] = hi;
              lp[e] = pack_bf16x2(u0 - bf16_lo(hi), u1 - bf16_hi(hi));
            }
            sts128(sV(vst) + off, w);
            sts128(sUlo + off, wl);
          }
          fence_proxy_async_smem();
          tc_fence_before();
          mbar_arrive(bar(U_U));
          UPD_TRACE(tr, 3200 + 8 * c + 5);
        }
      }
      mbar_wait(bar(U_MMA), (nchunks - 1) & 1);
      tc_fence_after();
      // every load and MMA of this CTA is complete: the K/V rings can hold the partial
      constexpr int CPT = 128 / PARTS;  // value columns per thread
      float* prow = (DELTA ? red : part) + (long long)row * 128 + CPT * hh;
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
      if (hh == 0) (DELTA ? red : part)[128 * 128 + row] = __uint_as_float(zr);
    }
    tc_fence_before();
    __syncthreads();
    if (warp == NCW + 1) {
      __syncwarp();
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  }
  if (!DELTA) return;
  // ------------------------------------------------------------ delta: cluster reduction
  __syncthreads();
  cluster_sync();  // every CTA of the head has staged its partial
  {
    constexpr int E4 = (128 * 128 + 128) / 4;  // float4 elements of [M | z]
    const int per = (E4 + a.G - 1) / a.G;
    const int e4_begin = grp * per, e4_end = min(E4, e4_begin + per);
    const uint32_t red_addr = smem_u32(red);
    for (int e4 = e4_begin + (int)threadIdx.x; e4 < e4_end; e4 += blockDim.x) {
      const int e = 4 * e4;
      float4* st = e < 16384 ? reinterpret_cast<float4*>(&a.M[(long long)bh * 16384 + e])
                             : reinterpret_cast<float4*>(&a.z[(long long)bh * 128 + (e - 16384)]);
      float4 acc = *st;
      for (int g = 0; g < a.G; ++g) {
        const float4 v = ld_dsmem_f4(mapa_shared(red_addr + 16u * (uint32_t)e4, (uint32_t)g));
        acc.x += v.x;
        acc.y += v.y;
        acc.z += v.z;
        acc.w += v.w;
      }
      *st = acc;
    }
  }
  cluster_sync();  // peers have finished reading this CTA's shared memory
}

}  // namespace tc
}  // namespace infini
