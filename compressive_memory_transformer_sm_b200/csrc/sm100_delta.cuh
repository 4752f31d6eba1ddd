// delta_update_tc_kernel: one segment of the delta-rule memory update
// ("Leave No Context Behind", section 2.1.2, Eq. 9) on the sm_100a tensor
// cores:
//   M_s = M_{s-1} + sigma(K)^T (V - sigma(K) M_{s-1} / (sigma(K) z_{s-1}))
//   z_s = z_{s-1} + sum_t sigma(K_t)
//
// The products run transposed, so that M_{s-1} and U = V - R / den live in
// tensor memory as the A operand and only K, sigma(K)_lo and V tiles occupy
// shared memory (48 KB per 64-token chunk): deep enough rings that the
// chunks of a CTA overlap.  Per chunk c of 64 tokens:
//   sigma pass (CUDA cores, thread = a quarter-row of 16 columns):
//     sigma(K) = ELU + 1, split into bf16 hi (in place of K) + lo parts;
//     den_t = sigma(K_t) . z_{s-1} in fp32; dz += sigma(K) in fp32 registers
//   R^T  = M_{s-1}^T sigma(K)_hi^T                   (A: M^T bf16 in TMEM, B: K-major)
//   U pass (CUDA cores, thread = one value column d = one TMEM lane, 16 tokens):
//     U = V - R / den in fp32, split into bf16 hi + lo, written to TMEM as U^T
//   dM^T += U_hi^T sigma(K)_hi + U_hi^T sigma(K)_lo + U_lo^T sigma(K)_hi
//                                                    (A: U^T in TMEM, B: MN-major)
// The lo parts keep the accumulated update within ~2^-16 relative of fp32
// arithmetic; R uses bf16 M_{s-1}, as the memory read does.
//
// Software pipeline: the compute warps run sigma(c + 1) before U(c), and the
// MMA warp issues R(c + 1) before dM(c), so the R product of the next chunk
// runs under the U pass of this one and the dM products under the next
// sigma pass.  Double-buffered R and U in TMEM (448 of 512 columns).
//
// The G CTAs of a head (token ranges of the segment) form one cluster: each
// stages its partial [dM | dz] in shared memory; after a cluster barrier CTA g
// adds slice g of every partial, in rank order (deterministic), to the
// running M, z.  Every CTA first writes its slice of the snapshot of M_{s-1}
// that the attention kernel reads.
#pragma once

#include "sm100_common.cuh"
#include "sm100_update.cuh"

namespace infini {
namespace tc {

constexpr int kDChunk = 64;           // tokens per chunk
constexpr uint32_t kDBox = 8192;      // 64 rows x 128 B
constexpr uint32_t kDTile = 16384;    // 64 tokens x 128 bf16: two boxes
constexpr int kDeltaThreads = 576;    // 16 compute warps, a TMA warp, an MMA warp

struct DeltaSmem {
  static constexpr int KST = 6;  // K ring (sigma(K)_hi in place): loaded -> dM done
  static constexpr int LST = 3;  // sigma(K)_lo ring: sigma pass -> dM done
  static constexpr int VST = 4;  // V ring: loaded -> U pass done
  static constexpr uint32_t K0 = 0;
  static constexpr uint32_t KL0 = K0 + KST * kDTile;
  static constexpr uint32_t V0 = KL0 + LST * kDTile;
  static constexpr uint32_t Z = V0 + VST * kDTile;  // z_{s-1}, 128 floats
  // [LST][64] 1 / den of a chunk's tokens: sigma(c + LST) rewrites buffer c % LST
  // only after its lo-buffer wait (dM(c) done, so every warp's U(c) has read it)
  static constexpr uint32_t RINV = Z + 512u;
  static constexpr uint32_t BAR = RINV + 1024u;
  static_assert(LST * 64 * 4 <= 1024, "1 / den buffers");
  static constexpr uint32_t SLOT = BAR + 512u;
  static constexpr uint32_t BYTES = SLOT + 16u + 1024u;
  static_assert(BYTES <= 232448, "delta update kernel exceeds 227 KB of shared memory");
  // after the last chunk, over the rings: the partial [dM (128 x 128) | dz (128)]
  // (66,048 B from 0) and the 16 warps' dz sums (8 KB)
  static constexpr uint32_t RED = 0;
  static constexpr uint32_t DZS = 69632u;
  static_assert(DZS + 16u * 128u * 4u <= V0, "epilogue scratch must lie in the K / lo rings");
};

enum : int {
  D_KF = 0, D_KE = 6, D_LE = 12, D_VF = 15, D_VE = 19, D_SK = 23, D_RF = 25, D_UR = 27, D_UE = 29, D_MT = 31,
  D_DONE = 32, D_COUNT = 33
};

// 16-byte chunk c (0..15) of row r of a 64-row tile (two 8 KB boxes)
__device__ __forceinline__ uint32_t dswz(int r, int c) {
  return (uint32_t)(c >> 3) * kDBox + (uint32_t)r * 128u + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}
// K-major operand of 64 rows (the B of R^T: sigma(K) rows, 16 dk per step)
__device__ __forceinline__ uint64_t dkmajor_desc(uint32_t tile, int kk) {
  return smem_desc_sw128(tile, 16u, 1024u) + (uint64_t)((uint32_t)(kk >> 2) * (kDBox >> 4) + (uint32_t)(kk & 3) * 2u);
}
// MN-major operand of 64 K-rows x 128 (the B of dM^T: sigma(K) [t][dk], 16 tokens per step)
__device__ __forceinline__ uint64_t dmnmajor_desc(uint32_t tile, int kk) {
  return smem_desc_sw128(tile, kDBox, 1024u) + (uint64_t)((uint32_t)kk * (2048u >> 4));
}
__device__ __forceinline__ float lds_bf16(uint32_t a) {
  unsigned short v;
  asm volatile("ld.shared.u16 %0, [%1];" : "=h"(v) : "r"(a));
  return __uint_as_float((uint32_t)v << 16);
}

__global__ void __launch_bounds__(kDeltaThreads, 1)
    delta_update_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                           const UpdArgs a) {
  using SL = DeltaSmem;
  constexpr int KST = SL::KST, LST = SL::LST, VST = SL::VST;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const int grp = blockIdx.x % a.G;
  const int bh = blockIdx.x / a.G;
  const int s = a.seg0;
  const int b = bh / a.H, h = bh % a.H;
  const long long seg_start = (long long)s * a.N;
  const int n_s = (int)min((long long)a.N, a.L - seg_start);
  const int t_begin = grp * a.cpb * kTile;
  const int t_end = min(n_s, t_begin + a.cpb * kTile);
  const int nch = t_begin < t_end ? (t_end - t_begin + kDChunk - 1) / kDChunk : 0;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  float* red = reinterpret_cast<float*>(gbase + SL::RED);
  const float* Mh = a.M + (long long)bh * 16384;

  // Snapshot of M_{s-1}, z_{s-1} for the attention (and the backward): CTA
  // grp writes slice grp.  The running M, z change only after the cluster
  // barrier below, once every CTA of the head has read them.
  {
    const int per = (2048 + a.G - 1) / a.G;  // 16-byte chunks of the bf16 snapshot per CTA
    const int c_lo = grp * per, c_hi = min(2048, c_lo + per);
    __nv_bfloat16* snap = a.snapM + ((long long)bh * a.S + s) * 16384;
    for (int ch = c_lo + (int)threadIdx.x; ch < c_hi; ch += blockDim.x) {
      const int r = ch >> 4, cc = ch & 15;
      const float4 f0 = *reinterpret_cast<const float4*>(Mh + r * 128 + 8 * cc);
      const float4 f1 = *reinterpret_cast<const float4*>(Mh + r * 128 + 8 * cc + 4);
      if (a.snapM != nullptr)
        *reinterpret_cast<uint4*>(snap + r * 128 + 8 * cc) = make_uint4(
            pack_bf16x2(f0.x, f0.y), pack_bf16x2(f0.z, f0.w), pack_bf16x2(f1.x, f1.y), pack_bf16x2(f1.z, f1.w));
      if (a.snapM32 != nullptr) {
        float4* s32 = reinterpret_cast<float4*>(a.snapM32 + ((long long)bh * a.S + s) * 16384 + r * 128 + 8 * cc);
        s32[0] = f0;
        s32[1] = f1;
      }
    }
    if (grp == 0 && threadIdx.x < 128 && a.snapzw != nullptr)
      a.snapzw[((long long)bh * a.S + s) * 128 + threadIdx.x] = a.z[(long long)bh * 128 + threadIdx.x];
  }

  if (nch == 0) {  // group past the end of a short segment: contributes nothing
    for (int e = threadIdx.x; e < 128 * 128 + 128; e += blockDim.x) red[e] = 0.f;
  } else {
    auto bar = [&](int i) { return base + SL::BAR + 8u * (uint32_t)i; };
    auto sK = [&](int st) { return base + SL::K0 + (uint32_t)st * kDTile; };
    auto sL = [&](int st) { return base + SL::KL0 + (uint32_t)st * kDTile; };
    auto sV = [&](int st) { return base + SL::V0 + (uint32_t)st * kDTile; };
    const float* zs = reinterpret_cast<const float*>(gbase + SL::Z);
    float* rinv = reinterpret_cast<float*>(gbase + SL::RINV);
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + SL::SLOT);
    if (threadIdx.x == 0) {
      for (int i = 0; i < KST; ++i) {
        mbar_init(bar(D_KF + i), 1);
        mbar_init(bar(D_KE + i), 1);
      }
      for (int i = 0; i < LST; ++i) mbar_init(bar(D_LE + i), 1);
      for (int i = 0; i < VST; ++i) {
        mbar_init(bar(D_VF + i), 1);
        mbar_init(bar(D_VE + i), 16);
      }
      for (int i = 0; i < 2; ++i) {
        mbar_init(bar(D_SK + i), 16);
        mbar_init(bar(D_RF + i), 1);
        mbar_init(bar(D_UR + i), 16);
        mbar_init(bar(D_UE + i), 1);
      }
      mbar_init(bar(D_MT), 16);
      mbar_init(bar(D_DONE), 1);
      fence_barrier_init();
    }
    if (threadIdx.x < 128) reinterpret_cast<float*>(gbase + SL::Z)[threadIdx.x] = a.z[(long long)bh * 128 + threadIdx.x];
    if (warp == 17) {
      tmem_alloc(smem_u32(tmem_slot), 512);
      tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    // TMEM columns: M^T (bf16 pairs) 0-63, R^T buffers 64-191, U^T buffers
    // (hi 32 + lo 32 columns each) 192-319, dM^T 320-447
    const uint32_t tMT = tmem, tD = tmem + 320u;
    auto tR = [&](int rb) { return tmem + 64u + 64u * (uint32_t)rb; };
    auto tU = [&](int ub) { return tmem + 192u + 64u * (uint32_t)ub; };

    if (warp == 16) {
      if (lane == 0) {
        // ---------------------------------------------------------- producer
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        for (int c = 0; c < nch; ++c) {
          const int lt = (int)(seg_start + t_begin + (long long)c * kDChunk);
          const int ks = c % KST, vs = c % VST;
          if (c >= KST) mbar_wait(bar(D_KE + ks), ((c / KST) - 1) & 1);
          mbar_expect_tx(bar(D_KF + ks), kDTile);
          tma_load_4d(sK(ks), &tm_k, bar(D_KF + ks), 0, lt, h, b);
          tma_load_4d(sK(ks) + kDBox, &tm_k, bar(D_KF + ks), 64, lt, h, b);
          if (c >= VST) mbar_wait(bar(D_VE + vs), ((c / VST) - 1) & 1);
          mbar_expect_tx(bar(D_VF + vs), kDTile);
          tma_load_4d(sV(vs), &tm_v, bar(D_VF + vs), 0, lt, h, b);
          tma_load_4d(sV(vs) + kDBox, &tm_v, bar(D_VF + vs), 64, lt, h, b);
        }
      }
    } else if (warp == 17) {
      if (lane == 0) {
        // ---------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc_r = idesc_bf16(128, 64, 0, 0);   // A = M^T (TMEM), B = sigma(K)_hi K-major
        constexpr uint32_t idesc_d = idesc_bf16(128, 128, 0, 1);  // A = U^T (TMEM), B = sigma(K) MN-major
        mbar_wait(bar(D_MT), 0);
        auto issue_r = [&](int c) {
          const int rb = c & 1, ks = c % KST;
          mbar_wait(bar(D_SK + rb), (c >> 1) & 1);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 8; ++kk) mma_ts(tR(rb), tMT + 8u * (uint32_t)kk, dkmajor_desc(sK(ks), kk), idesc_r, kk > 0 ? 1u : 0u);
          mma_commit(bar(D_RF + rb));
        };
        issue_r(0);
        for (int c = 0; c < nch; ++c) {
          if (c + 1 < nch) issue_r(c + 1);
          const int ub = c & 1, ks = c % KST, ls = c % LST;
          mbar_wait(bar(D_UR + ub), (c >> 1) & 1);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t bH = dmnmajor_desc(sK(ks), kk), bL = dmnmajor_desc(sL(ls), kk);
            const uint32_t aH = tU(ub) + 8u * (uint32_t)kk, aL = aH + 32u;
            mma_ts(tD, aH, bH, idesc_d, (c > 0 || kk > 0) ? 1u : 0u);
            mma_ts(tD, aH, bL, idesc_d, 1u);
            mma_ts(tD, aL, bH, idesc_d, 1u);
          }
          mma_commit(bar(D_KE + ks));
          mma_commit(bar(D_LE + ls));
          mma_commit(bar(D_UE + ub));
        }
        mma_commit(bar(D_DONE));
      }
    } else {
      // ------------------------------------------------------------ compute warps
      const int q = warp & 3, g = warp >> 2;
      const uint32_t lq = (uint32_t)(32 * q) << 16;  // this warp's TMEM lane quarter
      const int d = 32 * q + lane;                   // U pass: value column = TMEM lane
      {
        // M_{s-1}^T into TMEM: lane d, column j = (M[2j][d], M[2j+1][d]) for
        // this warp's 32 rows k of M
        uint32_t mw[16];
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          const int k = 32 * g + 2 * j;
          mw[j] = pack_bf16x2(Mh[k * 128 + d], Mh[(k + 1) * 128 + d]);
        }
        tmem_st16(tMT + lq + 16u * (uint32_t)g, mw);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(D_MT));
      }
      // sigma pass: row rr of the chunk, 16-byte chunks p (columns 8p..8p+7)
      // and 8 + p (columns 64 + 8p..)
      const int rr = 4 * warp + (lane >> 3), p = lane & 7;
      float dz[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) dz[i] = 0.f;
      auto sigma_pass = [&](int c) {
        const int ks = c % KST, ls = c % LST, rb = c & 1;
        mbar_wait(bar(D_KF + ks), (c / KST) & 1);
        const bool valid = t_begin + c * kDChunk + rr < t_end;
        uint4 w[2], lo[2];
        w[0] = lds128(sK(ks) + dswz(rr, p));
        w[1] = lds128(sK(ks) + dswz(rr, 8 + p));
        float dp = 0.f;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const float4 za = *reinterpret_cast<const float4*>(zs + 64 * i + 8 * p);
          const float4 zb = *reinterpret_cast<const float4*>(zs + 64 * i + 8 * p + 4);
          const float zz[8] = {za.x, za.y, za.z, za.w, zb.x, zb.y, zb.z, zb.w};
          uint32_t* wp = reinterpret_cast<uint32_t*>(&w[i]);
          uint32_t* lp = reinterpret_cast<uint32_t*>(&lo[i]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float s0 = valid ? elu1(bf16_lo(wp[e])) : 0.f;
            const float s1 = valid ? elu1(bf16_hi(wp[e])) : 0.f;
            dp = fmaf(s0, zz[2 * e], dp);
            dp = fmaf(s1, zz[2 * e + 1], dp);
            dz[8 * i + 2 * e] += s0;
            dz[8 * i + 2 * e + 1] += s1;
            const uint32_t hi = pack_bf16x2(s0, s1);
            wp[e] = hi;
            lp[e] = pack_bf16x2(s0 - bf16_lo(hi), s1 - bf16_hi(hi));
          }
        }
        sts128(sK(ks) + dswz(rr, p), w[0]);
        sts128(sK(ks) + dswz(rr, 8 + p), w[1]);
        if (c >= LST) mbar_wait(bar(D_LE + ls), ((c / LST) - 1) & 1);  // dM(c - LST) released the lo buffer
        sts128(sL(ls) + dswz(rr, p), lo[0]);
        sts128(sL(ls) + dswz(rr, 8 + p), lo[1]);
        // den of the row: the 8 lanes of the row in a fixed butterfly (every lane gets the same sum)
        dp += __shfl_xor_sync(0xffffffffu, dp, 1);
        dp += __shfl_xor_sync(0xffffffffu, dp, 2);
        dp += __shfl_xor_sync(0xffffffffu, dp, 4);
        if (p == 0) rinv[64 * ls + rr] = dp != 0.f ? 1.f / dp : 0.f;
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(D_SK + rb));
      };
      // U pass: value column d, tokens 16g..16g+15 of the chunk
      auto u_pass = [&](int c) {
        const int rb = c & 1, vs = c % VST;
        mbar_wait(bar(D_SK + rb), (c >> 1) & 1);  // every warp's 1 / den of chunk c
        mbar_wait(bar(D_RF + rb), (c >> 1) & 1);
        tc_fence_after();
        uint32_t r[16];
        tmem_ld16(tR(rb) + lq + 16u * (uint32_t)g, r);
        float ri[16];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const float4 f = *reinterpret_cast<const float4*>(rinv + 64 * (c % LST) + 16 * g + 4 * i);
          ri[4 * i] = f.x; ri[4 * i + 1] = f.y; ri[4 * i + 2] = f.z; ri[4 * i + 3] = f.w;
        }
        mbar_wait(bar(D_VF + vs), (c / VST) & 1);
        float v[16];
        const uint32_t vcol = (uint32_t)(d >> 6) * kDBox + (uint32_t)(d & 7) * 2u;
#pragma unroll
        for (int t = 0; t < 16; ++t) {
          const int tt = 16 * g + t;
          v[t] = lds_bf16(sV(vs) + vcol + (uint32_t)tt * 128u + ((uint32_t)(((d >> 3) & 7) ^ (tt & 7)) << 4));
        }
        tmem_ld_wait();
        uint32_t hw[8], lw[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          const float u0 = v[2 * j] - __uint_as_float(r[2 * j]) * ri[2 * j];
          const float u1 = v[2 * j + 1] - __uint_as_float(r[2 * j + 1]) * ri[2 * j + 1];
          hw[j] = pack_bf16x2(u0, u1);
          lw[j] = pack_bf16x2(u0 - bf16_lo(hw[j]), u1 - bf16_hi(hw[j]));
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(D_VE + vs));  // every lane's V values are in registers
        if (c >= 2) mbar_wait(bar(D_UE + rb), ((c >> 1) - 1) & 1);  // dM(c - 2) released the U buffer
        tc_fence_after();
        tmem_st8(tU(rb) + lq + 8u * (uint32_t)g, hw);
        tmem_st8(tU(rb) + lq + 32u + 8u * (uint32_t)g, lw);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(D_UR + rb));
      };
      sigma_pass(0);
      for (int c = 0; c < nch; ++c) {
        if (c + 1 < nch) sigma_pass(c + 1);
        u_pass(c);
      }
      mbar_wait(bar(D_DONE), 0);
      tc_fence_after();
      // every load and MMA of this CTA is complete: the rings hold the partial.
      // dM[k][d] = dM^T[d][k]: lane d, columns k = 32g..32g+31
      {
        uint32_t rw[32];
        tmem_ld32(tD + lq + 32u * (uint32_t)g, rw);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) red[(32 * g + j) * 128 + d] = __uint_as_float(rw[j]);
      }
      // dz: the 4 rows of the warp (lanes p, p + 8, p + 16, p + 24), then the 16 warps in order
      float* dzs = reinterpret_cast<float*>(gbase + SL::DZS);
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        dz[i] += __shfl_xor_sync(0xffffffffu, dz[i], 8);
        dz[i] += __shfl_xor_sync(0xffffffffu, dz[i], 16);
      }
      if (lane < 8) {
#pragma unroll
        for (int i = 0; i < 16; ++i) dzs[warp * 128 + 64 * (i >> 3) + 8 * p + (i & 7)] = dz[i];
      }
      named_bar_sync(1, 512);
      if (threadIdx.x < 128) {
        float t = 0.f;
        for (int w2 = 0; w2 < 16; ++w2) t += dzs[w2 * 128 + threadIdx.x];
        red[16384 + threadIdx.x] = t;
      }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 17) {
      __syncwarp();
      tc_fence_after();
      tmem_dealloc(tmem, 512);
    }
  }
  // ------------------------------------------------------------ cluster reduction
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
      for (int g2 = 0; g2 < a.G; ++g2) {
        const float4 v = ld_dsmem_f4(mapa_shared(red_addr + 16u * (uint32_t)e4, (uint32_t)g2));
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
