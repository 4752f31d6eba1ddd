// delta_update_tc_kernel: one segment of the delta-rule memory update
// ("Leave No Context Behind", section 2.1.2, Eq. 9) on the sm_100a tensor
// cores:
//   M_s = M_{s-1} + sigma(K)^T (V - sigma(K) M_{s-1} / (sigma(K) z_{s-1}))
//   z_s = z_{s-1} + sum_t sigma(K_t)
//
// M_{s-1} is fixed for the whole segment, so the retrieval term factors out
// of the sum over tokens:
//   sum_t sigma(K_t)^T sigma(K_t) M_{s-1} / den_t = G M_{s-1},
//   G = sum_t sigma(K_t)^T sigma(K_t) / den_t      ([dk][dk]),
// and dM = sigma(K)^T V - G M_{s-1}: every chunk's work is products that
// read only shared memory, with no retrieval product and no round trip
// through the CUDA cores between products, plus one G M_{s-1} product per
// CTA at the end.  (The sums of Eq. 9, reassociated; with the hi + lo splits
// below the result is closer to fp64 than a retrieval through a bf16 M_{s-1}.)
//
// Per chunk c of 64 tokens:
//   sigma pass (CUDA cores; thread = row rr of the chunk, 16 of its columns):
//     sigma(K) = ELU + 1 in fp32, split into bf16 hi (in place of K) + lo;
//     den_t = sigma(K_t) . z_{s-1} (fp32); S_t = sigma(K_t) / den_t (0 where
//     den_t = 0) in bf16; dz += sigma(K) in fp32 registers
//   tensor cores (transposed, fp32 accumulators in TMEM):
//     VM^T += V^T sigma_hi + V^T sigma_lo           (V exact in bf16)
//     G    += S^T sigma_hi
// After the last chunk: dM^T = VM^T + M^T (-G^T), with M^T in TMEM (hi + lo
// parts, the A operand) and -G^T written to shared memory as bf16 hi + lo.
// sigma^T V and the final product keep ~2^-16 relative accuracy; G's bf16
// roundings are independent across tokens and average out in the sum, so
// that the state stays within ~2e-5 relative of fp64 over many segments,
// closer than a retrieval through a bf16 M_{s-1} (fp32 accumulation).
//
// The G CTAs of a head (token ranges of the segment) form one cluster.  Once
// every CTA of the cluster is past its chunks (a cluster barrier), each
// stores slice g of its partial [dM | dz] into CTA g's shared memory; after a
// second barrier CTA g adds the G partials of slice g, in rank order
// (deterministic), to the running M, z.  Every CTA first writes its slice of
// the snapshot of M_{s-1} that the attention kernel reads.
#pragma once

#include "sm100_common.cuh"
#include "sm100_update.cuh"

namespace infini {
namespace tc {

// Phase timestamps of one CTA (block INFINI_DELTA_TRACE) for tuning builds;
// shares the attention kernel's trace array (slots 3200 and up): 3200-3209
// phases of thread 0, 3210 + c its sigma pass of chunk c, 3280 + c the MMA
// warp's chunk c, 3350 + c the producer's chunk c, 3420-3421 the reduction.
#if defined(INFINI_DELTA_TRACE) && defined(INFINI_ATTN_TRACE)
#define DELTA_TRACE(cond, slot)                                                                         \
  do {                                                                                                  \
    if ((cond) && blockIdx.x == INFINI_DELTA_TRACE && (slot) < 4096) g_attn_trace[(slot)] = clock64(); \
  } while (0)
#else
#define DELTA_TRACE(cond, slot) \
  do {                          \
  } while (0)
#endif

constexpr int kDChunk = 64;         // tokens per chunk
constexpr uint32_t kDBox = 8192;    // 64 rows x 128 B
constexpr uint32_t kDTile = 16384;  // 64 tokens x 128 bf16: two boxes
constexpr int kDeltaThreads = 608;  // 16 compute warps, a K-load warp, an MMA warp, a V-load warp

struct DeltaSmem {
  static constexpr int KST = 5;  // K ring (sigma(K)_hi in place): loaded -> chunk products done
  static constexpr int VST = 4;  // V ring: loaded -> chunk products done
  static constexpr int LST = 2;  // sigma_lo, S: sigma pass -> chunk products done
  static constexpr uint32_t K0 = 0;
  static constexpr uint32_t V0 = K0 + KST * kDTile;
  static constexpr uint32_t W0 = V0 + VST * kDTile;  // LST x [sigma_lo | S]
  static constexpr uint32_t END = W0 + LST * 2 * kDTile;  // end of the rings
  static constexpr uint32_t BAR = END;
  static constexpr uint32_t SLOT = BAR + 256u;
  static constexpr uint32_t BYTES = SLOT + 16u + 1024u;
  static_assert(BYTES <= 232448, "delta update kernel exceeds 227 KB of shared memory");
  // after the last chunk, over the rings: -G^T as bf16 hi and lo K-major
  // tiles (128 x 128, two 16 KB boxes each), the landing area of this CTA's
  // slice of the G partials (G x slice <= 4135 float4), the 16 warps' dz sums
  // (8 KB) and this CTA's partial [dM | dz] staged for sending (66,048 B),
  // before it M_{s-1} as bf16 hi and lo MN-major tiles (the A operand M^T of
  // the final product) in the same place
  static constexpr uint32_t GH = 0;
  static constexpr uint32_t GL = 32768u;
  static constexpr uint32_t LAND = 65536u;
  static constexpr uint32_t DZS = LAND + 66560u;
  static constexpr uint32_t RED = DZS + 16u * 128u * 4u;
  static constexpr uint32_t MH = RED;
  static constexpr uint32_t ML = RED + 32768u;
  static_assert(RED % 1024u == 0 && ML + 32768u <= RED + 66048u, "M tiles");
  static_assert(RED + 66048u <= END, "epilogue scratch must lie in the rings");
};

enum : int {
  D_KF = 0, D_KE = 5, D_VF = 10, D_VE = 14, D_LE = 18, D_SK = 20, D_ACC = 22, D_GR = 23, D_FIN = 24, D_RX = 25,
  D_COUNT = 26
};
constexpr int kDeltaE4 = (128 * 128 + 128) / 4;  // float4 elements of [M | z]

// 16-byte chunk c (0..15) of row r of a 64-row tile (two 8 KB boxes)
__device__ __forceinline__ uint32_t dswz(int r, int c) {
  return (uint32_t)(c >> 3) * kDBox + (uint32_t)r * 128u + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}
// MN-major operand of 64 K-rows (tokens) x 128 M/N columns, 16 tokens per step
__device__ __forceinline__ uint64_t dmn_desc(uint32_t tile, int kk) {
  return smem_desc_sw128(tile, kDBox, 1024u) + (uint64_t)((uint32_t)kk * (2048u >> 4));
}
// Rows of M owned by CTA grp of G for the snapshot: k with k * G / 128 = grp.
__device__ __forceinline__ int delta_row_lo(int grp, int G) { return (grp * 128 + G - 1) / G; }

// Snapshot rows [r_lo, r_hi) of M_{s-1} (bf16 for the attention; fp32 when
// asked, for the backward) and, from CTA 0, z_{s-1}, by `nthr` threads.
__device__ __forceinline__ void delta_snapshot(const UpdArgs& a, const float* Mh, int bh, int s, int grp, int tid,
                                               int nthr) {
  const int c_lo = 16 * delta_row_lo(grp, a.G), c_hi = 16 * delta_row_lo(grp + 1, a.G);  // 16-byte bf16 chunks
  __nv_bfloat16* snap = a.snapM + ((long long)bh * a.S + s) * 16384;
  for (int ch = c_lo + tid; ch < c_hi; ch += nthr) {
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
  if (grp == 0 && tid < 128 && a.snapzw != nullptr)
    a.snapzw[((long long)bh * a.S + s) * 128 + tid] = a.z[(long long)bh * 128 + tid];
}

// bf16 hi and lo parts of (x0, x1): hi = bf16(x), lo = bf16(x - hi)
__device__ __forceinline__ void split2(float x0, float x1, uint32_t& hi, uint32_t& lo) {
  hi = pack_bf16x2(x0, x1);
  float l0, l1;
  fma2(l0, l1, bf16_lo(hi), bf16_hi(hi), -1.f, -1.f, x0, x1);
  lo = pack_bf16x2(l0, l1);
}


__global__ void __launch_bounds__(kDeltaThreads, 1)
    delta_update_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                           const UpdArgs a) {
  using SL = DeltaSmem;
  constexpr int KST = SL::KST, VST = SL::VST, LST = SL::LST;
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
  const float* Mh = a.M + (long long)bh * 16384;
  const int per = (kDeltaE4 + a.G - 1) / a.G;  // float4 elements of [M | z] in a slice
  const int e4_begin = grp * per, e4_end = min(kDeltaE4, e4_begin + per);  // this CTA's slice
  auto has_tokens = [&](int g2) { return g2 * a.cpb * kTile < n_s; };   // CTA g2 of the head has chunks
  auto bar = [&](int i) { return base + SL::BAR + 8u * (uint32_t)i; };
  [[maybe_unused]] const bool t0 = threadIdx.x == 0;
  DELTA_TRACE(t0, 3200);
  if (threadIdx.x == 0) {
    // receive barrier: this CTA's slice from every other CTA of the head
    // with tokens, armed before this CTA's arrival on the cluster barrier
    // (peers copy only after it)
    int senders = 0;
    for (int g2 = 0; g2 < a.G; ++g2) senders += g2 != grp && has_tokens(g2);
    mbar_init(bar(D_RX), 1);
    fence_barrier_init();
    mbar_expect_tx(bar(D_RX), (uint32_t)(senders * (e4_end - e4_begin) * 16));
  }
  // Launched as a programmatic dependent of the previous segment's update,
  // whose outputs are M, z and their snapshots only: the next segment's grid
  // may start its setup and its K, V loads now; every read or write of M, z
  // and the snapshots comes after griddep_wait().
  griddep_launch_dependents();

  if (nch == 0) {
    // a group past the end of a short segment: its snapshot slice; it sends nothing
    griddep_wait();
    delta_snapshot(a, Mh, bh, s, grp, threadIdx.x, blockDim.x);
    cluster_arrive();
    cluster_wait();
  } else {
    auto sK = [&](int st) { return base + SL::K0 + (uint32_t)st * kDTile; };
    auto sV = [&](int st) { return base + SL::V0 + (uint32_t)st * kDTile; };
    auto sLo = [&](int st) { return base + SL::W0 + (uint32_t)(2 * st) * kDTile; };
    auto sS = [&](int st) { return base + SL::W0 + (uint32_t)(2 * st + 1) * kDTile; };
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + SL::SLOT);
    if (threadIdx.x == 0) {
      for (int i = 0; i < KST; ++i) {
        mbar_init(bar(D_KF + i), 1);
        mbar_init(bar(D_KE + i), 1);
      }
      for (int i = 0; i < VST; ++i) {
        mbar_init(bar(D_VF + i), 1);
        mbar_init(bar(D_VE + i), 1);
      }
      for (int i = 0; i < LST; ++i) {
        mbar_init(bar(D_LE + i), 1);
        mbar_init(bar(D_SK + i), 16);
      }
      mbar_init(bar(D_ACC), 1);
      mbar_init(bar(D_GR), 16);
      mbar_init(bar(D_FIN), 1);
      fence_barrier_init();
    }
    if (warp == 17) {
      tmem_alloc(smem_u32(tmem_slot), 256);
      tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    DELTA_TRACE(t0, 3202);
    // TMEM columns: VM^T (then dM^T) 0-127, G 128-255
    const uint32_t tVM = tmem, tG = tmem + 128u;

    if (warp == 16 || warp == 18) {
      // ------------------------------------------------------------ producers
      // warp 16 loads K, warp 18 V: the K ring runs ahead of the V ring, whose
      // stages the chunk products release later than the sigma pass needs
      // the next keys
      if (lane == 0) {
        const bool kw = warp == 16;
        const CUtensorMap* tm = kw ? &tm_k : &tm_v;
        const int nst = kw ? KST : VST;
        const int full = kw ? D_KF : D_VF, empty = kw ? D_KE : D_VE;
        const uint32_t ring = kw ? base + SL::K0 : base + SL::V0;
        prefetch_tensormap(tm);
        auto load_chunk = [&](int c) {
          const int lt = (int)(seg_start + t_begin + (long long)c * kDChunk);
          const int st = c % nst;
          if (c >= nst) mbar_wait_parked(bar(empty + st), ((c / nst) - 1) & 1);
          mbar_expect_tx(bar(full + st), kDTile);
          tma_load_4d(ring + (uint32_t)st * kDTile, tm, bar(full + st), 0, lt, h, b);
          tma_load_4d(ring + (uint32_t)st * kDTile + kDBox, tm, bar(full + st), 64, lt, h, b);
          DELTA_TRACE(!kw && c < 64, 3350 + c);
        };
        for (int c = 0; c < nch; ++c) load_chunk(c);
      }
      __syncwarp();
      if (warp == 18) {
        // idle until the end: bring M_{s-1} (read by the epilogue) into L2
        griddep_wait();
        for (int i = lane; i < 512; i += 32) prefetch_l2(Mh + 32 * i);
      }
      cluster_arrive();  // every load lands before the chunk products complete
      cluster_wait();
    } else if (warp == 17) {
      if (lane == 0) {
        // ---------------------------------------------------------- MMA issuer
        constexpr uint32_t idesc_c = idesc_bf16(128, 128, 1, 1);  // chunk products: A, B MN-major
        for (int c = 0; c < nch; ++c) {
          const int ks = c % KST, vs = c % VST, ls = c % LST;
          mbar_wait_parked(bar(D_SK + ls), (c / LST) & 1);
          mbar_wait_parked(bar(D_VF + vs), (c / VST) & 1);
          tc_fence_after();
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint32_t acc = (c > 0 || kk > 0) ? 1u : 0u;
            const uint64_t bH = dmn_desc(sK(ks), kk), bL = dmn_desc(sLo(ls), kk);
            const uint64_t aV = dmn_desc(sV(vs), kk), aS = dmn_desc(sS(ls), kk);
            mma_ss(tVM, aV, bH, idesc_c, acc);
            mma_ss(tVM, aV, bL, idesc_c, 1u);
            mma_ss(tG, aS, bH, idesc_c, acc);
          }
          mma_commit(bar(D_KE + ks));
          mma_commit(bar(D_VE + vs));
          mma_commit(bar(D_LE + ls));
          DELTA_TRACE(c < 64, 3280 + c);
        }
        mma_commit(bar(D_ACC));
      }
      __syncwarp();
      cluster_arrive();  // the rings are released by the compute warps' arrivals after ACC
      if (lane == 0) {
        constexpr uint32_t idesc_f = idesc_bf16(128, 128, 1, 0);  // final: A = M^T MN-major, B = -G^T K-major
        mbar_wait_parked(bar(D_GR), 0);
        tc_fence_after();
        const uint32_t gh = base + SL::GH, gl = base + SL::GL, mh = base + SL::MH, ml = base + SL::ML;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
          mma_ss(tVM, mnmajor_desc(mh, kk), kmajor_desc(gh, kk), idesc_f, 1u);
          mma_ss(tVM, mnmajor_desc(mh, kk), kmajor_desc(gl, kk), idesc_f, 1u);
          mma_ss(tVM, mnmajor_desc(ml, kk), kmajor_desc(gh, kk), idesc_f, 1u);
        }
        mma_commit(bar(D_FIN));
      }
      __syncwarp();
      cluster_wait();
    } else {
      // ------------------------------------------------------------ compute warps
      const int q = warp & 3, g = warp >> 2;
      const uint32_t lq = (uint32_t)(32 * q) << 16;  // this warp's TMEM lane quarter
      const int d = 32 * q + lane;                   // TMEM lane: a dv (M^T, dM^T) or dk (G) index
      // M_{s-1} is needed only by the final product: the chunks start as
      // soon as z_{s-1} (the previous segment's update) is available
      griddep_wait();
      if (grp == 0 && threadIdx.x < 128 && a.snapzw != nullptr)
        a.snapzw[((long long)bh * a.S + s) * 128 + threadIdx.x] = a.z[(long long)bh * 128 + threadIdx.x];
      DELTA_TRACE(t0, 3201);
      // sigma pass: row rr of the chunk, 16-byte chunks p (columns 8p..8p+7)
      // and 8 + p (columns 64 + 8p..)
      const int rr = 4 * warp + (lane >> 3), p = lane & 7;
      float zz[16], dz[16];
      {
        const float* zh = a.z + (long long)bh * 128;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          zz[i] = zh[64 * (i >> 3) + 8 * p + (i & 7)];
          dz[i] = 0.f;
        }
      }
      // ring stages and phase parities of chunk c, advanced incrementally
      int ks = 0, ls = 0;
      uint32_t kph = 0, lph = 0;
      for (int c = 0; c < nch; ++c) {
        mbar_wait_parked(bar(D_KF + ks), kph);
        DELTA_TRACE(t0 && c < 64, 3430 + c);
        uint4 w[2];
        w[0] = lds128(sK(ks) + dswz(rr, p));
        w[1] = lds128(sK(ks) + dswz(rr, 8 + p));
        // sigma = max(x, 0) + 2^(min(x, 0) log2 e), pairs of columns in f32x2
        float sg[16];
        float dp0 = 0.f, dp1 = 0.f;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          const uint32_t* wp = reinterpret_cast<const uint32_t*>(&w[i]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const int j = 8 * i + 2 * e;
            const float x0 = bf16_lo(wp[e]), x1 = bf16_hi(wp[e]);
            float m0, m1;
            mul2(m0, m1, fminf(x0, 0.f), fminf(x1, 0.f), 1.4426950408889634f, 1.4426950408889634f);
            add2(sg[j], sg[j + 1], fmaxf(x0, 0.f), fmaxf(x1, 0.f), ex2_approx(m0), ex2_approx(m1));
          }
        }
        if (t_begin + c * kDChunk + rr >= t_end) {  // a token past the segment's end (last chunk only)
#pragma unroll
          for (int j = 0; j < 16; ++j) sg[j] = 0.f;
        }
#pragma unroll
        for (int j = 0; j < 16; j += 2) {
          fma2(dp0, dp1, sg[j], sg[j + 1], zz[j], zz[j + 1], dp0, dp1);
          add2(dz[j], dz[j + 1], dz[j], dz[j + 1], sg[j], sg[j + 1]);
        }
        // den of the row: the 8 lanes of the row in a fixed butterfly (every lane gets the same sum)
        float dp = dp0 + dp1;
        dp += __shfl_xor_sync(0xffffffffu, dp, 1);
        dp += __shfl_xor_sync(0xffffffffu, dp, 2);
        dp += __shfl_xor_sync(0xffffffffu, dp, 4);
        const float rinv = dp != 0.f ? rcp_approx(dp) : 0.f;
        uint4 hi[2], lo[2], sv[2];
#pragma unroll
        for (int i = 0; i < 2; ++i) {
          uint32_t* hp = reinterpret_cast<uint32_t*>(&hi[i]);
          uint32_t* lp = reinterpret_cast<uint32_t*>(&lo[i]);
          uint32_t* sp = reinterpret_cast<uint32_t*>(&sv[i]);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = sg[8 * i + 2 * e], x1 = sg[8 * i + 2 * e + 1];
            hp[e] = pack_bf16x2(x0, x1);
            float l0, l1, s0, s1;
            fma2(l0, l1, bf16_lo(hp[e]), bf16_hi(hp[e]), -1.f, -1.f, x0, x1);
            lp[e] = pack_bf16x2(l0, l1);
            mul2(s0, s1, x0, x1, rinv, rinv);
            sp[e] = pack_bf16x2(s0, s1);
          }
        }
        sts128(sK(ks) + dswz(rr, p), hi[0]);
        sts128(sK(ks) + dswz(rr, 8 + p), hi[1]);
        if (c >= LST) mbar_wait_parked(bar(D_LE + ls), lph ^ 1u);  // products of chunk c - LST are done
        DELTA_TRACE(t0 && c < 64, 3500 + c);
        sts128(sLo(ls) + dswz(rr, p), lo[0]);
        sts128(sLo(ls) + dswz(rr, 8 + p), lo[1]);
        sts128(sS(ls) + dswz(rr, p), sv[0]);
        sts128(sS(ls) + dswz(rr, 8 + p), sv[1]);
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(bar(D_SK + ls));
        DELTA_TRACE(t0 && c < 64, 3210 + c);
        if (++ks == KST) {
          ks = 0;
          kph ^= 1u;
        }
        if (++ls == LST) {
          ls = 0;
          lph ^= 1u;
        }
      }
      mbar_wait_parked(bar(D_ACC), 0);
      tc_fence_after();
      __syncwarp();
      cluster_arrive();  // every load and chunk product of this CTA is complete: the rings are free
      DELTA_TRACE(t0, 3204);
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
      // M_{s-1} for the final product and the snapshot: 16-byte chunks
      // qq = tid + 512 i of the bf16 tiles (row k = qq / 16, columns
      // 8 (qq % 16) ..).  M is still M_{s-1}: no CTA of the head reduces
      // before this CTA's partial has reached it.
      float4 mv[8];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int qq = threadIdx.x + 512 * i;
        const float4* src = reinterpret_cast<const float4*>(Mh + (qq >> 4) * 128 + 8 * (qq & 15));
        mv[2 * i] = src[0];
        mv[2 * i + 1] = src[1];
      }
      // -G^T as the K-major B operand of the final product: row n = k holds
      // -G[k][k'] along k', i.e. TMEM lane k of G; this warp writes columns
      // 32g..32g+31
      {
        uint32_t rw[32];
        tmem_ld32(tG + lq + 32u * (uint32_t)g, rw);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint4 vh, vl;
          uint32_t* hp = reinterpret_cast<uint32_t*>(&vh);
          uint32_t* lp = reinterpret_cast<uint32_t*>(&vl);
#pragma unroll
          for (int e = 0; e < 4; ++e)
            split2(-__uint_as_float(rw[8 * i + 2 * e]), -__uint_as_float(rw[8 * i + 2 * e + 1]), hp[e], lp[e]);
          sts128(base + SL::GH + swz_chunk(d, 4 * g + i), vh);
          sts128(base + SL::GL + swz_chunk(d, 4 * g + i), vl);
        }
      }
      // M^T as the MN-major A operand: row k of M, columns d contiguous, in
      // hi and lo tiles; this CTA's rows of the snapshot from the same values
      {
        const int r_lo = delta_row_lo(grp, a.G), r_hi = delta_row_lo(grp + 1, a.G);
        __nv_bfloat16* snap = a.snapM + ((long long)bh * a.S + s) * 16384;
        float* snap32 = a.snapM32 + ((long long)bh * a.S + s) * 16384;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int qq = threadIdx.x + 512 * i, k = qq >> 4, cc = qq & 15;
          const float4 f0 = mv[2 * i], f1 = mv[2 * i + 1];
          uint4 vh, vl;
          split2(f0.x, f0.y, vh.x, vl.x);
          split2(f0.z, f0.w, vh.y, vl.y);
          split2(f1.x, f1.y, vh.z, vl.z);
          split2(f1.z, f1.w, vh.w, vl.w);
          sts128(base + SL::MH + swz_chunk(k, cc), vh);
          sts128(base + SL::ML + swz_chunk(k, cc), vl);
          if (k >= r_lo && k < r_hi) {
            if (a.snapM != nullptr) *reinterpret_cast<uint4*>(snap + k * 128 + 8 * cc) = vh;
            if (a.snapM32 != nullptr) {
              reinterpret_cast<float4*>(snap32 + k * 128 + 8 * cc)[0] = f0;
              reinterpret_cast<float4*>(snap32 + k * 128 + 8 * cc)[1] = f1;
            }
          }
        }
      }
      fence_proxy_async_smem();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(bar(D_GR));
      DELTA_TRACE(t0, 3205);
      named_bar_sync(1, 512);
      float dzt = 0.f;
      if (threadIdx.x < 128)
        for (int w2 = 0; w2 < 16; ++w2) dzt += dzs[w2 * 128 + threadIdx.x];
      DELTA_TRACE(t0, 3206);
      // dM[k][d] = dM^T[d][k]: lane d, columns k = 32g..32g+31, staged in
      // this CTA's shared memory as [dM | dz]
      mbar_wait_parked(bar(D_FIN), 0);
      tc_fence_after();
      float* red = reinterpret_cast<float*>(gbase + SL::RED);
      {
        uint32_t rw[32];
        tmem_ld32(tVM + lq + 32u * (uint32_t)g, rw);
        tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < 32; ++j) red[(32 * g + j) * 128 + d] = __uint_as_float(rw[j]);
        if (threadIdx.x < 128) red[16384 + threadIdx.x] = dzt;
      }
      fence_proxy_async_smem();  // the bulk copies read the staged partial
      named_bar_sync(1, 512);
      DELTA_TRACE(t0, 3207);
      cluster_wait();  // every CTA of the cluster is past its chunks: its landing area is free
      DELTA_TRACE(t0, 3208);
      // slice r of the partial to CTA r (slot grp of its landing area); this
      // CTA's own slice stays in place
      const int r = threadIdx.x;
      if (r < a.G && r != grp) {
        const int len = min(per, kDeltaE4 - r * per);
        bulk_copy_to_peer(mapa_shared(base + SL::LAND + 16u * (uint32_t)(grp * per), (uint32_t)r),
                          base + SL::RED + 16u * (uint32_t)(r * per), (uint32_t)(16 * len),
                          mapa_shared(bar(D_RX), (uint32_t)r));
        bulk_commit();
        bulk_wait_read();  // the source stays valid until it has been read
      }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 17) {
      __syncwarp();
      tc_fence_after();
      tmem_dealloc(tmem, 256);
    }
  }
  // ------------------------------------------------------------ cluster reduction
  // This CTA's slice of M, z (no other CTA writes it) is loaded while the
  // partials land: at most 7 float4 per thread (a slice of <= 4128 float4).
  auto state4 = [&](int e4) {
    const int e = 4 * e4;
    return e < 16384 ? reinterpret_cast<float4*>(&a.M[(long long)bh * 16384 + e])
                     : reinterpret_cast<float4*>(&a.z[(long long)bh * 128 + (e - 16384)]);
  };
  constexpr int kIt = (kDeltaE4 + kDeltaThreads - 1) / kDeltaThreads;
  float4 acc[kIt];
  griddep_wait();  // (complete long since for the threads that read M above)
#pragma unroll
  for (int it = 0; it < kIt; ++it) {
    const int e4 = e4_begin + (int)threadIdx.x + it * kDeltaThreads;
    if (e4 < e4_end) acc[it] = *state4(e4);
  }
  mbar_wait_parked(bar(D_RX), 0);  // every other CTA's partial of this slice has landed
  DELTA_TRACE(t0, 3209);
  {
    const float4* lf = reinterpret_cast<const float4*>(gbase + SL::LAND);
    const float4* own = reinterpret_cast<const float4*>(gbase + SL::RED);  // this CTA's partial (nch > 0)
#pragma unroll
    for (int it = 0; it < kIt; ++it) {
      const int e4 = e4_begin + (int)threadIdx.x + it * kDeltaThreads;
      if (e4 < e4_end) {
        for (int g2 = 0; g2 < a.G; ++g2) {
          if (g2 == grp ? nch == 0 : !has_tokens(g2)) continue;
          const float4 v = g2 != grp ? lf[g2 * per + (e4 - e4_begin)] : own[e4];
          acc[it].x += v.x;
          acc[it].y += v.y;
          acc[it].z += v.z;
          acc[it].w += v.w;
        }
        *state4(e4) = acc[it];
      }
    }
  }
  DELTA_TRACE(t0, 3420);
}

}  // namespace tc
}  // namespace infini
