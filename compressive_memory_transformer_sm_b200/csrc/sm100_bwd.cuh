// Tensor-core (tcgen05 / TMEM / TMA) kernels of the backward pass for bf16
// tensors with d_key = d_value = 128: the local attention's gradients (Eq. 6)
//
//   P = 2^(c' S - lse2) with S = Q K^T, c' = scale * log2(e), lse2 the row's
//   log2-sum-exp2 from the forward;  dP' = dO V^T;  D'_i = dO_i . A_dot_i;
//   dS' = P (dP' - D');  dQ = scale (1 - g) dS' K;  dK = scale (1 - g) dS'^T Q;
//   dV = (1 - g) P^T dO
//
// (the gate's (1 - g) of d_dot = (1 - g) dA is applied once, at the end), each
// kernel adding the memory terms computed on CUDA cores (dq_mem; dk_upd,
// dv_upd) before its single bf16 store.
//
// Both kernels: one CTA per work tile, 192 threads -- warps 0-3 a compute
// warpgroup (thread = tile row = TMEM lane), warp 4 loads (TMA, 128-byte
// swizzle), warp 5 issues the MMAs (one elected lane) and owns the 512 TMEM
// columns.  P and dS are packed to bf16 in place over the fp32 tile they are
// computed from (chunk c of 32 columns is read before its 16 packed columns
// are written, and chunk c writes only columns chunks <= c have read) and feed
// the next products from TMEM as the A operand.  Every wait is bounded.
#pragma once

#include "sm100_common.cuh"

namespace infini {
namespace tc {

struct BwdTcArgs {
  const float* lse2;     // [BH*L]
  const float* Dp;       // [BH*L]: dO_i . A_dot_i
  const float* beta;
  const float* mem_q;    // dq kernel: [BH*L][128] fp32 dq_mem
  const float* mem_k;    // dkdv kernel: [BH*L][128] fp32 dk_upd
  const float* mem_v;    // dkdv kernel: [BH*L][128] fp32 dv_upd
  __nv_bfloat16* out0;   // dq, or dk
  __nv_bfloat16* out1;   // dv
  int B, H, S, T;        // T: 128-row tiles per full segment
  long long L;
  int N;
  float scale, scale_log2;
};

constexpr int kBwdThreads = 192;
constexpr uint32_t kBT = 32768;  // one 128 x 128 bf16 tile (two 64-column boxes)

// ---------------------------------------------------------------- dQ
// Work tile: query tile t of (b, h, segment s); key tiles j = 0 .. t.
// TMEM: S [0, 128), dP of key tile j in [128 + 128 (j & 1), ...), dQ [384, 512).
// Shared memory: Q, dO, a 2-stage K ring, a 2-stage V ring.
enum : int { DQ_QD = 0, DQ_KF0 = 1, DQ_KE0 = 3, DQ_VF0 = 5, DQ_VE0 = 7, DQ_SF = 9, DQ_SE = 10, DQ_PF0 = 11,
             DQ_DSF0 = 13, DQ_DONE = 15, DQ_COUNT = 16 };
constexpr uint32_t kDQ_Q = 0, kDQ_DO = kBT, kDQ_K0 = 2 * kBT, kDQ_V0 = 4 * kBT, kDQ_BAR = 6 * kBT;
constexpr uint32_t kDQ_SLOT = kDQ_BAR + 8 * DQ_COUNT;
constexpr uint32_t kDQSmem = kDQ_SLOT + 16 + 1024;
static_assert(kDQSmem <= 232448, "dq kernel exceeds 227 KB of shared memory");

__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dq_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                     const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                     const BwdTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NS = a.B * a.H * a.S;
  const int t = a.T - 1 - (int)(blockIdx.x / NS);  // heaviest tiles first
  const int seg = (int)(blockIdx.x % NS);
  const int bh = seg / a.S, s = seg % a.S;
  const int b = bh / a.H, h = bh % a.H;
  const long long seg0 = (long long)s * a.N;
  const int n_s = (int)min((long long)a.N, a.L - seg0);
  if (t * 128 >= n_s) return;
  const int nk = t + 1;
  auto bar = [&](int i) { return base + kDQ_BAR + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kDQ_SLOT);
  if (threadIdx.x == 0) {
    mbar_init(bar(DQ_QD), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(DQ_KF0 + i), 1);
      mbar_init(bar(DQ_KE0 + i), 1);
      mbar_init(bar(DQ_VF0 + i), 1);
      mbar_init(bar(DQ_VE0 + i), 1);
      mbar_init(bar(DQ_PF0 + i), 1);
      mbar_init(bar(DQ_DSF0 + i), 128);
    }
    mbar_init(bar(DQ_SF), 1);
    mbar_init(bar(DQ_SE), 128);
    mbar_init(bar(DQ_DONE), 1);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int row0 = (int)(seg0 + (long long)t * 128);

  if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      prefetch_tensormap(&tm_do);
      int issued = 0;
      mbar_expect_tx(bar(DQ_QD), 2 * kBT);
      tma_load_4d(base + kDQ_Q, &tm_q, bar(DQ_QD), 0, row0, h, b);
      tma_load_4d(base + kDQ_Q + kBox, &tm_q, bar(DQ_QD), 64, row0, h, b);
      tma_load_4d(base + kDQ_DO, &tm_do, bar(DQ_QD), 0, row0, h, b);
      tma_load_4d(base + kDQ_DO + kBox, &tm_do, bar(DQ_QD), 64, row0, h, b);
      for (int j = 0; j < nk; ++j) {
        const int st = j & 1;
        const uint32_t ph = (uint32_t)((j >> 1) & 1);
        if (!mbar_wait(bar(DQ_KE0 + st), ph ^ 1u) || !mbar_wait(bar(DQ_VE0 + st), ph ^ 1u)) break;
        const int kr = (int)(seg0 + (long long)j * 128);
        const uint32_t sk = base + kDQ_K0 + (uint32_t)st * kBT, sv = base + kDQ_V0 + (uint32_t)st * kBT;
        mbar_expect_tx(bar(DQ_KF0 + st), kBT);
        tma_load_4d(sk, &tm_k, bar(DQ_KF0 + st), 0, kr, h, b);
        tma_load_4d(sk + kBox, &tm_k, bar(DQ_KF0 + st), 64, kr, h, b);
        mbar_expect_tx(bar(DQ_VF0 + st), kBT);
        tma_load_4d(sv, &tm_v, bar(DQ_VF0 + st), 0, kr, h, b);
        tma_load_4d(sv + kBox, &tm_v, bar(DQ_VF0 + st), 64, kr, h, b);
        issued = j + 1;
      }
      if (device_aborted()) {
        // a wait gave up: let the copies still in flight land before the CTA exits
        mbar_drain(bar(DQ_QD), 0);
        for (int j = max(0, issued - 2); j < issued; ++j) {
          mbar_drain(bar(DQ_KF0 + (j & 1)), (uint32_t)((j >> 1) & 1));
          mbar_drain(bar(DQ_VF0 + (j & 1)), (uint32_t)((j >> 1) & 1));
        }
      }
    }
  } else if (warp == 5) {
    // -------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc_kk = idesc_bf16(128, 128, 0, 0);  // A, B K-major
    constexpr uint32_t idesc_ts = idesc_bf16(128, 128, 0, 1);  // A from TMEM, B MN-major
    const uint32_t tS = tmem, tDQ = tmem + 384;
    auto tP = [&](int j) { return tmem + 128u + 128u * (uint32_t)(j & 1); };
    auto sK = [&](int j) { return base + kDQ_K0 + (uint32_t)(j & 1) * kBT; };
    auto sV = [&](int j) { return base + kDQ_V0 + (uint32_t)(j & 1) * kBT; };
    bool ok = mbar_wait(bar(DQ_QD), 0);
    // dQ += dS(j) K(j): A = dS (bf16, TMEM columns 0-63 of dP(j)), B = K(j) MN-major
    auto issue_dq = [&](int j) {
      if (!mbar_wait(bar(DQ_DSF0 + (j & 1)), (uint32_t)((j >> 1) & 1))) return false;
      tc_fence_after();
      const uint64_t db = mnmajor_base(sK(j));
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tDQ, tP(j) + (uint32_t)kk * 8u, db + mnmajor_step(kk), idesc_ts, (j > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar(DQ_KE0 + (j & 1)));
      }
      __syncwarp();
      return true;
    };
    for (int j = 0; ok && j < nk; ++j) {
      const uint32_t ph = (uint32_t)((j >> 1) & 1);
      ok = mbar_wait(bar(DQ_KF0 + (j & 1)), ph) && mbar_wait(bar(DQ_VF0 + (j & 1)), ph);
      if (ok && j > 0) ok = mbar_wait(bar(DQ_SE), (uint32_t)((j - 1) & 1));  // S(j-1) read out
      if (!ok) break;
      tc_fence_after();
      {
        const uint64_t da = kmajor_base(base + kDQ_Q), db = kmajor_base(sK(j));
        const uint64_t da2 = kmajor_base(base + kDQ_DO), db2 = kmajor_base(sV(j));
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tS, da + kmajor_step(kk), db + kmajor_step(kk), idesc_kk, kk > 0 ? 1u : 0u);
          mma_commit(bar(DQ_SF));
          // dP(j) overwrites dS(j-2), which dQ(j-2), issued earlier, has consumed
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tP(j), da2 + kmajor_step(kk), db2 + kmajor_step(kk), idesc_kk, kk > 0 ? 1u : 0u);
          mma_commit(bar(DQ_PF0 + (j & 1)));
          mma_commit(bar(DQ_VE0 + (j & 1)));
        }
        __syncwarp();
      }
      if (j > 0) ok = issue_dq(j - 1);
    }
    if (ok) ok = issue_dq(nk - 1);
    // every product issued has completed before the epilogue reads dQ and TMEM is released
    if (elect_one()) mma_commit(bar(DQ_DONE));
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- compute warpgroup
    const int row = warp * 32 + lane;  // query row in the tile = TMEM lane
    const uint32_t lrow = (uint32_t)(warp * 32) << 16;
    const int qrow = t * 128 + row;
    const bool valid = qrow < n_s;
    const long long grow = (long long)bh * a.L + seg0 + qrow;
    const float lse = valid ? a.lse2[grow] : 0.f;
    const float Dv = valid ? a.Dp[grow] : 0.f;
    const float c = a.scale_log2;
    bool ok = true;
    for (int j = 0; j < nk && ok; ++j) {
      ok = mbar_wait(bar(DQ_SF), (uint32_t)(j & 1)) && mbar_wait(bar(DQ_PF0 + (j & 1)), (uint32_t)((j >> 1) & 1));
      if (!ok) break;
      tc_fence_after();
      const uint32_t tS = tmem + lrow, tP = tmem + lrow + 128u + 128u * (uint32_t)(j & 1);
      const bool diag = j == t;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sv[32], pv[32];
        tmem_ld32(tS + 32u * cc, sv);
        tmem_ld32(tP + 32u * cc, pv);
        tmem_ld_wait();
        if (cc == 3) {  // all of S(j) is in registers: S(j + 1) may be issued
          tc_fence_before();
          mbar_arrive(bar(DQ_SE));
        }
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float d[2];
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const int key = 32 * cc + 2 * e + x;  // key inside the tile
            const float p = (diag && key > row) ? 0.f : ex2_approx(__uint_as_float(sv[2 * e + x]) * c - lse);
            d[x] = p * (__uint_as_float(pv[2 * e + x]) - Dv);
          }
          w[e] = pack_bf16x2(d[0], d[1]);
        }
        tmem_st16(tP + 16u * cc, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(DQ_DSF0 + (j & 1)));
    }
    if (ok && mbar_wait(bar(DQ_DONE), 0)) {
      tc_fence_after();
      const float gw = 1.f / (1.f + __expf(-a.beta[h]));
      const float f = a.scale * (1.f - gw);
      const float4* mq = reinterpret_cast<const float4*>(a.mem_q + grow * 128);
      uint4* dst = reinterpret_cast<uint4*>(a.out0 + grow * 128);
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t r[32];
        tmem_ld32(tmem + lrow + 384u + 32u * cc, r);
        tmem_ld_wait();
        if (valid) {
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float4 m0 = mq[8 * cc + 2 * e], m1 = mq[8 * cc + 2 * e + 1];
            dst[4 * cc + e] = make_uint4(
                pack_bf16x2(f * __uint_as_float(r[8 * e]) + m0.x, f * __uint_as_float(r[8 * e + 1]) + m0.y),
                pack_bf16x2(f * __uint_as_float(r[8 * e + 2]) + m0.z, f * __uint_as_float(r[8 * e + 3]) + m0.w),
                pack_bf16x2(f * __uint_as_float(r[8 * e + 4]) + m1.x, f * __uint_as_float(r[8 * e + 5]) + m1.y),
                pack_bf16x2(f * __uint_as_float(r[8 * e + 6]) + m1.z, f * __uint_as_float(r[8 * e + 7]) + m1.w));
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    if (elect_one()) mbar_drain(bar(DQ_DONE), 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// ---------------------------------------------------------------- dK, dV
// Work tile: key tile j of (b, h, segment s); query tiles i = j .. nq - 1.
// TMEM: S^T [0, 128), dP^T [128, 256), dV [256, 384), dK [384, 512).
// Shared memory: K, V, a 2-stage Q ring, a 2-stage dO ring, and the query
// tile's lse2 and D' (two buffers).  MMA order per query tile u:
// S^T(u), dK(u - 1), dP^T(u), dV(u): the P pass of u overlaps dK(u - 1) and
// dP^T(u), the dS pass of u overlaps dV(u) and S^T(u + 1).
enum : int { KV_KV = 0, KV_QF0 = 1, KV_QE0 = 3, KV_OF0 = 5, KV_OE0 = 7, KV_SF = 9, KV_PW = 10, KV_PF = 11,
             KV_DSF = 12, KV_DONE = 13, KV_COUNT = 14 };
constexpr uint32_t kKV_K = 0, kKV_V = kBT, kKV_Q0 = 2 * kBT, kKV_O0 = 4 * kBT, kKV_LD = 6 * kBT;
constexpr uint32_t kKV_BAR = kKV_LD + 2048;
constexpr uint32_t kKV_SLOT = kKV_BAR + 8 * KV_COUNT;
constexpr uint32_t kKVSmem = kKV_SLOT + 16 + 1024;
static_assert(kKVSmem <= 232448, "dk/dv kernel exceeds 227 KB of shared memory");

__global__ void __launch_bounds__(kBwdThreads, 1)
    bwd_dkdv_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                       const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                       const BwdTcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int NS = a.B * a.H * a.S;
  const int jt = (int)(blockIdx.x / NS);  // key tile: the low ones have the most query tiles, they go first
  const int seg = (int)(blockIdx.x % NS);
  const int bh = seg / a.S, s = seg % a.S;
  const int b = bh / a.H, h = bh % a.H;
  const long long seg0 = (long long)s * a.N;
  const int n_s = (int)min((long long)a.N, a.L - seg0);
  if (jt * 128 >= n_s) return;
  const int nq = (n_s + 127) / 128;
  const int nu = nq - jt;  // query tiles jt .. nq - 1
  auto bar = [&](int i) { return base + kKV_BAR + 8u * (uint32_t)i; };
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kKV_SLOT);
  float* ld = reinterpret_cast<float*>(gbase + kKV_LD);  // [2 buffers][lse2 128 | D' 128]
  if (threadIdx.x == 0) {
    mbar_init(bar(KV_KV), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(KV_QF0 + i), 1);
      mbar_init(bar(KV_QE0 + i), 1);
      mbar_init(bar(KV_OF0 + i), 1);
      mbar_init(bar(KV_OE0 + i), 1);
    }
    mbar_init(bar(KV_SF), 1);
    mbar_init(bar(KV_PW), 128);
    mbar_init(bar(KV_PF), 1);
    mbar_init(bar(KV_DSF), 128);
    mbar_init(bar(KV_DONE), 1);
    fence_barrier_init();
  }
  if (warp == 5) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const int krow0 = (int)(seg0 + (long long)jt * 128);

  if (warp == 4) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      prefetch_tensormap(&tm_do);
      int issued = 0;
      mbar_expect_tx(bar(KV_KV), 2 * kBT);
      tma_load_4d(base + kKV_K, &tm_k, bar(KV_KV), 0, krow0, h, b);
      tma_load_4d(base + kKV_K + kBox, &tm_k, bar(KV_KV), 64, krow0, h, b);
      tma_load_4d(base + kKV_V, &tm_v, bar(KV_KV), 0, krow0, h, b);
      tma_load_4d(base + kKV_V + kBox, &tm_v, bar(KV_KV), 64, krow0, h, b);
      for (int u = 0; u < nu; ++u) {
        const int st = u & 1;
        const uint32_t ph = (uint32_t)((u >> 1) & 1);
        if (!mbar_wait(bar(KV_QE0 + st), ph ^ 1u) || !mbar_wait(bar(KV_OE0 + st), ph ^ 1u)) break;
        const int qr = (int)(seg0 + (long long)(jt + u) * 128);
        const uint32_t sq = base + kKV_Q0 + (uint32_t)st * kBT, so = base + kKV_O0 + (uint32_t)st * kBT;
        mbar_expect_tx(bar(KV_QF0 + st), kBT);
        tma_load_4d(sq, &tm_q, bar(KV_QF0 + st), 0, qr, h, b);
        tma_load_4d(sq + kBox, &tm_q, bar(KV_QF0 + st), 64, qr, h, b);
        mbar_expect_tx(bar(KV_OF0 + st), kBT);
        tma_load_4d(so, &tm_do, bar(KV_OF0 + st), 0, qr, h, b);
        tma_load_4d(so + kBox, &tm_do, bar(KV_OF0 + st), 64, qr, h, b);
        issued = u + 1;
      }
      if (device_aborted()) {
        mbar_drain(bar(KV_KV), 0);
        for (int u = max(0, issued - 2); u < issued; ++u) {
          mbar_drain(bar(KV_QF0 + (u & 1)), (uint32_t)((u >> 1) & 1));
          mbar_drain(bar(KV_OF0 + (u & 1)), (uint32_t)((u >> 1) & 1));
        }
      }
    }
  } else if (warp == 5) {
    // -------------------------------------------------------------- MMA issuer
    constexpr uint32_t idesc_kk = idesc_bf16(128, 128, 0, 0);
    constexpr uint32_t idesc_ts = idesc_bf16(128, 128, 0, 1);
    const uint32_t tS = tmem, tP = tmem + 128, tDV = tmem + 256, tDK = tmem + 384;
    auto sQ = [&](int u) { return base + kKV_Q0 + (uint32_t)(u & 1) * kBT; };
    auto sO = [&](int u) { return base + kKV_O0 + (uint32_t)(u & 1) * kBT; };
    // dK += dS^T(u) Q(u): A = dS^T (bf16 in dP^T's columns 0-63), B = Q(u) MN-major
    auto issue_dk = [&](int u) {
      if (!mbar_wait(bar(KV_DSF), (uint32_t)(u & 1))) return false;
      tc_fence_after();
      const uint64_t db = mnmajor_base(sQ(u));
      if (elect_one()) {
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tDK, tP + (uint32_t)kk * 8u, db + mnmajor_step(kk), idesc_ts, (u > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar(KV_QE0 + (u & 1)));
      }
      __syncwarp();
      return true;
    };
    bool ok = mbar_wait(bar(KV_KV), 0);
    for (int u = 0; ok && u < nu; ++u) {
      const uint32_t ph = (uint32_t)((u >> 1) & 1);
      ok = mbar_wait(bar(KV_QF0 + (u & 1)), ph) && mbar_wait(bar(KV_OF0 + (u & 1)), ph);
      if (!ok) break;
      tc_fence_after();
      // S^T(u) = K Q(u)^T (overwrites P^T(u - 1), which dV(u - 1), issued earlier, consumed)
      {
        const uint64_t da = kmajor_base(base + kKV_K), db = kmajor_base(sQ(u));
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tS, da + kmajor_step(kk), db + kmajor_step(kk), idesc_kk, kk > 0 ? 1u : 0u);
          mma_commit(bar(KV_SF));
        }
        __syncwarp();
      }
      if (u > 0 && !(ok = issue_dk(u - 1))) break;
      // dP^T(u) = V dO(u)^T (overwrites dS^T(u - 1), consumed by dK(u - 1) just issued)
      {
        const uint64_t da = kmajor_base(base + kKV_V), db = kmajor_base(sO(u));
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ss(tP, da + kmajor_step(kk), db + kmajor_step(kk), idesc_kk, kk > 0 ? 1u : 0u);
          mma_commit(bar(KV_PF));
        }
        __syncwarp();
      }
      // dV += P^T(u) dO(u) once P^T(u) is packed
      if (!(ok = mbar_wait(bar(KV_PW), (uint32_t)(u & 1)))) break;
      tc_fence_after();
      {
        const uint64_t db = mnmajor_base(sO(u));
        if (elect_one()) {
#pragma unroll
          for (int kk = 0; kk < 8; ++kk)
            mma_ts(tDV, tS + (uint32_t)kk * 8u, db + mnmajor_step(kk), idesc_ts, (u > 0 || kk > 0) ? 1u : 0u);
          mma_commit(bar(KV_OE0 + (u & 1)));
        }
        __syncwarp();
      }
    }
    if (ok) ok = issue_dk(nu - 1);
    if (elect_one()) mma_commit(bar(KV_DONE));
    __syncwarp();
  } else {
    // ---------------------------------------------------------------- compute warpgroup
    const int row = warp * 32 + lane;  // key row in the tile = TMEM lane
    const uint32_t lrow = (uint32_t)(warp * 32) << 16;
    const int krow = jt * 128 + row;
    const float c = a.scale_log2;
    bool ok = true;
    for (int u = 0; u < nu && ok; ++u) {
      const int qt = jt + u;
      float* ldb = ld + 256 * (u & 1);
      {
        // lse2 and D' of the query tile's rows (rows past the segment: masked below)
        const int qr = qt * 128 + row;
        const long long g = (long long)bh * a.L + seg0 + qr;
        ldb[row] = qr < n_s ? a.lse2[g] : 0.f;
        ldb[128 + row] = qr < n_s ? a.Dp[g] : 0.f;
        named_bar_sync(1, 128);
      }
      const int qlim = n_s - qt * 128;  // query columns < qlim are real
      const bool diag = u == 0;
      if (!(ok = mbar_wait(bar(KV_SF), (uint32_t)(u & 1)))) break;
      tc_fence_after();
      uint32_t pk[64];  // P^T(u) of this key row, bf16 pairs
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t sv[32];
        tmem_ld32(tmem + lrow + 32u * cc, sv);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float p[2];
#pragma unroll
          for (int x = 0; x < 2; ++x) {
            const int qi = 32 * cc + 2 * e + x;  // query column inside the tile
            const bool live = qi < qlim && !(diag && qi < row);
            p[x] = live ? ex2_approx(__uint_as_float(sv[2 * e + x]) * c - ldb[qi]) : 0.f;
          }
          pk[16 * cc + e] = pack_bf16x2(p[0], p[1]);
        }
        tmem_st16(tmem + lrow + 16u * cc, *reinterpret_cast<uint32_t(*)[16]>(&pk[16 * cc]));
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(KV_PW));
      if (!(ok = mbar_wait(bar(KV_PF), (uint32_t)(u & 1)))) break;
      tc_fence_after();
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t dv[32];
        tmem_ld32(tmem + lrow + 128u + 32u * cc, dv);
        tmem_ld_wait();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int qi = 32 * cc + 2 * e;
          const uint32_t pw = pk[16 * cc + e];
          const float d0 = bf16_lo(pw) * (__uint_as_float(dv[2 * e]) - ldb[128 + qi]);
          const float d1 = bf16_hi(pw) * (__uint_as_float(dv[2 * e + 1]) - ldb[128 + qi + 1]);
          w[e] = pack_bf16x2(d0, d1);
        }
        tmem_st16(tmem + lrow + 128u + 16u * cc, w);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(KV_DSF));
    }
    if (ok && mbar_wait(bar(KV_DONE), 0)) {
      tc_fence_after();
      const float gw = 1.f / (1.f + __expf(-a.beta[h]));
      const bool valid = krow < n_s;
      const long long grow = (long long)bh * a.L + seg0 + krow;
      // dv = (1 - g) P^T dO + dv_upd, dk = scale (1 - g) dS'^T Q + dk_upd
#pragma unroll 1
      for (int which = 0; which < 2; ++which) {
        const float f = which ? (1.f - gw) : a.scale * (1.f - gw);
        const float4* mm = reinterpret_cast<const float4*>((which ? a.mem_v : a.mem_k) + grow * 128);
        uint4* dst = reinterpret_cast<uint4*>((which ? a.out1 : a.out0) + grow * 128);
        const uint32_t tacc = tmem + lrow + (which ? 256u : 384u);
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t r[32];
          tmem_ld32(tacc + 32u * cc, r);
          tmem_ld_wait();
          if (valid) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float4 m0 = mm[8 * cc + 2 * e], m1 = mm[8 * cc + 2 * e + 1];
              dst[4 * cc + e] = make_uint4(
                  pack_bf16x2(f * __uint_as_float(r[8 * e]) + m0.x, f * __uint_as_float(r[8 * e + 1]) + m0.y),
                  pack_bf16x2(f * __uint_as_float(r[8 * e + 2]) + m0.z, f * __uint_as_float(r[8 * e + 3]) + m0.w),
                  pack_bf16x2(f * __uint_as_float(r[8 * e + 4]) + m1.x, f * __uint_as_float(r[8 * e + 5]) + m1.y),
                  pack_bf16x2(f * __uint_as_float(r[8 * e + 6]) + m1.z, f * __uint_as_float(r[8 * e + 7]) + m1.w));
            }
          }
        }
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    if (elect_one()) mbar_drain(bar(KV_DONE), 0);
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace infini
