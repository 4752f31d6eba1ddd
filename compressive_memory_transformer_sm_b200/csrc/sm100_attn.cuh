// attn_tc_kernel: A_dot (Eq. 6) + A_mem (Eq. 7) + gate (Eq. 10) of the
// Infini-attention forward, fused, on the sm_100a tensor cores: one CTA per
// (b, h, segment, pair of 128-row query tiles).
#pragma once

#include "sm100_common.cuh"

// Softmax tuning knobs (compile time): every INFINI_POLY_EVERY-th pair of
// exponentials runs on the FMA pipe (0 = none), and P is packed to bf16 on the
// integer pipe when INFINI_PACK_ALU is 1.
#ifndef INFINI_POLY_EVERY
#define INFINI_POLY_EVERY 0
#endif
#ifndef INFINI_PACK_ALU
#define INFINI_PACK_ALU 0
#endif
// 1: scale-and-subtract and the row sum use packed fp32x2 instructions.
#ifndef INFINI_F32X2
#define INFINI_F32X2 1
#endif

namespace infini {
namespace tc {

// Pipeline timestamps of one CTA (block INFINI_ATTN_TRACE) for tuning builds:
// slot = 8 * (tile) + event; softmax warpgroup k writes at 1024 * k, the MMA
// thread at 2048.  Compiled out unless INFINI_ATTN_TRACE is defined.
#ifdef INFINI_ATTN_TRACE
__device__ unsigned long long g_attn_trace[4096];
#define ATTN_TRACE(cond, slot)                                                                   \
  do {                                                                                           \
    if ((cond) && blockIdx.x == INFINI_ATTN_TRACE && (slot) < 4096) g_attn_trace[(slot)] = clock64(); \
  } while (0)
#else
#define ATTN_TRACE(cond, slot) \
  do {                         \
  } while (0)
#endif

struct AttnArgs {
  const float* beta;
  const float* snapz;     // [BH][S][128] fp32: z_{s-1}
  __nv_bfloat16* out;
  int B, H, S, T;         // T = query tiles per full segment
  int P;                  // work items per full segment: ceil(T / 2) pairs, or T tiles when `single`
  int GS;                 // segments per scheduling group
  int single;             // 1: one query tile per CTA (small grids), warpgroup 1 idle
  long long L;
  int N;
  float scale_log2;       // softmax scale * log2(e)
  long long os[3];        // element strides of out
};

// Shared memory of the attention kernel (offsets from a 1024-aligned base).
constexpr int kKStages = 3;          // K ring depth (V ring: 2)
constexpr uint32_t kA_Q0 = 0;
constexpr uint32_t kA_Q1 = 32768;
constexpr uint32_t kA_K0 = 65536;    // K ring: 3 stages of 32 KB
constexpr uint32_t kA_V0 = kA_K0 + kKStages * 32768u;  // V ring: 2 stages of 32 KB
constexpr uint32_t kA_Z = kA_V0 + 2 * 32768u;  // z_{s-1}, one copy per softmax warpgroup
constexpr uint32_t kA_BAR = kA_Z + 1024;
constexpr int kAttnThreads = 384;
// Register split: the kernel launches with 168 registers per thread (384 x 168
// = 64512); the load/MMA warpgroup gives back to 88 and the two softmax
// warpgroups take 208: 2 x 128 x 208 + 128 x 88 = 64512 (the split with no
// spills on either side).  The build checks
// that ptxas allocated exactly kAttnLaunchRegs, else an increase could wait
// forever.
constexpr uint32_t kAttnLaunchRegs = 168, kAttnSoftmaxRegs = 208, kAttnOtherRegs = 88;
static_assert(2 * 128 * kAttnSoftmaxRegs + 128 * kAttnOtherRegs == kAttnThreads * kAttnLaunchRegs,
              "register split must add up to the launch allocation");

// Barrier indices.
enum : int {
  B_Q = 0,
  B_KF0 = 1,   // K stage full (2)
  B_VF0 = 3,   // V stage full (2)
  B_KE0 = 5,   // K stage free: both S products of that key tile done (2)
  B_SF0 = 7,   // S of query tile k ready (2)
  B_PF0 = 9,   // P of query tile k written (2, 128 arrivals)
  B_SQ0 = 11,  // sigma(Q) of query tile k written (2, 128 arrivals)
  B_MEM0 = 13, // sigma(Q_k) M_{s-1} ready (2)
  B_VE0 = 15,  // V stage free: both P V products of that key tile done (2)
  B_KF2 = 17,  // third K stage full
  B_KE2 = 18,  // third K stage free
  B_COUNT = 19
};
constexpr uint32_t kA_TMEMSLOT = kA_BAR + 8 * B_COUNT;
constexpr uint32_t kAttnSmem = kA_TMEMSLOT + 16 + 1024;  // + alignment slack
static_assert(kAttnSmem <= 232448, "attention kernel exceeds 227 KB of shared memory");

// One CTA computes two adjacent 128-row query tiles (2m, 2m+1) of one
// (b, h, segment), sharing every K/V tile load between them.
// Warps 0-3: softmax warpgroup of query tile 2m; warps 4-7: of tile 2m+1
// (thread = query row = TMEM lane).  Warp 8 loads (TMA), warp 9 issues the
// MMAs and owns TMEM, warps 10-11 only complete their warpgroup.  TMEM columns: S of tile 2m [0,128), S of tile 2m+1
// [128,256), O of tile 2m [256,384), O of tile 2m+1 [384,512).  P (bf16)
// overwrites the first 64 columns of its S buffer and feeds the P V product
// from TMEM; after the last P V product the S buffer receives sigma(Q) M_{s-1}.
//
// MMA issue order (k = query tile): S_0(0) S_1(0) | PV_0(j-1) S_0(j) PV_1(j-1)
// S_1(j) | ... : the strict alternation keeps the two softmax warpgroups half
// a period apart, so one works while the tensor cores serve the other, and
// "S_k(j) complete" implies "PV_k(j-1) complete": the O rescale of the
// softmax needs no extra wait.
//
// CTAs are ordered by groups of GS segments (about one wave of CTAs per
// group, so the group's K/V stays in L2), heaviest pair first inside a group.
__global__ void __launch_bounds__(kAttnThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_mt,
                   const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  ATTN_TRACE(threadIdx.x == 0, 3000);

  // ---- work item: (pair m, segment) from the grouped schedule
  const int NS = a.B * a.H * a.S;
  const int per_group = a.GS * a.P;
  const int grp = (int)(blockIdx.x / per_group);
  const int r = (int)(blockIdx.x % per_group);
  const int gsz = min(a.GS, NS - grp * a.GS);
  if (r >= gsz * a.P) return;  // padding of the last group
  const int m = a.P - 1 - r / gsz;       // pair index, or tile index when single
  const int seg = grp * a.GS + r % gsz;  // = bh * S + s
  const int bh = seg / a.S, s = seg % a.S;
  const int b = bh / a.H, h = bh % a.H;
  const long long seg0 = (long long)s * a.N;
  const int n_s = (int)min((long long)a.N, a.L - seg0);
  const bool single = a.single != 0;
  const int tq0 = single ? m : 2 * m;    // query tile of warpgroup 0 (warpgroup 1: tq0 + 1)
  if (tq0 * kTile >= n_s) return;        // tail segment: the tile(s) are empty
  const int nk1 = tq0 + (single ? 1 : 2); // K/V tiles of the CTA's last query tile
  const int nk0 = tq0 + 1;               // K/V tiles of query tile tq0

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  auto sQ = [&](int k) { return base + (k ? kA_Q1 : kA_Q0); };
  auto sK = [&](int st) { return base + kA_K0 + (uint32_t)st * kTileBytes; };
  auto sV = [&](int st) { return base + kA_V0 + (uint32_t)st * kTileBytes; };
  auto bar = [&](int i) { return base + kA_BAR + 8u * (uint32_t)i; };
  // K tile j lives in stage j % 3; its barriers (full / free) and their phase (j / 3) & 1
  auto kfull = [&](int j) { const int st = j % kKStages; return bar(st < 2 ? B_KF0 + st : B_KF2); };
  auto kfree = [&](int j) { const int st = j % kKStages; return bar(st < 2 ? B_KE0 + st : B_KE2); };
  auto kph = [&](int j) { return (uint32_t)((j / kKStages) & 1); };
  auto sKt = [&](int j) { return sK(j % kKStages); };
  float* zs = reinterpret_cast<float*>(gbase + kA_Z);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kA_TMEMSLOT);

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_KF0 + i), 1);
      mbar_init(bar(B_VF0 + i), 1);
      mbar_init(bar(B_KE0 + i), 1);
      mbar_init(bar(B_VE0 + i), 1);
      if (i == 0) {
        mbar_init(bar(B_KF2), 1);
        mbar_init(bar(B_KE2), 1);
      }
      mbar_init(bar(B_SF0 + i), 1);
      mbar_init(bar(B_PF0 + i), 128);
      mbar_init(bar(B_SQ0 + i), 128);
      mbar_init(bar(B_MEM0 + i), 1);
    }
    fence_barrier_init();
  }
  if (warp == 9) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  ATTN_TRACE(threadIdx.x == 0, 3001);

  if (warp >= 8) {
  regs_decrease<kAttnOtherRegs>();
  if (warp == 8) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      prefetch_tensormap(&tm_mt);
      const int lq = (int)(seg0 + (long long)tq0 * kTile);
      mbar_expect_tx(bar(B_Q), (single ? 1 : 2) * kTileBytes);
      tma_load_4d(sQ(0), &tm_q, bar(B_Q), 0, lq, h, b);
      tma_load_4d(sQ(0) + kBox, &tm_q, bar(B_Q), 64, lq, h, b);
      if (!single) {
        tma_load_4d(sQ(1), &tm_q, bar(B_Q), 0, lq + kTile, h, b);
        tma_load_4d(sQ(1) + kBox, &tm_q, bar(B_Q), 64, lq + kTile, h, b);
      }
      // K tile j goes in once the S products of key tile j-2 are done; V trails
      // K by one tile (V tile j once the P V products of key tile j-2 are
      // done), so that a pending V never holds back the next K.
      for (int j = 0; j <= nk1; ++j) {
        if (j < nk1) {
          const int lk = (int)(seg0 + (long long)j * kTile);
          if (j >= kKStages) mbar_wait(kfree(j), kph(j - kKStages));
          mbar_expect_tx(kfull(j), kTileBytes);
          tma_load_4d(sKt(j), &tm_k, kfull(j), 0, lk, h, b);
          tma_load_4d(sKt(j) + kBox, &tm_k, kfull(j), 64, lk, h, b);
        }
        if (j >= 1) {
          const int jv = j - 1, st = jv & 1;
          const int lk = (int)(seg0 + (long long)jv * kTile);
          if (jv >= 2) mbar_wait(bar(B_VE0 + st), ((jv - 2) >> 1) & 1);
          mbar_expect_tx(bar(B_VF0 + st), kTileBytes);
          tma_load_4d(sV(st), &tm_v, bar(B_VF0 + st), 0, lk, h, b);
          tma_load_4d(sV(st) + kBox, &tm_v, bar(B_VF0 + st), 64, lk, h, b);
        }
      }
      // M_{s-1} (bf16 snapshot, [dk][dv]) enters the K ring as tile nk1.
      if (nk1 >= kKStages) mbar_wait(kfree(nk1), kph(nk1 - kKStages));
      mbar_expect_tx(kfull(nk1), kTileBytes);
      tma_load_2d(sKt(nk1), &tm_mt, kfull(nk1), 0, seg * 128);
      tma_load_2d(sKt(nk1) + kBox, &tm_mt, kfull(nk1), 64, seg * 128);
    }
  } else if (warp == 9) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_kk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 128, 0, 1);
      auto issue_s = [&](int k, int j) {
        const uint32_t kt = sKt(j);
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + (uint32_t)k * 128u, kmajor_desc(sQ(k), kk), kmajor_desc(kt, kk), idesc_kk,
                 kk > 0 ? 1u : 0u);
        mma_commit(bar(B_SF0 + k));
      };
      auto issue_pv = [&](int k, int j) {  // P of tile k, key tile j; call in order j = 0, 1, ...
        const int st = j & 1;
        mbar_wait(bar(B_PF0 + k), j & 1);
        ATTN_TRACE(true, 2048 + 8 * (j + 1) + 3 + k);
        mbar_wait(bar(B_VF0 + st), (j >> 1) & 1);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + 256u + (uint32_t)k * 128u, tmem + (uint32_t)k * 128u + (uint32_t)kk * 8u,
                 mnmajor_desc(sV(st), kk), idesc_pv, (j > 0 || kk > 0) ? 1u : 0u);
      };
      mbar_wait(bar(B_Q), 0);
      mbar_wait(kfull(0), 0);
      tc_fence_after();
      issue_s(0, 0);
      if (!single) issue_s(1, 0);
      mma_commit(kfree(0));
      for (int j = 1; j < nk1; ++j) {
        mbar_wait(kfull(j), kph(j));
        ATTN_TRACE(true, 2048 + 8 * j + 0);
        tc_fence_after();
        if (j - 1 < nk0) issue_pv(0, j - 1);
        ATTN_TRACE(true, 2048 + 8 * j + 1);
        if (j < nk0) issue_s(0, j);
        ATTN_TRACE(true, 2048 + 8 * j + 5);
        if (!single) issue_pv(1, j - 1);
        ATTN_TRACE(true, 2048 + 8 * j + 2);
        mma_commit(bar(B_VE0 + ((j - 1) & 1)));
        if (!single) issue_s(1, j);
        mma_commit(kfree(j));
      }
      issue_pv(single ? 0 : 1, nk1 - 1);
      mma_commit(bar(B_VE0 + ((nk1 - 1) & 1)));
      // memory read: sigma(Q_k) (written over Q_k by the softmax warps) times M_{s-1}
      mbar_wait(kfull(nk1), kph(nk1));
      const uint32_t mt = sKt(nk1);  // M_{s-1} [dk][dv]: MN-major B operand (like V)
      constexpr uint32_t idesc_mem = idesc_bf16(128, 128, 0, 1);
#pragma unroll 1
      for (int k = 0; k < (single ? 1 : 2); ++k) {
        mbar_wait(bar(B_SQ0 + k), 0);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + (uint32_t)k * 128u, kmajor_desc(sQ(k), kk), mnmajor_desc(mt, kk), idesc_mem,
                 kk > 0 ? 1u : 0u);
        mma_commit(bar(B_MEM0 + k));
      }
    }
  }
  } else {
    regs_increase<kAttnSoftmaxRegs>();
    // -------------------------------------------------------------- softmax WGs
    const int k = warp >> 2;            // query tile tq0 + k
    if (!(single && k == 1)) {
    const int row = (warp & 3) * 32 + lane;  // query row in the tile = TMEM lane
    const uint32_t lrow = (uint32_t)((warp & 3) * 32) << 16;
    const uint32_t tS = tmem + lrow + (uint32_t)k * 128u;
    const uint32_t tO = tmem + lrow + 256u + (uint32_t)k * 128u;
    const int nk = nk0 + k;             // its K/V tiles; the last one is its diagonal
    const float c = a.scale_log2;
    float m_ref = 0.f, l = 0.f;
    const bool tr = (row == 0);
    const float zrow = a.snapz[(long long)seg * 128 + row];  // used after the loop
    for (int j = 0; j < nk; ++j) {
      ATTN_TRACE(tr, 1024 * k + 8 * j + 0);
      mbar_wait(bar(B_SF0 + k), j & 1);
      ATTN_TRACE(tr, 1024 * k + 8 * j + 1);
      tc_fence_after();
      uint32_t x[128];
      {
        uint32_t (&x0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&x[0]);
        uint32_t (&x1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&x[32]);
        uint32_t (&x2)[32] = *reinterpret_cast<uint32_t(*)[32]>(&x[64]);
        uint32_t (&x3)[32] = *reinterpret_cast<uint32_t(*)[32]>(&x[96]);
        tmem_ld32(tS, x0);
        tmem_ld32(tS + 32u, x1);
        tmem_ld32(tS + 64u, x2);
        tmem_ld32(tS + 96u, x3);
        tmem_ld_wait();
      }
      if (j == nk - 1) {  // diagonal tile: key e is visible to query row iff e <= row
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (e > row) x[e] = __float_as_uint(-INFINITY);
      }
      float mx[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) mx[i] = __uint_as_float(x[i]);
#pragma unroll
      for (int e = 4; e < 128; ++e) mx[e & 3] = fmaxf(mx[e & 3], __uint_as_float(x[e]));
      const float mxs = fmaxf(fmaxf(mx[0], mx[1]), fmaxf(mx[2], mx[3])) * c;
      ATTN_TRACE(tr, 1024 * k + 8 * j + 2);
      // Move the reference max only when the row max grows by more than 2^8:
      // O / l stays exact for any reference, and p stays below 256.
      const float m_new = (j == 0) ? mxs : (mxs > m_ref + 8.f ? mxs : m_ref);
      const bool resc = (j > 0) && (m_new != m_ref);
      if (__any_sync(0xffffffffu, resc)) {
        // S_k(j) complete implies P V of tile j-1 complete (issue order), so O is final here.
        const float alpha = resc ? ex2_approx(m_ref - m_new) : 1.f;
        l *= alpha;
        uint32_t o[16];
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
          tmem_ld16(tO + 16u * cc, o);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 16; ++e) o[e] = __float_as_uint(__uint_as_float(o[e]) * alpha);
          tmem_st16(tO + 16u * cc, o);
        }
        tmem_st_wait();
      }
      m_ref = m_new;
      const float nm = -m_ref;
      float ls[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int e = 0; e < 64; ++e) {
        float a0, a1;
        if (INFINI_F32X2) {
          fma2(a0, a1, __uint_as_float(x[2 * e]), __uint_as_float(x[2 * e + 1]), c, c, nm, nm);
        } else {
          a0 = fmaf(__uint_as_float(x[2 * e]), c, nm);
          a1 = fmaf(__uint_as_float(x[2 * e + 1]), c, nm);
        }
        float p0, p1;
        if (INFINI_POLY_EVERY > 0 && (e % (INFINI_POLY_EVERY > 0 ? INFINI_POLY_EVERY : 1)) == INFINI_POLY_EVERY - 1) {
          p0 = exp2_poly(a0);
          p1 = exp2_poly(a1);
        } else {
          p0 = ex2_approx(a0);
          p1 = ex2_approx(a1);
        }
        if (INFINI_F32X2) {
          if ((e & 1) == 0) {
            add2(ls[0], ls[1], ls[0], ls[1], p0, p1);
          } else {
            add2(ls[2], ls[3], ls[2], ls[3], p0, p1);
          }
        } else {
          ls[e & 3] += p0 + p1;
        }
        x[e] = INFINI_PACK_ALU ? pack_bf16x2_alu(p0, p1) : pack_bf16x2(p0, p1);
      }
      l += (ls[0] + ls[1]) + (ls[2] + ls[3]);
      ATTN_TRACE(tr, 1024 * k + 8 * j + 3);
      {
        uint32_t (&p0)[32] = *reinterpret_cast<uint32_t(*)[32]>(&x[0]);
        uint32_t (&p1)[32] = *reinterpret_cast<uint32_t(*)[32]>(&x[32]);
        tmem_st32(tS, p0);
        tmem_st32(tS + 32u, p1);
      }
      tmem_st_wait();
      tc_fence_before();
      mbar_arrive(bar(B_PF0 + k));
      ATTN_TRACE(tr, 1024 * k + 8 * j + 4);
    }
    // Every Q_k K^T product has completed: overwrite this row of Q_k with
    // sigma(Q_k) (bf16) for the memory read, and form the fp32 denominator
    // sigma(q) . z_{s-1} from the unrounded sigma.
    float den = 0.f;
    {
      float* zk = zs + 128 * k;
      zk[row] = zrow;
      named_bar_sync(1 + k, 128);
      ATTN_TRACE(row == 0, 3008 + 8 * k + 3);
      const uint32_t q = sQ(k);
      uint4 w[16];
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) w[cc] = lds128(q + swz_chunk(row, cc));
      ATTN_TRACE(row == 0, 3008 + 8 * k + 4);
      float dp[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) {
        uint32_t* wp = reinterpret_cast<uint32_t*>(&w[cc]);
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float s0 = elu1(bf16_lo(wp[e])), s1 = elu1(bf16_hi(wp[e]));
          dp[e] = fmaf(s0, zk[8 * cc + 2 * e], dp[e]);
          dp[e] = fmaf(s1, zk[8 * cc + 2 * e + 1], dp[e]);
          wp[e] = pack_bf16x2(s0, s1);
        }
      }
      ATTN_TRACE(row == 0, 3008 + 8 * k + 5);
#pragma unroll
      for (int cc = 0; cc < 16; ++cc) sts128(q + swz_chunk(row, cc), w[cc]);
      den = (dp[0] + dp[1]) + (dp[2] + dp[3]);
      ATTN_TRACE(row == 0, 3008 + 8 * k + 6);
      fence_proxy_async_smem();
      mbar_arrive(bar(B_SQ0 + k));
      ATTN_TRACE(row == 0, 3008 + 8 * k + 0);
    }
    // ---------------------------------------------------------------- epilogue
    mbar_wait(bar(B_MEM0 + k), 0);  // also implies the last P V product of tile k is complete
    ATTN_TRACE(row == 0, 3008 + 8 * k + 1);
    tc_fence_after();
    const float gw = 1.f / (1.f + __expf(-a.beta[h]));
    const float wdot = (1.f - gw) / l;
    const float wmem = den != 0.f ? gw / den : 0.f;
    const int qrow = (tq0 + k) * kTile + row;
    const bool valid = qrow < n_s;
    __nv_bfloat16* orow = a.out + b * a.os[0] + h * a.os[1] + (seg0 + qrow) * a.os[2];
#pragma unroll
    for (int cc = 0; cc < 4; ++cc) {
      uint32_t ro[32], rm[32];
      tmem_ld32(tO + 32u * cc, ro);
      tmem_ld32(tS + 32u * cc, rm);
      tmem_ld_wait();
      uint32_t pk[16];
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const float v0 = wmem * __uint_as_float(rm[2 * e]) + wdot * __uint_as_float(ro[2 * e]);
        const float v1 = wmem * __uint_as_float(rm[2 * e + 1]) + wdot * __uint_as_float(ro[2 * e + 1]);
        pk[e] = pack_bf16x2(v0, v1);
      }
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(orow + 32 * cc);
#pragma unroll
        for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
      }
    }
    ATTN_TRACE(row == 0, 3008 + 8 * k + 2);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 9) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

}  // namespace tc
}  // namespace infini
