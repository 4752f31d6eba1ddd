// Tensor-core (tcgen05 / TMEM / TMA) kernels of the Infini-attention forward
// for bf16 inputs with d_key = d_value = 128 on sm_100a.
//
//   attn_tc_kernel        A_dot (Eq. 6) + A_mem (Eq. 7) + gate (Eq. 10), fused:
//                         one CTA per (b, h, segment, 128-row query tile).
//   mem_update_tc_kernel  the segment's share of sigma(K)^T U and sum_t sigma(K_t)
//                         for the linear (Eq. 8, U = V) or delta (Eq. 9,
//                         U = V - sigma(K) M_{s-1} / (sigma(K) z_{s-1})) rule.
//
// Operand tiles are 128 rows x 128 bf16 columns, held in shared memory as two
// TMA boxes of 128 rows x 64 columns (16 KB each) with the 128-byte swizzle:
// 16-byte chunk c of row r sits at chunk position c ^ (r % 8) of the row.
// A tile is K-major when its rows are the MMA's M/N index (Q, K, sigma(Q),
// M^T); it is MN-major when its rows are the MMA's K index (V, U, sigma(K)
// read as sigma(K)^T).
#pragma once

#include "common.cuh"

namespace infini {
namespace tc {

constexpr int kTile = 128;
constexpr uint32_t kBox = 16384;        // 128 rows x 128 B
constexpr uint32_t kTileBytes = 32768;  // two boxes

// Descriptor of K-step kk (16 elements along K) of a K-major tile.
__device__ __forceinline__ uint64_t kmajor_desc(uint32_t tile, int kk) {
  return smem_desc_sw128(tile + (uint32_t)(kk >> 2) * kBox + (uint32_t)(kk & 3) * 32u, 16u, 1024u);
}
// Descriptor of K-step kk (16 rows along K) of an MN-major tile.
__device__ __forceinline__ uint64_t mnmajor_desc(uint32_t tile, int kk) {
  return smem_desc_sw128(tile + (uint32_t)kk * 2048u, kBox, 1024u);
}
// Descriptor of K-step kk of the 16-row K-major block of ones (two 2 KB boxes).
__device__ __forceinline__ uint64_t ones_desc(uint32_t tile, int kk) {
  return smem_desc_sw128(tile + (uint32_t)(kk >> 2) * 2048u + (uint32_t)(kk & 3) * 32u, 16u, 1024u);
}
// Byte offset of 16-byte chunk c (0..15, 8 bf16 each) of row r inside a tile.
__device__ __forceinline__ uint32_t swz_chunk(int r, int c) {
  return (uint32_t)(c >> 3) * kBox + (uint32_t)r * 128u + ((uint32_t)((c & 7) ^ (r & 7)) << 4);
}

__device__ __forceinline__ uint4 lds128(uint32_t a) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(a));
  return v;
}
__device__ __forceinline__ void sts128(uint32_t a, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}

struct AttnArgs {
  const float* beta;
  const float* snapz;     // [BH][S][128] fp32: z_{s-1}
  __nv_bfloat16* out;
  int B, H, S, T;         // T = query tiles per full segment
  long long L;
  int N;
  float scale_log2;       // softmax scale * log2(e)
  long long os[3];        // element strides of out
};

// Shared memory of the attention kernel (offsets from a 1024-aligned base).
constexpr uint32_t kA_Q = 0;
constexpr uint32_t kA_K0 = 32768;
constexpr uint32_t kA_V0 = 98304;
constexpr uint32_t kA_Z = 163840;
constexpr uint32_t kA_BAR = kA_Z + 512;
constexpr uint32_t kA_TMEMSLOT = kA_BAR + 256;
constexpr uint32_t kAttnSmem = kA_TMEMSLOT + 16 + 1024;  // + alignment slack

// Barrier indices.
enum : int {
  B_Q = 0, B_KF0 = 1, B_VF0 = 3, B_KVE0 = 5, B_SF0 = 7, B_PF0 = 9, B_O0 = 11, B_SQ = 13, B_MEM = 14, B_COUNT = 15
};

// Warp roles: warp 0 loads (TMA), warp 1 issues MMAs and owns TMEM, warps 2-5
// (one warpgroup, thread = query row = TMEM lane) run the softmax and the
// epilogue.  TMEM columns: S/P double buffer [0,128) and [128,256), O
// accumulator [256,384), sigma(Q) M_{s-1} [384,512).  P (bf16) overwrites the
// first 64 columns of its S buffer and feeds the P V product from TMEM.
__global__ void __launch_bounds__(192, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_mt,
                   const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);

  const int BHS = a.B * a.H * a.S;
  const int it = a.T - 1 - (int)(blockIdx.x / BHS);  // longest query tiles first
  const int rem = (int)(blockIdx.x % BHS);
  const int bh = rem / a.S, s = rem % a.S;
  const int b = bh / a.H, h = bh % a.H;
  const long long seg0 = (long long)s * a.N;
  const int n_s = (int)min((long long)a.N, a.L - seg0);
  if (it * kTile >= n_s) return;  // tail segment: this tile is empty
  const int nk = it + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t sQ = base + kA_Q;
  auto sK = [&](int st) { return base + kA_K0 + (uint32_t)st * kTileBytes; };
  auto sV = [&](int st) { return base + kA_V0 + (uint32_t)st * kTileBytes; };
  auto bar = [&](int i) { return base + kA_BAR + 8u * (uint32_t)i; };
  float* zs = reinterpret_cast<float*>(gbase + kA_Z);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kA_TMEMSLOT);

  if (threadIdx.x == 0) {
    mbar_init(bar(B_Q), 1);
    for (int i = 0; i < 2; ++i) {
      mbar_init(bar(B_KF0 + i), 1);
      mbar_init(bar(B_VF0 + i), 1);
      mbar_init(bar(B_KVE0 + i), 1);
      mbar_init(bar(B_SF0 + i), 1);
      mbar_init(bar(B_PF0 + i), 128);
      mbar_init(bar(B_O0 + i), 1);
    }
    mbar_init(bar(B_SQ), 128);
    mbar_init(bar(B_MEM), 1);
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  if (warp >= 2) zs[threadIdx.x - 64] = a.snapz[((long long)bh * a.S + s) * 128 + (threadIdx.x - 64)];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      prefetch_tensormap(&tm_q);
      prefetch_tensormap(&tm_k);
      prefetch_tensormap(&tm_v);
      prefetch_tensormap(&tm_mt);
      const int lq = (int)(seg0 + (long long)it * kTile);
      mbar_expect_tx(bar(B_Q), kTileBytes);
      tma_load_4d(sQ, &tm_q, bar(B_Q), 0, lq, h, b);
      tma_load_4d(sQ + kBox, &tm_q, bar(B_Q), 64, lq, h, b);
      for (int j = 0; j < nk; ++j) {
        const int st = j & 1;
        if (j >= 2) mbar_wait(bar(B_KVE0 + st), ((j - 2) >> 1) & 1);
        const int lk = (int)(seg0 + (long long)j * kTile);
        mbar_expect_tx(bar(B_KF0 + st), kTileBytes);
        tma_load_4d(sK(st), &tm_k, bar(B_KF0 + st), 0, lk, h, b);
        tma_load_4d(sK(st) + kBox, &tm_k, bar(B_KF0 + st), 64, lk, h, b);
        mbar_expect_tx(bar(B_VF0 + st), kTileBytes);
        tma_load_4d(sV(st), &tm_v, bar(B_VF0 + st), 0, lk, h, b);
        tma_load_4d(sV(st) + kBox, &tm_v, bar(B_VF0 + st), 64, lk, h, b);
      }
      // M_{s-1}^T (bf16 snapshot) enters the K ring as tile nk.
      const int st = nk & 1;
      if (nk >= 2) mbar_wait(bar(B_KVE0 + st), ((nk - 2) >> 1) & 1);
      const int row = (bh * a.S + s) * 128;
      mbar_expect_tx(bar(B_KF0 + st), kTileBytes);
      tma_load_2d(sK(st), &tm_mt, bar(B_KF0 + st), 0, row);
      tma_load_2d(sK(st) + kBox, &tm_mt, bar(B_KF0 + st), 64, row);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      constexpr uint32_t idesc_kk = idesc_bf16(128, 128, 0, 0);
      constexpr uint32_t idesc_pv = idesc_bf16(128, 128, 0, 1);
      auto issue_pv = [&](int jj) {
        const int st = jj & 1, ph = (jj >> 1) & 1;
        mbar_wait(bar(B_PF0 + st), ph);
        mbar_wait(bar(B_VF0 + st), ph);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ts(tmem + 256, tmem + (uint32_t)st * 128u + (uint32_t)kk * 8u, mnmajor_desc(sV(st), kk), idesc_pv,
                 (jj > 0 || kk > 0) ? 1u : 0u);
        mma_commit(bar(B_KVE0 + st));
        mma_commit(bar(B_O0 + st));
      };
      mbar_wait(bar(B_Q), 0);
      for (int j = 0; j < nk; ++j) {
        const int st = j & 1, ph = (j >> 1) & 1;
        mbar_wait(bar(B_KF0 + st), ph);
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < 8; ++kk)
          mma_ss(tmem + (uint32_t)st * 128u, kmajor_desc(sQ, kk), kmajor_desc(sK(st), kk), idesc_kk,
                 kk > 0 ? 1u : 0u);
        mma_commit(bar(B_SF0 + st));
        if (j >= 1) issue_pv(j - 1);
      }
      issue_pv(nk - 1);
      // memory read: sigma(Q) (written over Q by the softmax warps) times M_{s-1}
      mbar_wait(bar(B_SQ), 0);
      const int st = nk & 1;
      mbar_wait(bar(B_KF0 + st), (nk >> 1) & 1);
      tc_fence_after();
#pragma unroll
      for (int kk = 0; kk < 8; ++kk)
        mma_ss(tmem + 384, kmajor_desc(sQ, kk), kmajor_desc(sK(st), kk), idesc_kk, kk > 0 ? 1u : 0u);
      mma_commit(bar(B_MEM));
    }
  } else {
    // -------------------------------------------------------------- softmax WG
    const int wq = warp & 3;
    const int row = wq * 32 + lane;  // query row in the tile = TMEM lane
    const uint32_t lrow = (uint32_t)(wq * 32) << 16;
    float m_ref = 0.f, l = 0.f, den = 0.f;
    for (int j = 0; j < nk; ++j) {
      const int st = j & 1, ph = (j >> 1) & 1;
      mbar_wait(bar(B_SF0 + st), ph);
      tc_fence_after();
      const uint32_t tS = tmem + lrow + (uint32_t)st * 128u;
      float x[128];
      {
        uint32_t r[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(tS + 32u * c, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) x[32 * c + e] = __uint_as_float(r[e]) * a.scale_log2;
        }
      }
      if (j == nk - 1) {  // diagonal tile: key kk is visible to query row iff kk <= row
#pragma unroll
        for (int e = 0; e < 128; ++e)
          if (e > row) x[e] = -INFINITY;
      }
      float mx = x[0];
#pragma unroll
      for (int e = 1; e < 128; ++e) mx = fmaxf(mx, x[e]);
      // Rescale only when the running max grows by more than 2^8: the final
      // O / l is exact for any reference max, and values stay below 256.
      const float m_new = (j == 0) ? mx : (mx > m_ref + 8.f ? mx : m_ref);
      const bool resc = (j > 0) && (m_new != m_ref);
      const float alpha = resc ? ex2_approx(m_ref - m_new) : 1.f;
      if (__any_sync(0xffffffffu, resc)) {
        const int jj = j - 1;
        mbar_wait(bar(B_O0 + (jj & 1)), (jj >> 1) & 1);
        tc_fence_after();
        uint32_t r[32];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          tmem_ld32(tmem + lrow + 256u + 32u * c, r);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
          tmem_st32(tmem + lrow + 256u + 32u * c, r);
        }
        tmem_st_wait();
      }
      m_ref = m_new;
      l *= alpha;
      {
        uint32_t pk[32];
#pragma unroll
        for (int half = 0; half < 2; ++half) {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const float p0 = ex2_approx(x[64 * half + 2 * e] - m_ref);
            const float p1 = ex2_approx(x[64 * half + 2 * e + 1] - m_ref);
            l += p0 + p1;
            pk[e] = pack_bf16x2(p0, p1);
          }
          tmem_st32(tS + 32u * half, pk);
        }
        tmem_st_wait();
      }
      tc_fence_before();
      mbar_arrive(bar(B_PF0 + st));
      if (j == nk - 1) {
        // Every Q K^T product has completed: overwrite this row of Q with
        // sigma(Q) (bf16) for the memory read, and form the fp32
        // denominator sigma(q) . z_{s-1} from the unrounded sigma.
#pragma unroll
        for (int c = 0; c < 16; ++c) {
          const uint32_t ad = sQ + swz_chunk(row, c);
          uint4 w = lds128(ad);
          uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float s0 = elu1(bf16_lo(wp[e])), s1 = elu1(bf16_hi(wp[e]));
            den = fmaf(s0, zs[8 * c + 2 * e], den);
            den = fmaf(s1, zs[8 * c + 2 * e + 1], den);
            wp[e] = pack_bf16x2(s0, s1);
          }
          sts128(ad, w);
        }
        fence_proxy_async_smem();
        mbar_arrive(bar(B_SQ));
      }
    }
    // ---------------------------------------------------------------- epilogue
    {
      const int jj = nk - 1;
      mbar_wait(bar(B_O0 + (jj & 1)), (jj >> 1) & 1);
      mbar_wait(bar(B_MEM), 0);
      tc_fence_after();
      const float gw = 1.f / (1.f + __expf(-a.beta[h]));
      const float wdot = (1.f - gw) / l;
      const float wmem = den != 0.f ? gw / den : 0.f;
      const int qrow = it * kTile + row;
      const bool valid = qrow < n_s;
      __nv_bfloat16* orow = a.out + b * a.os[0] + h * a.os[1] + (seg0 + qrow) * a.os[2];
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint32_t ro[32], rm[32];
        tmem_ld32(tmem + lrow + 256u + 32u * c, ro);
        tmem_ld32(tmem + lrow + 384u + 32u * c, rm);
        tmem_ld_wait();
        uint32_t pk[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float v0 = wmem * __uint_as_float(rm[2 * e]) + wdot * __uint_as_float(ro[2 * e]);
          const float v1 = wmem * __uint_as_float(rm[2 * e + 1]) + wdot * __uint_as_float(ro[2 * e + 1]);
          pk[e] = pack_bf16x2(v0, v1);
        }
        if (valid) {
          uint4* dst = reinterpret_cast<uint4*>(orow + 32 * c);
#pragma unroll
          for (int e = 0; e < 4; ++e) dst[e] = make_uint4(pk[4 * e], pk[4 * e + 1], pk[4 * e + 2], pk[4 * e + 3]);
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
