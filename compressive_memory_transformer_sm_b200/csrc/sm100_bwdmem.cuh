// The memory read's backward (Eq. 7) on the sm_100a tensor cores, for bf16
// tensors with d_key = d_value = 128: the memory-read terms that bwd_q_kernel
// (bwd_simt.cuh) computes on the other paths, with two products on tcgen05.
// For 128 query rows of one (b, h, segment), with M = M^(s), z = z^(s) the
// state entering the segment:
//   den = sigma(q) . z (fp32), num = sigma(q) M (product 1), A_mem = num / den,
//   D'_i = dO_i . A_dot_i, the dbeta row term dO_i . (A_mem_i - A_dot_i),
//   d_num = g dO / den, d_den = -g dO . A_mem / den (zero where den = 0),
//   dq_mem = sigma'(q) (d_num M^T + d_den z) (product 2).
// Both products take fp32 operands split into bf16 hi + lo parts
// (x_hi y_hi + x_hi y_lo + x_lo y_hi, fp32 in TMEM: ~2^-16 relative).  M's
// hi and lo tiles are stored once, row-major [dk][dv] with the 128-byte
// swizzle: the MN-major B operand of sigma(q) M and, read as K-major, the B
// operand M^T of d_num M^T.  The A tiles hold sigma(q), then d_num.
//
// 512 threads: thread (row r = TMEM lane, quarter qq) handles columns
// [32 qq, 32 qq + 32) of query row r; one thread issues the products.
#pragma once

#include "sm100_common.cuh"

namespace infini {
namespace tc {

constexpr int kQmThreads = 512;
constexpr uint32_t kQmAH = 0, kQmAL = 32768, kQmMH = 65536, kQmML = 98304;  // 128 x 128 bf16 tiles
constexpr uint32_t kQmZ = 131072;        // z, 128 floats
constexpr uint32_t kQmX = kQmZ + 512;    // [4 quantities][4 column quarters][128 rows] partial row sums
constexpr uint32_t kQmBAR = kQmX + 8 * 1024;
constexpr uint32_t kQmSLOT = kQmBAR + 16;
constexpr uint32_t kQmSmem = kQmSLOT + 16 + 1024;

// 16 fp32 values -> the bf16 hi and lo parts of two 16-byte chunks each
__device__ __forceinline__ void qm_split8(const float* x, uint4& hi, uint4& lo) {
  uint32_t* h = reinterpret_cast<uint32_t*>(&hi);
  uint32_t* l = reinterpret_cast<uint32_t*>(&lo);
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    h[e] = pack_bf16x2(x[2 * e], x[2 * e + 1]);
    l[e] = pack_bf16x2(x[2 * e] - bf16_lo(h[e]), x[2 * e + 1] - bf16_hi(h[e]));
  }
}

__global__ void __launch_bounds__(kQmThreads, 1)
    bwd_qmem_tc_kernel(const __nv_bfloat16* __restrict__ q, const __nv_bfloat16* __restrict__ dout,
                       const float* __restrict__ adot, const float* __restrict__ beta,
                       const float* __restrict__ snapM, const float* __restrict__ snapz, int B, int H, int S,
                       int N, long long L, int blocks_per_seg, float* __restrict__ dq_mem, float* __restrict__ Dp,
                       float* __restrict__ brow, float* __restrict__ dnum, float* __restrict__ dden) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int idx = blockIdx.x;
  const int blk = idx % blocks_per_seg;
  idx /= blocks_per_seg;
  const int s = idx % S;
  const int bh = idx / S;
  const int h = bh % H;
  const long long seg_start = (long long)s * N;
  const int n_s = (int)min((long long)N, L - seg_start);
  const int r0 = blk * 128;
  if (r0 >= n_s) return;
  const int nr = min(128, n_s - r0);
  const long long row0 = (long long)bh * L + seg_start + r0;
  const float gw = 1.f / (1.f + expf(-beta[h]));
  float* zs = reinterpret_cast<float*>(gbase + kQmZ);
  float* xs = reinterpret_cast<float*>(gbase + kQmX);  // [den | d_den | dbeta | D'][4 quarters][128 rows]
  const uint32_t bar = base + kQmBAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kQmSLOT);

  const int row = 32 * (warp & 3) + lane, qq = warp >> 2;  // query row (TMEM lane), column quarter
  const int c0 = 32 * qq;                                   // first column of this thread
  const uint32_t lq = (uint32_t)(32 * (warp & 3)) << 16;
  const bool valid = row < nr;
  const long long grow = row0 + row;  // global row (meaningful when valid)

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  // this thread's q chunks now, and dO, A_dot (read after product 1) into L2
  uint4 qw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    qw[i] = valid ? __ldg(reinterpret_cast<const uint4*>(q + grow * 128 + c0) + i) : make_uint4(0u, 0u, 0u, 0u);
  if (valid) {
    if ((qq & 1) == 0) prefetch_l2(dout + grow * 128 + c0);
    prefetch_l2(adot + grow * 128 + c0);
  }
  if (tid < 128) zs[tid] = snapz[((long long)bh * S + s) * 128 + tid];
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  // M [dk][dv] (fp32) -> hi / lo tiles: 2048 chunks of 8 values, 4 per thread
  {
    const float* Mp = snapM + ((long long)bh * S + s) * 16384;
#pragma unroll
    for (int ch = tid; ch < 2048; ch += kQmThreads) {
      const int i = ch >> 4, c = ch & 15;
      const float4 f0 = __ldg(reinterpret_cast<const float4*>(Mp + i * 128 + 8 * c));
      const float4 f1 = __ldg(reinterpret_cast<const float4*>(Mp + i * 128 + 8 * c + 4));
      const float x[8] = {f0.x, f0.y, f0.z, f0.w, f1.x, f1.y, f1.z, f1.w};
      uint4 hi, lo;
      qm_split8(x, hi, lo);
      sts128(base + kQmMH + swz_chunk(i, c), hi);
      sts128(base + kQmML + swz_chunk(i, c), lo);
    }
  }
  __syncthreads();  // z staged
  // sigma(q) of this thread's 32 columns -> A tiles; partial den
  {
    float dpart = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = 4 * qq + i;  // 16-byte chunk of the row
      float x[8];
      const uint32_t wp[4] = {qw[i].x, qw[i].y, qw[i].z, qw[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        x[2 * e] = valid ? elu1_accurate(bf16_lo(wp[e])) : 0.f;
        x[2 * e + 1] = valid ? elu1_accurate(bf16_hi(wp[e])) : 0.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) dpart = fmaf(x[e], zs[8 * c + e], dpart);
      uint4 hi, lo;
      qm_split8(x, hi, lo);
      sts128(base + kQmAH + swz_chunk(row, c), hi);
      sts128(base + kQmAL + swz_chunk(row, c), lo);
    }
    xs[qq * 128 + row] = dpart;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tP1 = tmem, tP2 = tmem + 128u;
  // a row quantity from its four column quarters, in a fixed order
  auto rowsum = [&](int quantity) {
    const float* x4 = xs + quantity * 512 + row;
    return ((x4[0] + x4[128]) + x4[256]) + x4[384];
  };
  const float den = rowsum(0);
  // product 1: num = sigma(q) M (A K-major, B = M MN-major)
  if (tid == 0) {
    constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 1);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t aH = kmajor_desc(base + kQmAH, kk), aL = kmajor_desc(base + kQmAL, kk);
      const uint64_t bH = mnmajor_desc(base + kQmMH, kk), bL = mnmajor_desc(base + kQmML, kk);
      mma_ss(tP1, aH, bH, idesc, kk > 0 ? 1u : 0u);
      mma_ss(tP1, aH, bL, idesc, 1u);
      mma_ss(tP1, aL, bH, idesc, 1u);
    }
    mma_commit(bar);
  }
  mbar_wait(bar, 0);
  tc_fence_after();
  // row terms over this thread's 32 columns; d_num -> A tiles (product 1 has read them)
  float bt = 0.f, dp = 0.f, dd = 0.f;
  {
    uint32_t nm[32];
    tmem_ld32(tP1 + lq + (uint32_t)c0, nm);
    tmem_ld_wait();
    float dA[32], ad[32];
    if (valid) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(dout + grow * 128 + c0) + i);
        const uint32_t wp[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          dA[8 * i + 2 * e] = bf16_lo(wp[e]);
          dA[8 * i + 2 * e + 1] = bf16_hi(wp[e]);
        }
      }
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 f = __ldg(reinterpret_cast<const float4*>(adot + grow * 128 + c0) + i);
        ad[4 * i] = f.x; ad[4 * i + 1] = f.y; ad[4 * i + 2] = f.z; ad[4 * i + 3] = f.w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) dA[e] = ad[e] = 0.f;
    }
    float w[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float am = den != 0.f ? __uint_as_float(nm[e]) / den : 0.f;
      bt = fmaf(dA[e], am - ad[e], bt);
      dp = fmaf(dA[e], ad[e], dp);
      w[e] = 0.f;
      if (den != 0.f) {
        w[e] = gw * dA[e] / den;
        dd = fmaf(gw * dA[e], am, dd);
      }
    }
    if (valid) {
      float4* dst = reinterpret_cast<float4*>(dnum + grow * 128 + c0);
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[i] = make_float4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint4 hi, lo;
      qm_split8(w + 8 * i, hi, lo);
      sts128(base + kQmAH + swz_chunk(row, 4 * qq + i), hi);
      sts128(base + kQmAL + swz_chunk(row, 4 * qq + i), lo);
    }
  }
  xs[512 + qq * 128 + row] = dd;
  xs[1024 + qq * 128 + row] = bt;
  xs[1536 + qq * 128 + row] = dp;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const float d_den = den != 0.f ? -rowsum(1) / den : 0.f;
  if (qq == 0 && valid) {
    Dp[grow] = rowsum(3);
    brow[grow] = rowsum(2);
    dden[grow] = d_den;
  }
  // product 2: d_num M^T (A K-major, B = M read K-major)
  if (tid == 0) {
    constexpr uint32_t idesc = idesc_bf16(128, 128, 0, 0);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t aH = kmajor_desc(base + kQmAH, kk), aL = kmajor_desc(base + kQmAL, kk);
      const uint64_t bH = kmajor_desc(base + kQmMH, kk), bL = kmajor_desc(base + kQmML, kk);
      mma_ss(tP2, aH, bH, idesc, kk > 0 ? 1u : 0u);
      mma_ss(tP2, aH, bL, idesc, 1u);
      mma_ss(tP2, aL, bH, idesc, 1u);
    }
    mma_commit(bar);
  }
  mbar_wait(bar, 1);
  tc_fence_after();
  // dq_mem = sigma'(q) (d_num M^T + d_den z): sigma'(x) = 1 above zero, e^x at or below
  {
    uint32_t pr[32];
    tmem_ld32(tP2 + lq + (uint32_t)c0, pr);
    tmem_ld_wait();
    if (valid) {
      float o[32];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(q + grow * 128 + c0) + i);  // L2
        const uint32_t wp[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 8 * i + 2 * e;
          const float x0 = bf16_lo(wp[e]), x1 = bf16_hi(wp[e]);
          const float s0 = x0 > 0.f ? 1.f : expf(x0), s1 = x1 > 0.f ? 1.f : expf(x1);
          o[j] = s0 * fmaf(d_den, zs[c0 + j], __uint_as_float(pr[j]));
          o[j + 1] = s1 * fmaf(d_den, zs[c0 + j + 1], __uint_as_float(pr[j + 1]));
        }
      }
      float4* dst = reinterpret_cast<float4*>(dq_mem + grow * 128 + c0);
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

// The update's backward (Eq. 8 / 9) on the tensor cores: the quantities of
// bwd_upd_kernel for 128 key rows of one (b, h, segment), with G = dLoss/dM
// and gz = dLoss/dz after the segment:
//   dU = sigma(K) G (product 1), written as the dv term;
//   delta rule: R = sigma(K) M^(s) / den_k (product 2), U = V - R,
//     d_num_r = -dU / den_k, d_den_r = dU . R / den_k (rows written);
//   dsigma(K) = U G^T (product 3) (+ d_num_r M^T, product 4, into the same
//   accumulator) + gz (+ d_den_r z), written as sigma'(k) dsigma(K).
// fp32 operands in bf16 hi + lo parts (V is exact in bf16: two products for
// V G^T).  G's and M's tiles are stored row-major [dk][dv]: the MN-major B
// operand of sigma(K) G and sigma(K) M and, read as K-major, G^T and M^T.
// The A tiles hold sigma(K), then U (or V), then d_num_r.  512 threads:
// thread (row r = TMEM lane, quarter qq) handles columns [32 qq, 32 qq + 32)
// of key row r; one thread issues the products.
constexpr uint32_t kUpAH = 0, kUpAL = 32768, kUpGH = 65536, kUpGL = 98304, kUpMH = 131072, kUpML = 163840;
constexpr uint32_t kUpZ = 196608;           // gz, then z (2 x 128 floats)
constexpr uint32_t kUpX = kUpZ + 1024;      // [2 quantities][4 column quarters][128 rows]
constexpr uint32_t kUpBAR = kUpX + 4096;
constexpr uint32_t kUpSLOT = kUpBAR + 16;
constexpr uint32_t kUpSmem = kUpSLOT + 16 + 1024;
constexpr int kUpThreads = 512;

__global__ void __launch_bounds__(kUpThreads, 1)
    bwd_upd_tc_kernel(const __nv_bfloat16* __restrict__ k, const __nv_bfloat16* __restrict__ v, int B, int H, int S,
                      int N, long long L, int seg0, const float* __restrict__ gstate, long long gstride_s,
                      long long gstride_bh, const float* __restrict__ snapM, const float* __restrict__ snapz,
                      float* __restrict__ dk_upd, float* __restrict__ dv_upd, float* __restrict__ dnum_r,
                      float* __restrict__ dden_r, int blocks_per_seg) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool delta = snapM != nullptr;
  // as a programmatic dependent (the delta rule's reverse steps), nothing the
  // previous kernel reads or writes is touched before it has completed
  griddep_launch_dependents();
  griddep_wait();
  int idx = blockIdx.x;
  const int blk = idx % blocks_per_seg;
  idx /= blocks_per_seg;
  const int sl = idx % (delta ? 1 : S);
  const int bh = idx / (delta ? 1 : S);
  const int s = seg0 + sl;
  const long long seg_start = (long long)s * N;
  const int n_s = (int)min((long long)N, L - seg_start);
  const int r0 = blk * 128;
  if (r0 >= n_s) return;
  const int nr = min(128, n_s - r0);
  const long long row0 = (long long)bh * L + seg_start + r0;
  float* gz = reinterpret_cast<float*>(gbase + kUpZ);
  float* zs = gz + 128;
  float* xs = reinterpret_cast<float*>(gbase + kUpX);  // [den | d_den][4 quarters][128 rows]
  const uint32_t bar = base + kUpBAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kUpSLOT);
  const int row = 32 * (warp & 3) + lane, qq = warp >> 2;  // key row (TMEM lane), column quarter
  const uint32_t lq = (uint32_t)(32 * (warp & 3)) << 16;
  const bool valid = row < nr;
  const long long grow = row0 + row;
  const float* gp = gstate + (long long)bh * gstride_bh + (long long)s * gstride_s;
  const float* Mp = delta ? snapM + ((long long)bh * S + s) * 16384 : nullptr;

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  // this thread's k chunks now, and v (read after the first products) into L2
  uint4 kw[4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
    kw[i] = valid ? __ldg(reinterpret_cast<const uint4*>(k + grow * 128) + 4 * qq + i) : make_uint4(0u, 0u, 0u, 0u);
  if (valid && (qq & 1) == 0) prefetch_l2(v + grow * 128 + 32 * qq);
  if (tid < 128) {
    gz[tid] = gp[16384 + tid];
    zs[tid] = delta ? snapz[((long long)bh * S + s) * 128 + tid] : 0.f;
  }
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 512);
    tmem_relinquish();
  }
  // G (and M) [dk][dv] fp32 -> hi / lo tiles
#pragma unroll
  for (int ch = tid; ch < 2048; ch += kUpThreads) {
    const int i = ch >> 4, c = ch & 15;
    float x[8];
    {
      const float4 f0 = __ldg(reinterpret_cast<const float4*>(gp + i * 128 + 8 * c));
      const float4 f1 = __ldg(reinterpret_cast<const float4*>(gp + i * 128 + 8 * c + 4));
      x[0] = f0.x; x[1] = f0.y; x[2] = f0.z; x[3] = f0.w; x[4] = f1.x; x[5] = f1.y; x[6] = f1.z; x[7] = f1.w;
    }
    uint4 hi, lo;
    qm_split8(x, hi, lo);
    sts128(base + kUpGH + swz_chunk(i, c), hi);
    sts128(base + kUpGL + swz_chunk(i, c), lo);
    if (delta) {
      const float4 f0 = __ldg(reinterpret_cast<const float4*>(Mp + i * 128 + 8 * c));
      const float4 f1 = __ldg(reinterpret_cast<const float4*>(Mp + i * 128 + 8 * c + 4));
      x[0] = f0.x; x[1] = f0.y; x[2] = f0.z; x[3] = f0.w; x[4] = f1.x; x[5] = f1.y; x[6] = f1.z; x[7] = f1.w;
      qm_split8(x, hi, lo);
      sts128(base + kUpMH + swz_chunk(i, c), hi);
      sts128(base + kUpML + swz_chunk(i, c), lo);
    }
  }
  __syncthreads();  // gz, z staged
  // sigma(K) of this thread's 32 columns -> A tiles; partial den_k (delta)
  {
    float dpart = 0.f;
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = 4 * qq + i;
      float x[8];
      if (valid) {
        const uint4 w = kw[i];
        const uint32_t wp[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          x[2 * e] = elu1_accurate(bf16_lo(wp[e]));
          x[2 * e + 1] = elu1_accurate(bf16_hi(wp[e]));
        }
      } else {
#pragma unroll
        for (int e = 0; e < 8; ++e) x[e] = 0.f;
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) dpart = fmaf(x[e], zs[8 * c + e], dpart);
      uint4 hi, lo;
      qm_split8(x, hi, lo);
      sts128(base + kUpAH + swz_chunk(row, c), hi);
      sts128(base + kUpAL + swz_chunk(row, c), lo);
    }
    xs[qq * 128 + row] = dpart;
  }
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tDU = tmem, tR = tmem + 128u, tDS = tmem + 256u;
  // a row quantity from its four column quarters, in a fixed order
  auto rowsum = [&](int quantity) {
    const float* x4 = xs + quantity * 512 + row;
    return ((x4[0] + x4[128]) + x4[256]) + x4[384];
  };
  const float den = delta ? rowsum(0) : 0.f;
  // d (+)= A B in hi / lo parts: aH bH + aH bL (+ aL bH when `alo`); B MN-major or K-major
  auto issue3 = [&](uint32_t d, uint32_t aH, uint32_t aL, bool alo, uint32_t bH, uint32_t bL, bool bmn, bool acc0) {
    const uint32_t idesc = bmn ? idesc_bf16(128, 128, 0, 1) : idesc_bf16(128, 128, 0, 0);
#pragma unroll
    for (int kk = 0; kk < 8; ++kk) {
      const uint64_t dbH = bmn ? mnmajor_desc(bH, kk) : kmajor_desc(bH, kk);
      const uint64_t dbL = bmn ? mnmajor_desc(bL, kk) : kmajor_desc(bL, kk);
      mma_ss(d, kmajor_desc(aH, kk), dbH, idesc, (acc0 || kk > 0) ? 1u : 0u);
      mma_ss(d, kmajor_desc(aH, kk), dbL, idesc, 1u);
      if (alo) mma_ss(d, kmajor_desc(aL, kk), dbH, idesc, 1u);
    }
  };
  // products 1 (and 2): sigma(K) G, sigma(K) M
  if (tid == 0) {
    issue3(tDU, base + kUpAH, base + kUpAL, true, base + kUpGH, base + kUpGL, true, false);
    if (delta) issue3(tR, base + kUpAH, base + kUpAL, true, base + kUpMH, base + kUpML, true, false);
    mma_commit(bar);
  }
  mbar_wait(bar, 0);
  tc_fence_after();
  // dU -> dv term; U = V (- R) -> A tiles; delta: d_num_r, d_den_r
  float dd = 0.f;
  {
    const int c0 = 32 * qq;
    uint32_t du[32], rr[32];
    tmem_ld32(tDU + lq + (uint32_t)c0, du);
    if (delta) tmem_ld32(tR + lq + (uint32_t)c0, rr);
    tmem_ld_wait();
    float u[32], w[32];
    if (valid) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 vv = __ldg(reinterpret_cast<const uint4*>(v + grow * 128 + c0) + i);
        const uint32_t wp[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          u[8 * i + 2 * e] = bf16_lo(wp[e]);
          u[8 * i + 2 * e + 1] = bf16_hi(wp[e]);
        }
      }
      float4* dvd = reinterpret_cast<float4*>(dv_upd + grow * 128 + c0);
#pragma unroll
      for (int i = 0; i < 8; ++i)
        dvd[i] = make_float4(__uint_as_float(du[4 * i]), __uint_as_float(du[4 * i + 1]), __uint_as_float(du[4 * i + 2]),
                             __uint_as_float(du[4 * i + 3]));
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) u[e] = 0.f;
    }
    if (delta) {
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const float R = den != 0.f ? __uint_as_float(rr[e]) / den : 0.f;
        if (valid) u[e] -= R;
        w[e] = (valid && den != 0.f) ? -__uint_as_float(du[e]) / den : 0.f;
        dd = fmaf(__uint_as_float(du[e]), R, dd);
      }
      if (valid) {
        float4* dn = reinterpret_cast<float4*>(dnum_r + grow * 128 + c0);
#pragma unroll
        for (int i = 0; i < 8; ++i) dn[i] = make_float4(w[4 * i], w[4 * i + 1], w[4 * i + 2], w[4 * i + 3]);
      }
    }
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      uint4 hi, lo;
      qm_split8(u + 8 * i, hi, lo);  // linear: V exact, lo = 0
      sts128(base + kUpAH + swz_chunk(row, c0 / 8 + i), hi);
      if (delta) sts128(base + kUpAL + swz_chunk(row, c0 / 8 + i), lo);
    }
  }
  if (delta) xs[512 + qq * 128 + row] = dd;
  fence_proxy_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const float d_den = (delta && den != 0.f) ? rowsum(1) / den : 0.f;
  if (delta && qq == 0 && valid) dden_r[grow] = d_den;
  // product 3: U G^T (linear: V G^T, V exact)
  if (tid == 0) {
    issue3(tDS, base + kUpAH, base + kUpAL, delta, base + kUpGH, base + kUpGL, false, false);
    mma_commit(bar);
  }
  mbar_wait(bar, 1);
  tc_fence_after();
  if (delta) {
    // product 4: d_num_r M^T into the same accumulator; d_num_r back from global (just written)
    {
      const int c0 = 32 * qq;
      float w[32];
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 f = valid ? __ldg(reinterpret_cast<const float4*>(dnum_r + grow * 128 + c0) + i)
                               : make_float4(0.f, 0.f, 0.f, 0.f);
        w[4 * i] = f.x; w[4 * i + 1] = f.y; w[4 * i + 2] = f.z; w[4 * i + 3] = f.w;
      }
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 hi, lo;
        qm_split8(w + 8 * i, hi, lo);
        sts128(base + kUpAH + swz_chunk(row, c0 / 8 + i), hi);
        sts128(base + kUpAL + swz_chunk(row, c0 / 8 + i), lo);
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      issue3(tDS, base + kUpAH, base + kUpAL, true, base + kUpMH, base + kUpML, false, true);
      mma_commit(bar);
    }
    mbar_wait(bar, 0);
    tc_fence_after();
  }
  // dk term: sigma'(k) (dsigma(K) + gz + d_den_r z)
  {
    const int c0 = 32 * qq;
    uint32_t ds[32];
    tmem_ld32(tDS + lq + (uint32_t)c0, ds);
    tmem_ld_wait();
    if (valid) {
      float o[32];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 kw = __ldg(reinterpret_cast<const uint4*>(k + grow * 128 + c0) + i);
        const uint32_t wp[4] = {kw.x, kw.y, kw.z, kw.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int j = 8 * i + 2 * e;
          const float x0 = bf16_lo(wp[e]), x1 = bf16_hi(wp[e]);
          const float s0 = x0 > 0.f ? 1.f : expf(x0), s1 = x1 > 0.f ? 1.f : expf(x1);
          o[j] = s0 * (__uint_as_float(ds[j]) + gz[c0 + j] + d_den * zs[c0 + j]);
          o[j + 1] = s1 * (__uint_as_float(ds[j + 1]) + gz[c0 + j + 1] + d_den * zs[c0 + j + 1]);
        }
      }
      float4* dst = reinterpret_cast<float4*>(dk_upd + grow * 128 + c0);
#pragma unroll
      for (int i = 0; i < 8; ++i) dst[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// The memory gradient's partial sums sigma(X)^T Y (dk x dv) and
// sigma(X)^T y0 (dk) over the rows of one (b, h, segment, row group) on the
// tensor cores, for bf16 X with d_key = d_value = 128: the quantity
// bwd_outer_kernel (bwd_mem.cuh) computes on CUDA cores, same partial layout
// [BH][nseg][G][dk * dv + dk].  X = Q with Y = d_num, y0 = d_den (the memory
// read's terms, Eq. 7) or X = K with Y = d_num_r, y0 = d_den_r (the delta
// rule's retrieval, Eq. 9).  Per 128-row block:
//   sigma(X) (fp32, the accurate ELU + 1) and Y as bf16 hi + lo tiles, rows
//   = the product's K index: sigma^T is the MN-major A operand, Y the MN-major
//   B operand; D += s_hi^T Y_hi + s_hi^T Y_lo + s_lo^T Y_hi (~2^-16
//   relative, fp32 in TMEM);
//   y0's hi and lo parts as rows 0 and 1 of a 16-row K-major B tile (rows
//   2-15 zero): Dz += (s_hi + s_lo)^T [y0_hi | y0_lo | 0], and
//   sigma^T y0 = Dz[:, 0] + Dz[:, 1].
// 512 threads: thread (row r = TMEM lane, quarter qq) stages columns
// [32 qq, 32 qq + 32) of row r and writes those of row r's partial; thread 0
// issues the products.  A group with no rows writes a zero partial.
constexpr int kOtThreads = 512;
constexpr uint32_t kOtAH = 0, kOtAL = 32768, kOtYH = 65536, kOtYL = 98304;  // 128 x 128 bf16 tiles
constexpr uint32_t kOtY0 = 131072;       // 16 x 128 bf16 K-major (two 2 KB boxes)
constexpr uint32_t kOtBAR = kOtY0 + 4096;
constexpr uint32_t kOtSLOT = kOtBAR + 16;
constexpr uint32_t kOtSmem = kOtSLOT + 16 + 1024;

__device__ __forceinline__ void sts16(uint32_t a, unsigned short v) {
  asm volatile("st.shared.u16 [%0], %1;" ::"r"(a), "h"(v) : "memory");
}

__global__ void __launch_bounds__(kOtThreads, 1)
    bwd_outer_tc_kernel(const __nv_bfloat16* __restrict__ x, const float* __restrict__ Y,
                        const float* __restrict__ y0, int N, long long L, int seg0, int nseg, int G, int cpb,
                        float* __restrict__ partial) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  uint8_t* gbase = smem_raw + (base - raw);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  // as a programmatic dependent (the delta rule's reverse steps), nothing the
  // previous kernel reads or writes is touched before it has completed
  griddep_launch_dependents();
  griddep_wait();
  int idx = blockIdx.x;
  const int grp = idx % G;
  idx /= G;
  const int sl = idx % nseg;
  const int bh = idx / nseg;
  const long long seg_start = (long long)(seg0 + sl) * N;
  const int n_s = (int)min((long long)N, L - seg_start);
  const int t_begin = grp * cpb * 128;
  const int t_end = min(n_s, t_begin + cpb * 128);
  const int nblk = t_begin < t_end ? (t_end - t_begin + 127) / 128 : 0;
  const uint32_t bar = base + kOtBAR;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(gbase + kOtSLOT);
  const int row = 32 * (warp & 3) + lane, qq = warp >> 2;  // row of the block (TMEM lane: dk index), column quarter
  const uint32_t lq = (uint32_t)(32 * (warp & 3)) << 16;

  if (tid == 0) {
    mbar_init(bar, 1);
    fence_barrier_init();
  }
  if (tid < 256) sts128(base + kOtY0 + 16u * (uint32_t)tid, make_uint4(0u, 0u, 0u, 0u));  // the y0 tile, 4 KB
  if (warp == 0) {
    tmem_alloc(smem_u32(tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t tD = tmem, tZ = tmem + 128u;

#pragma unroll 1
  for (int blk = 0; blk < nblk; ++blk) {
    const int r0 = t_begin + 128 * blk;
    const bool valid = row < t_end - r0;
    const long long grow = (long long)bh * L + seg_start + r0 + row;
    if (row < t_end - r0 - 128) {  // the next block's row: into L2 while this one is staged and multiplied
      if ((qq & 1) == 0) prefetch_l2(x + (grow + 128) * 128 + 32 * qq);
      prefetch_l2(Y + (grow + 128) * 128 + 32 * qq);
    }
    // this thread's x and Y chunks, all loads issued before any store (and
    // while the previous block's products run)
    uint4 xw[4];
    float4 yf[8];
#pragma unroll
    for (int i = 0; i < 4; ++i)
      xw[i] = valid ? __ldg(reinterpret_cast<const uint4*>(x + grow * 128) + 4 * qq + i) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      yf[i] = valid ? __ldg(reinterpret_cast<const float4*>(Y + grow * 128 + 32 * qq) + i)
                    : make_float4(0.f, 0.f, 0.f, 0.f);
    if (blk > 0) {
      mbar_wait(bar, (uint32_t)(blk - 1) & 1u);  // the previous block's products have read the tiles
      tc_fence_after();
    }
    // sigma(x) of this thread's 32 columns (rows past the end: sigma = 0)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = 4 * qq + i;
      float v[8];
      const uint32_t wp[4] = {xw[i].x, xw[i].y, xw[i].z, xw[i].w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        v[2 * e] = valid ? elu1_accurate(bf16_lo(wp[e])) : 0.f;
        v[2 * e + 1] = valid ? elu1_accurate(bf16_hi(wp[e])) : 0.f;
      }
      uint4 hi, lo;
      qm_split8(v, hi, lo);
      sts128(base + kOtAH + swz_chunk(row, c), hi);
      sts128(base + kOtAL + swz_chunk(row, c), lo);
    }
    // Y of this thread's 32 columns
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int c = 4 * qq + i;
      const float v[8] = {yf[2 * i].x, yf[2 * i].y, yf[2 * i].z, yf[2 * i].w,
                          yf[2 * i + 1].x, yf[2 * i + 1].y, yf[2 * i + 1].z, yf[2 * i + 1].w};
      uint4 hi, lo;
      qm_split8(v, hi, lo);
      sts128(base + kOtYH + swz_chunk(row, c), hi);
      sts128(base + kOtYL + swz_chunk(row, c), lo);
    }
    // y0 of this row: element (n, k = row) of the K-major tile, n = 0 (hi), 1 (lo)
    if (qq == 0) {
      const float v = valid ? y0[grow] : 0.f;
      const __nv_bfloat16 vh = __float2bfloat16_rn(v);
      const __nv_bfloat16 vl = __float2bfloat16_rn(v - __bfloat162float(vh));
      const int c = row >> 3;
#pragma unroll
      for (int n = 0; n < 2; ++n) {
        const uint32_t a = base + kOtY0 + (uint32_t)(c >> 3) * 2048u + (uint32_t)n * 128u +
                           ((uint32_t)((c & 7) ^ n) << 4) + (uint32_t)(row & 7) * 2u;
        sts16(a, __bfloat16_as_ushort(n == 0 ? vh : vl));
      }
    }
    fence_proxy_async_smem();
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (tid == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, 128, 1, 1);  // A = sigma^T, B = Y: both MN-major
      constexpr uint32_t idesc_z = idesc_bf16(128, 16, 1, 0);  // B = the y0 tile, K-major
#pragma unroll
      for (int kk = 0; kk < 8; ++kk) {
        const uint32_t acc = (blk > 0 || kk > 0) ? 1u : 0u;
        const uint64_t aH = mnmajor_desc(base + kOtAH, kk), aL = mnmajor_desc(base + kOtAL, kk);
        const uint64_t bH = mnmajor_desc(base + kOtYH, kk), bL = mnmajor_desc(base + kOtYL, kk);
        const uint64_t bz = ones_desc(base + kOtY0, kk);
        mma_ss(tD, aH, bH, idesc, acc);
        mma_ss(tD, aH, bL, idesc, 1u);
        mma_ss(tD, aL, bH, idesc, 1u);
        mma_ss(tZ, aH, bz, idesc_z, acc);
        mma_ss(tZ, aL, bz, idesc_z, 1u);
      }
      mma_commit(bar);
    }
  }
  if (nblk > 0) {
    mbar_wait(bar, (uint32_t)(nblk - 1) & 1u);
    tc_fence_after();
  }
  // row `row` (a dk index) of the partial: columns [32 qq, 32 qq + 32), and
  // (qq = 0) its sigma^T y0 entry
  float* out = partial + (((long long)bh * nseg + sl) * G + grp) * (long long)(16384 + 128);
  {
    const int c0 = 32 * qq;
    uint32_t v[32];
    if (nblk > 0) {
      tmem_ld32(tD + lq + (uint32_t)c0, v);
      tmem_ld_wait();
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = 0u;
    }
    float4* dst = reinterpret_cast<float4*>(out + row * 128 + c0);
#pragma unroll
    for (int i = 0; i < 8; ++i)
      dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]), __uint_as_float(v[4 * i + 2]),
                           __uint_as_float(v[4 * i + 3]));
  }
  if (qq == 0) {
    float zsum = 0.f;
    if (nblk > 0) {
      uint32_t v[16];
      tmem_ld16(tZ + lq, v);
      tmem_ld_wait();
      zsum = __uint_as_float(v[0]) + __uint_as_float(v[1]);
    }
    out[16384 + row] = zsum;
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 0) {
    tc_fence_after();
    tmem_dealloc(tmem, 256);
  }
}

}  // namespace tc
}  // namespace infini
