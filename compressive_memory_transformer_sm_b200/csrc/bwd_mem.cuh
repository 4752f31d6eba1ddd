// The memory branch of the backward on CUDA cores, in fp32: the update's
// gradient (Eq. 8 / 9, for tensors the tensor-core kernels do not take; see
// sm100_bwdmem.cuh for those and for the memory read's) and the
// sigma(X)^T [Y | y0] partials that feed the memory-gradient chain (see
// bwd_simt.cuh for the formulas).  Every product here is a small dense one per (b, h, segment) --
// rows x 128 times 128 x 128 -- so each block stages its operands in shared
// memory and computes them with a register-tiled block product: thread
// (tx, ty) = (tid % 16, tid / 16) owns output rows 16 i + ty and columns
// 16 j + tx, and each k step loads RI + 8 operands for 8 RI fused
// multiply-adds (one load per 4-8 FMAs instead of one per FMA).  Operands are
// zero-padded to 128, so any head size up to 128 runs the same code.
#pragma once

#include "bwd_simt.cuh"

namespace infini {

constexpr int kMP = 129;  // padded row of a 128-wide fp32 tile in shared memory (conflict-free columns)

// acc[i][j] += sum_{k < K} A(16 i + ty, k) B(k, 16 j + tx), with A(m, k) at
// A[m * am + k * ak] and B(k, n) at B[k * bk + n * bn] (shared memory).
template <int RI>
__device__ __forceinline__ void mm_tile(const float* __restrict__ A, int am, int ak, const float* __restrict__ B,
                                        int bk, int bn, int K, float (&acc)[RI][8], int ty, int tx) {
#pragma unroll 2
  for (int k = 0; k < K; ++k) {
    float a[RI], b[8];
#pragma unroll
    for (int i = 0; i < RI; ++i) a[i] = A[(16 * i + ty) * am + k * ak];
#pragma unroll
    for (int j = 0; j < 8; ++j) b[j] = B[k * bk + (16 * j + tx) * bn];
#pragma unroll
    for (int i = 0; i < RI; ++i)
#pragma unroll
      for (int j = 0; j < 8; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
  }
}

// Sum over the 16 threads that share an output row (lanes with the same ty).
__device__ __forceinline__ float row16_sum(float x) {
#pragma unroll
  for (int o = 8; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// sigma'(x) from sigma(x): 1 above zero (sigma > 1), e^x = sigma at or below.
__device__ __forceinline__ float sigma_prime_of(float sg) { return sg > 1.f ? 1.f : sg; }

// Stage rows x cols of a row-major fp32 matrix (row stride `cols`) into a
// [rows_tile][kMP] shared tile, zero beyond nrows x cols (the tile is
// rows_tile x 128).  float4 loads when cols % 4 == 0 and src is 16-byte aligned.
__device__ __forceinline__ void stage_f32(float* __restrict__ dst, const float* __restrict__ src, int rows_tile,
                                          int nrows, int cols) {
  const bool vec = (cols & 3) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0;
  if (vec) {
    for (int e = threadIdx.x; e < rows_tile * 32; e += blockDim.x) {
      const int r = e >> 5, c = (e & 31) * 4;
      float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
      if (r < nrows && c < cols) x = __ldg(reinterpret_cast<const float4*>(src + (long long)r * cols + c));
      float* d = dst + r * kMP + c;
      d[0] = x.x;
      d[1] = x.y;
      d[2] = x.z;
      d[3] = x.w;
    }
  } else {
    for (int e = threadIdx.x; e < rows_tile * 128; e += blockDim.x) {
      const int r = e >> 7, c = e & 127;
      dst[r * kMP + c] = (r < nrows && c < cols) ? src[(long long)r * cols + c] : 0.f;
    }
  }
}

// Stage sigma(x) of rows x cols elements of a row-major T matrix (row stride
// `cols`) into a [rows_tile][kMP] shared tile, zero elsewhere; 16-byte loads
// when a row is a whole number of 16-byte chunks and src is aligned.
template <typename T>
__device__ __forceinline__ void stage_sigma(float* __restrict__ dst, const T* __restrict__ src, int rows_tile,
                                            int nrows, int cols) {
  constexpr int PER = 16 / (int)sizeof(T);  // elements per 16 bytes
  const bool vec = cols % PER == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0;
  if (vec) {
    constexpr int CH = 128 / PER;  // 16-byte chunks per 128 columns
    for (int e = threadIdx.x; e < rows_tile * CH; e += blockDim.x) {
      const int r = e / CH, c = (e % CH) * PER;
      float x[PER];
      if (r < nrows && c < cols) {
        const uint4 w = __ldg(reinterpret_cast<const uint4*>(src + (long long)r * cols + c));
        if constexpr (sizeof(T) == 2) {
          const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            x[2 * i] = elu1_accurate(bf16_lo(u[i]));
            x[2 * i + 1] = elu1_accurate(bf16_hi(u[i]));
          }
        } else {
          x[0] = elu1_accurate(__uint_as_float(w.x));
          x[1] = elu1_accurate(__uint_as_float(w.y));
          x[2] = elu1_accurate(__uint_as_float(w.z));
          x[3] = elu1_accurate(__uint_as_float(w.w));
        }
      } else {
#pragma unroll
        for (int i = 0; i < PER; ++i) x[i] = 0.f;
      }
#pragma unroll
      for (int i = 0; i < PER; ++i) dst[r * kMP + c + i] = x[i];
    }
  } else {
    for (int e = threadIdx.x; e < rows_tile * 128; e += blockDim.x) {
      const int r = e >> 7, c = e & 127;
      dst[r * kMP + c] = (r < nrows && c < cols) ? elu1_accurate(to_f32(src[(long long)r * cols + c])) : 0.f;
    }
  }
}

// Partials sigma(X)^T Y (dk x dy) and sigma(X)^T y0 (dk) over the rows of one
// (b, h, segment, token group), layout [BH][nseg][G][dk * dy + dk]; rows of X
// contiguous [B*H*L][dk], Y fp32 [B*H*L][dy], y0 fp32 [B*H*L].  The rows are
// staged 64 at a time; the product's K index is the token.
template <typename T>
__global__ void __launch_bounds__(256, 1) bwd_outer_kernel(const T* __restrict__ x, const float* __restrict__ Y,
                                                           const float* __restrict__ y0, BwdGeo g, int dy, int seg0,
                                                           int nseg, int G, int cpb, float* __restrict__ partial) {
  extern __shared__ float sm[];
  const int dk = g.dk, tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  int idx = blockIdx.x;
  const int grp = idx % G;
  idx /= G;
  const int sl = idx % nseg;
  const int bh = idx / nseg;
  const int s = seg0 + sl;
  const long long seg_start = (long long)s * g.N;
  const int n_s = (int)min((long long)g.N, g.L - seg_start);
  const int t_begin = grp * cpb * 128;
  const int t_end = min(n_s, t_begin + cpb * 128);
  constexpr int LY = 130;
  float* Sx = sm;              // [64][kMP] sigma(x)[t][i]
  float* Sy = Sx + 64 * kMP;   // [64][LY]  Y[t][j], y0 in column 128
  float acc[8][8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) acc[i][j] = 0.f;
  float accz = 0.f;
  for (int t0 = t_begin; t0 < t_end; t0 += 64) {
    const int nt = min(64, t_end - t0);
    const long long rb = (long long)bh * g.L + seg_start + t0;
    __syncthreads();
    stage_sigma<T>(Sx, x + rb * dk, 64, nt, dk);
    for (int e = tid; e < 64 * 128; e += 256) {
      const int t = e >> 7, c = e & 127;
      Sy[t * LY + c] = (t < nt && c < dy) ? Y[(rb + t) * dy + c] : 0.f;
    }
    if (tid < 64) Sy[tid * LY + 128] = tid < nt ? y0[rb + tid] : 0.f;
    __syncthreads();
    mm_tile<8>(Sx, 1, kMP, Sy, LY, 1, nt, acc, ty, tx);
    if (tid < 128)
      for (int t = 0; t < nt; ++t) accz = fmaf(Sx[t * kMP + tid], Sy[t * LY + 128], accz);
  }
  const int E = dk * dy;
  float* out = partial + (((long long)bh * nseg + sl) * G + grp) * (long long)(E + dk);
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const int r = 16 * i + ty;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = 16 * j + tx;
      if (r < dk && c < dy) out[r * dy + c] = acc[i][j];
    }
  }
  if (tid < dk) out[E + tid] = accz;
}

// The update's gradient terms for 64 key rows of one (b, h, segment), with
// G = dLoss/dM after the segment and gz = dLoss/dz after it (gstate):
//   dU = sigma(K) G (product 1), written as the dv term;
//   delta rule: R = sigma(K) M^(s) / den_k (product 2), U = V - R,
//     d_num_r = -dU / den_k, d_den_r = dU . R / den_k (rows written);
//   dsigma(K) = U G^T (+ d_num_r M^T) (products 3, 4) + gz (+ d_den_r z),
//   written as the dk term sigma'(k) dsigma(K).
template <typename T>
__global__ void __launch_bounds__(256, 1)
    bwd_upd_kernel(const T* __restrict__ k, const T* __restrict__ v, BwdGeo g, int seg0,
                   const float* __restrict__ gstate, long long gstride_s, long long gstride_bh,
                   const float* __restrict__ snapM, const float* __restrict__ snapz, float* __restrict__ dk_upd,
                   float* __restrict__ dv_upd, float* __restrict__ dnum_r, float* __restrict__ dden_r,
                   int blocks_per_seg) {
  extern __shared__ float sm[];
  const int dk = g.dk, dv = g.dv, tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
  const bool delta = snapM != nullptr;
  int idx = blockIdx.x;
  const int blk = idx % blocks_per_seg;
  idx /= blocks_per_seg;
  const int sl = idx % (delta ? 1 : g.S);
  const int bh = idx / (delta ? 1 : g.S);
  const int s = seg0 + sl;
  const long long seg_start = (long long)s * g.N;
  const int n_s = (int)min((long long)g.N, g.L - seg_start);
  const int r0 = blk * 64;
  if (r0 >= n_s) return;
  const int nr = min(64, n_s - r0);
  const long long row0 = (long long)bh * g.L + seg_start + r0;
  float* Gs = sm;                                   // [128][kMP] G[i][j]
  float* Ms = Gs + 128 * kMP;                       // [128][kMP] M[i][j] (delta)
  float* Sk = Ms + (delta ? 128 * kMP : 0);         // [64][kMP] sigma(k), then U
  float* W = Sk + 64 * kMP;                         // [64][kMP] d_num_r (delta)
  float* gz = W + (delta ? 64 * kMP : 0);           // [128]
  float* zs = gz + 128;                             // [128]
  float* dens = zs + 128;                           // [64]
  float* ddr = dens + 64;                           // [64]
  const float* gp = gstate + (long long)bh * gstride_bh + (long long)s * gstride_s;
  const float* Mp = delta ? snapM + ((long long)bh * g.S + s) * dk * dv : nullptr;
  stage_f32(Gs, gp, 128, dk, dv);
  if (delta) stage_f32(Ms, Mp, 128, dk, dv);
  stage_sigma<T>(Sk, k + row0 * dk, 64, nr, dk);
  if (tid < 128) {
    gz[tid] = tid < dk ? gp[dk * dv + tid] : 0.f;
    zs[tid] = (delta && tid < dk) ? snapz[((long long)bh * g.S + s) * dk + tid] : 0.f;
  }
  __syncthreads();
  if (delta && tid < 64) {
    float d = 0.f;
    for (int i = 0; i < dk; ++i) d = fmaf(Sk[tid * kMP + i], zs[i], d);
    dens[tid] = d;
  }
  float du[4][8], rr[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) du[i][j] = rr[i][j] = 0.f;
  mm_tile<4>(Sk, kMP, 1, Gs, kMP, 1, dk, du, ty, tx);  // dU = sigma(K) G
  if (delta) mm_tile<4>(Sk, kMP, 1, Ms, kMP, 1, dk, rr, ty, tx);  // sigma(K) M
  __syncthreads();  // sigma(K) is read out: its buffer takes U; the denominators are in place
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 16 * i + ty;
    const float den = delta ? dens[r] : 0.f;
    float dd = 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = 16 * j + tx;
      const bool in = r < nr && c < dv;
      const long long o = (row0 + r) * dv + c;
      float u = in ? to_f32(v[o]) : 0.f;
      if (in) dv_upd[o] = du[i][j];
      if (delta) {
        const float R = den != 0.f ? rr[i][j] / den : 0.f;
        u -= in ? R : 0.f;
        const float w = (in && den != 0.f) ? -du[i][j] / den : 0.f;
        W[r * kMP + c] = w;
        if (in) dnum_r[o] = w;
        dd = fmaf(du[i][j], R, dd);
      }
      Sk[r * kMP + c] = u;
    }
    if (delta) {
      dd = row16_sum(dd);
      const float d_den = den != 0.f ? dd / den : 0.f;
      if (tx == 0) {
        ddr[r] = d_den;
        if (r < nr) dden_r[row0 + r] = d_den;
      }
    }
  }
  __syncthreads();
  float ds[4][8];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 8; ++j) ds[i][j] = 0.f;
  mm_tile<4>(Sk, kMP, 1, Gs, 1, kMP, dv, ds, ty, tx);  // U G^T
  if (delta) mm_tile<4>(W, kMP, 1, Ms, 1, kMP, dv, ds, ty, tx);  // + d_num_r M^T
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = 16 * i + ty;
    if (r >= nr) continue;
    const float dr = delta ? ddr[r] : 0.f;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const int c = 16 * j + tx;
      if (c < dk) {
        const long long o = (row0 + r) * dk + c;
        const float sg = elu1_accurate(to_f32(k[o]));
        dk_upd[o] = sigma_prime_of(sg) * (ds[i][j] + gz[c] + dr * zs[c]);
      }
    }
  }
}

}  // namespace infini
