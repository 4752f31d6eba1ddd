// decode_kernel: token-level streaming decode of the Infini-attention layer.
// One new query row per (b, h) against the cached keys 0..n-1 of its current
// segment (local causal attention, Eq. 6, for one row), the memory read with
// the live M, z = M_{s-1}, z_{s-1} (Eq. 7) and the gate (Eq. 10), in fp32 on
// CUDA cores.  The work is one matrix-vector product per (b, h): bound by
// reading the n (dk + dv) cached elements, and by latency at small B * H.
#pragma once

#include "common.cuh"
#include "simt.cuh"

namespace infini {

constexpr int kDecodeWarps = 8;

// Block = 8 warps per (b, h): warp w takes keys w, w + 8, ...; lanes split the
// head dimensions (lane + 32 c); each warp keeps its own running max, sum and
// output row, merged in a fixed order at the end (deterministic).
template <typename T>
__global__ void __launch_bounds__(32 * kDecodeWarps)
    decode_kernel(const T* __restrict__ q, const T* __restrict__ kc, const T* __restrict__ vc,
                  const float* __restrict__ beta, const float* __restrict__ M, const float* __restrict__ z,
                  T* __restrict__ out, int H, int N, int n, int dk, int dv, float scale) {
  __shared__ float qs[128], sq[128];
  __shared__ float wm[kDecodeWarps], wl[kDecodeWarps], wacc[kDecodeWarps][128];
  __shared__ float den_s;
  const int bh = blockIdx.x, h = bh % H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const T* qrow = q + (long long)bh * dk;
  for (int i = tid; i < dk; i += blockDim.x) {
    const float x = to_f32(qrow[i]);
    qs[i] = x;
    sq[i] = elu1_accurate(x);
  }
  __syncthreads();
  const T* kb = kc + (long long)bh * N * dk;
  const T* vb = vc + (long long)bh * N * dv;
  float m = -INFINITY, l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int j = warp; j < n; j += kDecodeWarps) {
    float s = 0.f;
    for (int i = lane; i < dk; i += 32) s = fmaf(qs[i], to_f32(kb[(long long)j * dk + i]), s);
    s = warp_sum(s) * scale;
    const float mn = fmaxf(m, s);
    const float alpha = expf(m - mn);  // 0 for the first key (m = -inf)
    const float p = expf(s - mn);
    l = l * alpha + p;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int d = lane + 32 * c;
      if (d < dv) acc[c] = fmaf(p, to_f32(vb[(long long)j * dv + d]), acc[c] * alpha);
    }
    m = mn;
  }
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = l;
  }
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    const int d = lane + 32 * c;
    if (d < dv) wacc[warp][d] = acc[c];
  }
  const float* Mh = M + (long long)bh * dk * dv;
  const float* zh = z + (long long)bh * dk;
  if (warp == 0) {
    float d = 0.f;
    for (int i = lane; i < dk; i += 32) d = fmaf(sq[i], zh[i], d);
    d = warp_sum(d);
    if (lane == 0) den_s = d;
  }
  __syncthreads();
  float gm = -INFINITY;
  for (int w = 0; w < kDecodeWarps; ++w) gm = fmaxf(gm, wm[w]);
  float gl = 0.f;
  for (int w = 0; w < kDecodeWarps; ++w) gl += wl[w] * expf(wm[w] - gm);  // a warp without keys adds 0
  const float g = 1.f / (1.f + expf(-beta[h]));
  const float den = den_s;
  for (int c = tid; c < dv; c += blockDim.x) {
    float num = 0.f;
    for (int i = 0; i < dk; ++i) num = fmaf(sq[i], Mh[(long long)i * dv + c], num);
    float o = 0.f;
    for (int w = 0; w < kDecodeWarps; ++w) o = fmaf(wacc[w][c], expf(wm[w] - gm), o);
    const float a_mem = den != 0.f ? num / den : 0.f;
    out[(long long)bh * dv + c] = from_f32<T>(g * a_mem + (1.f - g) * (o / gl));
  }
}

}  // namespace infini
