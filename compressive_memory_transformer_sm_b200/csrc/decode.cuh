// Token-level streaming decode of the Infini-attention layer: one new query
// row per (b, h) against the cached keys 0..n-1 of its current segment (local
// causal attention, Eq. 6, for one row), the memory read with the live
// M, z = M_{s-1}, z_{s-1} (Eq. 7) and the gate (Eq. 10), in fp32 on CUDA
// cores.  The work is one matrix-vector product per (b, h): bound by reading
// the n (dk + dv) cached elements, and by latency at small B * H.
#pragma once

#include "common.cuh"
#include "simt.cuh"

namespace infini {


// ------------------------------------------------------------------ split decode
// The same step spread over many CTAs: the keys 0..n-1 of a (b, h) are cut
// into `splits` ranges, one CTA each (grid B*H x splits), so a short batch
// still fills the GPU.  Each range yields a partial softmax state -- running
// max m, sum l and unnormalised output o -- that decode_merge_kernel combines
// in a fixed order (deterministic), adding the memory read and the gate.
// Key n - 1 is the new token: read from k_t, v_t, which CTA 0 of the (b, h)
// also appends to the caches (row n - 1); no CTA of the launch reads that row.
template <typename T>
__global__ void __launch_bounds__(256)
    decode_part_kernel(const T* __restrict__ q, const T* __restrict__ k_t, const T* __restrict__ v_t,
                       T* __restrict__ kc, T* __restrict__ vc, int N, int n, int dk, int dv, float scale, int per,
                       float* __restrict__ part) {
  __shared__ float qs[128];
  __shared__ float wm[8], wl[8], wacc[8][128];
  const int bh = blockIdx.x, split = blockIdx.y;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long BH = gridDim.x;
  if (split == 0) {  // append the token to the caches
    for (int i = tid; i < dk; i += 256) kc[((long long)bh * N + n - 1) * dk + i] = k_t[(long long)bh * dk + i];
    for (int i = tid; i < dv; i += 256) vc[((long long)bh * N + n - 1) * dv + i] = v_t[(long long)bh * dv + i];
  }
  for (int i = tid; i < dk; i += 256) qs[i] = to_f32(q[(long long)bh * dk + i]);
  __syncthreads();
  const int j0 = split * per, j1 = min(n, j0 + per);
  const T* kb = kc + (long long)bh * N * dk;
  const T* vb = vc + (long long)bh * N * dv;
  // warp w: keys j0 + 32 w' + lane for w' = w, w + 8, ... (a lane per key for the
  // scores, then a lane per column for the weighted sum of the 32 value rows)
  float m = -INFINITY, l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int jb = j0 + 32 * warp; jb < j1; jb += 256) {
    const int j = jb + lane;
    float s = -INFINITY;
    if (j < j1) {
      const T* kr = j == n - 1 ? k_t + (long long)bh * dk : kb + (long long)j * dk;
      float d = 0.f;
      for (int i = 0; i < dk; ++i) d = fmaf(qs[i], to_f32(kr[i]), d);
      s = d * scale;
    }
    const float mx = warp_max(s);
    const float mn = fmaxf(m, mx);
    const float alpha = expf(m - mn);  // 0 while m = -inf
    const float p = j < j1 ? expf(s - mn) : 0.f;
    l = l * alpha + warp_sum(p);
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] *= alpha;
    const int cnt = min(32, j1 - jb);
    for (int jj = 0; jj < cnt; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const int key = jb + jj;
      const T* vr = key == n - 1 ? v_t + (long long)bh * dv : vb + (long long)key * dv;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int d = lane + 32 * c;
        if (d < dv) acc[c] = fmaf(pj, to_f32(vr[d]), acc[c]);
      }
    }
    m = mn;
  }
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = l;
  }
#pragma unroll
  for (int c = 0; c < 4; ++c)
    if (lane + 32 * c < dv) wacc[warp][lane + 32 * c] = acc[c];
  __syncthreads();
  // the block's state: merge the eight warps in order
  float gm = -INFINITY;
  for (int w = 0; w < 8; ++w) gm = fmaxf(gm, wm[w]);
  float* out = part + ((long long)split * BH + bh) * (dv + 2);
  if (tid == 0) {
    float gl = 0.f;
    for (int w = 0; w < 8; ++w) gl += gm == -INFINITY ? 0.f : wl[w] * expf(wm[w] - gm);
    out[0] = gm;
    out[1] = gl;
  }
  for (int c = tid; c < dv; c += 256) {
    float o = 0.f;
    for (int w = 0; w < 8; ++w) o += gm == -INFINITY ? 0.f : wacc[w][c] * expf(wm[w] - gm);
    out[2 + c] = o;
  }
}

// One block per (b, h), a thread per output column: the ranges' states merged
// in split order, the memory read sigma(q) M / sigma(q) z (Eq. 7, 0 when the
// denominator is 0) and the gate (Eq. 10).
template <typename T>
__global__ void __launch_bounds__(128)
    decode_merge_kernel(const T* __restrict__ q, const float* __restrict__ beta, const float* __restrict__ M,
                        const float* __restrict__ z, const float* __restrict__ part, int splits, int H, int dk, int dv,
                        T* __restrict__ out) {
  __shared__ float sq[128];
  __shared__ float red[4];
  const int bh = blockIdx.x, h = bh % H, tid = threadIdx.x;
  const long long BH = gridDim.x;
  for (int i = tid; i < dk; i += 128) sq[i] = elu1_accurate(to_f32(q[(long long)bh * dk + i]));
  __syncthreads();
  const float* zh = z + (long long)bh * dk;
  float d = 0.f;
  for (int i = tid; i < dk; i += 128) d = fmaf(sq[i], zh[i], d);
  d = warp_sum(d);
  if ((tid & 31) == 0) red[tid >> 5] = d;
  __syncthreads();
  const float den = (red[0] + red[1]) + (red[2] + red[3]);
  float gm = -INFINITY;
  for (int sp = 0; sp < splits; ++sp) gm = fmaxf(gm, part[((long long)sp * BH + bh) * (dv + 2)]);
  float gl = 0.f;
  for (int sp = 0; sp < splits; ++sp) {
    const float* ps = part + ((long long)sp * BH + bh) * (dv + 2);
    gl += ps[0] == -INFINITY ? 0.f : ps[1] * expf(ps[0] - gm);
  }
  const float g = 1.f / (1.f + expf(-beta[h]));
  const float* Mh = M + (long long)bh * dk * dv;
  for (int c = tid; c < dv; c += 128) {
    float o = 0.f;
    for (int sp = 0; sp < splits; ++sp) {
      const float* ps = part + ((long long)sp * BH + bh) * (dv + 2);
      o += ps[0] == -INFINITY ? 0.f : ps[2 + c] * expf(ps[0] - gm);
    }
    float num = 0.f;
    for (int i = 0; i < dk; ++i) num = fmaf(sq[i], Mh[(long long)i * dv + c], num);
    const float a_mem = den != 0.f ? num / den : 0.f;
    out[(long long)bh * dv + c] = from_f32<T>(g * a_mem + (1.f - g) * (o / gl));
  }
}

}  // namespace infini

namespace infini {

// ------------------------------------------------------------------ fused decode
// The split decode in one launch: the CTAs of the key ranges of one (b, h)
// form a thread-block cluster (grid splits x B*H, cluster splits x 1); each
// computes its range's softmax state into its own shared memory, and after a
// cluster barrier rank 0 reads the others' states through distributed shared
// memory, merges them in rank order (deterministic), adds the memory read
// (Eq. 7) and the gate (Eq. 10) and writes the row; a second barrier keeps
// every CTA's shared memory alive until rank 0 is done.  No global scratch.
// The memory read is spread the same way: CTA r forms sigma(q) M and
// sigma(q) z over its slice of M's rows, before its key range, and rank 0
// adds the slices in rank order.  CTA 0 also appends k_t, v_t to row n - 1 of
// the caches (no CTA reads it).
constexpr int kDecodeMaxSplits = 16;

// q . k for one cached key row of dk elements: 16-byte vector loads when
// `vec` (dk a multiple of 8 for bf16 / 4 for fp32 and 16-byte aligned rows),
// scalar loads otherwise.
template <typename T>
__device__ __forceinline__ float decode_dot(const float* qs, const T* kr, int dk, bool vec) {
  float d = 0.f;
  if (vec) {
    const uint4* k4 = reinterpret_cast<const uint4*>(kr);
    if constexpr (sizeof(T) == 2) {
#pragma unroll 8
      for (int c = 0; c < dk / 8; ++c) {
        const uint4 w = __ldg(k4 + c);
        const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          d = fmaf(qs[8 * c + 2 * e], bf16_lo(u[e]), d);
          d = fmaf(qs[8 * c + 2 * e + 1], bf16_hi(u[e]), d);
        }
      }
    } else {
#pragma unroll 8
      for (int c = 0; c < dk / 4; ++c) {
        const float4 w = __ldg(reinterpret_cast<const float4*>(k4 + c));
        d = fmaf(qs[4 * c], w.x, d);
        d = fmaf(qs[4 * c + 1], w.y, d);
        d = fmaf(qs[4 * c + 2], w.z, d);
        d = fmaf(qs[4 * c + 3], w.w, d);
      }
    }
  } else {
    for (int i = 0; i < dk; ++i) d = fmaf(qs[i], to_f32(kr[i]), d);
  }
  return d;
}

template <typename T>
__global__ void __launch_bounds__(256)
    decode_fused_kernel(const T* __restrict__ q, const T* __restrict__ k_t, const T* __restrict__ v_t,
                        T* __restrict__ kc, T* __restrict__ vc, const float* __restrict__ beta,
                        const float* __restrict__ M, const float* __restrict__ z, T* __restrict__ out, int H, int N,
                        int n, int dk, int dv, float scale, int per, int vec) {
  __shared__ float qs[128];
  __shared__ float wm[8], wl[8], wacc[8][128];
  __shared__ __align__(16) float st[2 + 128];  // this range's state: m, l, o[dv]
  __shared__ __align__(16) float mr[2][129];   // this slice's sigma(q) M [dv] and sigma(q) z, per thread half
  __shared__ float sq[128];
  const int split = blockIdx.x, bh = blockIdx.y, splits = gridDim.x;
  const int h = bh % H;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  if (split == 0) {
    for (int i = tid; i < dk; i += 256) kc[((long long)bh * N + n - 1) * dk + i] = k_t[(long long)bh * dk + i];
    for (int i = tid; i < dv; i += 256) vc[((long long)bh * N + n - 1) * dv + i] = v_t[(long long)bh * dv + i];
  }
  for (int i = tid; i < dk; i += 256) {
    qs[i] = to_f32(q[(long long)bh * dk + i]);
    sq[i] = elu1_accurate(qs[i]);
  }
  __syncthreads();
  {
    // the memory read over rows [i0, i1) of M, z: thread (column c, half hf)
    // takes every other row; 16 independent sums keep 16 loads in flight
    const int i0 = split * dk / splits, i1 = (split + 1) * dk / splits;
    const int c = tid & 127, hf = tid >> 7;
    const float* Mh = M + (long long)bh * dk * dv;
    float nm[16];
#pragma unroll
    for (int u = 0; u < 16; ++u) nm[u] = 0.f;
    if (c < dv) {
      int i = i0 + hf;
      for (; i + 30 < i1; i += 32) {
#pragma unroll
        for (int u = 0; u < 16; ++u) nm[u] = fmaf(sq[i + 2 * u], Mh[(long long)(i + 2 * u) * dv + c], nm[u]);
      }
      for (int u = 0; i < i1; i += 2, ++u) nm[u & 15] = fmaf(sq[i], Mh[(long long)i * dv + c], nm[u & 15]);
      float t = 0.f;
#pragma unroll
      for (int u = 0; u < 16; ++u) t += nm[u];
      mr[hf][c] = t;
    }
    if (tid < 32) {  // sigma(q) z over the slice: lanes stride the rows, then the warp
      float d = 0.f;
      for (int i = i0 + tid; i < i1; i += 32) d = fmaf(sq[i], z[(long long)bh * dk + i], d);
      d = warp_sum(d);
      if (tid == 0) mr[0][128] = d;
    }
  }
  const int j0 = split * per, j1 = min(n, j0 + per);
  const T* kb = kc + (long long)bh * N * dk;
  const T* vb = vc + (long long)bh * N * dv;
  float m = -INFINITY, l = 0.f, acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int jb = j0 + 32 * warp; jb < j1; jb += 256) {
    const int j = jb + lane;
    float s = -INFINITY;
    if (j < j1) {
      const T* kr = j == n - 1 ? k_t + (long long)bh * dk : kb + (long long)j * dk;
      s = decode_dot<T>(qs, kr, dk, vec != 0) * scale;
    }
    const float mn = fmaxf(m, warp_max(s));
    const float alpha = expf(m - mn);  // 0 while m = -inf
    const float p = j < j1 ? expf(s - mn) : 0.f;
    l = l * alpha + warp_sum(p);
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[c] *= alpha;
    const int cnt = min(32, j1 - jb);
#pragma unroll 8
    for (int jj = 0; jj < cnt; ++jj) {
      const float pj = __shfl_sync(0xffffffffu, p, jj);
      const int key = jb + jj;
      const T* vr = key == n - 1 ? v_t + (long long)bh * dv : vb + (long long)key * dv;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int d = lane + 32 * c;
        if (d < dv) acc[c] = fmaf(pj, to_f32(vr[d]), acc[c]);
      }
    }
    m = mn;
  }
  if (lane == 0) {
    wm[warp] = m;
    wl[warp] = l;
  }
#pragma unroll
  for (int c = 0; c < 4; ++c)
    if (lane + 32 * c < dv) wacc[warp][lane + 32 * c] = acc[c];
  __syncthreads();
  {
    float gm = -INFINITY;
    for (int w = 0; w < 8; ++w) gm = fmaxf(gm, wm[w]);
    if (tid == 0) {
      float gl = 0.f;
      for (int w = 0; w < 8; ++w) gl += gm == -INFINITY ? 0.f : wl[w] * expf(wm[w] - gm);
      st[0] = gm;
      st[1] = gl;
    }
    for (int c = tid; c < dv; c += 256) {
      float o = 0.f;
      for (int w = 0; w < 8; ++w) o += gm == -INFINITY ? 0.f : wacc[w][c] * expf(wm[w] - gm);
      st[2 + c] = o;
    }
  }
  cluster_sync();  // every range's state is in its CTA's shared memory
  if (split == 0) {
    const uint32_t sbase = smem_u32(st), mbase = smem_u32(&mr[0][0]);
    // den = sigma(q) . z: the slices in rank order
    float den = 0.f;
    for (int r = 0; r < splits; ++r) den += ld_dsmem_f32(mapa_shared(mbase + 4u * 128u, (uint32_t)r));
    float gm = -INFINITY;
    for (int r = 0; r < splits; ++r) gm = fmaxf(gm, ld_dsmem_f32(mapa_shared(sbase, (uint32_t)r)));
    float gl = 0.f;
    for (int r = 0; r < splits; ++r) {
      const uint32_t a = mapa_shared(sbase, (uint32_t)r);
      const float mx = ld_dsmem_f32(a);
      gl += mx == -INFINITY ? 0.f : ld_dsmem_f32(a + 4u) * expf(mx - gm);
    }
    const float g = 1.f / (1.f + expf(-beta[h]));
    for (int c = tid; c < dv; c += 256) {
      float o = 0.f, num = 0.f;
      for (int r = 0; r < splits; ++r) {
        const uint32_t a = mapa_shared(sbase, (uint32_t)r);
        const float mx = ld_dsmem_f32(a);
        o += mx == -INFINITY ? 0.f : ld_dsmem_f32(a + 4u * (uint32_t)(2 + c)) * expf(mx - gm);
        const uint32_t b = mapa_shared(mbase + 4u * (uint32_t)c, (uint32_t)r);
        num += ld_dsmem_f32(b) + ld_dsmem_f32(b + 4u * 129u);  // the slice's two halves
      }
      const float a_mem = den != 0.f ? num / den : 0.f;
      out[(long long)bh * dv + c] = from_f32<T>(g * a_mem + (1.f - g) * (o / gl));
    }
  }
  cluster_sync();  // rank 0 has read every state
}

}  // namespace infini
