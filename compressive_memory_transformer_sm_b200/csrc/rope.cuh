// rope_kernel: rotary position embeddings of q and k for the local attention
// only (section 4.1 of "Leave No Context Behind", quoted on the explainer
// page: the dot-product attention's Q, K carry position embeddings, the
// compressive memory's do not).  Writes rotated copies of q and k; the
// attention kernels read them for Q K^T, while sigma(Q) of the memory read and
// the memory update keep reading the un-rotated tensors.
//
// Rotation: the pair (x_2i, x_2i+1) of the row at position p turns by the
// angle p * base^(-2i/dk):  (x_2i cos - x_2i+1 sin, x_2i sin + x_2i+1 cos).
// The angle is formed in fp64 and reduced to [-pi, pi] before the fp32
// sine and cosine, so positions up to 2^31 keep ~1e-7 rad of accuracy (a
// product p * f formed in fp32 would carry an error of p * 2^-24 rad).
//
// HBM-bound: one read and one write of q and k.  Each thread handles E
// consecutive elements (E / 2 pairs) of the same position in q and in k, so a
// cosine / sine pair serves both tensors (and every head, when the grid has
// fewer rows than B * H).
#pragma once

#include "common.cuh"

namespace infini {

constexpr int kRopeMaxPairs = 64;  // dk <= 128

struct RopeArgs {
  const void* q;
  const void* k;
  void* qr;                 // contiguous [B, H, L, dk] rotated q
  void* kr;                 // contiguous [B, H, L, dk] rotated k
  long long qs[3], ks[3];   // element strides of the (B, H, L) dimensions of q, k
  long long L;
  long long offset;         // position of token 0
  int B, H, dk;
  double inv_freq[kRopeMaxPairs];  // base^(-2i/dk), i < dk / 2
};

template <typename T, int E>
__device__ __forceinline__ void rope_load(const T* p, float (&x)[E]) {
  if constexpr (E == 8 && sizeof(T) == 2) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      x[2 * e] = bf16_lo(w[e]);
      x[2 * e + 1] = bf16_hi(w[e]);
    }
  } else if constexpr (E == 8 && sizeof(T) == 4) {
    const float4 a = __ldg(reinterpret_cast<const float4*>(p));
    const float4 b = __ldg(reinterpret_cast<const float4*>(p) + 1);
    x[0] = a.x; x[1] = a.y; x[2] = a.z; x[3] = a.w;
    x[4] = b.x; x[5] = b.y; x[6] = b.z; x[7] = b.w;
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) x[e] = to_f32(p[e]);
  }
}

template <typename T, int E>
__device__ __forceinline__ void rope_store(T* p, const float (&x)[E]) {
  if constexpr (E == 8 && sizeof(T) == 2) {
    *reinterpret_cast<uint4*>(p) =
        make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]), pack_bf16x2(x[6], x[7]));
  } else if constexpr (E == 8 && sizeof(T) == 4) {
    reinterpret_cast<float4*>(p)[0] = make_float4(x[0], x[1], x[2], x[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(x[4], x[5], x[6], x[7]);
  } else {
#pragma unroll
    for (int e = 0; e < E; ++e) p[e] = from_f32<T>(x[e]);
  }
}

// cos and sin of pos * f: the product and its reduction modulo 2 pi in fp64,
// then the fast fp32 sine and cosine on [-pi, pi] (absolute error ~4e-7).
__device__ __forceinline__ void rope_angle(long long pos, double f, float& c, float& s) {
  const double th = (double)pos * f;
  const double turns = rint(th * 0.15915494309189535);  // th / (2 pi), nearest integer
  const double r = fma(-turns, 6.283185307179586, th);
  __sincosf((float)r, &s, &c);
}

// Thread (x, y) of block (bx, by): element group x (E elements) of token
// t = bx * blockDim.y + y of head by (then by + gridDim.y, ... when B * H
// exceeds the grid), so that no index needs a division.  E = 8 needs
// dk % 8 == 0 and vector-aligned rows, E = 2 (one pair) only an even dk.
template <typename T, int E>
__global__ void __launch_bounds__(256) rope_kernel(const __grid_constant__ RopeArgs a) {
  // the frequencies in shared memory: lanes of a warp index different pairs,
  // which a constant-bank read would serialise
  __shared__ double fr[kRopeMaxPairs];
  const int tid = threadIdx.y * blockDim.x + threadIdx.x;
  if (tid < a.dk / 2) fr[tid] = a.inv_freq[tid];
  __syncthreads();
  const int j = threadIdx.x;
  const long long t = (long long)blockIdx.x * blockDim.y + threadIdx.y;
  if (t >= a.L) return;
  const long long pos = a.offset + t;
  // the rotation of this thread's pairs, shared by q and k of every head it serves
  float cs[E / 2], sn[E / 2];
#pragma unroll
  for (int e = 0; e < E / 2; ++e) rope_angle(pos, fr[j * (E / 2) + e], cs[e], sn[e]);
  // the rotated copies are workspace buffers, never the inputs: with the
  // pointers marked so, the loads of several heads are in flight together
  const T* __restrict__ q = static_cast<const T*>(a.q);
  const T* __restrict__ k = static_cast<const T*>(a.k);
  T* __restrict__ qr = static_cast<T*>(a.qr);
  T* __restrict__ kr = static_cast<T*>(a.kr);
  const int BH = a.B * a.H;
#pragma unroll 4
  for (int bh = blockIdx.y; bh < BH; bh += gridDim.y) {
    const int b = bh / a.H, h = bh - b * a.H;
    const long long row = (long long)bh * a.L + t;
    float xq[E], xk[E];
    rope_load<T, E>(q + b * a.qs[0] + h * a.qs[1] + t * a.qs[2] + j * E, xq);
    rope_load<T, E>(k + b * a.ks[0] + h * a.ks[1] + t * a.ks[2] + j * E, xk);
#pragma unroll
    for (int e = 0; e < E; e += 2) {
      const float c = cs[e / 2], s = sn[e / 2];
      const float q0 = xq[e], q1 = xq[e + 1], k0 = xk[e], k1 = xk[e + 1];
      xq[e] = q0 * c - q1 * s;
      xq[e + 1] = q0 * s + q1 * c;
      xk[e] = k0 * c - k1 * s;
      xk[e + 1] = k0 * s + k1 * c;
    }
    rope_store<T, E>(qr + row * a.dk + j * E, xq);
    rope_store<T, E>(kr + row * a.dk + j * E, xk);
  }
}

}  // namespace infini
