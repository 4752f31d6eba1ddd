// CUDA-core kernels of the Infini-attention forward: any head size up to
// 128, fp32 or bf16 inputs, fp32 arithmetic throughout.  They serve the fp32
// inputs (where tensor-core rounding would not meet an fp32 tolerance) and
// every shape the tensor-core kernels do not cover.
//
// The decomposition is the same as on the tensor-core path:
//   1. update partials  -- per (b, h, segment, token group): the group's share
//      of sigma(K)^T U with U = V (linear rule, Eq. 8) or
//      U = V - sigma(K) M_{s-1} / (sigma(K) z_{s-1}) (delta rule, Eq. 9),
//      and of sum_t sigma(K_t);
//   2. state kernel     -- adds the partials to the running (M, z) in a fixed
//      order and writes the per-segment snapshots (M_{s-1}, z_{s-1});
//   3. attention kernel -- A_dot (Eq. 6), A_mem from the snapshot (Eq. 7) and
//      the gate (Eq. 10), fused, one output write.
#pragma once

#include "common.cuh"

namespace infini {

struct Geo {
  int B, H;
  long long L;
  int N, dk, dv, S;
  long long qs[3], ks[3], vs[3], os[3];  // element strides of (B, H, L)
  long long qms[3];                       // strides of the attention kernel's un-rotated q (qm)
};

__device__ __forceinline__ long long off3(const long long (&st)[3], int b, int h, long long l) {
  return b * st[0] + h * st[1] + l * st[2];
}

__device__ __forceinline__ float warp_max(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, o));
  return x;
}
__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
  return x;
}

// Partial layout: [BH][nseg][G][dk*dv + dk] fp32; M part row-major [dk][dv].
//
// Grid: BH * nseg * G blocks of 256 threads.  Block (bh, segment seg0 + sl,
// group grp) covers tokens [grp*cpb*128, min((grp+1)*cpb*128, n_s)) of the
// segment.  snapM / snapz hold M_{s-1}, z_{s-1} (fp32 [BH][S][dk][dv] and
// [BH][S][dk]); snapM == nullptr selects the linear rule.
template <typename T>
__global__ void __launch_bounds__(256) simt_update_kernel(const T* __restrict__ k, const T* __restrict__ v, Geo g,
                                                          int seg0, int nseg, int G, int cpb,
                                                          const float* __restrict__ snapM,
                                                          const float* __restrict__ snapz,
                                                          float* __restrict__ partial) {
  extern __shared__ float sm[];
  const int dk = g.dk, dv = g.dv, tid = threadIdx.x;
  int idx = blockIdx.x;
  const int grp = idx % G;
  idx /= G;
  const int sl = idx % nseg;
  const int bh = idx / nseg;
  const int s = seg0 + sl;
  const int b = bh / g.H, h = bh % g.H;
  const long long seg_start = (long long)s * g.N;
  const int n_s = (int)min((long long)g.N, g.L - seg_start);
  const int t_begin = grp * cpb * 128;
  const int t_end = min(n_s, t_begin + cpb * 128);
  const bool delta = snapM != nullptr;

  float* sk = sm;             // [32][dk]
  float* u = sk + 32 * dk;    // [32][dv]
  float* den = u + 32 * dv;   // [32]
  float* Mp = den + 32;       // [dk][dv]  (delta)
  float* zp = Mp + dk * dv;   // [dk]      (delta)
  if (delta) {
    const float* Ms = snapM + ((long long)bh * g.S + s) * dk * dv;
    for (int e = tid; e < dk * dv; e += 256) Mp[e] = Ms[e];
    for (int e = tid; e < dk; e += 256) zp[e] = snapz[((long long)bh * g.S + s) * dk + e];
  }

  const int E = dk * dv;
  float acc[64];
#pragma unroll
  for (int r = 0; r < 64; ++r) acc[r] = 0.f;
  float accz = 0.f;

  for (int t0 = t_begin; t0 < t_end; t0 += 32) {
    const int nt = min(32, t_end - t0);
    __syncthreads();
    for (int e = tid; e < 32 * dk; e += 256) {
      const int tt = e / dk, i = e - tt * dk;
      float x = 0.f;
      if (tt < nt) x = elu1_accurate(to_f32(k[off3(g.ks, b, h, seg_start + t0 + tt) + i]));
      sk[e] = x;
    }
    for (int e = tid; e < 32 * dv; e += 256) {
      const int tt = e / dv, j = e - tt * dv;
      u[e] = tt < nt ? to_f32(v[off3(g.vs, b, h, seg_start + t0 + tt) + j]) : 0.f;
    }
    __syncthreads();
    if (delta) {
      if (tid < 32) {
        float d = 0.f;
        for (int i = 0; i < dk; ++i) d = fmaf(sk[tid * dk + i], zp[i], d);
        den[tid] = d;
      }
      __syncthreads();
      // U = V - sigma(K) M_{s-1} / (sigma(K) z_{s-1}); a zero denominator retrieves zero.
      for (int e = tid; e < 32 * dv; e += 256) {
        const int tt = e / dv, j = e - tt * dv;
        const float d = den[tt];
        if (d != 0.f) {
          float r = 0.f;
          for (int i = 0; i < dk; ++i) r = fmaf(sk[tt * dk + i], Mp[i * dv + j], r);
          u[e] -= r / d;
        }
      }
      __syncthreads();
    }
#pragma unroll
    for (int r = 0; r < 64; ++r) {
      const int e = tid + 256 * r;
      if (e < E) {
        const int i = e / dv, j = e - i * dv;
        float a = acc[r];
        for (int tt = 0; tt < nt; ++tt) a = fmaf(sk[tt * dk + i], u[tt * dv + j], a);
        acc[r] = a;
      }
    }
    if (tid < dk)
      for (int tt = 0; tt < nt; ++tt) accz += sk[tt * dk + tid];
  }
  float* out = partial + (((long long)bh * nseg + sl) * G + grp) * (long long)(E + dk);
#pragma unroll
  for (int r = 0; r < 64; ++r) {
    const int e = tid + 256 * r;
    if (e < E) out[e] = acc[r];
  }
  if (tid < dk) out[E + tid] = accz;
}

// Running state and snapshots.  Thread e of block (x, bh) owns element e of
// the concatenation [M (dk*dv) | z (dk)] of head bh.
//   op 0 (linear scan): for each segment sl < nseg, snapshot then add the
//        segment's G partials; finally store the state (M_S, z_S).
//   op 1 (delta step of segment s): add the G partials of the one segment
//        in `partial`, store, and snapshot as segment s + 1 if it exists.
//   op 2 (snapshot only): snapshot the state as segment s.
// Snapshots are fp32 [BH][S][dk][dv] (snapM32) and/or, for the tensor-core
// kernels, bf16 [BH][S][dk][dv] (snapM16); z snapshots fp32.  `counter`, when
// given (op 2), is set to zero (the next attention launch's work counter); a
// programmatic dependent launch may start as soon as every block has begun.
__global__ void __launch_bounds__(256) state_kernel(float* __restrict__ M, float* __restrict__ z,
                                                    const float* __restrict__ partial, int dk, int dv, int S, int op,
                                                    int s, int nseg, int G, float* __restrict__ snapM32,
                                                    __nv_bfloat16* __restrict__ snapM16,
                                                    float* __restrict__ snapz, unsigned int* __restrict__ counter) {
  griddep_launch_dependents();
  const int bh = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  const int E = dk * dv;
  if (e >= E + dk) return;
  float* st = e < E ? &M[(long long)bh * E + e] : &z[(long long)bh * dk + (e - E)];
  float acc = *st;
  const long long pstride = E + dk;
  auto snap = [&](int seg, float val) {
    const long long base = (long long)bh * S + seg;
    if (e < E) {
      if (snapM32) snapM32[base * E + e] = val;
      if (snapM16) snapM16[base * E + e] = __float2bfloat16_rn(val);
    } else if (snapz) {
      snapz[base * dk + (e - E)] = val;
    }
  };
  if (op == 0) {
    // eight segments at a time: their partial sums are loaded together, so
    // the scan waits on memory once per eight segments rather than per segment
    for (int s8 = 0; s8 < nseg; s8 += 8) {
      float d[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        d[u] = 0.f;
        if (s8 + u < nseg) {
          const float* p = partial + ((long long)bh * nseg + s8 + u) * G * pstride + e;
          for (int gi = 0; gi < G; ++gi) d[u] += p[gi * pstride];
        }
      }
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        if (s8 + u < nseg) {
          snap(s8 + u, acc);
          acc += d[u];
        }
      }
    }
    *st = acc;
  } else if (op == 1) {
    const float* p = partial + (long long)bh * G * pstride + e;
    for (int gi = 0; gi < G; ++gi) acc += p[gi * pstride];
    *st = acc;
    if (s + 1 < S) snap(s + 1, acc);
  } else {
    snap(s, acc);
    if (counter != nullptr && e == 0 && bh == 0) *counter = 0u;
  }
}

// Fused A_dot + A_mem + gate on CUDA cores.  Block = 8 warps handling 32
// query rows of one (b, h, segment); warp w owns rows 4w .. 4w+3.  Key /
// value tiles of 32 rows are staged in shared memory; the online softmax
// keeps a running max and sum per row; the memory read uses the fp32
// snapshot M_{s-1}, z_{s-1} of the segment.
template <typename T>
__global__ void __launch_bounds__(256, 3) simt_attn_kernel(const T* __restrict__ q, const T* __restrict__ k,
                                                        const T* __restrict__ v, const float* __restrict__ beta,
                                                        T* __restrict__ out, Geo g, float scale, int QT,
                                                        const float* __restrict__ snapM,
                                                        const float* __restrict__ snapz,
                                                        const T* __restrict__ qm, float* __restrict__ adot_out,
                                                        float* __restrict__ lse_out) {
  extern __shared__ float sm[];
  const int dk = g.dk, dv = g.dv, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BHS = g.B * g.H * g.S;
  const int qb = QT - 1 - (int)(blockIdx.x / BHS);  // heaviest query blocks first
  const int rem = (int)(blockIdx.x % BHS);
  const int bh = rem / g.S, s = rem % g.S;
  const int b = bh / g.H, h = bh % g.H;
  const long long seg_start = (long long)s * g.N;
  const int n_s = (int)min((long long)g.N, g.L - seg_start);
  const int q0 = qb * 32;
  if (q0 >= n_s) return;
  const int qlast = min(n_s, q0 + 32) - 1;

  float* Ks = sm;                  // [32][dk+1]
  float* Vs = Ks + 32 * (dk + 1);  // [32][dv]
  float* Qs = Vs + 32 * dv;        // [32][dk]
  for (int e = tid; e < 32 * dk; e += 256) {
    const int r = e / dk, i = e - r * dk;
    Qs[e] = (q0 + r < n_s) ? to_f32(q[off3(g.qs, b, h, seg_start + q0 + r) + i]) : 0.f;
  }

  float o[4][4], m_i[4], l_i[4];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    m_i[rr] = -INFINITY;
    l_i[rr] = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) o[rr][c] = 0.f;
  }
  const int nkt = qlast / 32 + 1;
  for (int kt = 0; kt < nkt; ++kt) {
    __syncthreads();
    for (int e = tid; e < 32 * dk; e += 256) {
      const int r = e / dk, i = e - r * dk;
      const int kk = kt * 32 + r;
      Ks[r * (dk + 1) + i] = kk < n_s ? to_f32(k[off3(g.ks, b, h, seg_start + kk) + i]) : 0.f;
    }
    for (int e = tid; e < 32 * dv; e += 256) {
      const int r = e / dv, j = e - r * dv;
      const int kk = kt * 32 + r;
      Vs[e] = kk < n_s ? to_f32(v[off3(g.vs, b, h, seg_start + kk) + j]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = warp * 4 + rr;
      const int qi = q0 + r;
      if (qi > qlast) continue;  // warp-uniform
      if (kt * 32 > qi) continue;
      const int key = kt * 32 + lane;
      float sc = -INFINITY;
      if (key <= qi) {
        float d = 0.f;
        for (int i = 0; i < dk; ++i) d = fmaf(Qs[r * dk + i], Ks[lane * (dk + 1) + i], d);
        sc = d * scale;
      }
      const float mx = warp_max(sc);
      const float m_new = fmaxf(m_i[rr], mx);
      const float p = key <= qi ? expf(sc - m_new) : 0.f;
      const float alpha = expf(m_i[rr] - m_new);
      l_i[rr] = l_i[rr] * alpha + warp_sum(p);
      m_i[rr] = m_new;
#pragma unroll
      for (int c = 0; c < 4; ++c) o[rr][c] *= alpha;
      const int jmax = min(31, qi - kt * 32);
      for (int jj = 0; jj <= jmax; ++jj) {
        const float pj = __shfl_sync(0xffffffffu, p, jj);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = lane + 32 * c;
          if (col < dv) o[rr][c] = fmaf(pj, Vs[jj * dv + col], o[rr][c]);
        }
      }
    }
  }

  if (qm != nullptr) {
    // q and k carry rotary position embeddings for the scores above; the
    // memory read takes sigma of the un-rotated rows
    __syncthreads();
    for (int e = tid; e < 32 * dk; e += 256) {
      const int r = e / dk, i = e - r * dk;
      Qs[e] = (q0 + r < n_s) ? to_f32(qm[off3(g.qms, b, h, seg_start + q0 + r) + i]) : 0.f;
    }
    __syncthreads();
  }
  const float gw = 1.f / (1.f + expf(-beta[h]));
  const float* Mp = snapM + ((long long)bh * g.S + s) * dk * dv;
  const float* zp = snapz + ((long long)bh * g.S + s) * dk;
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = warp * 4 + rr;
    const int qi = q0 + r;
    if (qi > qlast) continue;
    float num[4] = {0.f, 0.f, 0.f, 0.f};
    float den = 0.f;
    for (int i = 0; i < dk; ++i) {
      const float sq = elu1_accurate(Qs[r * dk + i]);
      den = fmaf(sq, zp[i], den);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col = lane + 32 * c;
        if (col < dv) num[c] = fmaf(sq, Mp[i * dv + col], num[c]);
      }
    }
    const float inv_l = 1.f / l_i[rr];
    T* orow = out + off3(g.os, b, h, seg_start + qi);
    // for the backward's recomputation: A_dot and log-sum-exp of the row,
    // [B*H*L][dv] and [B*H*L] (contiguous), when asked for
    const long long xrow = (long long)bh * g.L + seg_start + qi;
    if (lse_out != nullptr && lane == 0) lse_out[xrow] = m_i[rr] + logf(l_i[rr]);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int col = lane + 32 * c;
      if (col < dv) {
        const float a_mem = den != 0.f ? num[c] / den : 0.f;
        orow[col] = from_f32<T>(gw * a_mem + (1.f - gw) * (o[rr][c] * inv_l));
        if (adot_out != nullptr) adot_out[xrow * dv + col] = o[rr][c] * inv_l;
      }
    }
  }
}

}  // namespace infini
