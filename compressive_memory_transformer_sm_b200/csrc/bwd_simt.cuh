// Backward of the Infini-attention forward on CUDA cores (fp32 arithmetic,
// bf16 or fp32 tensors, any head size up to 128): the gradients of a scalar
// loss with respect to q, k, v, beta and the initial memory (M_0, z_0), given
// its gradients with respect to the output and the final memory (M_S, z_S).
// Back-propagation through time over the compressive memory (explainer page
// "Leave No Context Behind", section 3, "Training infrastructure"), written
// out by the chain rule through Eq. 6-10, segment by segment:
//
//   forward quantities, recomputed:   M^(s), z^(s) entering segment s (fp32),
//                                     A_dot and lse = log sum exp of each row
//   gate (Eq. 10):      d_dot = (1 - g) dA,  d_mem = g dA,
//                       dbeta = g (1 - g) sum dA . (A_mem - A_dot)
//   local (Eq. 6):      D_i = d_dot_i . A_dot_i,  p_ij = exp(c q_i.k_j - lse_i),
//                       ds_ij = p_ij (d_dot_i . v_j - D_i),
//                       dq_i = c sum_j ds_ij k_j,  dk_j = c sum_i ds_ij q_i,
//                       dv_j = sum_i p_ij d_dot_i
//   memory read (Eq. 7): den = sigma(q).z, A_mem = sigma(q) M / den,
//                       d_num = d_mem / den, d_den = -d_mem . A_mem / den,
//                       dsigma(q) = d_num M^T + d_den z^T  (zero where den = 0),
//                       and into the memory: dM^(s) += sigma(Q)^T d_num,
//                       dz^(s) += sigma(Q)^T d_den
//   update (Eq. 8/9):   with G = dLoss/dM^(s+1), gz = dLoss/dz^(s+1),
//                       U = V (linear) or V - R, R = sigma(K) M^(s) / den_k,
//                       dV += sigma(K) G,  dsigma(K) += U G^T + 1 gz^T,
//                       delta: dR = -sigma(K) G, d_num_r = dR / den_k,
//                       d_den_r = -dR . R / den_k,
//                       dsigma(K) += d_num_r M^(s)T + d_den_r z^(s)T,
//                       dM^(s) += sigma(K)^T d_num_r, dz^(s) += sigma(K)^T d_den_r
//   chain:              dM^(s) = dM^(s+1) + (the two memory terms above),
//                       dz^(s) likewise; dM^(S), dz^(S) are given.
//   sigma'(x) = 1 above zero, e^x at or below.
//
// Kernels (all deterministic: fixed summation orders, no atomics):
//   bwd_q_kernel     per (b, h, segment, 32 query rows): dq (local + memory
//                    read), D, the dbeta row terms, d_num and d_den rows
//   bwd_outer_kernel per (b, h, segment, token group): sigma(X)^T [Y | y0]
//                    partials (X = Q with d_num / d_den, or K with the delta
//                    rule's d_num_r / d_den_r)
//   bwd_state_kernel the memory-gradient chain: a reverse scan of the
//                    partials (linear rule) or one reverse step (delta rule)
//   bwd_upd_kernel   per (b, h, segment, 128 key rows): the update's dk, dv
//                    terms (and the delta rule's d_num_r, d_den_r rows)
//   bwd_kv_kernel    per (b, h, segment, 32 key rows): dk, dv of the local
//                    attention plus the update terms, one write
//   bwd_beta_kernel  dbeta per head in a fixed order
#pragma once

#include "simt.cuh"

namespace infini {

__device__ __forceinline__ float sigma_prime(float x) { return x > 0.f ? 1.f : expf(fminf(x, 0.f)); }

struct BwdGeo {
  int B, H, S, N, dk, dv;
  long long L;
};
__device__ __forceinline__ long long bwd_row(const BwdGeo& g, int bh, long long t) { return (long long)bh * g.L + t; }

// dq and the per-row terms.  Block = 8 warps, 32 query rows of one
// (b, h, segment); warp w owns rows 4w .. 4w+3; lane = key inside a key tile
// (scores) or column (accumulators).
template <typename T>
__global__ void __launch_bounds__(256, 2)
    bwd_q_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, const T* __restrict__ dout,
                 const float* __restrict__ beta, const float* __restrict__ adot, const float* __restrict__ lse,
                 const float* __restrict__ snapM, const float* __restrict__ snapz, BwdGeo g, float scale, int QT,
                 T* __restrict__ dq, float* __restrict__ Drow, float* __restrict__ brow, float* __restrict__ dnum,
                 float* __restrict__ dden) {
  extern __shared__ float sm[];
  const int dk = g.dk, dv = g.dv, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BHS = g.B * g.H * g.S;
  const int qb = QT - 1 - (int)(blockIdx.x / BHS);
  const int rem = (int)(blockIdx.x % BHS);
  const int bh = rem / g.S, s = rem % g.S;
  const int h = bh % g.H;
  const long long seg_start = (long long)s * g.N;
  const int n_s = (int)min((long long)g.N, g.L - seg_start);
  const int q0 = qb * 32;
  if (q0 >= n_s) return;
  const int qlast = min(n_s, q0 + 32) - 1;
  const float gw = 1.f / (1.f + expf(-beta[h]));

  float* Ks = sm;                  // [32][dk+1]
  float* Vs = Ks + 32 * (dk + 1);  // [32][dv]
  float* Qs = Vs + 32 * dv;        // [32][dk]
  float* Dd = Qs + 32 * dk;        // [32][dv] d_dot rows
  float* Wr = Dd + 32 * dv;        // [32][dv] per-row vector (d_num)
  for (int e = tid; e < 32 * dk; e += 256) {
    const int r = e / dk, i = e - r * dk;
    Qs[e] = (q0 + r < n_s) ? to_f32(q[bwd_row(g, bh, seg_start + q0 + r) * dk + i]) : 0.f;
  }
  for (int e = tid; e < 32 * dv; e += 256) {
    const int r = e / dv, j = e - r * dv;
    Dd[e] = (q0 + r < n_s) ? (1.f - gw) * to_f32(dout[bwd_row(g, bh, seg_start + q0 + r) * dv + j]) : 0.f;
  }
  __syncthreads();
  float Di[4], li[4], dqa[4][4];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = warp * 4 + rr, qi = q0 + r;
    float d = 0.f;
    li[rr] = 0.f;
    if (qi <= qlast) {
      const long long row = bwd_row(g, bh, seg_start + qi);
      for (int j = lane; j < dv; j += 32) d = fmaf(Dd[r * dv + j], adot[row * dv + j], d);
      li[rr] = lse[row];
    }
    Di[rr] = warp_sum(d);
#pragma unroll
    for (int c = 0; c < 4; ++c) dqa[rr][c] = 0.f;
  }
  const int nkt = qlast / 32 + 1;
  for (int kt = 0; kt < nkt; ++kt) {
    __syncthreads();
    for (int e = tid; e < 32 * dk; e += 256) {
      const int r = e / dk, i = e - r * dk;
      const int kk = kt * 32 + r;
      Ks[r * (dk + 1) + i] = kk < n_s ? to_f32(k[bwd_row(g, bh, seg_start + kk) * dk + i]) : 0.f;
    }
    for (int e = tid; e < 32 * dv; e += 256) {
      const int r = e / dv, j = e - r * dv;
      const int kk = kt * 32 + r;
      Vs[e] = kk < n_s ? to_f32(v[bwd_row(g, bh, seg_start + kk) * dv + j]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = warp * 4 + rr, qi = q0 + r;
      if (qi > qlast || kt * 32 > qi) continue;  // warp-uniform
      const int key = kt * 32 + lane;
      float ds = 0.f;
      if (key <= qi) {
        float sc = 0.f, dp = 0.f;
        for (int i = 0; i < dk; ++i) sc = fmaf(Qs[r * dk + i], Ks[lane * (dk + 1) + i], sc);
        for (int j = 0; j < dv; ++j) dp = fmaf(Dd[r * dv + j], Vs[lane * dv + j], dp);
        const float p = expf(sc * scale - li[rr]);
        ds = p * (dp - Di[rr]);
      }
      const int jmax = min(31, qi - kt * 32);
      for (int jj = 0; jj <= jmax; ++jj) {
        const float dsj = __shfl_sync(0xffffffffu, ds, jj);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = lane + 32 * c;
          if (col < dk) dqa[rr][c] = fmaf(dsj, Ks[jj * (dk + 1) + col], dqa[rr][c]);
        }
      }
    }
  }
  // memory read (Eq. 7) and the gate's beta term, row by row
  const float* Mp = snapM + ((long long)bh * g.S + s) * dk * dv;
  const float* zp = snapz + ((long long)bh * g.S + s) * dk;
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int r = warp * 4 + rr, qi = q0 + r;
    if (qi > qlast) continue;
    const long long row = bwd_row(g, bh, seg_start + qi);
    float den = 0.f;
    for (int i = 0; i < dk; ++i) den = fmaf(elu1_accurate(Qs[r * dk + i]), zp[i], den);
    float amem[4] = {0.f, 0.f, 0.f, 0.f}, dn[4] = {0.f, 0.f, 0.f, 0.f};
    if (den != 0.f) {
      for (int i = 0; i < dk; ++i) {
        const float sq = elu1_accurate(Qs[r * dk + i]);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = lane + 32 * c;
          if (col < dv) amem[c] = fmaf(sq, Mp[i * dv + col], amem[c]);
        }
      }
    }
    float dd = 0.f, bterm = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int col = lane + 32 * c;
      if (col < dv) {
        const float dA = to_f32(dout[row * dv + col]);
        const float am = den != 0.f ? amem[c] / den : 0.f;
        bterm = fmaf(dA, am - adot[row * dv + col], bterm);
        if (den != 0.f) {
          const float dmem = gw * dA;
          dn[c] = dmem / den;
          dd = fmaf(dmem, am, dd);
        }
        Wr[r * dv + col] = dn[c];
        dnum[row * dv + col] = dn[c];
      }
    }
    const float d_den = den != 0.f ? -warp_sum(dd) / den : 0.f;
    bterm = warp_sum(bterm);
    if (lane == 0) {
      Drow[row] = Di[rr];
      brow[row] = bterm;
      dden[row] = d_den;
    }
    __syncwarp();
    // dq = c * local + sigma'(q) (d_num M^T + d_den z)
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int col = lane + 32 * c;
      if (col < dk) {
        float ds = d_den * zp[col];
        if (den != 0.f)
          for (int j = 0; j < dv; ++j) ds = fmaf(Wr[r * dv + j], Mp[col * dv + j], ds);
        dq[row * dk + col] = from_f32<T>(scale * dqa[rr][c] + sigma_prime(Qs[r * dk + col]) * ds);
      }
    }
  }
}

// The memory read's backward (Eq. 7) and the per-row terms for the tensor-core
// path, where the local attention's gradients come from the tcgen05 kernels:
// for 128 query rows of one (b, h, segment) (four passes of 32; warp w: rows
// 4w .. 4w+3 of a pass, lane = column), D'_i = dO_i . A_dot_i (A_dot from the
// forward's recomputation), the dbeta row term dO_i . (A_mem_i - A_dot_i), and
// dq_mem = sigma'(q) (d_num M^T + d_den z) with d_num, d_den rows written for
// the memory chain.  M^(s) is staged in shared memory once per block.
template <typename T>
__global__ void __launch_bounds__(256, 2) bwd_qmem_kernel(const T* __restrict__ q, const T* __restrict__ dout,
                                                       const float* __restrict__ adot,
                                                       const float* __restrict__ beta,
                                                       const float* __restrict__ snapM,
                                                       const float* __restrict__ snapz, BwdGeo g,
                                                       int blocks_per_seg, float* __restrict__ dq_mem,
                                                       float* __restrict__ Dp, float* __restrict__ brow,
                                                       float* __restrict__ dnum, float* __restrict__ dden) {
  extern __shared__ float sm[];
  const int dk = g.dk, dv = g.dv, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  int idx = blockIdx.x;
  const int blk = idx % blocks_per_seg;
  idx /= blocks_per_seg;
  const int s = idx % g.S;
  const int bh = idx / g.S;
  const int h = bh % g.H;
  const long long seg_start = (long long)s * g.N;
  const int n_s = (int)min((long long)g.N, g.L - seg_start);
  const int r0 = blk * 128;
  if (r0 >= n_s) return;
  const int rend = min(n_s, r0 + 128);
  const float gw = 1.f / (1.f + expf(-beta[h]));
  float* Ms = sm;                  // [dk][dv + 1]
  float* zs = Ms + dk * (dv + 1);  // [dk]
  float* sq = zs + dk;             // [8 warps][dk] sigma(q) of the warp's current row
  float* wn = sq + 8 * dk;         // [8 warps][dv] d_num of the warp's current row
  const float* Mp = snapM + ((long long)bh * g.S + s) * dk * dv;
  for (int e = tid; e < dk * dv; e += 256) Ms[(e / dv) * (dv + 1) + e % dv] = Mp[e];
  for (int e = tid; e < dk; e += 256) zs[e] = snapz[((long long)bh * g.S + s) * dk + e];
  __syncthreads();
  float* sqw = sq + warp * dk;
  float* wnw = wn + warp * dv;
  for (int t = r0 + warp; t < rend; t += 8) {  // one row per warp at a time
    const long long row = bwd_row(g, bh, seg_start + t);
    float xq[4];
    float dpart = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = lane + 32 * c;
      xq[c] = i < dk ? to_f32(q[row * dk + i]) : 0.f;
      if (i < dk) {
        const float sg = elu1_accurate(xq[c]);
        sqw[i] = sg;
        dpart = fmaf(sg, zs[i], dpart);
      }
    }
    const float den = warp_sum(dpart);
    __syncwarp();
    float num[4] = {0.f, 0.f, 0.f, 0.f};
    if (den != 0.f) {
      for (int i = 0; i < dk; ++i) {
        const float si = sqw[i];
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (lane + 32 * c < dv) num[c] = fmaf(si, Ms[i * (dv + 1) + lane + 32 * c], num[c]);
      }
    }
    float dd = 0.f, bterm = 0.f, dpr = 0.f;
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int j = lane + 32 * c;
      if (j < dv) {
        const float dA = to_f32(dout[row * dv + j]);
        const float ad = adot[row * dv + j];
        const float am = den != 0.f ? num[c] / den : 0.f;
        dpr = fmaf(dA, ad, dpr);
        bterm = fmaf(dA, am - ad, bterm);
        float w = 0.f;
        if (den != 0.f) {
          w = gw * dA / den;
          dd = fmaf(gw * dA, am, dd);
        }
        wnw[j] = w;
        dnum[row * dv + j] = w;
      }
    }
    const float d_den = den != 0.f ? -warp_sum(dd) / den : 0.f;
    dpr = warp_sum(dpr);
    bterm = warp_sum(bterm);
    if (lane == 0) {
      Dp[row] = dpr;
      brow[row] = bterm;
      dden[row] = d_den;
    }
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int i = lane + 32 * c;
      if (i < dk) {
        float a = d_den * zs[i];
        if (den != 0.f)
          for (int j = 0; j < dv; ++j) a = fmaf(wnw[j], Ms[i * (dv + 1) + j], a);
        dq_mem[row * dk + i] = sigma_prime(xq[c]) * a;
      }
    }
    __syncwarp();
  }
}

// Partials of sigma(X)^T Y (dk x dy) and sigma(X)^T y0 (dk) for the rows of
// one (b, h, segment, token group); layout [BH][nseg][G][dk*dy + dk] like the
// forward's update partials.  Rows of X: element strides given by rows of
// length dk (contiguous [B, H, L, dk]); Y: fp32 [BH*L][dy]; y0: fp32 [BH*L].
template <typename T>
__global__ void __launch_bounds__(256) bwd_outer_kernel(const T* __restrict__ x, const float* __restrict__ Y,
                                                        const float* __restrict__ y0, BwdGeo g, int dy, int seg0,
                                                        int nseg, int G, int cpb, float* __restrict__ partial) {
  extern __shared__ float sm[];
  const int dk = g.dk, tid = threadIdx.x;
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
  float* sx = sm;            // [32][dk]
  float* sy = sx + 32 * dk;  // [32][dy + 1]: Y then y0
  const int E = dk * dy;
  float acc[64];
#pragma unroll
  for (int r = 0; r < 64; ++r) acc[r] = 0.f;
  float accz = 0.f;
  for (int t0 = t_begin; t0 < t_end; t0 += 32) {
    const int nt = min(32, t_end - t0);
    __syncthreads();
    for (int e = tid; e < 32 * dk; e += 256) {
      const int tt = e / dk, i = e - tt * dk;
      sx[e] = tt < nt ? elu1_accurate(to_f32(x[bwd_row(g, bh, seg_start + t0 + tt) * dk + i])) : 0.f;
    }
    for (int e = tid; e < 32 * (dy + 1); e += 256) {
      const int tt = e / (dy + 1), j = e - tt * (dy + 1);
      const long long row = bwd_row(g, bh, seg_start + t0 + tt);
      sy[e] = tt < nt ? (j < dy ? Y[row * dy + j] : y0[row]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int r = 0; r < 64; ++r) {
      const int e = tid + 256 * r;
      if (e < E) {
        const int i = e / dy, j = e - i * dy;
        float a = acc[r];
        for (int tt = 0; tt < nt; ++tt) a = fmaf(sx[tt * dk + i], sy[tt * (dy + 1) + j], a);
        acc[r] = a;
      }
    }
    if (tid < dk)
      for (int tt = 0; tt < nt; ++tt) accz = fmaf(sx[tt * dk + tid], sy[tt * (dy + 1) + dy], accz);
  }
  float* out = partial + (((long long)bh * nseg + sl) * G + grp) * (long long)(E + dk);
#pragma unroll
  for (int r = 0; r < 64; ++r) {
    const int e = tid + 256 * r;
    if (e < E) out[e] = acc[r];
  }
  if (tid < dk) out[E + tid] = accz;
}

// The memory-gradient chain.  Thread e of block (x, bh) owns element e of
// [dM (dk*dv) | dz (dk)] of head bh.
//   op 0 (linear, all segments): from the given dM^(S), dz^(S) (or zeros),
//        for s = S-1 .. 0: snapshot the running gradient as gsnap[s]
//        (= dLoss/d state after segment s), then add segment s's partials
//        (G groups); finally store dM^(0), dz^(0) into out0 (if given).
//   op 1 (delta, segment s): running += segment s's read partials (cpart,
//        G groups, all segments laid out) + the update partials (upart,
//        Gu groups, this segment only).
//   op 2: running = dM^(S), dz^(S) (or zeros).
//   op 3: out0 = running.
__global__ void __launch_bounds__(256) bwd_state_kernel(float* __restrict__ running, const float* __restrict__ init,
                                                        const float* __restrict__ initz, const float* __restrict__ cpart,
                                                        const float* __restrict__ upart, int dk, int dv, int S, int op,
                                                        int s, int G, int Gu, float* __restrict__ gsnap,
                                                        float* __restrict__ out0, float* __restrict__ out0z) {
  const int bh = blockIdx.y;
  const int e = blockIdx.x * 256 + threadIdx.x;
  const int E = dk * dv;
  if (e >= E + dk) return;
  const long long pst = E + dk;
  auto initial = [&]() -> float {
    if (e < E) return init ? init[(long long)bh * E + e] : 0.f;
    return initz ? initz[(long long)bh * dk + (e - E)] : 0.f;
  };
  auto store0 = [&](float val) {
    if (e < E) {
      if (out0) out0[(long long)bh * E + e] = val;
    } else if (out0z) {
      out0z[(long long)bh * dk + (e - E)] = val;
    }
  };
  if (op == 0) {
    float acc = initial();
    for (int si = S - 1; si >= 0; --si) {
      gsnap[((long long)bh * S + si) * pst + e] = acc;
      const float* p = cpart + ((long long)bh * S + si) * G * pst + e;
      for (int gi = 0; gi < G; ++gi) acc += p[gi * pst];
    }
    store0(acc);
  } else if (op == 1) {
    float acc = running[(long long)bh * pst + e];
    const float* p = cpart + ((long long)bh * S + s) * G * pst + e;
    for (int gi = 0; gi < G; ++gi) acc += p[gi * pst];
    const float* u = upart + (long long)bh * Gu * pst + e;
    for (int gi = 0; gi < Gu; ++gi) acc += u[gi * pst];
    running[(long long)bh * pst + e] = acc;
  } else if (op == 2) {
    running[(long long)bh * pst + e] = initial();
  } else {
    store0(running[(long long)bh * pst + e]);
  }
}

// The update's gradient terms for 128 key rows of one (b, h, segment), in
// four passes of 32 (warp w: rows 4w .. 4w+3 of a pass, lane = column).
// gst: [dM | dz] gradient after the segment (G, gz), fp32, dk*dv + dk.
// Writes dk_upd = sigma'(k) dsigma(K) and dv_upd (fp32 [BH*L][d]) and, for
// the delta rule (snapM != nullptr), the rows d_num_r, d_den_r.
template <typename T>
__global__ void __launch_bounds__(256) bwd_upd_kernel(const T* __restrict__ k, const T* __restrict__ v, BwdGeo g,
                                                      int seg0, const float* __restrict__ gstate, long long gstride_s,
                                                      long long gstride_bh, const float* __restrict__ snapM,
                                                      const float* __restrict__ snapz, float* __restrict__ dk_upd,
                                                      float* __restrict__ dv_upd, float* __restrict__ dnum_r,
                                                      float* __restrict__ dden_r, int blocks_per_seg) {
  extern __shared__ float sm[];
  const int dk = g.dk, dv = g.dv, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const bool delta = snapM != nullptr;
  int idx = blockIdx.x;
  const int blk = idx % blocks_per_seg;
  idx /= blocks_per_seg;
  const int sl = idx % (delta ? 1 : g.S);
  const int bh = idx / (delta ? 1 : g.S);
  const int s = seg0 + sl;
  const long long seg_start = (long long)s * g.N;
  const int n_s = (int)min((long long)g.N, g.L - seg_start);
  const int r0 = blk * 128;
  if (r0 >= n_s) return;
  float* Gs = sm;                     // [dk][dv + 1]
  float* Ms = Gs + dk * (dv + 1);     // [dk][dv + 1] (delta)
  float* gz = Ms + (delta ? dk * (dv + 1) : 0);  // [dk]
  float* zs = gz + dk;                // [dk] (delta)
  float* sk = zs + dk;                // [32][dk]
  float* U = sk + 32 * dk;            // [32][dv]
  float* W = U + 32 * dv;             // [32][dv]  dR / den (delta)
  const float* gp = gstate + (long long)bh * gstride_bh + (long long)s * gstride_s;
  for (int e = tid; e < dk * dv; e += 256) Gs[(e / dv) * (dv + 1) + e % dv] = gp[e];
  for (int e = tid; e < dk; e += 256) gz[e] = gp[dk * dv + e];
  const float* Mp = delta ? snapM + ((long long)bh * g.S + s) * dk * dv : nullptr;
  if (delta) {
    for (int e = tid; e < dk * dv; e += 256) Ms[(e / dv) * (dv + 1) + e % dv] = Mp[e];
    for (int e = tid; e < dk; e += 256) zs[e] = snapz[((long long)bh * g.S + s) * dk + e];
  }
  const int rend = min(n_s, r0 + 128);
  for (int t0 = r0; t0 < rend; t0 += 32) {
    __syncthreads();
    for (int e = tid; e < 32 * dk; e += 256) {
      const int tt = e / dk, i = e - tt * dk;
      sk[e] = t0 + tt < rend ? to_f32(k[bwd_row(g, bh, seg_start + t0 + tt) * dk + i]) : 0.f;
    }
    for (int e = tid; e < 32 * dv; e += 256) {
      const int tt = e / dv, j = e - tt * dv;
      U[e] = t0 + tt < rend ? to_f32(v[bwd_row(g, bh, seg_start + t0 + tt) * dv + j]) : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int r = warp * 4 + rr;
      const int t = t0 + r;
      if (t >= rend) continue;  // warp-uniform
      const long long row = bwd_row(g, bh, seg_start + t);
      float* kr = sk + r * dk;  // raw k, then sigma(k) below
      float* ur = U + r * dv;
      float* wr = W + r * dv;
      float xk[4];
#pragma unroll
      for (int c = 0; c < 4; ++c) xk[c] = lane + 32 * c < dk ? kr[lane + 32 * c] : 0.f;
      __syncwarp();
#pragma unroll
      for (int c = 0; c < 4; ++c)
        if (lane + 32 * c < dk) kr[lane + 32 * c] = elu1_accurate(xk[c]);
      __syncwarp();
      float den = 0.f;
      if (delta) {
        float d = 0.f;
        for (int i = lane; i < dk; i += 32) d = fmaf(kr[i], zs[i], d);
        den = warp_sum(d);
      }
      // dU = sigma(k) G (the dv_upd row), and R = sigma(k) M^(s) / den (delta)
      float du[4] = {0.f, 0.f, 0.f, 0.f}, rv[4] = {0.f, 0.f, 0.f, 0.f};
      for (int i = 0; i < dk; ++i) {
        const float ski = kr[i];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = lane + 32 * c;
          if (col < dv) {
            du[c] = fmaf(ski, Gs[i * (dv + 1) + col], du[c]);
            if (delta) rv[c] = fmaf(ski, Ms[i * (dv + 1) + col], rv[c]);
          }
        }
      }
      float dd = 0.f;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col = lane + 32 * c;
        if (col < dv) {
          dv_upd[row * dv + col] = du[c];
          if (delta) {
            const float R = den != 0.f ? rv[c] / den : 0.f;
            ur[col] -= R;  // U = V - R
            const float w = den != 0.f ? -du[c] / den : 0.f;  // d_num_r = dR / den, dR = -dU
            wr[col] = w;
            dnum_r[row * dv + col] = w;
            dd = fmaf(-du[c], R, dd);
          }
        }
      }
      const float d_den = delta && den != 0.f ? -warp_sum(dd) / den : 0.f;
      if (delta && lane == 0) dden_r[row] = d_den;
      __syncwarp();
      // dsigma(k)_i = sum_j U_j G_ij + gz_i (+ sum_j d_num_r_j M_ij + d_den_r z_i)
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const int col = lane + 32 * c;
        if (col < dk) {
          float a = gz[col];
          for (int j = 0; j < dv; ++j) a = fmaf(ur[j], Gs[col * (dv + 1) + j], a);
          if (delta) {
            for (int j = 0; j < dv; ++j) a = fmaf(wr[j], Ms[col * (dv + 1) + j], a);
            a = fmaf(d_den, zs[col], a);
          }
          dk_upd[row * dk + col] = sigma_prime(xk[c]) * a;
        }
      }
    }
  }
}

// dk, dv of the local attention for 32 keys of one (b, h, segment), plus the
// update's terms; one write.  Warp w owns keys 4w .. 4w+3; lane = query row
// inside a query tile (scores) or column (accumulators).
template <typename T>
__global__ void __launch_bounds__(256, 2)
    bwd_kv_kernel(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
                  const T* __restrict__ dout, const float* __restrict__ beta, const float* __restrict__ lse,
                  const float* __restrict__ Drow, const float* __restrict__ dk_upd, const float* __restrict__ dv_upd,
                  BwdGeo g, float scale, int KT, T* __restrict__ dk_out, T* __restrict__ dv_out) {
  extern __shared__ float sm[];
  const int dk = g.dk, dv = g.dv, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int BHS = g.B * g.H * g.S;
  const int kb = (int)(blockIdx.x / BHS);
  const int rem = (int)(blockIdx.x % BHS);
  const int bh = rem / g.S, s = rem % g.S;
  const int h = bh % g.H;
  const long long seg_start = (long long)s * g.N;
  const int n_s = (int)min((long long)g.N, g.L - seg_start);
  const int k0 = kb * 32;
  if (k0 >= n_s) return;
  const int klast = min(n_s, k0 + 32) - 1;
  const float gw = 1.f / (1.f + expf(-beta[h]));
  float* Ks = sm;                   // [32][dk]
  float* Vs = Ks + 32 * dk;         // [32][dv]
  float* Qs = Vs + 32 * dv;         // [32][dk + 1]
  float* Dd = Qs + 32 * (dk + 1);   // [32][dv + 1] d_dot rows
  float* LD = Dd + 32 * (dv + 1);   // [32][2]: lse, D
  for (int e = tid; e < 32 * dk; e += 256) {
    const int r = e / dk, i = e - r * dk;
    Ks[e] = k0 + r < n_s ? to_f32(k[bwd_row(g, bh, seg_start + k0 + r) * dk + i]) : 0.f;
  }
  for (int e = tid; e < 32 * dv; e += 256) {
    const int r = e / dv, j = e - r * dv;
    Vs[e] = k0 + r < n_s ? to_f32(v[bwd_row(g, bh, seg_start + k0 + r) * dv + j]) : 0.f;
  }
  float dka[4][4], dva[4][4];
#pragma unroll
  for (int rr = 0; rr < 4; ++rr)
#pragma unroll
    for (int c = 0; c < 4; ++c) dka[rr][c] = dva[rr][c] = 0.f;
  const int nqt = (n_s + 31) / 32;
  for (int qt = kb; qt < nqt; ++qt) {
    __syncthreads();
    const int q0 = qt * 32;
    for (int e = tid; e < 32 * dk; e += 256) {
      const int r = e / dk, i = e - r * dk;
      Qs[r * (dk + 1) + i] = q0 + r < n_s ? to_f32(q[bwd_row(g, bh, seg_start + q0 + r) * dk + i]) : 0.f;
    }
    for (int e = tid; e < 32 * dv; e += 256) {
      const int r = e / dv, j = e - r * dv;
      Dd[r * (dv + 1) + j] =
          q0 + r < n_s ? (1.f - gw) * to_f32(dout[bwd_row(g, bh, seg_start + q0 + r) * dv + j]) : 0.f;
    }
    if (tid < 32) {
      const bool ok = q0 + tid < n_s;
      const long long row = bwd_row(g, bh, seg_start + q0 + tid);
      LD[2 * tid] = ok ? lse[row] : 0.f;
      LD[2 * tid + 1] = ok ? Drow[row] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int rr = 0; rr < 4; ++rr) {
      const int kj = k0 + warp * 4 + rr;
      if (kj > klast) continue;  // warp-uniform
      const int qi = q0 + lane;
      float p = 0.f, ds = 0.f;
      if (qi < n_s && qi >= kj) {
        float sc = 0.f, dp = 0.f;
        const float* kr = Ks + (warp * 4 + rr) * dk;
        const float* vr = Vs + (warp * 4 + rr) * dv;
        for (int i = 0; i < dk; ++i) sc = fmaf(Qs[lane * (dk + 1) + i], kr[i], sc);
        for (int j = 0; j < dv; ++j) dp = fmaf(Dd[lane * (dv + 1) + j], vr[j], dp);
        p = expf(sc * scale - LD[2 * lane]);
        ds = p * (dp - LD[2 * lane + 1]);
      }
      for (int ii = 0; ii < 32; ++ii) {
        const float pi = __shfl_sync(0xffffffffu, p, ii);
        const float dsi = __shfl_sync(0xffffffffu, ds, ii);
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          const int col = lane + 32 * c;
          if (col < dv) dva[rr][c] = fmaf(pi, Dd[ii * (dv + 1) + col], dva[rr][c]);
          if (col < dk) dka[rr][c] = fmaf(dsi, Qs[ii * (dk + 1) + col], dka[rr][c]);
        }
      }
    }
  }
#pragma unroll
  for (int rr = 0; rr < 4; ++rr) {
    const int kj = k0 + warp * 4 + rr;
    if (kj > klast) continue;
    const long long row = bwd_row(g, bh, seg_start + kj);
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const int col = lane + 32 * c;
      if (col < dk) dk_out[row * dk + col] = from_f32<T>(scale * dka[rr][c] + dk_upd[row * dk + col]);
      if (col < dv) dv_out[row * dv + col] = from_f32<T>(dva[rr][c] + dv_upd[row * dv + col]);
    }
  }
}

// dbeta[h] = g (1 - g) * sum over batch rows and tokens of the row terms, in a
// fixed order (one block per head; a strided sum per thread, then a tree).
__global__ void __launch_bounds__(256) bwd_beta_kernel(const float* __restrict__ brow, const float* __restrict__ beta,
                                                       int B, int H, long long L, float* __restrict__ dbeta) {
  __shared__ float red[256];
  const int h = blockIdx.x;
  float acc = 0.f;
  for (int b = 0; b < B; ++b) {
    const float* p = brow + ((long long)b * H + h) * L;
    for (long long t = threadIdx.x; t < L; t += 256) acc += p[t];
  }
  red[threadIdx.x] = acc;
  __syncthreads();
  for (int w = 128; w > 0; w >>= 1) {
    if ((int)threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) {
    const float gw = 1.f / (1.f + expf(-beta[h]));
    dbeta[h] = gw * (1.f - gw) * red[0];
  }
}

}  // namespace infini
