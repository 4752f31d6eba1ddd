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
// Kernels (all deterministic: fixed summation orders, no atomics; the memory
// branch's register-tiled products -- bwd_outer_kernel, bwd_upd_kernel --
// are in bwd_mem.cuh, their tensor-core forms in sm100_bwdmem.cuh):
//   bwd_q_kernel     per (b, h, segment, 32 query rows): dq (local + memory
//                    read), D, the dbeta row terms, d_num and d_den rows
//   bwd_state_kernel the memory-gradient chain: a reverse scan of the
//                    partials (linear rule) or one reverse step (delta rule)
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
  // as a programmatic dependent (the delta rule's reverse steps), nothing the
  // previous kernel reads or writes is touched before it has completed
  griddep_launch_dependents();
  griddep_wait();
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
