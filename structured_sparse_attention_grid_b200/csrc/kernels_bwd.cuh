// Backward pass of the one-step Monarch attention (iters = 1, self-attention,
// optional frame-chunk causal mask), CUDA-core fp32 arithmetic for every
// element type.  The forward it differentiates (MonarchRT explainers §2.C:
// the factors need a single refinement step after finetuning) is
//   R step (per key tile c1):  R = softmax_c2(s q[c1,a2].k[c1,c2]),
//                              h = -sum R ln R,  k~ = R k,  z = R v
//   L step (per position a2):  L = softmax_c1(s q[a1,a2].k~[c1,a2] + h[c1,a2]),
//                              y[a1,a2] = sum_c1 L z[c1,a2].
// The L step is a softmax attention per position with an additive bias, so
// its backward has the usual form with D = rowsum(L * dL) = dy . y:
//   dS = L (dy.z - D),  dq = s dS k~,  dk~ = s dS^T q,  dz = L^T dy,  dh = colsum(dS).
// The R step's backward per tile, with G = dk~ k^T + dz v^T and the entropy
// term dh (ln R + 1) (its "+1" shifts a row of G by a constant and cancels):
//   dSr = R (G' - rowsum(R G')),  G' = G - dh ln R,
//   dk = R^T dk~ + s dSr^T q,  dv = R^T dz,  dq += s dSr k.
// Scores are kept in base-2 units (x = s log2(e) q.k), as in the forward.
#pragma once

#include "common.cuh"

namespace monarch {

// Workspace of one backward call (device memory, fp32).
struct BwdWork {
  float* dd;    // [BH][b2][b1q_pad]  D = dy . y per query row
  float* dqL;   // [BH][b2][b1q][d]   L-step part of dq, row (a1, a2)
  float* dkt;   // [BH][b2][b1k][d]   dk~[c1, a2]
  float* dz;    // [BH][b2][b1k][d]   dz[c1, a2]
  float* dh;    // [BH][b2][b1k_pad]  dh[c1, a2]
};

__device__ __forceinline__ void warp_sum2(float& a, float& b) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    a += __shfl_xor_sync(0xffffffffu, a, o);
    b += __shfl_xor_sync(0xffffffffu, b, o);
  }
}

// ---------------------------------------------------------------------------
// Row preparation: one warp per query row (a1, a2).  Online softmax over the
// visible key tiles gives the row's base-2 log-sum-exp and y = sum L z; the
// kernel keeps D = dy . y (y itself is not stored).
// grid (ceil(b1q/ROWS), b2, BH), block 32*ROWS.
template <typename T, typename TG, int D>
__global__ void __launch_bounds__(512)
l_bwd_prep_simt(const T* __restrict__ q, const TG* __restrict__ dy, Work w, BwdWork bw, Geo g) {
  constexpr int KC = 32;
  constexpr int PER = D / 32;
  __shared__ float sK[KC][D];
  __shared__ float sZ[KC][D];
  __shared__ float sH[KC];
  const int a2 = blockIdx.y, bh = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a1 = blockIdx.x * (blockDim.x >> 5) + warp;
  const bool valid = a1 < g.b1q;
  const long long tok = (long long)bh * g.Nq * D + (valid ? token_of(g, a1, a2) : 0) * D;
  float qv[PER], acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    qv[i] = valid ? to_f(q[tok + lane + 32 * i]) * g.sl2 : 0.f;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const long long base = ((long long)bh * g.b2 + a2) * g.b1k;
  const float* hrow = w.h + ((long long)bh * g.b2 + a2) * g.b1k_pad;
  const int rowlim = key_limit(g, valid ? a1 : 0);
  const int climit = key_limit(g, min(g.b1q - 1, (int)(blockIdx.x + 1) * (int)(blockDim.x >> 5) - 1));
  for (int c0 = 0; c0 < climit; c0 += KC) {
    const int nk = min(KC, g.b1k - c0);
    __syncthreads();
    for (int i = threadIdx.x; i < nk * D; i += blockDim.x) {
      const int j = i / D, c = i - j * D;
      sK[j][c] = w.kt[(base + c0 + j) * D + c];
      sZ[j][c] = w.z[(base + c0 + j) * D + c];
    }
    for (int j = threadIdx.x; j < nk; j += blockDim.x) sH[j] = hrow[c0 + j] * kLog2e;
    __syncthreads();
    for (int j = 0; j < nk && c0 + j < rowlim; ++j) {
      float p = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) p = fmaf(qv[i], sK[j][lane + 32 * i], p);
      const float sc = warp_sum(p) + sH[j];
      const float mn = fmaxf(m, sc);
      const float corr = exp2f(m - mn);
      const float e = exp2f(sc - mn);
      l = fmaf(l, corr, e);
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = fmaf(e, sZ[j][lane + 32 * i], acc[i] * corr);
      m = mn;
    }
  }
  if (!valid) return;
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) dot = fmaf(to_f(dy[tok + lane + 32 * i]), acc[i], dot);
  dot = warp_sum(dot);
  if (lane == 0) {
    const long long r = ((long long)bh * g.b2 + a2) * g.b1q_pad + a1;
    w.lse[r] = m + log2f(l);
    bw.dd[r] = dot / l;
  }
}

// ---------------------------------------------------------------------------
// dq of the L step: one warp per query row (a1, a2), a pass over its visible
// key tiles:  L = 2^(x - lse),  dS = L (dy.z - D),  dqL = s sum_c1 dS k~.
// grid (ceil(b1q/ROWS), b2, BH), block 32*ROWS.
template <typename T, typename TG, int D>
__global__ void __launch_bounds__(512)
l_bwd_dq_simt(const T* __restrict__ q, const TG* __restrict__ dy, Work w, BwdWork bw, Geo g) {
  constexpr int KC = 32;
  constexpr int PER = D / 32;
  __shared__ float sK[KC][D];
  __shared__ float sZ[KC][D];
  __shared__ float sH[KC];
  const int a2 = blockIdx.y, bh = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int a1 = blockIdx.x * (blockDim.x >> 5) + warp;
  const bool valid = a1 < g.b1q;
  const long long tok = (long long)bh * g.Nq * D + (valid ? token_of(g, a1, a2) : 0) * D;
  float qv[PER], dyv[PER], acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    qv[i] = valid ? to_f(q[tok + lane + 32 * i]) * g.sl2 : 0.f;
    dyv[i] = valid ? to_f(dy[tok + lane + 32 * i]) : 0.f;
    acc[i] = 0.f;
  }
  const long long r = ((long long)bh * g.b2 + a2) * g.b1q_pad + (valid ? a1 : 0);
  const float lse = w.lse[r], dd = bw.dd[r];
  const long long base = ((long long)bh * g.b2 + a2) * g.b1k;
  const float* hrow = w.h + ((long long)bh * g.b2 + a2) * g.b1k_pad;
  const int rowlim = key_limit(g, valid ? a1 : 0);
  const int climit = key_limit(g, min(g.b1q - 1, (int)(blockIdx.x + 1) * (int)(blockDim.x >> 5) - 1));
  for (int c0 = 0; c0 < climit; c0 += KC) {
    const int nk = min(KC, g.b1k - c0);
    __syncthreads();
    for (int i = threadIdx.x; i < nk * D; i += blockDim.x) {
      const int j = i / D, c = i - j * D;
      sK[j][c] = w.kt[(base + c0 + j) * D + c];
      sZ[j][c] = w.z[(base + c0 + j) * D + c];
    }
    for (int j = threadIdx.x; j < nk; j += blockDim.x) sH[j] = hrow[c0 + j] * kLog2e;
    __syncthreads();
    for (int j = 0; j < nk && c0 + j < rowlim; ++j) {
      float p = 0.f, dl = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        p = fmaf(qv[i], sK[j][lane + 32 * i], p);
        dl = fmaf(dyv[i], sZ[j][lane + 32 * i], dl);
      }
      warp_sum2(p, dl);
      const float ds = exp2f(p + sH[j] - lse) * (dl - dd);
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = fmaf(ds, sK[j][lane + 32 * i], acc[i]);
    }
  }
  if (!valid) return;
  const float s = g.sl2 * (1.f / kLog2e);
  float* dst = bw.dqL + (((long long)bh * g.b2 + a2) * g.b1q + a1) * D;
#pragma unroll
  for (int i = 0; i < PER; ++i) dst[lane + 32 * i] = acc[i] * s;
}

// ---------------------------------------------------------------------------
// dk~, dz, dh of the L step: one warp per key column (c1, a2), a pass over the
// query tiles that see it:  dz = sum_a1 L dy,  dk~ = s sum_a1 dS q,
// dh = sum_a1 dS.  grid (ceil(b1k/ROWS), b2, BH), block 32*ROWS.
template <typename T, typename TG, int D>
__global__ void __launch_bounds__(512)
l_bwd_dkv_simt(const T* __restrict__ q, const TG* __restrict__ dy, Work w, BwdWork bw, Geo g) {
  constexpr int QC = 32;
  constexpr int PER = D / 32;
  __shared__ float sQ[QC][D];
  __shared__ float sY[QC][D];
  __shared__ float sL[QC];
  __shared__ float sD[QC];
  const int a2 = blockIdx.y, bh = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int c1 = blockIdx.x * (blockDim.x >> 5) + warp;
  const bool valid = c1 < g.b1k;
  const long long kbase = ((long long)bh * g.b2 + a2) * g.b1k;
  float kv[PER], zv[PER], ak[PER], az[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    kv[i] = valid ? w.kt[(kbase + c1) * D + lane + 32 * i] * g.sl2 : 0.f;
    zv[i] = valid ? w.z[(kbase + c1) * D + lane + 32 * i] : 0.f;
    ak[i] = 0.f;
    az[i] = 0.f;
  }
  const long long hidx = ((long long)bh * g.b2 + a2) * g.b1k_pad + (valid ? c1 : 0);
  const float hb = w.h[hidx] * kLog2e;
  float dh = 0.f;
  const int qstart = query_start(g, valid ? c1 : 0);
  const int a_lo = query_start(g, min(g.b1k - 1, (int)blockIdx.x * (int)(blockDim.x >> 5)));
  const long long hq = (long long)bh * g.Nq * D;
  const long long lrow = ((long long)bh * g.b2 + a2) * g.b1q_pad;
  for (int a0 = a_lo; a0 < g.b1q; a0 += QC) {
    const int nq = min(QC, g.b1q - a0);
    __syncthreads();
    for (int i = threadIdx.x; i < nq * D; i += blockDim.x) {
      const int j = i / D, c = i - j * D;
      const long long t = hq + token_of(g, a0 + j, a2) * D + c;
      sQ[j][c] = to_f(q[t]);
      sY[j][c] = to_f(dy[t]);
    }
    for (int j = threadIdx.x; j < nq; j += blockDim.x) {
      sL[j] = w.lse[lrow + a0 + j];
      sD[j] = bw.dd[lrow + a0 + j];
    }
    __syncthreads();
    for (int j = 0; j < nq; ++j) {
      if (a0 + j < qstart) continue;
      float p = 0.f, dl = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        p = fmaf(kv[i], sQ[j][lane + 32 * i], p);
        dl = fmaf(zv[i], sY[j][lane + 32 * i], dl);
      }
      warp_sum2(p, dl);
      const float L = exp2f(p + hb - sL[j]);
      const float ds = L * (dl - sD[j]);
      dh += ds;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        az[i] = fmaf(L, sY[j][lane + 32 * i], az[i]);
        ak[i] = fmaf(ds, sQ[j][lane + 32 * i], ak[i]);
      }
    }
  }
  if (!valid) return;
  const float s = g.sl2 * (1.f / kLog2e);
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    bw.dkt[(kbase + c1) * D + lane + 32 * i] = ak[i] * s;
    bw.dz[(kbase + c1) * D + lane + 32 * i] = az[i];
  }
  if (lane == 0) bw.dh[hidx] = dh;
}

// ---------------------------------------------------------------------------
// R-step backward for one key tile c1 of one head (all positions at once):
// recomputes R from q and k, forms dSr, and writes dk, dv and the finished dq
// of the tile's tokens in grid order.  Shared rows are padded to d+1 floats
// so that the column-wise dot products hit distinct banks.
// grid (b1k, BH), block 256, dynamic smem r_bwd_smem_floats(b2, d) floats.
__host__ __device__ constexpr int r_bwd_smem_floats(int b2, int d) { return 5 * b2 * (d + 1) + 2 * b2 * (b2 + 1) + b2; }

template <typename T, typename TG>
__global__ void __launch_bounds__(256)
r_bwd_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, TG* __restrict__ dq,
           TG* __restrict__ dk, TG* __restrict__ dv, BwdWork bw, Geo g) {
  extern __shared__ float smem[];
  const int c1 = blockIdx.x, bh = blockIdx.y;
  const int d = g.d, b2 = g.b2, dp = d + 1, sp = b2 + 1;
  float* sK = smem;
  float* sV = sK + b2 * dp;
  float* sQ = sV + b2 * dp;
  float* sDK = sQ + b2 * dp;
  float* sDZ = sDK + b2 * dp;
  float* sR = sDZ + b2 * dp;   // [a2][c2]: scores, then R
  float* sG = sR + b2 * sp;    // [a2][c2]: G, then dSr
  float* sDH = sG + b2 * sp;
  const long long hq = (long long)bh * g.Nq * d;
  const long long hk = (long long)bh * g.Nk * d;
  for (int i = threadIdx.x; i < b2 * d; i += blockDim.x) {
    const int r = i / d, c = i - r * d;
    const long long tk = token_of(g, c1, r) * d + c;
    sK[r * dp + c] = to_f(k[hk + tk]);
    sV[r * dp + c] = to_f(v[hk + tk]);
    sQ[r * dp + c] = to_f(q[hq + tk]);
    const long long o = (((long long)bh * b2 + r) * g.b1k + c1) * d + c;
    sDK[r * dp + c] = bw.dkt[o];
    sDZ[r * dp + c] = bw.dz[o];
  }
  for (int r = threadIdx.x; r < b2; r += blockDim.x) sDH[r] = bw.dh[((long long)bh * b2 + r) * g.b1k_pad + c1];
  __syncthreads();

  // scores (base 2) and G = dk~ k^T + dz v^T
  for (int i = threadIdx.x; i < b2 * b2; i += blockDim.x) {
    const int a2 = i / b2, c2 = i - a2 * b2;
    const float* qa = sQ + a2 * dp;
    const float* ka = sDK + a2 * dp;
    const float* za = sDZ + a2 * dp;
    const float* kc = sK + c2 * dp;
    const float* vc = sV + c2 * dp;
    float sc = 0.f, gg = 0.f;
    for (int c = 0; c < d; ++c) {
      sc = fmaf(qa[c], kc[c], sc);
      gg = fmaf(ka[c], kc[c], fmaf(za[c], vc[c], gg));
    }
    sR[a2 * sp + c2] = sc * g.sl2;
    sG[a2 * sp + c2] = gg;
  }
  __syncthreads();

  // per row: R = softmax, ln R = ln2 (x - m) - ln l (finite where R underflows),
  // G' = G - dh ln R, dSr = R (G' - sum R G')
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr float kLn2 = 0.6931471805599453f;
  for (int a2 = warp; a2 < b2; a2 += blockDim.x >> 5) {
    float* xr = sR + a2 * sp;
    float* gr = sG + a2 * sp;
    float m = -INFINITY;
    for (int c2 = lane; c2 < b2; c2 += 32) m = fmaxf(m, xr[c2]);
    m = warp_max(m);
    float l = 0.f;
    for (int c2 = lane; c2 < b2; c2 += 32) l += exp2f(xr[c2] - m);
    l = warp_sum(l);
    const float inv = 1.f / l, lnl = logf(l), dh = sDH[a2];
    float rs = 0.f;
    for (int c2 = lane; c2 < b2; c2 += 32) {
      const float x = xr[c2] - m;
      const float R = exp2f(x) * inv;
      const float gp = gr[c2] - dh * (x * kLn2 - lnl);
      xr[c2] = R;
      gr[c2] = gp;
      rs = fmaf(R, gp, rs);
    }
    rs = warp_sum(rs);
    for (int c2 = lane; c2 < b2; c2 += 32) gr[c2] = xr[c2] * (gr[c2] - rs);
  }
  __syncthreads();

  const float s = g.sl2 * (1.f / kLog2e);
  // dk[c2] = sum_a2 R dk~[a2] + s dSr q[a2];  dv[c2] = sum_a2 R dz[a2]
  for (int i = threadIdx.x; i < b2 * d; i += blockDim.x) {
    const int c2 = i / d, c = i - c2 * d;
    float ak = 0.f, aq = 0.f, av = 0.f;
    for (int a2 = 0; a2 < b2; ++a2) {
      const float R = sR[a2 * sp + c2], ds = sG[a2 * sp + c2];
      ak = fmaf(R, sDK[a2 * dp + c], ak);
      aq = fmaf(ds, sQ[a2 * dp + c], aq);
      av = fmaf(R, sDZ[a2 * dp + c], av);
    }
    const long long t = token_of(g, c1, c2) * d + c;
    dk[hk + t] = from_f<TG>(fmaf(s, aq, ak));
    dv[hk + t] = from_f<TG>(av);
  }
  // dq[a2] = dqL[c1, a2] + s sum_c2 dSr k[c2]   (query tile c1 = key tile c1)
  for (int i = threadIdx.x; i < b2 * d; i += blockDim.x) {
    const int a2 = i / d, c = i - a2 * d;
    float a = 0.f;
    for (int c2 = 0; c2 < b2; ++c2) a = fmaf(sG[a2 * sp + c2], sK[c2 * dp + c], a);
    const float base = bw.dqL[(((long long)bh * b2 + a2) * g.b1q + c1) * d + c];
    dq[hq + token_of(g, c1, a2) * d + c] = from_f<TG>(fmaf(s, a, base));
  }
}

}  // namespace monarch
