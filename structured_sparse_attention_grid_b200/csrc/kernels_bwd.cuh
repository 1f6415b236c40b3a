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
// of the tile's tokens in grid order.  Positions are padded with zero rows to
// P4 = b2 rounded up to 4; shared rows of k, v, q, dk~, dz hold D + 4 floats
// and rows of R and dSr P4 floats, so that every shared access is a float4.
// The contractions run in register blocks: 4 x 4 (a2, c2) over a slice of the
// channels for the scores and G, 4 positions x 4 channels for dk/dv and for dq.
// grid (b1k, BH), block 256, dynamic smem r_bwd_smem_bytes(b2, D).
__host__ __device__ constexpr int r_bwd_p4(int b2) { return (b2 + 3) & ~3; }
__host__ __device__ constexpr size_t r_bwd_smem_bytes(int b2, int d) {
  return ((size_t)5 * r_bwd_p4(b2) * (d + 4) + 2 * (size_t)r_bwd_p4(b2) * r_bwd_p4(b2) + r_bwd_p4(b2)) * 4 +
         (size_t)b2 * 8;
}

template <typename T> __device__ __forceinline__ float4 load4(const T* p);
template <> __device__ __forceinline__ float4 load4<float>(const float* p) { return *reinterpret_cast<const float4*>(p); }
template <> __device__ __forceinline__ float4 load4<__nv_bfloat16>(const __nv_bfloat16* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xFFFF0000u));
}
template <> __device__ __forceinline__ float4 load4<__half>(const __half* p) {
  const uint2 u = *reinterpret_cast<const uint2*>(p);
  const float2 a = __half22float2(*reinterpret_cast<const __half2*>(&u.x));
  const float2 b = __half22float2(*reinterpret_cast<const __half2*>(&u.y));
  return make_float4(a.x, a.y, b.x, b.y);
}
template <typename T> __device__ __forceinline__ void store4(T* p, float4 v);
template <> __device__ __forceinline__ void store4<float>(float* p, float4 v) { *reinterpret_cast<float4*>(p) = v; }
template <> __device__ __forceinline__ void store4<__nv_bfloat16>(__nv_bfloat16* p, float4 v) {
  __nv_bfloat162 a = __floats2bfloat162_rn(v.x, v.y), b = __floats2bfloat162_rn(v.z, v.w);
  *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
}
template <> __device__ __forceinline__ void store4<__half>(__half* p, float4 v) {
  __half2 a = __floats2half2_rn(v.x, v.y), b = __floats2half2_rn(v.z, v.w);
  *reinterpret_cast<uint2*>(p) = make_uint2(*reinterpret_cast<uint32_t*>(&a), *reinterpret_cast<uint32_t*>(&b));
}
__device__ __forceinline__ float dot4(float4 a, float4 b, float acc) {
  return fmaf(a.x, b.x, fmaf(a.y, b.y, fmaf(a.z, b.z, fmaf(a.w, b.w, acc))));
}
__device__ __forceinline__ float4 axpy4(float a, float4 x, float4 y) {
  return make_float4(fmaf(a, x.x, y.x), fmaf(a, x.y, y.y), fmaf(a, x.z, y.z), fmaf(a, x.w, y.w));
}

template <typename T, typename TG, int D>
__global__ void __launch_bounds__(256, 3)
r_bwd_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v, TG* __restrict__ dq,
           TG* __restrict__ dk, TG* __restrict__ dv, BwdWork bw, Geo g) {
  extern __shared__ float4 smem4[];
  constexpr int DP = D + 4, C4 = D / 4;
  const int c1 = blockIdx.x, bh = blockIdx.y;
  const int b2 = g.b2, P4 = r_bwd_p4(b2);
  float* sK = reinterpret_cast<float*>(smem4);
  float* sV = sK + P4 * DP;
  float* sQ = sV + P4 * DP;
  float* sDK = sQ + P4 * DP;
  float* sDZ = sDK + P4 * DP;
  float* sR = sDZ + P4 * DP;   // [a2][c2], stride P4: scores, then R
  float* sG = sR + P4 * P4;    // [a2][c2], stride P4: G, then dSr
  float* sDH = sG + P4 * P4;   // [P4]
  long long* sTok = reinterpret_cast<long long*>(sDH + P4);
  const long long hq = (long long)bh * g.Nq * D;
  const long long hk = (long long)bh * g.Nk * D;
  for (int r = threadIdx.x; r < b2; r += blockDim.x) {
    sTok[r] = token_of(g, c1, r) * D;
    sDH[r] = bw.dh[((long long)bh * b2 + r) * g.b1k_pad + c1];
  }
  // zero the padding of R and dSr (rows and columns >= b2); the rest is written below
  for (int i = threadIdx.x; i < P4 * P4; i += blockDim.x) {
    const int r = i / P4, c = i - r * P4;
    if (r >= b2 || c >= b2) sR[i] = sG[i] = 0.f;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < P4 * C4; i += blockDim.x) {
    const int r = i / C4, c = (i - r * C4) * 4;
    float4 kk = make_float4(0.f, 0.f, 0.f, 0.f), vv = kk, qq = kk, dkk = kk, dzz = kk;
    if (r < b2) {
      const long long t = sTok[r] + c;
      kk = load4(k + hk + t);
      vv = load4(v + hk + t);
      qq = load4(q + hq + t);
      const long long o = (((long long)bh * b2 + r) * g.b1k + c1) * D + c;
      dkk = *reinterpret_cast<const float4*>(bw.dkt + o);
      dzz = *reinterpret_cast<const float4*>(bw.dz + o);
    }
    *reinterpret_cast<float4*>(sK + r * DP + c) = kk;
    *reinterpret_cast<float4*>(sV + r * DP + c) = vv;
    *reinterpret_cast<float4*>(sQ + r * DP + c) = qq;
    *reinterpret_cast<float4*>(sDK + r * DP + c) = dkk;
    *reinterpret_cast<float4*>(sDZ + r * DP + c) = dzz;
  }
  __syncthreads();

  // scores (base 2) and G = dk~ k^T + dz v^T in 4 x 4 blocks of (a2, c2): rows
  // {a + i nb} and columns {c + j nb}.  The channels are split into ds slices
  // (ds lanes per block, ds a power of two chosen to fill the CTA) whose
  // partial sums are added by shuffles.  Slice sl reads float4 columns
  // sl w + (u mod w) + 8 (u / w), w = 8 / ds, at step u: the 8 lanes of one
  // shared-memory phase (8 / ds blocks of neighbouring c, rows D + 4 floats
  // apart) then touch 8 distinct bank groups.
  {
    const int nb = P4 / 4, nblk = nb * nb;
    int ds = 1;
    while (ds < 8 && nblk * ds * 2 <= (int)blockDim.x) ds *= 2;
    const int w = 8 / ds, cs = C4 / ds, items = nblk * ds;
    const int lane = threadIdx.x & 31;
    // whole warps iterate together (the shuffles need every lane); a block's
    // ds lanes are all valid or all idle, since ds divides 32
    for (int base = threadIdx.x & ~31; base < items; base += blockDim.x) {
      const int item = base + lane;
      const bool live = item < items;
      const int blk = live ? item / ds : 0, sl = item & (ds - 1);
      const int a = blk / nb, c = blk - a * nb;
      float sc[4][4], gg[4][4];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) sc[i][j] = gg[i][j] = 0.f;
#pragma unroll 1
      for (int u = 0; u < cs; ++u) {
        const int cc = 4 * (sl * w + (u % w) + 8 * (u / w));
        float4 kc[4], x[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) kc[j] = *reinterpret_cast<const float4*>(sK + (c + j * nb) * DP + cc);
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = *reinterpret_cast<const float4*>(sQ + (a + i * nb) * DP + cc);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) sc[i][j] = dot4(x[i], kc[j], sc[i][j]);
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = *reinterpret_cast<const float4*>(sDK + (a + i * nb) * DP + cc);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) gg[i][j] = dot4(x[i], kc[j], gg[i][j]);
#pragma unroll
        for (int j = 0; j < 4; ++j) kc[j] = *reinterpret_cast<const float4*>(sV + (c + j * nb) * DP + cc);
#pragma unroll
        for (int i = 0; i < 4; ++i) x[i] = *reinterpret_cast<const float4*>(sDZ + (a + i * nb) * DP + cc);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) gg[i][j] = dot4(x[i], kc[j], gg[i][j]);
      }
      for (int o = 1; o < ds; o <<= 1)
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            sc[i][j] += __shfl_xor_sync(0xffffffffu, sc[i][j], o);
            gg[i][j] += __shfl_xor_sync(0xffffffffu, gg[i][j], o);
          }
      // lane sl of the block writes the entries e = 4 i + j with e mod ds = sl
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
          if (live && ((4 * i + j) & (ds - 1)) == sl && a + i * nb < b2 && c + j * nb < b2) {
            sR[(a + i * nb) * P4 + c + j * nb] = sc[i][j] * g.sl2;
            sG[(a + i * nb) * P4 + c + j * nb] = gg[i][j];
          }
    }
  }
  __syncthreads();

  // per row: R = softmax, ln R = ln2 (x - m) - ln l (finite where R underflows),
  // G' = G - dh ln R, dSr = R (G' - sum R G')
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  constexpr float kLn2 = 0.6931471805599453f;
  for (int a2 = warp; a2 < b2; a2 += blockDim.x >> 5) {
    float* xr = sR + a2 * P4;
    float* gr = sG + a2 * P4;
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
  const int n4 = P4 / 4;
  // dk[c2] = sum_a2 R dk~[a2] + s dSr q[a2];  dv[c2] = sum_a2 R dz[a2]
  // (4 positions c2 x 4 channels per thread)
  for (int i = threadIdx.x; i < n4 * C4; i += blockDim.x) {
    const int cg = i / C4, c = (i - cg * C4) * 4, c2b = 4 * cg;
    float4 ak[4], av[4];   // dk and dv of positions c2b .. c2b + 3
#pragma unroll
    for (int j = 0; j < 4; ++j) ak[j] = av[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int a2 = 0; a2 < b2; ++a2) {
      const float4 r4 = *reinterpret_cast<const float4*>(sR + a2 * P4 + c2b);
      const float4 d4 = *reinterpret_cast<const float4*>(sG + a2 * P4 + c2b);
      const float4 k4 = *reinterpret_cast<const float4*>(sDK + a2 * DP + c);
      const float4 q4 = *reinterpret_cast<const float4*>(sQ + a2 * DP + c);
      const float4 z4 = *reinterpret_cast<const float4*>(sDZ + a2 * DP + c);
      const float rr[4] = {r4.x, r4.y, r4.z, r4.w}, dd[4] = {s * d4.x, s * d4.y, s * d4.z, s * d4.w};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        ak[j] = axpy4(dd[j], q4, axpy4(rr[j], k4, ak[j]));
        av[j] = axpy4(rr[j], z4, av[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int c2 = c2b + j;
      if (c2 >= b2) break;
      const long long t = hk + sTok[c2] + c;
      store4(dk + t, ak[j]);
      store4(dv + t, av[j]);
    }
  }
  // dq[a2] = dqL[c1, a2] + s sum_c2 dSr k[c2]   (query tile c1 = key tile c1;
  // 4 positions a2 x 4 channels per thread; padded c2 rows are zero)
  for (int i = threadIdx.x; i < n4 * C4; i += blockDim.x) {
    const int ag = i / C4, c = (i - ag * C4) * 4, a2b = 4 * ag;
    float4 acc[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[j] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int c2 = 0; c2 < P4; c2 += 4) {
      float4 kr[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) kr[u] = *reinterpret_cast<const float4*>(sK + (c2 + u) * DP + c);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float4 d4 = *reinterpret_cast<const float4*>(sG + (a2b + j) * P4 + c2);
        acc[j] = axpy4(d4.x, kr[0], acc[j]);
        acc[j] = axpy4(d4.y, kr[1], acc[j]);
        acc[j] = axpy4(d4.z, kr[2], acc[j]);
        acc[j] = axpy4(d4.w, kr[3], acc[j]);
      }
    }
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int a2 = a2b + j;
      if (a2 >= b2) break;
      const float4 base = *reinterpret_cast<const float4*>(bw.dqL + (((long long)bh * b2 + a2) * g.b1q + c1) * D + c);
      store4(dq + hq + sTok[a2] + c, make_float4(fmaf(s, acc[j].x, base.x), fmaf(s, acc[j].y, base.y),
                                                 fmaf(s, acc[j].z, base.z), fmaf(s, acc[j].w, base.w)));
    }
  }
}

}  // namespace monarch
