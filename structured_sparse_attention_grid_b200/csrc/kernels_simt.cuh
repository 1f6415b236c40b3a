// CUDA-core kernels of the Monarch forward: fp32 arithmetic for every element
// type.  They are the f32 path (tensor-core TF32 cannot meet an fp32
// tolerance) and the general path for shapes the tensor-core kernels do not
// cover.  Grid gathers (the grid -> tile/position permutation) are fused into
// the loads and the inverse permutation into the output store.
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace monarch {

// ---------------------------------------------------------------------------
// Mean query per (head, position) over all query tiles: the q~ of cached key
// tiles in the first R step of a KV-cache call.  grid (b2, BH), block
// kQbarThreads.  The token offsets of the position's query tiles are computed
// once into shared memory; then thread (group, quad) sums the four columns
// `quad` over the query tiles group, group + groups, ... (a warp reads 32
// consecutive 4-column pieces of one token row), and the groups are added in
// shared memory.  Output: f32 [BH][b2][d] for f32 inputs; for bf16 / f16
// inputs the tensor-core R step's A operand, a high plane round(m) and a low
// plane round(m - high) of the input type, [2][BH][b2][d] (the same bytes).
constexpr int kQbarThreads = 512;
constexpr int kQbarMaxTiles = 4096;   // query tiles whose offsets fit the shared table

template <typename T>
__global__ void __launch_bounds__(kQbarThreads)
qbar_kernel(const T* __restrict__ q, void* __restrict__ qbar, Geo g) {
  __shared__ float4 part[kQbarThreads];
  __shared__ long long tok[kQbarMaxTiles];   // token offsets (elements) of this position's query tiles
  ptx::griddep_launch();
  ptx::griddep_wait();
  const int a2 = blockIdx.x, bh = blockIdx.y;
  const int nquad = g.d / 4, groups = kQbarThreads / nquad;
  const int quad = threadIdx.x % nquad, grp = threadIdx.x / nquad;
  const T* qh = q + (long long)bh * g.Nq * g.d + 4 * quad;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  for (int base = 0; base < g.b1q; base += kQbarMaxTiles) {
    const int n = min(kQbarMaxTiles, g.b1q - base);
    __syncthreads();   // the previous chunk's offsets are read
    for (int i = threadIdx.x; i < n; i += kQbarThreads) tok[i] = token_of(g, base + i, a2) * g.d;
    __syncthreads();
#pragma unroll 4
    for (int i = grp; i < n; i += groups) {
      const T* p = qh + tok[i];
      if constexpr (sizeof(T) == 4) {
        const float4 x = *reinterpret_cast<const float4*>(p);
        acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
      } else {
        const uint2 x = *reinterpret_cast<const uint2*>(p);
        const T* e = reinterpret_cast<const T*>(&x);
        acc.x += to_f(e[0]); acc.y += to_f(e[1]); acc.z += to_f(e[2]); acc.w += to_f(e[3]);
      }
    }
  }
  part[threadIdx.x] = acc;
  __syncthreads();
  if (grp == 0) {
    for (int i = 1; i < groups; ++i) {
      const float4 o = part[i * nquad + quad];
      acc.x += o.x; acc.y += o.y; acc.z += o.z; acc.w += o.w;
    }
    const float inv = 1.f / (float)g.b1q;
    const long long o = ((long long)bh * g.b2 + a2) * g.d + 4 * quad;
    const float m[4] = {acc.x * inv, acc.y * inv, acc.z * inv, acc.w * inv};
    if constexpr (sizeof(T) == 4) {
      float* dst = static_cast<float*>(qbar) + o;
      for (int e = 0; e < 4; ++e) dst[e] = m[e];
    } else {
      T* hi = static_cast<T*>(qbar) + o;
      T* lo = hi + (long long)g.BH * g.b2 * g.d;
      for (int e = 0; e < 4; ++e) {
        hi[e] = from_f<T>(m[e]);
        lo[e] = from_f<T>(m[e] - to_f(hi[e]));
      }
    }
  }
}

// ---------------------------------------------------------------------------
// R step for one key tile c1 of one head (all positions a2 at once):
//   R[a2,:] = softmax_c2(s q~[c1,a2].k[c1,c2]),  h = entropy(R[a2,:]),
//   k~[c1,a2] = sum_c2 R k[c1,c2],  z[c1,a2] = sum_c2 R v[c1,c2] (final step).
// grid (b1k, BH), block 128, dynamic smem (3*b2*d + b2*(b2+1)) floats.
template <typename T>
__global__ void __launch_bounds__(128)
r_step_simt(const T* __restrict__ q, const T* __restrict__ k, const T* __restrict__ v,
            Work w, Geo g, int mode, int final_step) {
  extern __shared__ float smem[];
  const int c1 = blockIdx.x, bh = blockIdx.y;
  const int d = g.d, b2 = g.b2;
  float* sK = smem;
  float* sQ = sK + b2 * d;
  float* sV = sQ + b2 * d;
  float* sS = sV + b2 * d;  // [b2][b2+1]
  const T* kh = k + (long long)bh * g.Nk * d;
  const T* vh = v + (long long)bh * g.Nk * d;
  const T* qh = q + (long long)bh * g.Nq * d;

  for (int i = threadIdx.x; i < b2 * d; i += blockDim.x) {
    const int c2 = i / d, c = i - c2 * d;
    const long long tk = token_of(g, c1, c2);
    sK[i] = to_f(kh[tk * d + c]);
    if (final_step) sV[i] = to_f(vh[tk * d + c]);
    float qv;
    if (mode == QT_IDENTITY) {
      qv = to_f(qh[token_of(g, c1, c2) * d + c]);
    } else if (mode == QT_KVINIT) {
      qv = (c1 >= g.off) ? to_f(qh[token_of(g, c1 - g.off, c2) * d + c])
                         : w.qbar[((long long)bh * b2 + c2) * d + c];
    } else {
      qv = w.qt[(((long long)bh * b2 + c2) * g.b1k + c1) * d + c];
    }
    sQ[i] = qv;  // row a2 = c2 index here: q~[c1, a2]
  }
  __syncthreads();

  // scores in base-2 units: s*log2(e) * q~[a2] . k[c2]
  for (int i = threadIdx.x; i < b2 * b2; i += blockDim.x) {
    const int a2 = i / b2, c2 = i - a2 * b2;
    const float* qa = sQ + a2 * d;
    const float* kc = sK + c2 * d;
    float acc = 0.f;
    for (int c = 0; c < d; ++c) acc = fmaf(qa[c], kc[c], acc);
    sS[a2 * (b2 + 1) + c2] = acc * g.sl2;
  }
  __syncthreads();

  // row softmax + entropy, one warp per row
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int a2 = warp; a2 < b2; a2 += blockDim.x >> 5) {
    float* row = sS + a2 * (b2 + 1);
    float m = -INFINITY;
    for (int c2 = lane; c2 < b2; c2 += 32) m = fmaxf(m, row[c2]);
    m = warp_max(m);
    float l = 0.f, sx = 0.f;
    for (int c2 = lane; c2 < b2; c2 += 32) {
      const float x = row[c2] - m;
      const float e = exp2f(x);
      row[c2] = e;
      l += e;
      sx += e * x;
    }
    l = warp_sum(l);
    sx = warp_sum(sx);
    const float inv = 1.f / l;
    for (int c2 = lane; c2 < b2; c2 += 32) row[c2] *= inv;
    // h = -sum R ln R = ln l - sum R (x ln 2)  with x in base-2 units
    if (lane == 0) w.h[((long long)bh * b2 + a2) * g.b1k_pad + c1] = logf(l) - (sx * inv) * 0.6931471805599453f;
  }
  __syncthreads();

  // k~[a2] = sum_c2 R[a2,c2] k[c2];  z[a2] = sum_c2 R[a2,c2] v[c2]
  for (int i = threadIdx.x; i < b2 * d; i += blockDim.x) {
    const int a2 = i / d, c = i - a2 * d;
    const float* r = sS + a2 * (b2 + 1);
    float ak = 0.f, av = 0.f;
    for (int c2 = 0; c2 < b2; ++c2) {
      ak = fmaf(r[c2], sK[c2 * d + c], ak);
      if (final_step) av = fmaf(r[c2], sV[c2 * d + c], av);
    }
    const long long o = (((long long)bh * b2 + a2) * g.b1k + c1) * d + c;
    w.kt[o] = ak;
    if (final_step) w.z[o] = av;
  }
}

// ---------------------------------------------------------------------------
// L step, row pass: one warp per query row (a1, a2); online softmax over the
// key tiles c1 of  s q[a1,a2].k~[c1,a2] + h[c1,a2].  Final step: writes
// out[token(a1,a2)] = sum_c1 L z / sum L (inverse permutation fused into the
// store); otherwise writes the row's base-2 log-sum-exp.
// grid (ceil(b1q/ROWS), b2, BH), block 32*ROWS.
template <typename T, typename TO, int D>
__global__ void __launch_bounds__(512)
l_row_simt(const T* __restrict__ q, TO* __restrict__ out, Work w, Geo g, int final_step) {
  constexpr int KC = 32;   // key tiles staged per chunk
  constexpr int PER = D / 32;
  __shared__ float sK[KC][D];
  __shared__ float sZ[KC][D];
  __shared__ float sH[KC];
  const int a2 = blockIdx.y, bh = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = blockDim.x >> 5;
  const int a1 = blockIdx.x * rows + warp;
  const bool valid = a1 < g.b1q;
  float qv[PER], acc[PER];
  const T* qrow = q + (long long)bh * g.Nq * D + (valid ? token_of(g, a1, a2) : 0) * D;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    qv[i] = valid ? to_f(qrow[lane + 32 * i]) * g.sl2 : 0.f;
    acc[i] = 0.f;
  }
  float m = -INFINITY, l = 0.f;
  const long long base = ((long long)bh * g.b2 + a2) * g.b1k;
  const int rowlim = key_limit(g, valid ? a1 : 0);   // visible key tiles [0, rowlim)
  for (int c0 = 0; c0 < g.b1k; c0 += KC) {
    const int nk = min(KC, g.b1k - c0);
    __syncthreads();
    for (int i = threadIdx.x; i < nk * D; i += blockDim.x) {
      const int j = i / D, c = i - j * D;
      sK[j][c] = w.kt[(base + c0 + j) * D + c];
      if (final_step) sZ[j][c] = w.z[(base + c0 + j) * D + c];
    }
    const float* hrow = w.h + ((long long)bh * g.b2 + a2) * g.b1k_pad;
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
      l = l * corr + e;
      if (final_step) {
#pragma unroll
        for (int i = 0; i < PER; ++i) acc[i] = fmaf(e, sZ[j][lane + 32 * i], acc[i] * corr);
      }
      m = mn;
    }
  }
  if (!valid) return;
  if (final_step) {
    const float inv = 1.f / l;
    TO* orow = out + (long long)bh * g.Nq * D + token_of(g, a1, a2) * D;
#pragma unroll
    for (int i = 0; i < PER; ++i) orow[lane + 32 * i] = from_f<TO>(acc[i] * inv);
  } else if (lane == 0) {
    w.lse[((long long)bh * g.b2 + a2) * g.b1q_pad + a1] = m + log2f(l);
  }
}

// ---------------------------------------------------------------------------
// L step, column pass (before a non-first R step): one warp per key tile
// (c1, a2);  L[a1,c1] = 2^(score - lse[a1]),
//   q~[c1,a2] = sum_a1 L q[a1,a2] / sum_a1 L.
// grid (ceil(b1k/ROWS), b2, BH), block 32*ROWS.
template <typename T, int D>
__global__ void __launch_bounds__(512)
l_col_simt(const T* __restrict__ q, Work w, Geo g) {
  constexpr int QC = 32;
  constexpr int PER = D / 32;
  __shared__ float sQ[QC][D];
  __shared__ float sL[QC];
  const int a2 = blockIdx.y, bh = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rows = blockDim.x >> 5;
  const int c1 = blockIdx.x * rows + warp;
  const bool valid = c1 < g.b1k;
  const long long kbase = ((long long)bh * g.b2 + a2) * g.b1k;
  float kv[PER], acc[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    kv[i] = valid ? w.kt[(kbase + c1) * D + lane + 32 * i] * g.sl2 : 0.f;
    acc[i] = 0.f;
  }
  const float hb = valid ? w.h[((long long)bh * g.b2 + a2) * g.b1k_pad + c1] * kLog2e : 0.f;
  float beta = 0.f, mc = -INFINITY;
  const int qstart = query_start(g, valid ? c1 : 0);   // queries that see this key tile: [qstart, b1q)
  const T* qh = q + (long long)bh * g.Nq * D;
  const float* lse = w.lse + ((long long)bh * g.b2 + a2) * g.b1q_pad;
  for (int a0 = 0; a0 < g.b1q; a0 += QC) {
    const int nq = min(QC, g.b1q - a0);
    __syncthreads();
    for (int i = threadIdx.x; i < nq * D; i += blockDim.x) {
      const int j = i / D, c = i - j * D;
      sQ[j][c] = to_f(qh[token_of(g, a0 + j, a2) * D + c]);
    }
    for (int j = threadIdx.x; j < nq; j += blockDim.x) sL[j] = lse[a0 + j];
    __syncthreads();
    for (int j = 0; j < nq; ++j) {
      if (a0 + j < qstart) continue;
      float p = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) p = fmaf(kv[i], sQ[j][lane + 32 * i], p);
      // x = log2 L[a1,c1] <= 0.  q~ is a ratio, so both sums carry a running
      // column shift mc (the largest x so far) and never underflow to 0/0.
      const float x = warp_sum(p) + hb - sL[j];
      const float mn = fmaxf(mc, x);
      const float corr = exp2f(mc - mn);
      const float e = exp2f(x - mn);
      beta = fmaf(beta, corr, e);
#pragma unroll
      for (int i = 0; i < PER; ++i) acc[i] = fmaf(e, sQ[j][lane + 32 * i], acc[i] * corr);
      mc = mn;
    }
  }
  if (!valid) return;
  const float inv = 1.f / beta;
#pragma unroll
  for (int i = 0; i < PER; ++i) w.qt[(kbase + c1) * D + lane + 32 * i] = acc[i] * inv;
}

}  // namespace monarch
