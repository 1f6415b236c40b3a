// Shared device-side definitions: geometry of the grid-aligned tiled Monarch
// factorisation and element-type helpers.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace monarch {

constexpr float kLog2e = 1.4426950408889634f;

// Geometry of one call.  Tile c1 = (t*(H/th) + y/th)*(W/tw) + x/tw spans the
// frames and the tiles of a frame; position c2 = (y%th)*tw + x%tw spans one
// tile (MonarchRT explainers, §2.A block alignment and §2.B tiling).
struct Geo {
  int BH;        // batch * heads
  int T, Tk;     // query frames, key frames
  int H, W, d;
  int th, tw;
  int ntx;       // tiles along x
  int P;         // tiles per frame
  int b2;        // positions per tile (th*tw)
  int b1q, b1k;  // query tiles, key tiles
  int off;       // key tile aligned with query tile 0: (Tk - T) * P
  int b1k_pad;   // row stride of h (b1k rounded up to 4: 16-byte rows for TMA)
  int b1q_pad;   // row stride of the row LSE
  long long Nq, Nk;
  float sl2;     // s * log2(e), s = 1/sqrt(d)
  int cq;        // key/query tiles per frame-chunk of the causal mask; 0 = no mask
  // Stacked positions (L step of small grids): pk positions of a head share
  // one row block, position p's tiles at rows [p pb1, (p + 1) pb1), so b2,
  // b1q, b1k above count stacked positions and rows; pb1q, pb1k are one
  // position's tiles.  pk = 1: no stacking.
  int pk, pb1q, pb1k;
};

// Frame-chunk causal mask (self-attention, chunks of C frames, cq = C * P
// tiles): query tile a1 sees the key tiles [0, key_limit(a1)) and key tile c1
// is seen by the query tiles [query_start(c1), b1q).  Chunks start at frame
// 0; the last one may be shorter.
__device__ __forceinline__ int key_limit(const Geo& g, int a1) {
  return g.cq ? min(g.b1k, (a1 / g.cq + 1) * g.cq) : g.b1k;
}
__device__ __forceinline__ int query_start(const Geo& g, int c1) { return g.cq ? (c1 / g.cq) * g.cq : 0; }

// The key rows that query row a1 sees: [lo, hi).  With stacked positions,
// the keys of the row's own position (and its causal window there).
__device__ __forceinline__ void row_keys(const Geo& g, int a1, int& lo, int& hi) {
  if (g.pk == 1) {
    lo = 0;
    hi = key_limit(g, a1);
    return;
  }
  const int p = a1 / g.pb1q, a = a1 - p * g.pb1q;
  lo = p * g.pb1k;
  hi = lo + (g.cq ? min(g.pb1k, (a / g.cq + 1) * g.cq) : g.pb1k);
}
// The query rows that see key row c1: [lo, hi).
__device__ __forceinline__ void col_queries(const Geo& g, int c1, int& lo, int& hi) {
  if (g.pk == 1) {
    lo = query_start(g, c1);
    hi = g.b1q;
    return;
  }
  const int p = c1 / g.pb1k, c = c1 - p * g.pb1k;
  lo = p * g.pb1q + (g.cq ? (c / g.cq) * g.cq : 0);
  hi = (p + 1) * g.pb1q;
}

// Token index (within one head) of tile c1, position c2.
__device__ __forceinline__ long long token_of(const Geo& g, int c1, int c2) {
  int t = c1 / g.P;
  int r = c1 - t * g.P;
  int ty = r / g.ntx;
  int tx = r - ty * g.ntx;
  int py = c2 / g.tw;
  int px = c2 - py * g.tw;
  return (long long)(t * g.H + ty * g.th + py) * g.W + tx * g.tw + px;
}

template <typename T> __device__ __forceinline__ float to_f(T x);
template <> __device__ __forceinline__ float to_f<float>(float x) { return x; }
template <> __device__ __forceinline__ float to_f<__nv_bfloat16>(__nv_bfloat16 x) { return __bfloat162float(x); }
template <> __device__ __forceinline__ float to_f<__half>(__half x) { return __half2float(x); }

template <typename T> __device__ __forceinline__ T from_f(float x);
template <> __device__ __forceinline__ float from_f<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float x) { return __float2bfloat16_rn(x); }
template <> __device__ __forceinline__ __half from_f<__half>(float x) { return __float2half_rn(x); }

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// How the R step obtains q~ (the L-weighted mean query of a key tile).
enum QtMode : int {
  QT_IDENTITY = 0,  // first step, self-attention: q~[c1] = q[c1]
  QT_KVINIT = 1,    // first step, KV cache: aligned tiles take q, cached ones the mean query
  QT_BUFFER = 2,    // later steps: q~ produced by the column pass
};

// Workspace of one call (device memory).  The SIMT kernels keep k~, z and q~
// in fp32; the tensor-core kernels store k~ and z as two fp16 planes (hi, lo)
// in the same bytes.
struct Work {
  float* kt;    // [BH][b2][b1k][d]  k~[c1,a2]
  float* z;     // [BH][b2][b1k][d]  z[c1,a2]
  float* qt;    // [BH][b2][b1k][d]  q~[c1,a2]
  float* h;     // [BH][b2][b1k_pad] entropy of R_{c1}[a2,:]
  float* lse;   // [BH][b2][b1q_pad] base-2 log-sum-exp of L rows
  float* qbar;  // [BH][b2][d]       mean query per position (KV init)
  void* qb;     // [BH][b2][b1q][d]  queries in block-major order (input type)
};

}  // namespace monarch
