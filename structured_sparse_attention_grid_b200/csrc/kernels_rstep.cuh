// R step for bf16 / f16 inputs on the tensor cores (warp-level mma.sync
// m16n8k16: the per-tile products are b2 x b2 x d with b2 <= 64, far below
// the 128-row tcgen05 tile, so a warp owns 16 positions of one key tile).
//
// For key tile c1 and positions a2 (16 per warp):
//   S[a2,c2] = s q~[c1,a2].k[c1,c2]      (q~ split hi+lo when it is computed)
//   R = softmax_c2(S), h = entropy(R)
//   k~[c1,a2] = sum_c2 R k[c1,c2]        (R split hi+lo; k~ stored as hi/lo planes)
//   z[c1,a2]  = sum_c2 R v[c1,c2]        (final step; stored as f16 hi/lo planes)
// k and v tiles are gathered from the grid layout straight into shared memory.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "kernels_tc.cuh"

namespace monarch {

namespace rs {

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1,
                                         int bf16) {
  if (bf16)
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
  else
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}

template <typename T>
__device__ __forceinline__ float2 load2(const T* p) {
  if constexpr (sizeof(T) == 4) {
    return *reinterpret_cast<const float2*>(p);
  } else {
    const uint32_t u = *reinterpret_cast<const uint32_t*>(p);
    return make_float2(to_f(*reinterpret_cast<const T*>(&u)), to_f(reinterpret_cast<const T*>(&u)[1]));
  }
}

}  // namespace rs

// Planes written by the tensor-core R step.
template <typename TQ>
struct TcPlanes {
  TQ* kt_hi;        // [BH][b2][b1k][d], then the lo plane at kt_hi + plane
  __half* z_hi;     // [BH][b2][b1k][d], then the lo plane
  long long plane;  // elements per plane
};

// grid (ceil(b1k / tiles_per_cta), BH), block 128, dynamic smem
// tiles_per_cta * 2 * (16*mt) * (D+8) * 2 bytes, mt = ceil(b2/16).
template <typename TQ, int D>
__global__ void __launch_bounds__(128)
r_step_tc(const TQ* __restrict__ q, const TQ* __restrict__ k, const TQ* __restrict__ v, Work w,
          TcPlanes<TQ> out, Geo g, int mode, int final_step) {
  constexpr int PITCH = D + 8;  // elements per shared row (16-byte pad: conflict-free ldmatrix)
  constexpr int bf16 = TcType<TQ>::kBf16;
  extern __shared__ uint8_t smem_raw[];
  TQ* smem = reinterpret_cast<TQ*>(smem_raw);
  const int mt = (g.b2 + 15) >> 4;  // 16-row m-tiles per key tile
  const int rows = mt * 16;
  const int tpc = 4 / mt;           // key tiles per CTA
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const TQ* kh = k + (long long)bh * g.Nk * D;
  const TQ* vh = v + (long long)bh * g.Nk * D;
  const TQ* qh = q + (long long)bh * g.Nq * D;

  // ---- gather k (and v) tiles: [tile][row][PITCH]
  const int nmat = final_step ? 2 : 1;
  const int chunks = D / 8;
  for (int i = tid; i < tpc * nmat * rows * chunks; i += blockDim.x) {
    const int ch = i % chunks;
    const int row = (i / chunks) % rows;
    const int mat = (i / (chunks * rows)) % nmat;
    const int tt = i / (chunks * rows * nmat);
    const int c1 = blockIdx.x * tpc + tt;
    const bool valid = row < g.b2 && c1 < g.b1k;
    const TQ* src = (mat ? vh : kh) + (valid ? token_of(g, c1, row) * D + ch * 8 : 0);
    TQ* dst = smem + ((tt * nmat + mat) * rows + row) * PITCH + ch * 8;
    ptx::cp_async_16(ptx::smem_u32(dst), src, valid ? 16u : 0u);
  }
  ptx::cp_async_commit();

  const int tt = warp / mt, mi = warp % mt;
  const int c1 = blockIdx.x * tpc + tt;
  const bool active = tt < tpc && c1 < g.b1k;
  const int r0 = mi * 16 + (lane >> 2), r1 = r0 + 8;  // positions a2 of this thread's rows
  const int qc = 2 * (lane & 3);                       // column pair inside an 8-wide block

  // ---- A fragments of q~ (rows r0, r1), split into hi + lo when computed
  uint32_t ahi[D / 16][4], alo[D / 16][4];
  bool split_q = false;
  if (active) {
    const float* qt_r0 = nullptr;
    const float* qt_r1 = nullptr;
    const TQ* qx_r0 = nullptr;
    const TQ* qx_r1 = nullptr;
    if (mode == QT_BUFFER) {
      if (r0 < g.b2) qt_r0 = w.qt + (((long long)bh * g.b2 + r0) * g.b1k + c1) * D;
      if (r1 < g.b2) qt_r1 = w.qt + (((long long)bh * g.b2 + r1) * g.b1k + c1) * D;
      split_q = true;
    } else if (mode == QT_KVINIT && c1 < g.off) {
      if (r0 < g.b2) qt_r0 = w.qbar + ((long long)bh * g.b2 + r0) * D;
      if (r1 < g.b2) qt_r1 = w.qbar + ((long long)bh * g.b2 + r1) * D;
      split_q = true;
    } else {
      const int cq = (mode == QT_KVINIT) ? c1 - g.off : c1;
      if (r0 < g.b2) qx_r0 = qh + token_of(g, cq, r0) * D;
      if (r1 < g.b2) qx_r1 = qh + token_of(g, cq, r1) * D;
    }
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      float2 v[4];
      const int cA = ks * 16 + qc, cB = cA + 8;
      if (split_q) {
        v[0] = qt_r0 ? rs::load2(qt_r0 + cA) : make_float2(0.f, 0.f);
        v[1] = qt_r1 ? rs::load2(qt_r1 + cA) : make_float2(0.f, 0.f);
        v[2] = qt_r0 ? rs::load2(qt_r0 + cB) : make_float2(0.f, 0.f);
        v[3] = qt_r1 ? rs::load2(qt_r1 + cB) : make_float2(0.f, 0.f);
      } else {
        v[0] = qx_r0 ? rs::load2(qx_r0 + cA) : make_float2(0.f, 0.f);
        v[1] = qx_r1 ? rs::load2(qx_r1 + cA) : make_float2(0.f, 0.f);
        v[2] = qx_r0 ? rs::load2(qx_r0 + cB) : make_float2(0.f, 0.f);
        v[3] = qx_r1 ? rs::load2(qx_r1 + cB) : make_float2(0.f, 0.f);
      }
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float hx = TcType<TQ>::round(v[e].x), hy = TcType<TQ>::round(v[e].y);
        ahi[ks][e] = TcType<TQ>::pack(hx, hy);
        alo[ks][e] = TcType<TQ>::pack(v[e].x - hx, v[e].y - hy);
      }
    }
  }
  ptx::cp_async_wait<0>();
  __syncthreads();
  if (!active) return;

  const TQ* sKt = smem + (tt * nmat) * rows * PITCH;
  const TQ* sVt = sKt + rows * PITCH;
  const uint32_t aK = ptx::smem_u32(sKt), aV = ptx::smem_u32(sVt);
  const int nt = rows / 8;  // n-tiles over c2 (even)
  // ldmatrix lane -> (row, column-block) map for x4 loads
  const int lr = lane & 7, lm = lane >> 3;

  // ---- S = q~ k^T  (B = k rows: "col-major" B, plain ldmatrix)
  float s[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      if (j < nt) {
        // matrices: (n-tile j, k lo), (j, k hi), (j+1, k lo), (j+1, k hi)
        const int row = (j + (lm >> 1)) * 8 + lr;
        const int col = ks * 16 + (lm & 1) * 8;
        uint32_t b0, b1, b2, b3;
        rs::ldsm_x4(aK + (row * PITCH + col) * 2, b0, b1, b2, b3);
        rs::mma16816(s[j], ahi[ks], b0, b1, bf16);
        rs::mma16816(s[j + 1], ahi[ks], b2, b3, bf16);
        if (split_q) {
          rs::mma16816(s[j], alo[ks], b0, b1, bf16);
          rs::mma16816(s[j + 1], alo[ks], b2, b3, bf16);
        }
      }
    }
  }

  // ---- softmax over c2 for rows r0 (s[.][0..1]) and r1 (s[.][2..3])
  float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const bool colok = j * 8 + qc + e < g.b2;
        s[j][e] = colok ? s[j][e] * g.sl2 : -INFINITY;
        s[j][2 + e] = colok ? s[j][2 + e] * g.sl2 : -INFINITY;
        m0 = fmaxf(m0, s[j][e]);
        m1 = fmaxf(m1, s[j][2 + e]);
      }
    }
  }
  m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
  m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
  m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
  m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
  float l0 = 0.f, l1 = 0.f, x0 = 0.f, x1 = 0.f;
#pragma unroll
  for (int j = 0; j < 8; ++j) {
    if (j < nt) {
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const float d0 = s[j][e] - m0, d1 = s[j][2 + e] - m1;
        const float p0 = ptx::ex2(d0), p1 = ptx::ex2(d1);
        s[j][e] = p0;
        s[j][2 + e] = p1;
        l0 += p0;
        l1 += p1;
        x0 += p0 > 0.f ? p0 * d0 : 0.f;
        x1 += p1 > 0.f ? p1 * d1 : 0.f;
      }
    }
  }
#pragma unroll
  for (int o = 1; o <= 2; o <<= 1) {
    l0 += __shfl_xor_sync(0xffffffffu, l0, o);
    l1 += __shfl_xor_sync(0xffffffffu, l1, o);
    x0 += __shfl_xor_sync(0xffffffffu, x0, o);
    x1 += __shfl_xor_sync(0xffffffffu, x1, o);
  }
  const float i0 = 1.f / l0, i1 = 1.f / l1;
  if ((lane & 3) == 0) {
    // h = -sum R ln R = ln l - ln2 * sum R (x - m)   (x in base-2 units)
    if (r0 < g.b2) w.h[((long long)bh * g.b2 + r0) * g.b1k + c1] = __logf(l0) - 0.6931471805599453f * x0 * i0;
    if (r1 < g.b2) w.h[((long long)bh * g.b2 + r1) * g.b1k + c1] = __logf(l1) - 0.6931471805599453f * x1 * i1;
  }
  // ---- R as A fragments (K = c2), split hi + lo
  uint32_t rhi[4][4], rlo[4][4];
#pragma unroll
  for (int kq = 0; kq < 4; ++kq) {
    if (2 * kq < nt) {
      const float v[8] = {s[2 * kq][0] * i0,     s[2 * kq][1] * i0,     s[2 * kq][2] * i1,
                          s[2 * kq][3] * i1,     s[2 * kq + 1][0] * i0, s[2 * kq + 1][1] * i0,
                          s[2 * kq + 1][2] * i1, s[2 * kq + 1][3] * i1};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const float hx = TcType<TQ>::round(v[2 * e]), hy = TcType<TQ>::round(v[2 * e + 1]);
        rhi[kq][e] = TcType<TQ>::pack(hx, hy);
        rlo[kq][e] = TcType<TQ>::pack(v[2 * e] - hx, v[2 * e + 1] - hy);
      }
    }
  }

  // ---- k~ = R k and z = R v  (B = tile rows [c2][d]: "row-major" B, ldmatrix.trans)
  for (int which = 0; which < (final_step ? 2 : 1); ++which) {
    const uint32_t aB = which ? aV : aK;
    float acc[D / 8][4];
#pragma unroll
    for (int j = 0; j < D / 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
#pragma unroll
    for (int kq = 0; kq < 4; ++kq) {
      if (2 * kq < nt) {
#pragma unroll
        for (int j = 0; j < D / 8; j += 2) {
          // matrices: (c2 lo, d-tile j), (c2 hi, j), (c2 lo, j+1), (c2 hi, j+1)
          const int row = kq * 16 + (lm & 1) * 8 + lr;
          const int col = (j + (lm >> 1)) * 8;
          uint32_t b0, b1, b2, b3;
          rs::ldsm_x4_t(aB + (row * PITCH + col) * 2, b0, b1, b2, b3);
          rs::mma16816(acc[j], rhi[kq], b0, b1, bf16);
          rs::mma16816(acc[j], rlo[kq], b0, b1, bf16);
          rs::mma16816(acc[j + 1], rhi[kq], b2, b3, bf16);
          rs::mma16816(acc[j + 1], rlo[kq], b2, b3, bf16);
        }
      }
    }
    // store rows r0 / r1 as hi + lo planes
#pragma unroll
    for (int half = 0; half < 2; ++half) {
      const int a2 = half ? r1 : r0;
      if (a2 >= g.b2) continue;
      const long long o = (((long long)bh * g.b2 + a2) * g.b1k + c1) * D;
#pragma unroll
      for (int j = 0; j < D / 8; ++j) {
        const float vx = acc[j][2 * half], vy = acc[j][2 * half + 1];
        const int col = j * 8 + qc;
        if (which == 0) {
          const float hx = TcType<TQ>::round(vx), hy = TcType<TQ>::round(vy);
          *reinterpret_cast<uint32_t*>(out.kt_hi + o + col) = TcType<TQ>::pack(hx, hy);
          *reinterpret_cast<uint32_t*>(out.kt_hi + out.plane + o + col) = TcType<TQ>::pack(vx - hx, vy - hy);
        } else {
          const float hx = TcType<__half>::round(vx), hy = TcType<__half>::round(vy);
          *reinterpret_cast<uint32_t*>(out.z_hi + o + col) = TcType<__half>::pack(hx, hy);
          *reinterpret_cast<uint32_t*>(out.z_hi + out.plane + o + col) = TcType<__half>::pack(vx - hx, vy - hy);
        }
      }
    }
  }
}

}  // namespace monarch
