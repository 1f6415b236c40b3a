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

// Split of a computed pair into hi + lo of type TQ (packed).
template <typename TQ>
__device__ __forceinline__ void split_pair(float x, float y, uint32_t& hi, uint32_t& lo) {
  hi = TcType<TQ>::pack(x, y);
  float hx, hy;
  if constexpr (TcType<TQ>::kBf16) {
    hx = __uint_as_float(hi << 16);
    hy = __uint_as_float(hi & 0xFFFF0000u);
  } else {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hi));
    hx = f.x;
    hy = f.y;
  }
  lo = TcType<TQ>::pack(x - hx, y - hy);
}

template <int D>
constexpr int r_step_tc_pitch() { return D + 8; }  // 16-bit elements per shared row (16-byte pad)

// Gathered [rows][PITCH] tiles per key tile: k always, v in the final step,
// the exact query rows in the first step.
__host__ __device__ inline int r_step_slots(int mode, int final_step) {
  return 1 + (final_step ? 1 : 0) + (mode != QT_BUFFER ? 1 : 0);
}

// Shared memory of r_step_tc: the gathered tiles plus a per-warp
// [2 planes][16 rows][PITCH] output stage and the row-offset table.
template <int D>
size_t r_step_tc_smem(int b2, int slots) {
  const int mt = (b2 + 15) / 16, rows = 16 * mt, tpc = 4 / mt;
  return (size_t)tpc * slots * rows * r_step_tc_pitch<D>() * 2 + 4 * 2 * 16 * r_step_tc_pitch<D>() * 2 + 64 * 4;
}

// grid (ceil(b1k / tiles_per_cta), BH), block 128 (4 warps; a warp owns 16
// positions of one key tile), tiles_per_cta = 4 / ceil(b2/16).
template <typename TQ, int D>
__global__ void __launch_bounds__(128, 3)
r_step_tc(const TQ* __restrict__ q, const TQ* __restrict__ k, const TQ* __restrict__ v, Work w,
          TcPlanes<TQ> out, Geo g, int mode, int final_step) {
  constexpr int PITCH = r_step_tc_pitch<D>();
  constexpr int CH = D / 8;     // 16-byte chunks per row
  constexpr int bf16 = TcType<TQ>::kBf16;
  extern __shared__ uint8_t smem_raw[];
  TQ* smem = reinterpret_cast<TQ*>(smem_raw);
  const int mt = (g.b2 + 15) >> 4;
  const int rows = mt * 16;
  const int tpc = 4 / mt;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int bh = blockIdx.y;
  const int slots = r_step_slots(mode, final_step);
  const int slot_v = 1, slot_x = final_step ? 2 : 1;
  TQ* stage = smem + tpc * slots * rows * PITCH + warp * 2 * 16 * PITCH;  // this warp's output stage
  int* roff = reinterpret_cast<int*>(smem + tpc * slots * rows * PITCH + 4 * 2 * 16 * PITCH);
  const TQ* kh = k + (long long)bh * g.Nk * D;
  const TQ* vh = v + (long long)bh * g.Nk * D;
  const TQ* qh = q + (long long)bh * g.Nq * D;

  // token offset of position c2 inside its tile: (c2 / tw) * W + c2 % tw
  if (tid < g.b2) roff[tid] = (tid / g.tw) * g.W + tid % g.tw;
  __syncthreads();

  // ---- gather k, v (final step) and the exact q rows (first step) of each tile
  for (int tt = 0; tt < tpc; ++tt) {
    const int c1 = blockIdx.x * tpc + tt;
    if (c1 >= g.b1k) break;
    const bool exact_q = mode != QT_BUFFER && !(mode == QT_KVINIT && c1 < g.off);
    const int cq = mode == QT_KVINIT ? c1 - g.off : c1;
    for (int mat = 0; mat < 3; ++mat) {
      if ((mat == 1 && !final_step) || (mat == 2 && !exact_q)) continue;
      const int ct = mat == 2 ? cq : c1;
      const long long tbase = token_of(g, ct, 0);
      const TQ* src0 = mat == 0 ? kh : (mat == 1 ? vh : qh);
      TQ* dst0 = smem + (tt * slots + (mat == 0 ? 0 : mat == 1 ? slot_v : slot_x)) * rows * PITCH;
      for (int row = tid / CH; row < rows; row += 128 / CH) {
        const int ch = tid % CH;
        const bool valid = row < g.b2;
        const TQ* src = src0 + (valid ? (tbase + roff[row]) * D + ch * 8 : 0);
        ptx::cp_async_16(ptx::smem_u32(dst0 + row * PITCH + ch * 8), src, valid ? 16u : 0u);
      }
    }
  }
  ptx::cp_async_commit();

  const int tt = warp / mt, mi = warp % mt;
  const int c1 = blockIdx.x * tpc + tt;
  const bool active = tt < tpc && c1 < g.b1k;
  const bool exact_q = mode != QT_BUFFER && !(mode == QT_KVINIT && c1 < g.off);
  const int r0 = mi * 16 + (lane >> 2), r1 = r0 + 8;  // positions a2 of this thread's rows
  const int qc = 2 * (lane & 3);
  const int lr = lane & 7, lm = lane >> 3;

  // ---- A fragments of a computed q~ (fp32 rows, split hi + lo); issued before the gather completes
  uint32_t ahi[D / 16][4], alo[D / 16][4];
  if (active && !exact_q) {
    const float* qr0 = nullptr;
    const float* qr1 = nullptr;
    if (mode == QT_BUFFER) {
      if (r0 < g.b2) qr0 = w.qt + (((long long)bh * g.b2 + r0) * g.b1k + c1) * D;
      if (r1 < g.b2) qr1 = w.qt + (((long long)bh * g.b2 + r1) * g.b1k + c1) * D;
    } else {
      if (r0 < g.b2) qr0 = w.qbar + ((long long)bh * g.b2 + r0) * D;
      if (r1 < g.b2) qr1 = w.qbar + ((long long)bh * g.b2 + r1) * D;
    }
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int cA = ks * 16 + qc, cB = cA + 8;
      const float2 v0 = qr0 ? *reinterpret_cast<const float2*>(qr0 + cA) : make_float2(0.f, 0.f);
      const float2 v1 = qr1 ? *reinterpret_cast<const float2*>(qr1 + cA) : make_float2(0.f, 0.f);
      const float2 v2 = qr0 ? *reinterpret_cast<const float2*>(qr0 + cB) : make_float2(0.f, 0.f);
      const float2 v3 = qr1 ? *reinterpret_cast<const float2*>(qr1 + cB) : make_float2(0.f, 0.f);
      split_pair<TQ>(v0.x, v0.y, ahi[ks][0], alo[ks][0]);
      split_pair<TQ>(v1.x, v1.y, ahi[ks][1], alo[ks][1]);
      split_pair<TQ>(v2.x, v2.y, ahi[ks][2], alo[ks][2]);
      split_pair<TQ>(v3.x, v3.y, ahi[ks][3], alo[ks][3]);
    }
  }
  ptx::cp_async_wait<0>();
  __syncthreads();

  // ---- first step: write the exact query rows in block-major order (coalesced)
  for (int t2 = 0; t2 < tpc; ++t2) {
    const int cc1 = blockIdx.x * tpc + t2;
    if (cc1 >= g.b1k) break;
    if (mode == QT_BUFFER || (mode == QT_KVINIT && cc1 < g.off)) continue;
    const int cq = mode == QT_KVINIT ? cc1 - g.off : cc1;
    const TQ* src0 = smem + (t2 * slots + slot_x) * rows * PITCH;
    TQ* qb = reinterpret_cast<TQ*>(w.qb);
    for (int i = tid; i < g.b2 * CH; i += 128) {
      const int row = i / CH, ch = i % CH;
      *reinterpret_cast<uint4*>(qb + (((long long)bh * g.b2 + row) * g.b1q + cq) * D + ch * 8) =
          *reinterpret_cast<const uint4*>(src0 + row * PITCH + ch * 8);
    }
  }
  if (!active) return;

  const uint32_t aK = ptx::smem_u32(smem + (tt * slots + 0) * rows * PITCH);
  const uint32_t aV = ptx::smem_u32(smem + (tt * slots + slot_v) * rows * PITCH);
  const uint32_t aX = ptx::smem_u32(smem + (tt * slots + slot_x) * rows * PITCH);
  if (exact_q) {
    // A fragments straight from the gathered exact rows: matrices (rows 0-7 | 8-15) x (k lo | k hi)
#pragma unroll
    for (int ks = 0; ks < D / 16; ++ks) {
      const int row = mi * 16 + (lm & 1) * 8 + lr;
      const int col = ks * 16 + (lm >> 1) * 8;
      rs::ldsm_x4(aX + (row * PITCH + col) * 2, ahi[ks][0], ahi[ks][1], ahi[ks][2], ahi[ks][3]);
    }
  }
  const int nt = rows / 8;  // n-tiles over c2 (even)

  // ---- S = q~ k^T
  float s[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) s[j][0] = s[j][1] = s[j][2] = s[j][3] = 0.f;
#pragma unroll
  for (int ks = 0; ks < D / 16; ++ks) {
#pragma unroll
    for (int j = 0; j < 8; j += 2) {
      if (j < nt) {
        const int row = (j + (lm >> 1)) * 8 + lr;
        const int col = ks * 16 + (lm & 1) * 8;
        uint32_t b0, b1, b2, b3;
        rs::ldsm_x4(aK + (row * PITCH + col) * 2, b0, b1, b2, b3);
        rs::mma16816(s[j], ahi[ks], b0, b1, bf16);
        rs::mma16816(s[j + 1], ahi[ks], b2, b3, bf16);
        if (!exact_q) {
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
    // h in bits: -sum R log2 R = log2 l - sum R (x - m)   (x in base-2 units)
    if (r0 < g.b2) w.h[((long long)bh * g.b2 + r0) * g.b1k_pad + c1] = log2f(l0) - x0 * i0;
    if (r1 < g.b2) w.h[((long long)bh * g.b2 + r1) * g.b1k_pad + c1] = log2f(l1) - x1 * i1;
  }
  // ---- R as A fragments (K = c2), split hi + lo
  uint32_t rhi[4][4], rlo[4][4];
#pragma unroll
  for (int kq = 0; kq < 4; ++kq) {
    if (2 * kq < nt) {
      split_pair<TQ>(s[2 * kq][0] * i0, s[2 * kq][1] * i0, rhi[kq][0], rlo[kq][0]);
      split_pair<TQ>(s[2 * kq][2] * i1, s[2 * kq][3] * i1, rhi[kq][1], rlo[kq][1]);
      split_pair<TQ>(s[2 * kq + 1][0] * i0, s[2 * kq + 1][1] * i0, rhi[kq][2], rlo[kq][2]);
      split_pair<TQ>(s[2 * kq + 1][2] * i1, s[2 * kq + 1][3] * i1, rhi[kq][3], rlo[kq][3]);
    }
  }

  // ---- k~ = R k and z = R v, staged per warp, then written as coalesced 16-byte rows
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
    __syncwarp();
    // stage rows (lane/4) and (lane/4 + 8) of this warp's 16, hi plane then lo plane
#pragma unroll
    for (int j = 0; j < D / 8; ++j) {
      uint32_t h0, l0w, h1, l1w;
      if (which == 0) {
        split_pair<TQ>(acc[j][0], acc[j][1], h0, l0w);
        split_pair<TQ>(acc[j][2], acc[j][3], h1, l1w);
      } else {
        split_pair<__half>(acc[j][0], acc[j][1], h0, l0w);
        split_pair<__half>(acc[j][2], acc[j][3], h1, l1w);
      }
      const int col = j * 8 + qc;
      const int ra = lane >> 2, rb = ra + 8;
      *reinterpret_cast<uint32_t*>(stage + ra * PITCH + col) = h0;
      *reinterpret_cast<uint32_t*>(stage + rb * PITCH + col) = h1;
      *reinterpret_cast<uint32_t*>(stage + (16 + ra) * PITCH + col) = l0w;
      *reinterpret_cast<uint32_t*>(stage + (16 + rb) * PITCH + col) = l1w;
    }
    __syncwarp();
    uint16_t* gbase = which ? reinterpret_cast<uint16_t*>(out.z_hi) : reinterpret_cast<uint16_t*>(out.kt_hi);
#pragma unroll
    for (int it = 0; it < (2 * 16 * CH) / 32; ++it) {
      const int idx = it * 32 + lane;
      const int plane = idx / (16 * CH);
      const int row = (idx / CH) % 16;
      const int ch = idx % CH;
      const int a2 = mi * 16 + row;
      if (a2 < g.b2) {
        const long long o = (((long long)bh * g.b2 + a2) * g.b1k + c1) * D + ch * 8;
        *reinterpret_cast<uint4*>(gbase + plane * out.plane + o) =
            *reinterpret_cast<const uint4*>(stage + (plane * 16 + row) * PITCH + ch * 8);
      }
    }
  }
}

}  // namespace monarch
