// R step for bf16 / f16 inputs (warp-level mma.sync m16n8k16: the per-tile
// products are b2 x b2 x d with b2 <= 64, far below the 128-row tcgen05 tile,
// so a warp owns 16 positions of one key tile).
//
// For key tile c1 and positions a2 (16 per warp):
//   S[a2,c2] = s q~[c1,a2].k[c1,c2]      (q~ split hi+lo when it is computed)
//   R = softmax_c2(S), h = entropy(R)
//   k~[c1,a2] = sum_c2 R k[c1,c2]        (R split hi+lo; k~ stored as hi/lo planes)
//   z[c1,a2]  = sum_c2 R v[c1,c2]        (final step; stored as f16 hi/lo planes)
//
// The kernel is persistent and HBM-bound: one warp issues TMA loads into a
// ring of shared-memory stages while four warps compute.  The grid-to-block
// permutation is done by the TMA box itself: a 4-D map over (d, W, H, frames)
// with box (64, tw, th, 1) lands one key tile as b2 consecutive rows in the
// in-tile order c2 = (y mod th) * tw + x mod tw.  q~ rows (one per a2, stride
// b1k*d) come through a 3-D map over the q~ buffer.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "kernels_tc.cuh"
#include "tc_common.cuh"

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


// Tensor maps of one R step (128-byte swizzle everywhere).
struct RMaps {
  CUtensorMap q;    // queries   {d, W, H, BH*T},    box {64, tw, th, 1}
  CUtensorMap k;    // keys      {d, W, H, BH*Tk},   box {64, tw, th, 1}
  CUtensorMap v;    // values    {d, W, H, BH*Tk},   box {64, tw, th, 1}
  CUtensorMap qt;   // q~ (f32)  {d, b1k, BH*b2},    box {32, 1, b2}
};

// Shared-memory layout of one key tile in a stage.  Every region is a stack
// of [r8 rows][128 B] swizzled boxes (r8 = b2 rounded up to 8, so each box
// starts on a 1024-byte boundary):
//   A  q~ as d/32 f32 boxes (step with a q~ buffer); afterwards this warp's
//      output stage, [plane][d/64][r8][128 B] of 16-bit values
//   K  keys, d/64 boxes;  V values (final step);  X exact query rows (first step)
struct RStepLayout {
  int r8, tp, offK, offV, offX, tile_bytes, stage_bytes;
};

__host__ __device__ inline RStepLayout r_step_layout(int b2, int d, int mode, int final_step) {
  RStepLayout L;
  L.r8 = (b2 + 7) & ~7;
  L.tp = 4 / ((b2 + 15) >> 4);
  L.offK = L.r8 * d * 4;
  L.offV = L.offK + L.r8 * d * 2;
  L.offX = L.offV + (final_step ? L.r8 * d * 2 : 0);
  L.tile_bytes = L.offX + (mode != QT_BUFFER ? L.r8 * d * 2 : 0);
  L.stage_bytes = L.tp * L.tile_bytes;
  return L;
}

constexpr int kRThreads = 160;           // 4 compute warps + 1 TMA warp
constexpr int kRMaxStages = 4;
constexpr int kRFixedSmem = 1024 + 128 + 2 * kRMaxStages * 8;  // alignment slack, zero row, barriers

// Byte offset of 16-byte chunk `ch` of row `r` in a [rows][128 B] swizzled box.
__device__ __forceinline__ uint32_t swz(int r, int ch) { return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4)); }

// grid: persistent (a multiple of the SM count); block kRThreads.  A work
// item is tp consecutive key tiles of one head; CTA b takes items b,
// b + gridDim.x, ...
template <typename TQ, int D>
__global__ void __launch_bounds__(kRThreads, 2)
r_step_tc(const __grid_constant__ RMaps maps, Work w, TcPlanes<TQ> out, Geo g, int mode, int final_step,
          int stages) {
  constexpr int CH = D / 8;     // 16-byte chunks per row
  constexpr int bf16 = TcType<TQ>::kBf16;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  const RStepLayout L = r_step_layout(g.b2, D, mode, final_step);
  uint8_t* zero = base + stages * L.stage_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(zero + 128);
  uint64_t* empty = full + kRMaxStages;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int n_groups = (g.b1k + L.tp - 1) / L.tp;
  const int n_items = g.BH * n_groups;

  if (tid < 32) reinterpret_cast<uint32_t*>(zero)[tid] = 0u;
  if (tid == 0) {
    for (int s = 0; s < stages; ++s) {
      ptx::mbar_init(full + s, 1);
      ptx::mbar_init(empty + s, 4);
    }
    ptx::fence_mbar_init();
  }
  __syncthreads();

  if (warp == 4) {
    // ------------------------------------------------------------- TMA producer
    if (lane == 0) {
      ptx::prefetch_tmap(&maps.k);
      if (mode == QT_BUFFER) ptx::prefetch_tmap(&maps.qt);
      int it = 0;
      for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
        const int s = it % stages;
        if (it >= stages && !ptx::mbar_wait(empty + s, ((it / stages) - 1) & 1)) break;
        const int bh = item / n_groups, c1_0 = (item - bh * n_groups) * L.tp;
        const int ntile = min(L.tp, g.b1k - c1_0);
        uint32_t bytes = 0;
        for (int tt = 0; tt < ntile; ++tt) {
          const int c1 = c1_0 + tt;
          const bool exact_q = mode != QT_BUFFER && !(mode == QT_KVINIT && c1 < g.off);
          bytes += g.b2 * D * ((mode == QT_BUFFER ? 4 : 0) + 2 + (final_step ? 2 : 0) + (exact_q ? 2 : 0));
        }
        ptx::mbar_expect_tx(full + s, bytes);
        for (int tt = 0; tt < ntile; ++tt) {
          const int c1 = c1_0 + tt;
          uint8_t* tb = base + s * L.stage_bytes + tt * L.tile_bytes;
          const int t = c1 / g.P, rem = c1 - t * g.P, ty = rem / g.ntx, tx = rem - ty * g.ntx;
          if (mode == QT_BUFFER)
            for (int qq = 0; qq < D / 32; ++qq)
              ptx::tma_load_3d(tb + qq * L.r8 * 128, &maps.qt, full + s, qq * 32, c1, bh * g.b2);
          for (int hf = 0; hf < D / 64; ++hf) {
            ptx::tma_load_4d(tb + L.offK + hf * L.r8 * 128, &maps.k, full + s, hf * 64, tx * g.tw, ty * g.th,
                             bh * g.Tk + t);
            if (final_step)
              ptx::tma_load_4d(tb + L.offV + hf * L.r8 * 128, &maps.v, full + s, hf * 64, tx * g.tw, ty * g.th,
                               bh * g.Tk + t);
          }
          const bool exact_q = mode != QT_BUFFER && !(mode == QT_KVINIT && c1 < g.off);
          if (exact_q) {
            const int tq = t - (g.Tk - g.T);   // the aligned query frame (== t without a cache)
            for (int hf = 0; hf < D / 64; ++hf)
              ptx::tma_load_4d(tb + L.offX + hf * L.r8 * 128, &maps.q, full + s, hf * 64, tx * g.tw, ty * g.th,
                               bh * g.T + tq);
          }
        }
      }
    }
    return;
  }

  // ------------------------------------------------------------ compute warps
  const int mt = (g.b2 + 15) >> 4;
  const int tt = warp / mt, mi = warp % mt;
  const int r0 = mi * 16 + (lane >> 2), r1 = r0 + 8;  // positions a2 of this thread's rows
  const int qc = 2 * (lane & 3);
  const int lr = lane & 7, lm = lane >> 3;
  const int nt = 2 * mt;                               // n-tiles of 8 over c2
  const uint32_t zaddr = ptx::smem_u32(zero);
  const uint32_t box = (uint32_t)L.r8 * 128;          // bytes of one swizzled box

  int it = 0;
  for (int item = blockIdx.x; item < n_items; item += gridDim.x, ++it) {
    const int s = it % stages;
    if (!ptx::mbar_wait(full + s, (it / stages) & 1)) break;
    const int bh = item / n_groups;
    const int c1 = (item - bh * n_groups) * L.tp + tt;
    uint8_t* tb = base + s * L.stage_bytes + tt * L.tile_bytes;
    if (tt < L.tp && c1 < g.b1k) {
      const bool exact_q = mode != QT_BUFFER && !(mode == QT_KVINIT && c1 < g.off);
      const int cq = mode == QT_KVINIT ? c1 - g.off : c1;
      const uint32_t aA = ptx::smem_u32(tb), aK = aA + L.offK, aV = aA + L.offV, aX = aA + L.offX;
      // address of the 16-byte chunk holding column col (a multiple of 8) of row `row` of a
      // 16-bit region; rows past b2 read the zero row
      auto rowaddr = [&](uint32_t region, int row, int col) -> uint32_t {
        return row < g.b2 ? region + (col >> 6) * box + swz(row, (col >> 3) & 7) : zaddr;
      };

      // ---- first step: the exact query rows of this tile, copied block-major
      if (exact_q) {
        TQ* qb = reinterpret_cast<TQ*>(w.qb);
        for (int i = mi * 32 + lane; i < g.b2 * CH; i += mt * 32) {
          const int row = i / CH, ch = i - row * CH;
          *reinterpret_cast<uint4*>(qb + (((long long)bh * g.b2 + row) * g.b1q + cq) * D + ch * 8) =
              *reinterpret_cast<const uint4*>(tb + L.offX + (ch >> 3) * box + swz(row, ch & 7));
        }
      }

      // element (r, c) of the f32 q~ boxes: box c/32, chunk (c mod 32)/4
      auto qrow = [&](int r, int c) -> float2 {
        if (r >= g.b2) return make_float2(0.f, 0.f);
        if (mode == QT_BUFFER)
          return *reinterpret_cast<const float2*>(tb + (c >> 5) * box + swz(r, (c & 31) >> 2) + (c & 3) * 4);
        return *reinterpret_cast<const float2*>(w.qbar + ((long long)bh * g.b2 + r) * D + c);
      };

      // ---- S = q~ k^T; the A fragments of each k-step (q~ rows split hi + lo, or
      // the exact query rows) are built just before use
      float sc[8][4];
#pragma unroll
      for (int j = 0; j < 8; ++j) sc[j][0] = sc[j][1] = sc[j][2] = sc[j][3] = 0.f;
#pragma unroll
      for (int ks = 0; ks < D / 16; ++ks) {
        uint32_t ahi[4], alo[4];
        if (exact_q) {
          rs::ldsm_x4(rowaddr(aX, mi * 16 + (lm & 1) * 8 + lr, ks * 16 + (lm >> 1) * 8), ahi[0], ahi[1], ahi[2],
                      ahi[3]);
        } else {
          const int cA = ks * 16 + qc, cB = cA + 8;
          const float2 v0 = qrow(r0, cA), v1 = qrow(r1, cA), v2 = qrow(r0, cB), v3 = qrow(r1, cB);
          split_pair<TQ>(v0.x, v0.y, ahi[0], alo[0]);
          split_pair<TQ>(v1.x, v1.y, ahi[1], alo[1]);
          split_pair<TQ>(v2.x, v2.y, ahi[2], alo[2]);
          split_pair<TQ>(v3.x, v3.y, ahi[3], alo[3]);
        }
#pragma unroll
        for (int j = 0; j < 8; j += 2) {
          if (j < nt) {
            uint32_t b0, b1, b2, b3;
            rs::ldsm_x4(rowaddr(aK, (j + (lm >> 1)) * 8 + lr, ks * 16 + (lm & 1) * 8), b0, b1, b2, b3);
            rs::mma16816(sc[j], ahi, b0, b1, bf16);
            rs::mma16816(sc[j + 1], ahi, b2, b3, bf16);
            if (!exact_q) {
              rs::mma16816(sc[j], alo, b0, b1, bf16);
              rs::mma16816(sc[j + 1], alo, b2, b3, bf16);
            }
          }
        }
      }

      // ---- softmax over c2 for rows r0 (sc[.][0..1]) and r1 (sc[.][2..3])
      float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (j < nt) {
#pragma unroll
          for (int e = 0; e < 2; ++e) {
            const bool colok = j * 8 + qc + e < g.b2;
            sc[j][e] = colok ? sc[j][e] * g.sl2 : -INFINITY;
            sc[j][2 + e] = colok ? sc[j][2 + e] * g.sl2 : -INFINITY;
            m0 = fmaxf(m0, sc[j][e]);
            m1 = fmaxf(m1, sc[j][2 + e]);
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
            const float d0 = sc[j][e] - m0, d1 = sc[j][2 + e] - m1;
            const float p0 = ptx::ex2(d0), p1 = ptx::ex2(d1);
            sc[j][e] = p0;
            sc[j][2 + e] = p1;
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
          split_pair<TQ>(sc[2 * kq][0] * i0, sc[2 * kq][1] * i0, rhi[kq][0], rlo[kq][0]);
          split_pair<TQ>(sc[2 * kq][2] * i1, sc[2 * kq][3] * i1, rhi[kq][1], rlo[kq][1]);
          split_pair<TQ>(sc[2 * kq + 1][0] * i0, sc[2 * kq + 1][1] * i0, rhi[kq][2], rlo[kq][2]);
          split_pair<TQ>(sc[2 * kq + 1][2] * i1, sc[2 * kq + 1][3] * i1, rhi[kq][3], rlo[kq][3]);
        }
      }
      // this warp's q~ rows are in registers: its rows of region A become the output stage
      __syncwarp();

      // ---- k~ = R k and z = R v, staged in region A, written as 16-byte rows
      for (int which = 0; which < (final_step ? 2 : 1); ++which) {
        const uint32_t aB = which ? aV : aK;
        const uint32_t lo_plane = (D / 64) * box;
#pragma unroll 1
        for (int hf = 0; hf < D / 64; ++hf) {  // 64 output columns at a time
          float acc[8][4];
#pragma unroll
          for (int j = 0; j < 8; ++j) acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f;
#pragma unroll
          for (int kq = 0; kq < 4; ++kq) {
            if (2 * kq < nt) {
#pragma unroll
              for (int j = 0; j < 8; j += 2) {
                uint32_t b0, b1, b2, b3;
                rs::ldsm_x4_t(rowaddr(aB, kq * 16 + (lm & 1) * 8 + lr, hf * 64 + (j + (lm >> 1)) * 8), b0, b1, b2,
                              b3);
                rs::mma16816(acc[j], rhi[kq], b0, b1, bf16);
                rs::mma16816(acc[j], rlo[kq], b0, b1, bf16);
                rs::mma16816(acc[j + 1], rhi[kq], b2, b3, bf16);
                rs::mma16816(acc[j + 1], rlo[kq], b2, b3, bf16);
              }
            }
          }
          // stage rows r0, r1: [plane][d/64][r8][128 B]
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            uint32_t h0, l0w, h1, l1w;
            if (which == 0) {
              split_pair<TQ>(acc[j][0], acc[j][1], h0, l0w);
              split_pair<TQ>(acc[j][2], acc[j][3], h1, l1w);
            } else {
              split_pair<__half>(acc[j][0], acc[j][1], h0, l0w);
              split_pair<__half>(acc[j][2], acc[j][3], h1, l1w);
            }
            const int ch = j, cb = qc * 2;  // chunk within the 128-byte row, byte within the chunk
            const uint32_t o0 = hf * box + swz(r0, ch) + cb;
            const uint32_t o1 = hf * box + swz(r1, ch) + cb;
            if (r0 < g.b2) {
              *reinterpret_cast<uint32_t*>(tb + o0) = h0;
              *reinterpret_cast<uint32_t*>(tb + lo_plane + o0) = l0w;
            }
            if (r1 < g.b2) {
              *reinterpret_cast<uint32_t*>(tb + o1) = h1;
              *reinterpret_cast<uint32_t*>(tb + lo_plane + o1) = l1w;
            }
          }
        }
        __syncwarp();
        uint16_t* gbase = which ? reinterpret_cast<uint16_t*>(out.z_hi) : reinterpret_cast<uint16_t*>(out.kt_hi);
#pragma unroll
        for (int k = 0; k < (2 * 16 * CH) / 32; ++k) {
          const int idx = k * 32 + lane;
          const int plane = idx / (16 * CH);
          const int row = (idx / CH) % 16;
          const int ch = idx % CH;
          const int a2 = mi * 16 + row;
          if (a2 < g.b2) {
            const long long o = (((long long)bh * g.b2 + a2) * g.b1k + c1) * D + ch * 8;
            *reinterpret_cast<uint4*>(gbase + plane * out.plane + o) = *reinterpret_cast<const uint4*>(
                tb + (plane * (D / 64) + (ch >> 3)) * box + swz(a2, ch & 7));
          }
        }
        __syncwarp();
      }
    }
    // every read of this stage by this warp is done
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(empty + s);
  }
}

// Shared memory of one r_step_tc launch with `stages` stages.
inline size_t r_step_smem(const RStepLayout& L, int stages) {
  return (size_t)stages * L.stage_bytes + kRFixedSmem;
}

}  // namespace monarch
