// Warp-specialised tcgen05 kernels of the L step (bf16 / f16 inputs).
//
// Block = 9 warps.  Warp 8 (one elected lane) issues every TMA load and every
// tcgen05.mma; warps 0-7 are softmax warps: row r of a 128-row tile belongs
// to TMEM lane r and is shared by warp (r/32) (columns 0-31 of each 64-wide
// block) and warp (r/32)+4 (columns 32-63).  Scores are double-buffered in
// TMEM so the tensor pipe computes block j+1 while the softmax warps work on
// block j; operand tiles arrive by TMA into double- or triple-buffered stages.
//
// Precision (see the header of kernels_tc.cuh): k~ and z as hi/lo planes, q
// exact, L split into hi/lo planes in the column pass, P single f16 with the
// rounded values summed, fp32 statistics.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "kernels_tc.cuh"

namespace monarch {
namespace v2 {

constexpr int kBlk = 64;            // keys (row pass) / queries (column pass) per block
constexpr int kBox = 8192;          // one [64 rows][128 B] swizzled box
constexpr int kThreads = 288;
constexpr int kMmaWarp = 8;

// ---- packed fp32 pairs (sm_100 f32x2 arithmetic)
__device__ __forceinline__ uint64_t f2u(float2 a) { return *reinterpret_cast<uint64_t*>(&a); }
__device__ __forceinline__ float2 u2f(uint64_t a) { return *reinterpret_cast<float2*>(&a); }
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(f2u(a)), "l"(f2u(b)), "l"(f2u(c)));
  return u2f(d);
}
__device__ __forceinline__ float2 add2(float2 a, float2 b) {
  uint64_t d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2u(a)), "l"(f2u(b)));
  return u2f(d);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2u(a)), "l"(f2u(b)));
  return u2f(d);
}

// hi = round(p) and lo = round(p - hi) of a pair, packed, in the operand type.
template <typename TQ>
__device__ __forceinline__ void split2(float2 p, uint32_t& hi, uint32_t& lo) {
  hi = TcType<TQ>::pack(p.x, p.y);
  float2 h;
  if constexpr (TcType<TQ>::kBf16) {
    h.x = __uint_as_float(hi << 16);
    h.y = __uint_as_float(hi & 0xFFFF0000u);
  } else {
    h = __half22float2(*reinterpret_cast<const __half2*>(&hi));
  }
  const float2 r = sub2(p, h);
  lo = TcType<TQ>::pack(r.x, r.y);
}

__device__ __forceinline__ void named_bar(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

__device__ __forceinline__ void sts128(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d) {
  asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, uint64_t* bar, int x, int y) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
      ::"r"(ptx::smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(ptx::smem_u32(bar)), "r"(x), "r"(y)
      : "memory");
}

struct Maps {
  CUtensorMap qb;   // block-major q  {d, b1q, BH*b2},      box {64, 64, 1}
  CUtensorMap kt;   // k~ planes      {d, b1k, 2*BH*b2},    box {64, 64, 1}
  CUtensorMap z;    // z planes       {d, b1k, 2*BH*b2},    box {64, 64, 1}
  CUtensorMap h;    // entropy        {b1k_pad, BH*b2},     box {64, 1}
  CUtensorMap lse;  // row LSE        {b1q_pad, BH*b2},     box {64, 1}
};

// ===========================================================================
// Row pass for one (head, position a2, 128 query rows), 64 key tiles per block.
//   OUT:  out[token(a1,a2)] = sum_c1 L z
//   !OUT: lse[a1] = log2 sum_c1 2^(s q.k~ + h)
template <typename TQ, typename TO, int D, bool OUT>
__global__ void __launch_bounds__(kThreads, OUT ? 1 : 2)
l_row(TO* __restrict__ out, const __grid_constant__ Maps maps, float* __restrict__ lse, Geo g) {
  constexpr int NH = D / 64;
  constexpr uint32_t kQ = 2 * NH * kBox;           // 128 query rows
  constexpr uint32_t kKst = 2 * NH * kBox;         // k~ hi+lo, 64 rows
  constexpr uint32_t kZst = 2 * NH * kBox;         // z hi+lo, 64 rows
  constexpr uint32_t kPst = 2 * kBox;              // P: 128 rows x 64 keys
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = sQ + kQ;                           // [2 stages]
  uint8_t* sZ = sK + 2 * kKst;                     // [2 stages] (OUT)
  uint8_t* sP = sZ + (OUT ? 2 * kZst : 0);         // [2 buffers] (OUT)
  float* sH = reinterpret_cast<float*>(sP + (OUT ? 2 * kPst : 0));  // [2][64]
  float* sX = sH + 2 * kBlk;                                         // [2][2][128] exchange
  uint64_t* bar = reinterpret_cast<uint64_t*>(sX + 2 * 2 * kTile);
  uint64_t* q_full = bar + 0;
  uint64_t* k_full = bar + 1;    // [2]
  uint64_t* z_full = bar + 3;    // [2]
  uint64_t* s_full = bar + 5;    // [2]
  uint64_t* s_free = bar + 7;    // [2]
  uint64_t* p_full = bar + 9;    // [2]
  uint64_t* pv_done = bar + 11;  // [2]
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bar + 13);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int a2 = blockIdx.y, bh = blockIdx.z;
  const int a1_base = blockIdx.x * kTile;
  const int zrow = bh * g.b2 + a2;
  const int plane_rows = g.BH * g.b2;
  const int nkb = (g.b1k + kBlk - 1) / kBlk;

  if (tid == 0) {
    ptx::mbar_init(q_full, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(k_full + i, 1);
      ptx::mbar_init(z_full + i, 1);
      ptx::mbar_init(s_full + i, 1);
      ptx::mbar_init(s_free + i, 8);
      ptx::mbar_init(p_full + i, 8);
      ptx::mbar_init(pv_done + i, 1);
    }
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(sTmem, 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t tO = tmem + 128;

  if (warp == kMmaWarp) {
    if (lane == 0) {
      // ------------------------------------------------ producer + MMA issuer
      auto load_k = [&](int blk, int st) {
        ptx::mbar_expect_tx(k_full + st, kKst + kBlk * 4);
        for (int p = 0; p < 2; ++p)
          for (int hf = 0; hf < NH; ++hf)
            ptx::tma_load_3d(sK + st * kKst + (p * NH + hf) * kBox, &maps.kt, k_full + st, hf * 64, blk * kBlk,
                             p * plane_rows + zrow);
        tma_load_2d(sH + st * kBlk, &maps.h, k_full + st, blk * kBlk, zrow);
      };
      auto load_z = [&](int blk, int st) {
        ptx::mbar_expect_tx(z_full + st, kZst);
        for (int p = 0; p < 2; ++p)
          for (int hf = 0; hf < NH; ++hf)
            ptx::tma_load_3d(sZ + st * kZst + (p * NH + hf) * kBox, &maps.z, z_full + st, hf * 64, blk * kBlk,
                             p * plane_rows + zrow);
      };
      ptx::prefetch_tmap(&maps.qb);
      ptx::prefetch_tmap(&maps.kt);
      ptx::mbar_expect_tx(q_full, kQ);
      for (int hf = 0; hf < NH; ++hf)
        for (int r = 0; r < 2; ++r)
          ptx::tma_load_3d(sQ + hf * 2 * kBox + r * kBox, &maps.qb, q_full, hf * 64, a1_base + r * kBlk, zrow);
      for (int s = 0; s < 2 && s < nkb; ++s) load_k(s, s);
      if (OUT)
        for (int s = 0; s < 2 && s < nkb; ++s) load_z(s, s);

      constexpr uint32_t idS = ptx::idesc_f16(128, kBlk, TcType<TQ>::kBf16, 0, 0);
      constexpr uint32_t idPV = ptx::idesc_f16(128, D, 0, 0, 1);
      const uint32_t aQ = ptx::smem_u32(sQ), aK = ptx::smem_u32(sK), aZ = ptx::smem_u32(sZ),
                     aP = ptx::smem_u32(sP);
      auto issue_s = [&](int blk) {
        const int st = blk & 1;
        const uint32_t tS = tmem + st * kBlk;
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t aoff = (kk >> 2) * 2 * kBox + (kk & 3) * 32;  // q: 128-row halves
            const uint32_t boff = (p * NH + (kk >> 2)) * kBox + (kk & 3) * 32;
            ptx::mma_f16_ss(tS, ptx::sw128_desc(aQ + aoff, 16, 1024),
                            ptx::sw128_desc(aK + st * kKst + boff, 16, 1024), idS, (p | kk) != 0);
          }
        ptx::mma_commit(s_full + st);
      };
      bool ok = ptx::mbar_wait(q_full, 0) && ptx::mbar_wait(k_full, 0);
      ptx::tc_fence_after();
      if (ok) issue_s(0);
      for (int j = 0; j < nkb && ok; ++j) {
        const int st = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        if (j + 1 < nkb) {
          const int sn = (j + 1) & 1;
          ok = ptx::mbar_wait(k_full + sn, ((j + 1) >> 1) & 1);
          if (ok && j + 1 >= 2) ok = ptx::mbar_wait(s_free + sn, ((j - 1) >> 1) & 1);
          ptx::tc_fence_after();
          if (ok) issue_s(j + 1);
        }
        // z stage (j+1)&1 held block j-1: refill it with block j+1 once L z (j-1)
        // is done.  Deferred to here so that the issuer never waits on the
        // product it has just issued.
        if (OUT && ok && j >= 1 && j + 1 < nkb) {
          ok = ptx::mbar_wait(pv_done + ((j - 1) & 1), ((j - 1) >> 1) & 1);
          if (ok) load_z(j + 1, (j + 1) & 1);
        }
        // k~ / h stage st is free once softmax(j) has read S(j) (and h)
        if (ok && j + 2 < nkb) {
          ok = ptx::mbar_wait(s_free + st, ph);
          if (ok) load_k(j + 2, st);
        }
        if (OUT && ok) {
          ok = ptx::mbar_wait(p_full + st, ph) && ptx::mbar_wait(z_full + st, ph);
          ptx::tc_fence_after();
          if (ok) {
#pragma unroll
            for (int p = 0; p < 2; ++p)
#pragma unroll
              for (int kk = 0; kk < kBlk / 16; ++kk)
                ptx::mma_f16_ss(tO, ptx::sw128_desc(aP + st * kPst + kk * 32, 16, 1024),
                                ptx::sw128_desc(aZ + st * kZst + p * NH * kBox + kk * 2048, kBox, 1024), idPV,
                                (j | p | kk) != 0);
            ptx::mma_commit(pv_done + st);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------- softmax warps
    const int r = 32 * (warp & 3) + lane;       // tile row / TMEM lane
    const int hf = warp >> 2;                   // column half of each block
    const int bid = 1 + (warp & 3);             // named barrier of the row pair
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    float m = -INFINITY, l = 0.f;
    bool ok = true;
    const float2 sl2 = make_float2(g.sl2, g.sl2);
    for (int j = 0; j < nkb; ++j) {
      const int st = j & 1;
      const uint32_t ph = (j >> 1) & 1;
      // after a timed-out wait (ok == false) the loop keeps its shape (every
      // named barrier is still reached by both threads of a row) but skips waits
      ok = ok && ptx::mbar_wait(s_full + st, ph) && ptx::mbar_wait(k_full + st, ph);
      ptx::tc_fence_after();
      uint32_t sr[32];
      ptx::tmem_ld32(tmem + st * kBlk + lane_off + hf * 32, sr);
      const float4* hv = reinterpret_cast<const float4*>(sH + st * kBlk + hf * 32);
      const int valid = min(kBlk, g.b1k - j * kBlk) - hf * 32;  // columns of this half that exist
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(s_free + st);
      float2 x[16];
      float mb = -INFINITY;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 h4 = hv[i];
        const float2 s0 = make_float2(__uint_as_float(sr[4 * i]), __uint_as_float(sr[4 * i + 1]));
        const float2 s1 = make_float2(__uint_as_float(sr[4 * i + 2]), __uint_as_float(sr[4 * i + 3]));
        x[2 * i] = fma2(s0, sl2, make_float2(h4.x * kLog2e, h4.y * kLog2e));
        x[2 * i + 1] = fma2(s1, sl2, make_float2(h4.z * kLog2e, h4.w * kLog2e));
      }
      if (valid < 32) {  // only the last block of a ragged row
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          if (2 * i >= valid) x[i].x = -INFINITY;
          if (2 * i + 1 >= valid) x[i].y = -INFINITY;
        }
      }
#pragma unroll
      for (int i = 0; i < 16; ++i) mb = fmaxf(mb, fmaxf(x[i].x, x[i].y));
      // row max over both halves
      float* xs = sX + st * 2 * kTile;
      xs[hf * kTile + r] = mb;
      named_bar(bid, 64);
      mb = fmaxf(mb, xs[(hf ^ 1) * kTile + r]);
      const bool move = mb > m + kLazyRescale;
      const float mn = move ? mb : m;
      const float corr = ptx::ex2(m - mn);
      const float2 nm = make_float2(-mn, -mn);
      float2 acc2 = make_float2(0.f, 0.f);
      if constexpr (OUT) {
        if (j > 0 && __any_sync(0xffffffffu, move)) {
          // PV(j-1) must be done writing O before it is rescaled
          ok = ok && ptx::mbar_wait(pv_done + ((j - 1) & 1), ((j - 1) >> 1) & 1);
          ptx::tc_fence_after();
#pragma unroll
          for (int cc = 0; cc < D / 64; ++cc) {
            uint32_t o[32];
            const uint32_t ta = tO + lane_off + hf * (D / 2) + cc * 32;
            ptx::tmem_ld32(ta, o);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
            ptx::tmem_st32(ta, o);
          }
          ptx::tmem_wait_st();
        }
        uint32_t pk[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 d = add2(x[i], nm);
          const __half2 hp = __floats2half2_rn(ptx::ex2(d.x), ptx::ex2(d.y));
          acc2 = add2(acc2, __half22float2(hp));
          pk[i] = *reinterpret_cast<const uint32_t*>(&hp);
        }
        // P buffer st was last read by PV(j-2), which finished before S(j)
        const uint32_t prow = ptx::smem_u32(sP + st * kPst);
#pragma unroll
        for (int c = 0; c < 4; ++c)
          sts128(prow + ptx::sw128_offset(r, hf * 4 + c), pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        ptx::fence_proxy_async();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(p_full + st);
      } else {
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float2 d = add2(x[i], nm);
          acc2 = add2(acc2, make_float2(ptx::ex2(d.x), ptx::ex2(d.y)));
        }
      }
      l = fmaf(l, corr, acc2.x + acc2.y);
      m = mn;
    }
    // combine the two halves' sums
    named_bar(bid, 64);
    float* xs = sX;
    xs[hf * kTile + r] = l;
    named_bar(bid, 64);
    const float lt = l + xs[(hf ^ 1) * kTile + r];
    const int a1 = a1_base + r;
    if constexpr (OUT) {
      const int last = nkb - 1;
      ok = ok && ptx::mbar_wait(pv_done + (last & 1), (last >> 1) & 1);
      ptx::tc_fence_after();
      const float inv = 1.f / lt;
      TO* orow = out + ((long long)bh * g.Nq + (a1 < g.b1q ? token_of(g, a1, a2) : 0)) * D + hf * (D / 2);
#pragma unroll
      for (int cc = 0; cc < D / 64; ++cc) {
        uint32_t o[32];
        ptx::tmem_ld32(tO + lane_off + hf * (D / 2) + cc * 32, o);
        ptx::tmem_wait_ld();
        if (a1 < g.b1q && ok) {
#pragma unroll
          for (int i = 0; i < 32; i += 4) {
            if constexpr (sizeof(TO) == 4) {
              *reinterpret_cast<float4*>(orow + cc * 32 + i) =
                  make_float4(__uint_as_float(o[i]) * inv, __uint_as_float(o[i + 1]) * inv,
                              __uint_as_float(o[i + 2]) * inv, __uint_as_float(o[i + 3]) * inv);
            } else {
              TO v4[4];
#pragma unroll
              for (int e = 0; e < 4; ++e) v4[e] = from_f<TO>(__uint_as_float(o[i + e]) * inv);
              *reinterpret_cast<uint2*>(orow + cc * 32 + i) = *reinterpret_cast<uint2*>(v4);
            }
          }
        }
      }
    } else if (hf == 0 && a1 < g.b1q) {
      lse[(long long)zrow * g.b1q_pad + a1] = m + log2f(lt);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 256);
}

template <int D, bool OUT>
constexpr size_t l_row_smem() {
  return 1024 + 2 * (D / 64) * kBox * (1 + 2 + (OUT ? 2 : 0)) + (OUT ? 2 * 2 * kBox : 0) + 2 * kBlk * 4 +
         4 * kTile * 4 + 16 * 8;
}

// ===========================================================================
// Column pass for one (head, position a2, 128 key tiles), 64 queries per block:
//   q~[c1,a2] = sum_a1 L q / sum_a1 L,  L = 2^(s q.k~ + h - lse[a1]).
// S^T = k~ q^T recomputed per block (A: k~ planes, B: q, K-major); the
// aggregate takes P^T_hi q + P^T_lo q (A: P^T planes, B: q, MN-major).
template <typename TQ, int D>
__global__ void __launch_bounds__(kThreads, 1)
l_col(const __grid_constant__ Maps maps, const float* __restrict__ hbuf, float* __restrict__ qt, Geo g) {
  constexpr int NH = D / 64;
  constexpr int QS = 3;                            // query stages
  constexpr uint32_t kK = 2 * 2 * NH * kBox;       // k~ hi+lo, 128 rows
  constexpr uint32_t kQst = NH * kBox;             // 64 query rows
  constexpr uint32_t kPst = 2 * 2 * kBox;          // P^T hi+lo, 128 rows x 64 queries
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base;
  uint8_t* sQ = sK + kK;                           // [QS]
  uint8_t* sP = sQ + QS * kQst;                    // [2]
  float* sL = reinterpret_cast<float*>(sP + 2 * kPst);  // [QS][64]
  float* sX = sL + QS * kBlk;                             // [2][128]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sX + 2 * kTile);
  uint64_t* k_full = bar + 0;
  uint64_t* q_full = bar + 1;    // [QS]
  uint64_t* s_full = bar + 4;    // [2]
  uint64_t* s_free = bar + 6;    // [2]
  uint64_t* p_full = bar + 8;    // [2]
  uint64_t* pq_done = bar + 10;  // [2]
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bar + 12);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int a2 = blockIdx.y, bh = blockIdx.z;
  const int kb = blockIdx.x * kTile;
  const int zrow = bh * g.b2 + a2;
  const int plane_rows = g.BH * g.b2;
  const int nqb = (g.b1q + kBlk - 1) / kBlk;

  if (tid == 0) {
    ptx::mbar_init(k_full, 1);
    for (int i = 0; i < QS; ++i) ptx::mbar_init(q_full + i, 1);
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(s_full + i, 1);
      ptx::mbar_init(s_free + i, 8);
      ptx::mbar_init(p_full + i, 8);
      ptx::mbar_init(pq_done + i, 1);
    }
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(sTmem, 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t tA = tmem + 128;

  if (warp == kMmaWarp) {
    if (lane == 0) {
      auto load_q = [&](int blk, int qs) {
        ptx::mbar_expect_tx(q_full + qs, kQst + kBlk * 4);
        for (int hf = 0; hf < NH; ++hf)
          ptx::tma_load_3d(sQ + qs * kQst + hf * kBox, &maps.qb, q_full + qs, hf * 64, blk * kBlk, zrow);
        tma_load_2d(sL + qs * kBlk, &maps.lse, q_full + qs, blk * kBlk, zrow);
      };
      ptx::prefetch_tmap(&maps.qb);
      ptx::prefetch_tmap(&maps.kt);
      ptx::mbar_expect_tx(k_full, kK);
      for (int p = 0; p < 2; ++p)
        for (int hf = 0; hf < NH; ++hf)
          for (int r = 0; r < 2; ++r)
            ptx::tma_load_3d(sK + (p * NH + hf) * 2 * kBox + r * kBox, &maps.kt, k_full, hf * 64, kb + r * kBlk,
                             p * plane_rows + zrow);
      for (int s = 0; s < QS && s < nqb; ++s) load_q(s, s);

      constexpr uint32_t idS = ptx::idesc_f16(128, kBlk, TcType<TQ>::kBf16, 0, 0);
      constexpr uint32_t idPQ = ptx::idesc_f16(128, D, TcType<TQ>::kBf16, 0, 1);
      const uint32_t aK = ptx::smem_u32(sK), aQ = ptx::smem_u32(sQ), aP = ptx::smem_u32(sP);
      auto issue_s = [&](int blk) {
        const int st = blk & 1, qs = blk % QS;
        const uint32_t tS = tmem + st * kBlk;
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
          for (int kk = 0; kk < D / 16; ++kk) {
            const uint32_t aoff = (p * NH + (kk >> 2)) * 2 * kBox + (kk & 3) * 32;  // k~: 128-row halves
            const uint32_t boff = qs * kQst + (kk >> 2) * kBox + (kk & 3) * 32;
            ptx::mma_f16_ss(tS, ptx::sw128_desc(aK + aoff, 16, 1024), ptx::sw128_desc(aQ + boff, 16, 1024), idS,
                            (p | kk) != 0);
          }
        ptx::mma_commit(s_full + st);
      };
      bool ok = ptx::mbar_wait(k_full, 0) && ptx::mbar_wait(q_full, 0);
      ptx::tc_fence_after();
      if (ok) issue_s(0);
      for (int i = 0; i < nqb && ok; ++i) {
        const int st = i & 1, qs = i % QS;
        const uint32_t ph = (i >> 1) & 1;
        if (i + 1 < nqb) {
          const int sn = (i + 1) & 1;
          ok = ptx::mbar_wait(q_full + (i + 1) % QS, ((i + 1) / QS) & 1);
          if (ok && i + 1 >= 2) ok = ptx::mbar_wait(s_free + sn, ((i - 1) >> 1) & 1);
          ptx::tc_fence_after();
          if (ok) issue_s(i + 1);
        }
        // query stage of block i-1 is free once P^T q (i-1) is done: refill it
        // with block i-1+QS (deferred so the issuer never waits on its last product)
        if (ok && i >= 1 && i - 1 + QS < nqb) {
          ok = ptx::mbar_wait(pq_done + ((i - 1) & 1), ((i - 1) >> 1) & 1);
          if (ok) load_q(i - 1 + QS, (i - 1) % QS);
        }
        ok = ok && ptx::mbar_wait(p_full + st, ph);
        ptx::tc_fence_after();
        if (ok) {
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int kk = 0; kk < kBlk / 16; ++kk)
              ptx::mma_f16_ss(tA, ptx::sw128_desc(aP + st * kPst + p * 2 * kBox + kk * 32, 16, 1024),
                              ptx::sw128_desc(aQ + qs * kQst + kk * 2048, kBox, 1024), idPQ, (i | p | kk) != 0);
          ptx::mma_commit(pq_done + st);
        }
      }
    }
  } else {
    const int r = 32 * (warp & 3) + lane;   // key tile row / TMEM lane
    const int hf = warp >> 2;               // query half of each block
    const int bid = 1 + (warp & 3);
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const int c1 = kb + r;
    const float hb = (c1 < g.b1k) ? hbuf[(long long)zrow * g.b1k_pad + c1] * kLog2e + kColShift : 0.f;
    const float2 sl2 = make_float2(g.sl2, g.sl2), hb2 = make_float2(hb, hb);
    float2 beta2 = make_float2(0.f, 0.f);
    bool ok = true;
    for (int i = 0; i < nqb; ++i) {
      const int st = i & 1, qs = i % QS;
      const uint32_t ph = (i >> 1) & 1;
      ok = ok && ptx::mbar_wait(s_full + st, ph) && ptx::mbar_wait(q_full + qs, (i / QS) & 1);
      ptx::tc_fence_after();
      uint32_t sr[32];
      ptx::tmem_ld32(tmem + st * kBlk + lane_off + hf * 32, sr);
      const float4* lv = reinterpret_cast<const float4*>(sL + qs * kBlk + hf * 32);
      const int valid = min(kBlk, g.b1q - i * kBlk) - hf * 32;
      ptx::tmem_wait_ld();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(s_free + st);
      uint32_t hi[16], lo[16];
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const float4 l4 = lv[e];
        float2 x0 = fma2(make_float2(__uint_as_float(sr[4 * e]), __uint_as_float(sr[4 * e + 1])), sl2, hb2);
        float2 x1 = fma2(make_float2(__uint_as_float(sr[4 * e + 2]), __uint_as_float(sr[4 * e + 3])), sl2, hb2);
        x0 = sub2(x0, make_float2(l4.x, l4.y));
        x1 = sub2(x1, make_float2(l4.z, l4.w));
        float2 p0 = make_float2(ptx::ex2(x0.x), ptx::ex2(x0.y));
        float2 p1 = make_float2(ptx::ex2(x1.x), ptx::ex2(x1.y));
        if (valid < 32) {  // only the last block of a ragged column
          if (4 * e >= valid) p0.x = 0.f;
          if (4 * e + 1 >= valid) p0.y = 0.f;
          if (4 * e + 2 >= valid) p1.x = 0.f;
          if (4 * e + 3 >= valid) p1.y = 0.f;
        }
        beta2 = add2(beta2, add2(p0, p1));
        split2<TQ>(p0, hi[2 * e], lo[2 * e]);
        split2<TQ>(p1, hi[2 * e + 1], lo[2 * e + 1]);
      }
      // P^T buffer st was last read by P^T q (i-2), which finished before S(i)
      const uint32_t prow = ptx::smem_u32(sP + st * kPst);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t off = ptx::sw128_offset(r, hf * 4 + c);
        sts128(prow + off, hi[4 * c], hi[4 * c + 1], hi[4 * c + 2], hi[4 * c + 3]);
        sts128(prow + 2 * kBox + off, lo[4 * c], lo[4 * c + 1], lo[4 * c + 2], lo[4 * c + 3]);
      }
      ptx::fence_proxy_async();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(p_full + st);
    }
    const float beta = beta2.x + beta2.y;
    sX[hf * kTile + r] = beta;
    named_bar(bid, 64);
    const float bt = beta + sX[(hf ^ 1) * kTile + r];
    const int last = nqb - 1;
    ok = ok && ptx::mbar_wait(pq_done + (last & 1), (last >> 1) & 1);
    ptx::tc_fence_after();
    const float inv = 1.f / bt;
    float* dst = qt + ((long long)zrow * g.b1k + (c1 < g.b1k ? c1 : 0)) * D + hf * (D / 2);
#pragma unroll
    for (int cc = 0; cc < D / 64; ++cc) {
      uint32_t o[32];
      ptx::tmem_ld32(tA + lane_off + hf * (D / 2) + cc * 32, o);
      ptx::tmem_wait_ld();
      if (c1 < g.b1k && ok) {
#pragma unroll
        for (int e = 0; e < 32; e += 4)
          *reinterpret_cast<float4*>(dst + cc * 32 + e) =
              make_float4(__uint_as_float(o[e]) * inv, __uint_as_float(o[e + 1]) * inv,
                          __uint_as_float(o[e + 2]) * inv, __uint_as_float(o[e + 3]) * inv);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 256);
}

template <int D>
constexpr size_t l_col_smem() {
  return 1024 + 2 * 2 * (D / 64) * kBox + 3 * (D / 64) * kBox + 2 * 2 * 2 * kBox + 3 * kBlk * 4 + 2 * kTile * 4 +
         16 * 8;
}

}  // namespace v2
}  // namespace monarch
