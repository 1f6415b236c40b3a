// The L step of a non-final iteration for small grids (at most 256 query
// tiles and 256 key tiles): the LSE pass and the column pass of one (head,
// position a2) in one CTA, with q, both k~ planes and h resident in shared
// memory for both passes.
//
//   phase A  lse[a1] = log2 sum_c1 2^(s q.k~_hi + h)        (rows of L)
//   phase B  q~[c1]  = sum_a1 L q / sum_a1 L,  L = 2^(s q.k~ + h - lse[a1])
//
// Phase A is the arithmetic of l_lse: S = q k~_hi^T (f16, N = 128 keys per
// MMA group), two column halves per row with their own running shift, merged
// at the end, one exponential pair in four on the FMA pipe; the row LSE
// goes to shared memory (and to the workspace).  Phase B is the arithmetic of
// l_col for the CTA's single item: S^T = k~_hi q^T + k~_lo q^T per 128-query
// block, L^T = 2^(x - lse + 15) split into f16 hi / lo over S^T in TMEM,
// acc += L^T_hi q + L^T_lo q, then q~ = acc / beta as hi / lo planes of the
// input type.  Every query block and key tile is loaded once, by TMA, at the
// start; the two passes share the operands (q is the A operand of phase A and
// the B operand of phase B, both K-major and, for L^T q, MN-major).  On the
// stacked geometry of the smallest grids (several positions of a head in one
// 128-row block) each row's window of keys, or each key row's window of
// queries, is its own position's (row_keys, col_queries).
//
// TMEM (512 columns).  Phase A: S(query tile t, key block b) at 256 t + 128 b,
// all four issued at once.  Phase B: key tile t at 256 t, S^T in [0, 128)
// (L^T written over it per 32-query chunk as [hi 16 | lo 16] columns), the
// accumulator in [128, 128 + D).  Phase B's first MMA is issued once every
// softmax warp has read phase A's scores (mbarrier a_done).
//
// Warps 0-15 are softmax warps: in phase A warp w takes query tile w / 8, lane
// quadrant w mod 4 and key half (w / 4) mod 2 of each block; in phase B key
// tile w / 8 and query half (w / 4) mod 2 of each block.  Warp 16 issues the
// MMAs and warp 17 the loads, each from one lane.
#pragma once

#include "tc_common.cuh"
#include "kernels_l.cuh"

namespace monarch {
namespace tc {

template <int D>
struct LsecolLayout {
  static constexpr int NH = D / 64;
  static constexpr uint32_t kKt = 2 * NH * 2 * kBox;   // k~ of one 128-row key tile: [plane][d half][2 x 64 rows]
  static constexpr uint32_t kQb = NH * 2 * kBox;       // one 128-query block: [d half][2 x 64 rows]
  static constexpr uint32_t oK = 0;
  static constexpr uint32_t oQ = oK + 2 * kKt;
  static constexpr uint32_t oH = oQ + 2 * kQb;          // h of 256 key tiles (f32)
  static constexpr uint32_t oL = oH + 2 * kTile * 4;    // lse of 256 queries (f32)
  static constexpr uint32_t oX = oL + 2 * kTile * 4;    // exchange: [tile][4][128] f32
  static constexpr uint32_t oBar = oX + 2 * 4 * kTile * 4;
  static constexpr uint32_t kBytes = oBar + 24 * 8;
  static constexpr size_t smem() { return kBytes > kExclusiveSmem ? kBytes : kExclusiveSmem; }
};

// grid (b2, BH), kThreads threads; b1q <= 256 and b1k <= 256.
template <typename TQ, int D>
__global__ void __launch_bounds__(kThreads, 1)
l_lsecol(const __grid_constant__ Maps maps, float* __restrict__ lse, TQ* __restrict__ qt, Geo g) {
  using Lay = LsecolLayout<D>;
  constexpr int NH = Lay::NH;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_misaligned(smem_raw)) return;
  uint8_t* sK = smem_raw + Lay::oK;
  uint8_t* sQ = smem_raw + Lay::oQ;
  float* sH = reinterpret_cast<float*>(smem_raw + Lay::oH);
  float* sL = reinterpret_cast<float*>(smem_raw + Lay::oL);
  float* sX = reinterpret_cast<float*>(smem_raw + Lay::oX);
  uint64_t* bar = reinterpret_cast<uint64_t*>(smem_raw + Lay::oBar);
  uint64_t* q_full = bar + 0;    // [query block]
  uint64_t* k_full = bar + 2;    // [key tile]: k~ planes and h
  uint64_t* s_full = bar + 4;    // phase A: [query tile][key block]
  uint64_t* a_done = bar + 8;    // phase A's scores are read (16 warps)
  uint64_t* t_full = bar + 9;    // phase B: S^T of [key tile]
  uint64_t* p_full = bar + 11;   // phase B: L^T of [key tile] in TMEM
  uint64_t* o_done = bar + 13;   // phase B: accumulator of [key tile] complete
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bar + 15);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int a2 = blockIdx.x, bh = blockIdx.y;
  const int zrow = bh * g.b2 + a2;
  const int plane_rows = g.BH * g.b2;
  const int nq = (g.b1q + kTile - 1) / kTile;   // query tiles = query blocks (1 or 2)
  const int nk = (g.b1k + kTile - 1) / kTile;   // key tiles = key blocks (1 or 2)

  if (tid == 0) {
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(q_full + i, 1);
      ptx::mbar_init(k_full + i, 1);
      ptx::mbar_init(t_full + i, 1);
      ptx::mbar_init(p_full + i, 8);
      ptx::mbar_init(o_done + i, 1);
    }
    for (int i = 0; i < 4; ++i) ptx::mbar_init(s_full + i, 1);
    ptx::mbar_init(a_done, kSoftWarps);
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(sTmem, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // dependents may start once every CTA of this grid holds its TMEM
  ptx::griddep_launch();
  ptx::griddep_wait();   // set-up done: global data of the previous kernel from here on
  const uint32_t tmem = *sTmem;

  if (warp == kLoadWarp) {
    if (lane == 0) {
      // ------------------------------------------------ every operand, once
      ptx::prefetch_tmap(&maps.kt);
      ptx::prefetch_tmap(&maps.qb);
      for (int t = 0; t < nk; ++t) {
        ptx::mbar_expect_tx(k_full + t, Lay::kKt + kTile * 4);
        for (int p = 0; p < 2; ++p)
          for (int hf = 0; hf < NH; ++hf)
            for (int rh = 0; rh < 2; ++rh)
              ptx::tma_load_3d(sK + t * Lay::kKt + (p * NH + hf) * 2 * kBox + rh * kBox, &maps.kt, k_full + t,
                               hf * 64, t * kTile + rh * kBlk, p * plane_rows + zrow);
        for (int rh = 0; rh < 2; ++rh)
          tma_load_2d(sH + t * kTile + rh * kBlk, &maps.h, k_full + t, t * kTile + rh * kBlk, zrow);
      }
      for (int i = 0; i < nq; ++i) {
        ptx::mbar_expect_tx(q_full + i, Lay::kQb);
        for (int hf = 0; hf < NH; ++hf)
          for (int rh = 0; rh < 2; ++rh)
            ptx::tma_load_3d(sQ + i * Lay::kQb + hf * 2 * kBox + rh * kBox, &maps.qb, q_full + i, hf * 64,
                             i * kTile + rh * kBlk, zrow);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      // ----------------------------------------------------------- MMA issuer
      const uint32_t aQ = ptx::smem_u32(sQ), aK = ptx::smem_u32(sK);
      bool ok = true;
      // phase A: S(t, b) = q_t k~_hi(b)^T, both operands K-major
      {
        constexpr uint32_t idS = ptx::idesc_f16(128, kTile, 0, 0, 0);
        for (int b = 0; b < nk && ok; ++b) {
          ok = ptx::mbar_wait(k_full + b, 0);
          for (int t = 0; t < nq && ok; ++t) {
            ok = ptx::mbar_wait(q_full + t, 0);
            ptx::tc_fence_after();
            if (!ok) break;
            const uint64_t a0 = ptx::sw128_desc(aQ + t * Lay::kQb, 16, 1024);
            const uint64_t b0 = ptx::sw128_desc(aK + b * Lay::kKt, 16, 1024);
#pragma unroll
            for (int hf = 0; hf < NH; ++hf)
#pragma unroll
              for (int k4 = 0; k4 < 4; ++k4)
                ptx::mma_f16_ss(tmem + 256 * t + 128 * b, a0 + ((hf * 2 * kBox + k4 * 32) >> 4),
                                b0 + ((hf * 2 * kBox + k4 * 32) >> 4), idS, (hf | k4) != 0);
            ptx::mma_commit(s_full + 2 * t + b);
          }
        }
      }
      // phase B: S^T(t) = k~(t) q_i^T over both planes; acc(t) += L^T(t) q_i
      constexpr uint32_t idT = ptx::idesc_f16(128, kTile, 0, 0, 0);
      constexpr uint32_t idPQ = ptx::idesc_f16(128, D, 0, 0, 1);
      auto issue_t = [&](int t, int i) {
        const uint64_t a0 = ptx::sw128_desc(aK + t * Lay::kKt, 16, 1024);
        const uint64_t b0 = ptx::sw128_desc(aQ + i * Lay::kQb, 16, 1024);
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
          for (int hf = 0; hf < NH; ++hf)
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
              ptx::mma_f16_ss(tmem + 256 * t, a0 + (((p * NH + hf) * 2 * kBox + k4 * 32) >> 4),
                              b0 + ((hf * 2 * kBox + k4 * 32) >> 4), idT, (p | hf | k4) != 0);
        ptx::mma_commit(t_full + t);
      };
      ok = ok && ptx::mbar_wait(a_done, 0);
      ptx::tc_fence_after();
      if (ok)
        for (int t = 0; t < nk; ++t) issue_t(t, 0);
      for (int i = 0; i < nq && ok; ++i) {
        const uint64_t q0 = ptx::sw128_desc(aQ + i * Lay::kQb, 2 * kBox, 1024);
        for (int t = 0; t < nk && ok; ++t) {
          ok = ptx::mbar_wait(p_full + t, i & 1);
          ptx::tc_fence_after();
          if (!ok) break;
          const uint32_t tp = tmem + 256 * t;
#pragma unroll
          for (int p = 0; p < 2; ++p)
#pragma unroll
            for (int kk = 0; kk < kTile / 16; ++kk)
              ptx::mma_f16_ts(tp + 128, tp + (kk >> 1) * 32 + p * 16 + (kk & 1) * 8, q0 + ((kk * 2048) >> 4), idPQ,
                              (i | p | kk) != 0);
          // S^T(t, i + 1) overwrites L^T(t, i): the product above runs first
          if (i + 1 < nq) issue_t(t, i + 1);
          else ptx::mma_commit(o_done + t);
        }
      }
    }
  } else {
    const int t = warp >> 3;                 // phase A: query tile; phase B: key tile
    const int hf = (warp >> 2) & 1;          // column half of a block
    const int r = 32 * (warp & 3) + lane;    // TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const float2 sl2 = make_float2(g.sl2, g.sl2);
    float* xs = sX + t * 4 * kTile;          // this tile's exchange area
    bool ok = true;
    // ------------------------------------------------- phase A: row LSE
    if (t < nq) {
      const int a1 = t * kTile + r;
      int klo, khi;   // visible key rows [klo, khi)
      row_keys(g, min(a1, g.b1q - 1), klo, khi);
      float m = -INFINITY, l = 0.f;
      for (int b = 0; b < nk; ++b) {
        ok = ok && ptx::mbar_wait(s_full + 2 * t + b, 0) && ptx::mbar_wait(k_full + b, 0);
        ptx::tc_fence_after();
        const float4* hv = reinterpret_cast<const float4*>(sH + b * kTile + 64 * hf);
#pragma unroll
        for (int sb = 0; sb < 2; ++sb) {   // 32 keys at a time: an online update each
          uint32_t s[32];
          ptx::tmem_ld32(tmem + 256 * t + 128 * b + lane_off + 64 * hf + 32 * sb, s);
          ptx::tmem_wait_ld();
          float2 x[16];
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 h4 = hv[8 * sb + i];
            x[2 * i] = fma2(make_float2(__uint_as_float(s[4 * i]), __uint_as_float(s[4 * i + 1])), sl2,
                            make_float2(h4.x, h4.y));
            x[2 * i + 1] = fma2(make_float2(__uint_as_float(s[4 * i + 2]), __uint_as_float(s[4 * i + 3])), sl2,
                                make_float2(h4.z, h4.w));
          }
          // these 32 keys' visible part is [vlo, vhi)
          const int kb0 = b * kTile + 64 * hf + 32 * sb;
          const int vlo = klo - kb0, vhi = khi - kb0;
          if (vlo > 0 || vhi < 32) {
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              if (2 * i < vlo || 2 * i >= vhi) x[i].x = -INFINITY;
              if (2 * i + 1 < vlo || 2 * i + 1 >= vhi) x[i].y = -INFINITY;
            }
          }
          float mb = -INFINITY;
#pragma unroll
          for (int i = 0; i < 16; ++i) mb = fmaxf(mb, fmaxf(x[i].x, x[i].y));
          const bool move = mb > m + kLazyRescale;
          const float mn = move ? mb : m;
          const float corr = (mn == m) ? 1.f : ptx::ex2(m - mn);
          const float nmv = (mn == -INFINITY) ? 0.f : -mn;
          const float2 nm = make_float2(nmv, nmv);
          float2 acc2 = make_float2(0.f, 0.f);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 d = add2(x[i], nm);
            // one pair in four on the FMA pipe, the rest on the MUFU unit
            const float2 e = ((i & 3) == 3) ? ex2_fma2(d) : make_float2(ptx::ex2(d.x), ptx::ex2(d.y));
            acc2 = add2(acc2, e);
          }
          l = fmaf(l, corr, acc2.x + acc2.y);
          m = mn;
        }
      }
      // merge the halves: (m, l) of each, shifts may differ
      xs[hf * kTile + r] = m;
      xs[2 * kTile + hf * kTile + r] = l;
      ptx::named_bar(1 + t, kTileThreads);
      if (hf == 0) {
        const float mo = xs[kTile + r], lo = xs[3 * kTile + r];
        const float M = fmaxf(m, mo);
        const float L = (m == -INFINITY ? 0.f : l * ptx::ex2(m - M)) + (mo == -INFINITY ? 0.f : lo * ptx::ex2(mo - M));
        const float v = M + log2f(L);
        sL[a1] = v;
        if (a1 < g.b1q) lse[(long long)zrow * g.b1q_pad + a1] = v;
      }
    }
    // phase A's scores are read and the row LSE is in shared memory
    ptx::tc_fence_before();
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(a_done);
    // ------------------------------------------------- phase B: q~ per key tile
    if (t < nk) {
      // this thread reads h (loaded with the key tile) and the row LSE (stored
      // by other warps before a_done): wait on both barriers itself
      ok = ok && ptx::mbar_wait(k_full + t, 0) && ptx::mbar_wait(a_done, 0);
      const int c1 = t * kTile + r;
      int qlo, qhi;   // the query rows that see this key row: [qlo, qhi)
      col_queries(g, min(c1, g.b1k - 1), qlo, qhi);
      const float hb = (c1 < g.b1k) ? sH[c1] + kColShift : 0.f;
      const float2 hb2 = make_float2(hb, hb);
      float2 beta2 = make_float2(0.f, 0.f);
      for (int i = 0; i < nq; ++i) {
        ok = ok && ptx::mbar_wait(t_full + t, i & 1);
        ptx::tc_fence_after();
        const int valid = min(kTile, qhi - i * kTile);   // queries of this block at or past it are masked
        const int vlo = qlo - i * kTile;                   // and those below this
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {      // 32 queries at a time
          const int cb = 64 * hf + 32 * hh;   // first S^T column (query) of this chunk
          uint32_t sr[32];
          ptx::tmem_ld32(tmem + 256 * t + lane_off + cb, sr);
          const float4* lv = reinterpret_cast<const float4*>(sL + i * kTile + cb);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int q8 = 0; q8 < 2; ++q8) {    // 16 queries: 8 packed columns per plane
            uint32_t hi[8], lo[8];
#pragma unroll
            for (int e4 = 0; e4 < 4; ++e4) {
              const int e = 4 * q8 + e4;
              const float4 l4 = lv[e];
              float2 x0 = fma2(make_float2(__uint_as_float(sr[4 * e]), __uint_as_float(sr[4 * e + 1])), sl2, hb2);
              float2 x1 =
                  fma2(make_float2(__uint_as_float(sr[4 * e + 2]), __uint_as_float(sr[4 * e + 3])), sl2, hb2);
              x0 = sub2(x0, make_float2(l4.x, l4.y));
              x1 = sub2(x1, make_float2(l4.z, l4.w));
              float2 p0 = make_float2(ptx::ex2(x0.x), ptx::ex2(x0.y));
              float2 p1 = make_float2(ptx::ex2(x1.x), ptx::ex2(x1.y));
              if (valid < kTile || vlo > 0) {  // a ragged last block, or queries hidden by the mask
                const int q0 = cb + 4 * e;
                if (q0 >= valid || q0 < vlo) p0.x = 0.f;
                if (q0 + 1 >= valid || q0 + 1 < vlo) p0.y = 0.f;
                if (q0 + 2 >= valid || q0 + 2 < vlo) p1.x = 0.f;
                if (q0 + 3 >= valid || q0 + 3 < vlo) p1.y = 0.f;
              }
              beta2 = add2(beta2, add2(p0, p1));
              split2<__half>(p0, hi[2 * e4], lo[2 * e4]);
              split2<__half>(p1, hi[2 * e4 + 1], lo[2 * e4 + 1]);
            }
            // L^T of these queries over the chunk's own S^T columns (all read
            // already): hi in [cb, cb + 16), lo in [cb + 16, cb + 32)
            ptx::tmem_st8(tmem + 256 * t + lane_off + cb + 8 * q8, hi);
            ptx::tmem_st8(tmem + 256 * t + lane_off + cb + 16 + 8 * q8, lo);
          }
        }
        ptx::tmem_wait_st();
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(p_full + t);
      }
      // beta = the two halves' column sums
      ptx::named_bar(1 + t, kTileThreads);   // phase A's reads of this exchange area are done
      xs[hf * kTile + r] = beta2.x + beta2.y;
      ptx::named_bar(1 + t, kTileThreads);
      const float beta = beta2.x + beta2.y + xs[(hf ^ 1) * kTile + r];
      ok = ok && ptx::mbar_wait(o_done + t, 0);
      ptx::tc_fence_after();
      // beta = 0: every query gives this key tile a weight below 2^-141 (all
      // flushed to zero), and q~ = 0 replaces 0/0
      const float inv = beta > 0.f ? 1.f / beta : 0.f;
      const float2 inv2 = make_float2(inv, inv);
      const long long plane = (long long)g.BH * g.b2 * g.b1k * D;
      TQ* dst = qt + ((long long)zrow * g.b1k + (c1 < g.b1k ? c1 : 0)) * D + hf * (D / 2);
#pragma unroll 1
      for (int cc = 0; cc < D / 32; ++cc) {   // 16 columns at a time
        uint32_t o[16];
        ptx::tmem_ld16(tmem + 256 * t + 128 + lane_off + hf * (D / 2) + cc * 16, o);
        ptx::tmem_wait_ld();
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int e = 0; e < 8; ++e)
          split2<TQ>(mul2(make_float2(__uint_as_float(o[2 * e]), __uint_as_float(o[2 * e + 1])), inv2), hi[e], lo[e]);
        if (c1 < g.b1k && ok) {   // 32 bytes a store (rows are D elements, planes 256-byte aligned)
          ptx::st_global_v8(dst + cc * 16, hi);
          ptx::st_global_v8(dst + plane + cc * 16, lo);
        }
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 512);
}

}  // namespace tc
}  // namespace monarch
