// tcgen05 kernels of the L step for bf16 / f16 inputs (row pass, output pass,
// column pass).
//
// A CTA owns two 128-row tiles (A and B) of one (head, position a2) problem.
// Warps 0-7 run the softmax of tile A and warps 8-15 that of tile B.  Thread
// r of a tile's warps w and w + 4 owns row r of the tile (TMEM lane r, lane
// quadrant w mod 4); warp w takes the first half of the block's columns and
// warp w + 4 the second, so one tile's softmax finishes in about half the time
// it takes a single warp per row.  Warp 16 issues the MMAs and warp 17 the
// TMA loads, each from one lane.  The issuer alternates between the tiles, so
// one tile's MMAs run while the other's softmax works.
//
// Every MMA is N >= 128 wide: a single thread issues about one tcgen05.mma per
// 60 cycles, so an N = 64 instruction (32 cycles of math) would leave the
// tensor pipe half idle.
//   row pass     S = q [k~_hi ; k~_lo]^T   (N = 128: the two planes of a
//                64-key block side by side; the softmax adds the halves)
//   output pass  O += P z_hi + P z_lo      (A = P in TMEM over S, N = d)
//   column pass  S^T = k~_hi q^T + k~_lo q^T   (128-query blocks, N = 128)
//                acc += P^T_hi q + P^T_lo q     (A = P^T in TMEM over S^T, N = d)
// A new score tile is issued into TMEM columns that hold the previous P only
// after the MMA consuming that P: tcgen05 MMAs of a thread run in issue order
// and a commit arrives when every earlier MMA is complete, so "S(j+1) done"
// also means "P z (j) done".
//
// The two column halves of a row share one running shift in the output pass:
// they exchange block maxima through shared memory at a per-tile named
// barrier, which also orders every read of S before the P stores over it.  The
// LSE pass keeps a shift per half and merges the halves at the end; there the
// exponentials (one per score, as many as the score MMA has columns) are split
// between the MUFU unit and an FMA-pipe polynomial.
//
// Precision: k~ and z as hi/lo planes, q exact, L split into hi/lo planes in
// the column pass, P single f16 with the rounded values summed, fp32
// statistics; h arrives in bits (base-2 entropy).
#pragma once

#include "tc_common.cuh"

namespace monarch {
namespace tc {

constexpr int kSoftWarps = 16;  // 8 per tile: 4 lane quadrants x 2 column halves
constexpr int kThreads = 32 * (kSoftWarps + 2);   // + MMA warp + TMA warp
constexpr int kMmaWarp = kSoftWarps;
constexpr int kLoadWarp = kSoftWarps + 1;
constexpr int kTileThreads = 256;                  // softmax threads of one tile

// Exchange area of one tile between its two column halves (bytes):
//   output pass   bf16 block maxima [parity][half][128], then f32 row sums [half][128]
//   LSE pass      f32 [m, l][half][128]
//   column pass   f32 column sums [half][128]
template <int KIND> constexpr int xchg_tile_bytes() { return KIND == 1 ? 1024 : (KIND == 0 ? 2048 : 1024); }

constexpr int kKS = 3;          // k~ / h stages (row passes)
constexpr int kQS = 2;          // query / lse stages (column pass)
constexpr int kQBlk = 128;      // queries per column-pass block

// Both kernels allocate all 512 TMEM columns, so their shared-memory
// requests are at least 120 KB: one CTA per SM, none waits in tcgen05.alloc.
constexpr size_t kExclusiveSmem = 120 * 1024;

template <int D, bool OUT>
constexpr size_t row_smem() {
  constexpr int NH = D / 64;
  constexpr size_t need = (size_t)2 * NH * 2 * kBox /* q */ + (size_t)kKS * 2 * NH * kBox /* k~ */ +
                          (OUT ? (size_t)2 * 2 * NH * kBox : 0) /* z */ + kKS * kBlk * 4 +
                          2 * xchg_tile_bytes<OUT ? 1 : 0>() + 32 * 8;
  return need > kExclusiveSmem ? need : kExclusiveSmem;
}

// ===========================================================================
// Row pass over 64-key blocks for one (head, position a2, 256 query rows).
//   OUT:  out[token(a1,a2)] = sum_c1 L z     (inverse permutation in the store);
//         with LSE_OUT also lse[a1] (base 2) of the same scores
//   !OUT: lse[a1] = log2 sum_c1 2^(s q.k~ + h)
// TMEM, tile t at column 256 t.  OUT: S [0, 128) (q.k~_hi in [0, 64), q.k~_lo
// in [64, 128); P over [0, 32)), O [128, 128 + D).  !OUT: S buffers [0, 128),
// [128, 256).
// One row-pass item (query tiles a1_base, a1_base + 128 of head bh,
// position a2) run by all kThreads threads of the CTA on `smem_raw`
// (row_smem<D, OUT>() bytes, 1024-byte aligned) and 512 TMEM columns at
// `tmem`.  ready != nullptr: the load warp waits (bounded, acquire) for
// *ready >= ready_need before its first load, instead of the item waiting for
// the previous grid, so it may overlap the R-step items that produce its
// inputs (in the same grid or in the kernel before).
template <typename TQ, typename TO, int D, bool OUT, bool LSE_OUT>
__device__ __forceinline__ void l_row_item(TO* __restrict__ out, const Maps& maps, float* __restrict__ lse,
                                           const Geo& g, int a1_base, int a2, int bh, uint8_t* smem_raw,
                                           uint32_t tmem, const int* ready, int ready_need) {
  constexpr int NH = D / 64;
  constexpr uint32_t kQt = NH * 2 * kBox;    // q of one tile (128 rows)
  constexpr uint32_t kKst = 2 * NH * kBox;   // k~ hi+lo, 64 rows: [d half][plane][64 rows]
  constexpr uint32_t kZst = 2 * NH * kBox;   // z hi+lo, 64 rows:  [plane][d half][64 rows]
  uint8_t* sQ = smem_raw;                                             // [2 tiles]
  uint8_t* sK = sQ + 2 * kQt;                                         // [kKS]
  uint8_t* sZ = sK + kKS * kKst;                                      // [2] (OUT)
  float* sH = reinterpret_cast<float*>(sZ + (OUT ? 2 * kZst : 0));    // [kKS][64]
  constexpr int kXt = xchg_tile_bytes<OUT ? 1 : 0>();
  uint8_t* sX = reinterpret_cast<uint8_t*>(sH + kKS * kBlk);          // [tile][kXt bytes]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sX + 2 * kXt);
  uint64_t* q_full = bar + 0;
  uint64_t* k_full = bar + 1;    // [kKS]
  uint64_t* k_free = bar + 4;    // [kKS]
  uint64_t* z_full = bar + 7;    // [2]
  uint64_t* z_free = bar + 9;    // [2]
  uint64_t* s_full = bar + 11;   // [tile][buf]
  uint64_t* s_free = bar + 15;   // [tile][buf]   (!OUT)
  uint64_t* p_full = bar + 19;   // [tile]        (OUT)
  uint64_t* o_done = bar + 21;   // [tile]        (OUT)
  // bar + 23: the TMEM slot of a one-item kernel (row_tmem_slot)

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int zrow = bh * g.b2 + a2;
  const int plane_rows = g.BH * g.b2;
  // key blocks any row of this CTA sees (all of them without a causal mask);
  // the last row's window ends highest
  int klast_lo, kmax;
  row_keys(g, min(a1_base + 2 * kTile, g.b1q) - 1, klast_lo, kmax);
  const int nkb = (kmax + kBlk - 1) / kBlk;
  const int ntiles = (g.b1q - a1_base > kTile) ? 2 : 1;

  if (tid == 0) {
    ptx::mbar_init(q_full, 1);
    for (int i = 0; i < kKS; ++i) {
      ptx::mbar_init(k_full + i, 1);
      ptx::mbar_init(k_free + i, 8 * ntiles);
    }
    for (int i = 0; i < 2; ++i) {
      ptx::mbar_init(z_full + i, 1);
      ptx::mbar_init(z_free + i, 1);
    }
    for (int t = 0; t < 2; ++t) {
      ptx::mbar_init(p_full + t, 8);
      ptx::mbar_init(o_done + t, 1);
      for (int b = 0; b < 2; ++b) {
        ptx::mbar_init(s_full + 2 * t + b, 1);
        ptx::mbar_init(s_free + 2 * t + b, 8);
      }
    }
    ptx::fence_mbar_init();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // set-up done: global data of the previous kernel from here on (or of the
  // items counted in *ready, which the load warp waits for)
  if (!ready) ptx::griddep_wait();
  auto tS = [&](int t, int b) { return tmem + 256 * t + 128 * b; };
  auto tO = [&](int t) { return tmem + 256 * t + 128; };

  if (warp == kLoadWarp) {
    if (lane == 0) {
      // --------------------------------------------------------- TMA producer
      ptx::prefetch_tmap(&maps.kt);
      if (ready) {
        // the R-step items of this head are done: their TMA and h stores are
        // visible (acquire), and this thread's loads below come after it
        ptx::wait_count(ready, ready_need);
        ptx::fence_proxy_async_global();
      }
      ptx::mbar_expect_tx(q_full, 2 * kQt);
      for (int t = 0; t < 2; ++t)
        for (int hf = 0; hf < NH; ++hf)
          for (int rh = 0; rh < 2; ++rh)
            ptx::tma_load_3d(sQ + t * kQt + hf * 2 * kBox + rh * kBox, &maps.qb, q_full, hf * 64,
                             a1_base + t * kTile + rh * kBlk, zrow);
      bool ok = true;
      for (int blk = 0; blk < nkb && ok; ++blk) {
        const int ks = blk % kKS;
        if (blk >= kKS) ok = ptx::mbar_wait(k_free + ks, ((blk / kKS) - 1) & 1);
        if (!ok) break;
        ptx::mbar_expect_tx(k_full + ks, kKst + kBlk * 4);
        for (int hf = 0; hf < NH; ++hf)
          for (int p = 0; p < 2; ++p)
            ptx::tma_load_3d(sK + ks * kKst + (hf * 2 + p) * kBox, &maps.kt, k_full + ks, hf * 64, blk * kBlk,
                             p * plane_rows + zrow);
        tma_load_2d(sH + ks * kBlk, &maps.h, k_full + ks, blk * kBlk, zrow);
        if constexpr (OUT) {
          const int zs = blk & 1;
          if (blk >= 2) ok = ptx::mbar_wait(z_free + zs, ((blk >> 1) - 1) & 1);
          if (!ok) break;
          ptx::mbar_expect_tx(z_full + zs, kZst);
          for (int p = 0; p < 2; ++p)
            for (int hf = 0; hf < NH; ++hf)
              ptx::tma_load_3d(sZ + zs * kZst + (p * NH + hf) * kBox, &maps.z, z_full + zs, hf * 64, blk * kBlk,
                               p * plane_rows + zrow);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      // ----------------------------------------------------------- MMA issuer
      constexpr uint32_t idS = ptx::idesc_f16(128, 2 * kBlk, TcType<TQ>::kBf16, 0, 0);
      constexpr uint32_t idPV = ptx::idesc_f16(128, D, 0, 0, 1);
      const uint32_t aQ = ptx::smem_u32(sQ), aK = ptx::smem_u32(sK), aZ = ptx::smem_u32(sZ);
      // S(t, blk) into buffer b: A = q tile (K-major), B = [k~_hi ; k~_lo] of
      // one d half (128 rows).  Descriptors are built once; a byte offset adds
      // (offset >> 4) to the start-address field.
      auto issue_s = [&](int t, int blk, int b) {
        const uint64_t a0 = ptx::sw128_desc(aQ + t * kQt, 16, 1024);
        const uint64_t b0 = ptx::sw128_desc(aK + (blk % kKS) * kKst, 16, 1024);
        const uint32_t td = tS(t, b);
#pragma unroll
        for (int hf = 0; hf < NH; ++hf)
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            ptx::mma_f16_ss(td, a0 + ((hf * 2 * kBox + k4 * 32) >> 4), b0 + ((hf * 2 * kBox + k4 * 32) >> 4), idS,
                            (hf | k4) != 0);
        ptx::mma_commit(s_full + 2 * t + b);
      };
      bool ok = ptx::mbar_wait(q_full, 0) && ptx::mbar_wait(k_full, 0);
      ptx::tc_fence_after();
      if (ok) {
        for (int t = 0; t < ntiles; ++t) issue_s(t, 0, 0);
        if (!OUT && nkb > 1) {
          ok = ptx::mbar_wait(k_full + 1, 0);
          ptx::tc_fence_after();
          if (ok)
            for (int t = 0; t < ntiles; ++t) issue_s(t, 1, 1);
        }
      }
      for (int j = 0; j < nkb && ok; ++j) {
        if constexpr (OUT) {
          ok = ptx::mbar_wait(z_full + (j & 1), (j >> 1) & 1);
          const uint64_t z0 = ptx::sw128_desc(aZ + (j & 1) * kZst, kBox, 1024);
          for (int t = 0; t < ntiles && ok; ++t) {
            ok = ptx::mbar_wait(p_full + t, j & 1);
            ptx::tc_fence_after();
            if (!ok) break;
            const uint32_t tp = tS(t, 0);
#pragma unroll
            for (int p = 0; p < 2; ++p)
#pragma unroll
              for (int kk = 0; kk < kBlk / 16; ++kk)
                ptx::mma_f16_ts(tO(t), tp + kk * 8, z0 + ((p * NH * kBox + kk * 2048) >> 4), idPV,
                                (j | p | kk) != 0);
            if (t == ntiles - 1) ptx::mma_commit(z_free + (j & 1));
            if (j + 1 < nkb) {
              // S(t, j+1) overwrites P(t, j): the P z product above runs first
              ok = ptx::mbar_wait(k_full + (j + 1) % kKS, ((j + 1) / kKS) & 1);
              ptx::tc_fence_after();
              if (ok) issue_s(t, j + 1, 0);
            } else {
              ptx::mma_commit(o_done + t);
            }
          }
        } else {
          const int b = j & 1;
          const uint32_t ph = (j >> 1) & 1;
          for (int t = 0; t < ntiles && ok; ++t) {
            ok = ptx::mbar_wait(s_free + 2 * t + b, ph);
            if (ok && j + 2 < nkb) {
              ok = ptx::mbar_wait(k_full + (j + 2) % kKS, ((j + 2) / kKS) & 1);
              ptx::tc_fence_after();
              if (ok) issue_s(t, j + 2, b);
            }
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------- softmax warps
    const int t = warp >> 3;                 // tile
    const int hf = (warp >> 2) & 1;          // column half: keys 32 hf .. 32 hf + 31 of a block
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const int a1 = a1_base + t * kTile + r;
    int klo, khi;   // visible key rows [klo, khi)
    row_keys(g, min(a1, g.b1q - 1), klo, khi);
    if (t < ntiles) {
      float m = -INFINITY, l = 0.f;
      float lx = 0.f;   // LSE_OUT: the row sum of the unrounded exponentials
      bool ok = true;
      const float2 sl2 = make_float2(g.sl2, g.sl2);
      for (int j = 0; j < nkb; ++j) {
        const int ks = j % kKS;
        const int b = OUT ? 0 : (j & 1);
        const uint32_t ph = OUT ? (j & 1) : ((j >> 1) & 1);
        // after a timed-out wait the loop keeps its shape (and its named
        // barriers) but skips waits
        ok = ok && ptx::mbar_wait(s_full + 2 * t + b, ph) && ptx::mbar_wait(k_full + ks, (j / kKS) & 1);
        ptx::tc_fence_after();
        const float4* hv = reinterpret_cast<const float4*>(sH + ks * kBlk + 32 * hf);
        float2 x[16];   // x[i] = keys 32 hf + 2i, 32 hf + 2i + 1
#pragma unroll
        for (int hh = 0; hh < 2; ++hh) {  // 16 keys at a time
          uint32_t shi[16], slo[16];
          ptx::tmem_ld16(tS(t, b) + lane_off + 32 * hf + 16 * hh, shi);
          ptx::tmem_ld16(tS(t, b) + lane_off + 64 + 32 * hf + 16 * hh, slo);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            const float4 h4 = hv[4 * hh + i];
            const float2 s0 = add2(make_float2(__uint_as_float(shi[4 * i]), __uint_as_float(shi[4 * i + 1])),
                                   make_float2(__uint_as_float(slo[4 * i]), __uint_as_float(slo[4 * i + 1])));
            const float2 s1 = add2(make_float2(__uint_as_float(shi[4 * i + 2]), __uint_as_float(shi[4 * i + 3])),
                                   make_float2(__uint_as_float(slo[4 * i + 2]), __uint_as_float(slo[4 * i + 3])));
            x[8 * hh + 2 * i] = fma2(s0, sl2, make_float2(h4.x, h4.y));
            x[8 * hh + 2 * i + 1] = fma2(s1, sl2, make_float2(h4.z, h4.w));
          }
        }
        // S and h of this block are read: release the k~/h stage
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          ptx::mbar_arrive(k_free + ks);
          if (!OUT) ptx::mbar_arrive(s_free + 2 * t + b);
        }
        // this half's visible keys are [vlo, vhi) of its 32
        const int vlo = klo - (j * kBlk + 32 * hf), vhi = khi - (j * kBlk + 32 * hf);
        if (vlo > 0 || vhi < 32) {  // a ragged row end, or stacked positions
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            if (2 * i < vlo || 2 * i >= vhi) x[i].x = -INFINITY;
            if (2 * i + 1 < vlo || 2 * i + 1 >= vhi) x[i].y = -INFINITY;
          }
        }
        float mb = -INFINITY;
#pragma unroll
        for (int i = 0; i < 16; ++i) mb = fmaxf(mb, fmaxf(x[i].x, x[i].y));
        if constexpr (OUT) {
          // one shift per row: merge the two halves' block maxima.  The
          // barrier also orders every S read of this tile before the P stores.
          // Both halves use the maxima rounded up to bf16, so they agree on
          // the shift; rounding up keeps every exponent <= 8.
          __nv_bfloat16* xs = reinterpret_cast<__nv_bfloat16*>(sX + t * kXt) + (j & 1) * 2 * kTile;
          const __nv_bfloat16 mine = __float2bfloat16_ru(mb);
          xs[hf * kTile + r] = mine;
          ptx::tc_fence_before();
          ptx::named_bar(1 + t, kTileThreads);
          ptx::tc_fence_after();
          mb = fmaxf(__bfloat162float(mine), __bfloat162float(xs[(hf ^ 1) * kTile + r]));
        }
        // the running shift moves only when the max grows by more than 2^8
        const bool move = mb > m + kLazyRescale;
        const float mn = move ? mb : m;
        const float corr = (mn == m) ? 1.f : ptx::ex2(m - mn);
        const float nmv = (mn == -INFINITY) ? 0.f : -mn;   // a half with no key yet
        const float2 nm = make_float2(nmv, nmv);
        float2 acc2 = make_float2(0.f, 0.f);
        if constexpr (OUT) {
          // S(t, j) is complete, hence so is P z (j-1): O may be rescaled.
          // The decision is the same in both halves; each scales its half of O.
          if (j > 0 && __any_sync(0xffffffffu, move)) {
#pragma unroll
            for (int cc = 0; cc < D / 32; ++cc) {
              uint32_t o[16];
              ptx::tmem_ld16(tO(t) + lane_off + hf * (D / 2) + cc * 16, o);
              ptx::tmem_wait_ld();
#pragma unroll
              for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * corr);
              ptx::tmem_st16(tO(t) + lane_off + hf * (D / 2) + cc * 16, o);
            }
          }
          uint32_t pk[16];
          float2 accx = make_float2(0.f, 0.f);
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 d = add2(x[i], nm);
            const float2 e = make_float2(ptx::ex2(d.x), ptx::ex2(d.y));
            const __half2 hp = __floats2half2_rn(e.x, e.y);
            acc2 = add2(acc2, __half22float2(hp));
            if constexpr (LSE_OUT) accx = add2(accx, e);
            pk[i] = *reinterpret_cast<const uint32_t*>(&hp);
          }
          if constexpr (LSE_OUT) lx = fmaf(lx, corr, accx.x + accx.y);
          // P: keys 2c, 2c + 1 in column c of the first 32 columns of S
          ptx::tmem_st16(tS(t, 0) + lane_off + 16 * hf, pk);
          ptx::tmem_wait_st();
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(p_full + t);
        } else {
#pragma unroll
          for (int i = 0; i < 16; ++i) {
            const float2 d = add2(x[i], nm);
            // one pair in four on the FMA pipe, the rest on the MUFU unit
            const float2 e = ((i & 3) == 3) ? ex2_fma2(d) : make_float2(ptx::ex2(d.x), ptx::ex2(d.y));
            acc2 = add2(acc2, e);
          }
        }
        l = fmaf(l, corr, acc2.x + acc2.y);
        m = mn;
      }
      if constexpr (OUT) {
        // row sum = the two halves' sums (same shift); the first barrier ends
        // every read of the block maxima that share these bytes
        float* xs = reinterpret_cast<float*>(sX + t * kXt);
        ptx::named_bar(1 + t, kTileThreads);
        xs[hf * kTile + r] = l;
        ptx::named_bar(1 + t, kTileThreads);
        const float lt = l + xs[(hf ^ 1) * kTile + r];
        if constexpr (LSE_OUT) {
          // the row's base-2 log-sum-exp of the same scores, from the
          // unrounded exponentials (the backward's P sums to 1 with it)
          ptx::named_bar(1 + t, kTileThreads);
          xs[hf * kTile + r] = lx;
          ptx::named_bar(1 + t, kTileThreads);
          if (hf == 0 && a1 < g.b1q) lse[(long long)zrow * g.b1q_pad + a1] = m + log2f(lx + xs[kTile + r]);
        }
        ok = ok && ptx::mbar_wait(o_done + t, 0);
        ptx::tc_fence_after();
        const float inv = 1.f / lt;
        // row a1 of stacked position p: tile a1 mod pb1q of position a2 pk + p
        const int sp = a1 / g.pb1q;
        const long long tok = a1 < g.b1q ? token_of(g, a1 - sp * g.pb1q, a2 * g.pk + sp) : 0;
        TO* orow = out + ((long long)bh * g.Nq + tok) * D + hf * (D / 2);
        // 32-byte stores when the caller's buffer allows them (every row
        // offset is a multiple of 32 bytes; the ABI promises 16 for the base)
        const bool wide = (reinterpret_cast<uintptr_t>(out) & 31) == 0;
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t o[16];
          ptx::tmem_ld16(tO(t) + lane_off + hf * (D / 2) + cc * 16, o);
          ptx::tmem_wait_ld();
          if (a1 < g.b1q && ok) {
            if constexpr (sizeof(TO) == 4) {
#pragma unroll
              for (int i = 0; i < 16; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * inv);
              if (wide) {
                ptx::st_global_v8(orow + cc * 16, *reinterpret_cast<const uint32_t(*)[8]>(o));
                ptx::st_global_v8(orow + cc * 16 + 8, *reinterpret_cast<const uint32_t(*)[8]>(o + 8));
              } else {
#pragma unroll
                for (int i = 0; i < 16; i += 4)
                  *reinterpret_cast<uint4*>(orow + cc * 16 + i) = make_uint4(o[i], o[i + 1], o[i + 2], o[i + 3]);
              }
            } else {
              uint32_t pk[8];
#pragma unroll
              for (int e = 0; e < 8; ++e) {
                TO two[2] = {from_f<TO>(__uint_as_float(o[2 * e]) * inv), from_f<TO>(__uint_as_float(o[2 * e + 1]) * inv)};
                pk[e] = *reinterpret_cast<const uint32_t*>(two);
              }
              if (wide) {
                ptx::st_global_v8(orow + cc * 16, pk);
              } else {
#pragma unroll
                for (int i = 0; i < 8; i += 4)
                  *reinterpret_cast<uint4*>(orow + cc * 16 + 2 * i) = make_uint4(pk[i], pk[i + 1], pk[i + 2], pk[i + 3]);
              }
            }
          }
        }
      } else {
        // merge the halves: (m, l) of each, shifts may differ
        float* xs = reinterpret_cast<float*>(sX + t * kXt);   // [m, l][half][128]
        xs[hf * kTile + r] = m;
        xs[2 * kTile + hf * kTile + r] = l;
        ptx::named_bar(1 + t, kTileThreads);
        if (hf == 0 && a1 < g.b1q) {
          const float mo = xs[kTile + r], lo = xs[3 * kTile + r];
          const float M = fmaxf(m, mo);
          const float L = (m == -INFINITY ? 0.f : l * ptx::ex2(m - M)) + (mo == -INFINITY ? 0.f : lo * ptx::ex2(mo - M));
          lse[(long long)zrow * g.b1q_pad + a1] = M + log2f(L);
        }
      }
    }
  }
}

template <int D, bool OUT>
constexpr uint32_t row_tmem_slot() {
  constexpr int NH = D / 64;
  return (uint32_t)(2 * NH * 2 * kBox + kKS * 2 * NH * kBox + (OUT ? 2 * 2 * NH * kBox : 0) + kKS * kBlk * 4 +
                    2 * xchg_tile_bytes<OUT ? 1 : 0>() + 23 * 8);
}

// One row-pass item per CTA: grid (ceil(b1q / 256), b2, BH), kThreads threads.
template <typename TQ, typename TO, int D, bool OUT, bool LSE_OUT = false>
__global__ void __launch_bounds__(kThreads, 1)
l_row(TO* __restrict__ out, const __grid_constant__ Maps maps, float* __restrict__ lse, Geo g) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_misaligned(smem_raw)) return;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem_raw + row_tmem_slot<D, OUT>());
  if (threadIdx.x < 32) {
    ptx::tmem_alloc(sTmem, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // dependents may start once every CTA of this grid holds its TMEM, so none
  // of theirs can take the columns a CTA of this grid still has to allocate
  ptx::griddep_launch();
  const uint32_t tmem = *sTmem;
  l_row_item<TQ, TO, D, OUT, LSE_OUT>(out, maps, lse, g, blockIdx.x * 2 * kTile, blockIdx.y, blockIdx.z, smem_raw,
                                      tmem, nullptr, 0);
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) ptx::tmem_dealloc(tmem, 512);
}

// ===========================================================================
// LSE pass over 128-key blocks for one (head, position a2, 256 query rows):
//   lse[a1] = log2 sum_c1 2^(s q.k~ + h)
// with k~ rounded once to f16 (the hi plane) and q exact in f16: the row sums
// only weight whole rows in the column pass, and this rounding keeps the
// result within the tolerance (a fp64 replay of the GPU roundings shows it).
// S = q k~_hi^T is one N = 128 MMA group per (tile, block); TMEM: tile t,
// buffer b at column 256 t + 128 b, so block j + 1 is computed while the
// softmax reads block j.  The two column halves of a row keep their own
// running shift and sum and are merged at the end.  A quarter of the
// exponentials run on the FMA pipe (ex2_fma2): with one plane the score MMA
// has half the columns per exponential of the two-plane passes, so the MUFU
// unit alone would be the bound.
constexpr int kLBlk = 128;   // keys per LSE-pass block
constexpr int kLS = 3;       // k~ / h stages

template <int D>
constexpr size_t lse_smem() {
  constexpr int NH = D / 64;
  constexpr size_t need = (size_t)2 * NH * 2 * kBox /* q */ + (size_t)kLS * NH * 2 * kBox /* k~ hi */ +
                          kLS * kLBlk * 4 + 2 * xchg_tile_bytes<0>() + 32 * 8;
  return need > kExclusiveSmem ? need : kExclusiveSmem;
}

template <int D>
__global__ void __launch_bounds__(kThreads, 1)
l_lse(const __grid_constant__ Maps maps, float* __restrict__ lse, Geo g) {
  constexpr int NH = D / 64;
  constexpr uint32_t kQt = NH * 2 * kBox;    // q of one tile: [d half][128 rows]
  constexpr uint32_t kKst = NH * 2 * kBox;   // k~ hi of one block: [d half][128 keys]
  constexpr int kXt = xchg_tile_bytes<0>();
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_misaligned(smem_raw)) return;
  uint8_t* sQ = smem_raw;                                      // [2 tiles]
  uint8_t* sK = sQ + 2 * kQt;                                  // [kLS]
  float* sH = reinterpret_cast<float*>(sK + kLS * kKst);       // [kLS][128]
  uint8_t* sX = reinterpret_cast<uint8_t*>(sH + kLS * kLBlk);  // [tile][kXt bytes]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sX + 2 * kXt);
  uint64_t* q_full = bar + 0;
  uint64_t* k_full = bar + 1;    // [kLS]
  uint64_t* k_free = bar + 4;    // [kLS]
  uint64_t* s_full = bar + 7;    // [tile][buf]
  uint64_t* s_free = bar + 11;   // [tile][buf]
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bar + 15);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int a2 = blockIdx.y, bh = blockIdx.z;
  const int a1_base = blockIdx.x * 2 * kTile;
  const int zrow = bh * g.b2 + a2;
  // key blocks any row of this CTA sees (all of them without a causal mask)
  const int kmax = key_limit(g, min(a1_base + 2 * kTile, g.b1q) - 1);
  const int nkb = (kmax + kLBlk - 1) / kLBlk;
  const int ntiles = (g.b1q - a1_base > kTile) ? 2 : 1;

  if (tid == 0) {
    ptx::mbar_init(q_full, 1);
    for (int i = 0; i < kLS; ++i) {
      ptx::mbar_init(k_full + i, 1);
      ptx::mbar_init(k_free + i, 8 * ntiles);
    }
    for (int i = 0; i < 4; ++i) {
      ptx::mbar_init(s_full + i, 1);
      ptx::mbar_init(s_free + i, 8);
    }
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(sTmem, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // dependents may start once every CTA of this grid holds its TMEM, so none
  // of theirs can take the columns a CTA of this grid still has to allocate
  ptx::griddep_launch();
  ptx::griddep_wait();   // set-up done: global data of the previous kernel from here on
  const uint32_t tmem = *sTmem;
  auto tS = [&](int t, int b) { return tmem + 256 * t + 128 * b; };

  if (warp == kLoadWarp) {
    if (lane == 0) {
      // --------------------------------------------------------- TMA producer
      ptx::prefetch_tmap(&maps.kt);
      ptx::mbar_expect_tx(q_full, 2 * kQt);
      for (int t = 0; t < 2; ++t)
        for (int hf = 0; hf < NH; ++hf)
          for (int rh = 0; rh < 2; ++rh)
            ptx::tma_load_3d(sQ + t * kQt + hf * 2 * kBox + rh * kBox, &maps.qb, q_full, hf * 64,
                             a1_base + t * kTile + rh * kBlk, zrow);
      bool ok = true;
      for (int blk = 0; blk < nkb && ok; ++blk) {
        const int ks = blk % kLS;
        if (blk >= kLS) ok = ptx::mbar_wait(k_free + ks, ((blk / kLS) - 1) & 1);
        if (!ok) break;
        ptx::mbar_expect_tx(k_full + ks, kKst + kLBlk * 4);
        for (int hf = 0; hf < NH; ++hf)
          for (int rh = 0; rh < 2; ++rh)
            ptx::tma_load_3d(sK + ks * kKst + hf * 2 * kBox + rh * kBox, &maps.kt, k_full + ks, hf * 64,
                             blk * kLBlk + rh * kBlk, zrow);
        for (int rh = 0; rh < 2; ++rh)
          tma_load_2d(sH + ks * kLBlk + rh * kBlk, &maps.h, k_full + ks, blk * kLBlk + rh * kBlk, zrow);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      // ----------------------------------------------------------- MMA issuer
      constexpr uint32_t idS = ptx::idesc_f16(128, kLBlk, 0, 0, 0);
      const uint32_t aQ = ptx::smem_u32(sQ), aK = ptx::smem_u32(sK);
      auto issue_s = [&](int t, int blk, int b) {
        const uint64_t a0 = ptx::sw128_desc(aQ + t * kQt, 16, 1024);
        const uint64_t b0 = ptx::sw128_desc(aK + (blk % kLS) * kKst, 16, 1024);
#pragma unroll
        for (int hf = 0; hf < NH; ++hf)
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4)
            ptx::mma_f16_ss(tS(t, b), a0 + ((hf * 2 * kBox + k4 * 32) >> 4), b0 + ((hf * 2 * kBox + k4 * 32) >> 4),
                            idS, (hf | k4) != 0);
        ptx::mma_commit(s_full + 2 * t + b);
      };
      bool ok = ptx::mbar_wait(q_full, 0) && ptx::mbar_wait(k_full, 0);
      ptx::tc_fence_after();
      if (ok) {
        for (int t = 0; t < ntiles; ++t) issue_s(t, 0, 0);
        if (nkb > 1) {
          ok = ptx::mbar_wait(k_full + 1, 0);
          ptx::tc_fence_after();
          if (ok)
            for (int t = 0; t < ntiles; ++t) issue_s(t, 1, 1);
        }
      }
      for (int j = 0; j < nkb && ok; ++j) {
        const int b = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        for (int t = 0; t < ntiles && ok; ++t) {
          ok = ptx::mbar_wait(s_free + 2 * t + b, ph);
          if (ok && j + 2 < nkb) {
            ok = ptx::mbar_wait(k_full + (j + 2) % kLS, ((j + 2) / kLS) & 1);
            ptx::tc_fence_after();
            if (ok) issue_s(t, j + 2, b);
          }
        }
      }
    }
  } else {
    // ------------------------------------------------------- softmax warps
    const int t = warp >> 3;                 // tile
    const int hf = (warp >> 2) & 1;          // column half: keys 64 hf .. 64 hf + 63 of a block
    const int r = 32 * (warp & 3) + lane;
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const int a1 = a1_base + t * kTile + r;
    const int rowlim = key_limit(g, min(a1, g.b1q - 1));   // visible key tiles [0, rowlim)
    if (t < ntiles) {
      float m = -INFINITY, l = 0.f;
      bool ok = true;
      const float2 sl2 = make_float2(g.sl2, g.sl2);
      for (int j = 0; j < nkb; ++j) {
        const int ks = j % kLS;
        const int b = j & 1;
        const uint32_t ph = (j >> 1) & 1;
        ok = ok && ptx::mbar_wait(s_full + 2 * t + b, ph) && ptx::mbar_wait(k_full + ks, (j / kLS) & 1);
        ptx::tc_fence_after();
        const float4* hv = reinterpret_cast<const float4*>(sH + ks * kLBlk + 64 * hf);
#pragma unroll
        for (int sb = 0; sb < 2; ++sb) {   // 32 keys at a time: an online update each
          uint32_t s[32];
          ptx::tmem_ld32(tS(t, b) + lane_off + 64 * hf + 32 * sb, s);
          ptx::tmem_wait_ld();
          float2 x[16];   // x[i] = keys 64 hf + 32 sb + 2i, + 1
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 h4 = hv[8 * sb + i];
            x[2 * i] = fma2(make_float2(__uint_as_float(s[4 * i]), __uint_as_float(s[4 * i + 1])), sl2,
                            make_float2(h4.x, h4.y));
            x[2 * i + 1] = fma2(make_float2(__uint_as_float(s[4 * i + 2]), __uint_as_float(s[4 * i + 3])), sl2,
                                make_float2(h4.z, h4.w));
          }
          if (sb == 1) {
            // S and h of this block are read: release the k~/h stage and the S buffer
            ptx::tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              ptx::mbar_arrive(k_free + ks);
              ptx::mbar_arrive(s_free + 2 * t + b);
            }
          }
          const int valid = min(kLBlk, rowlim - j * kLBlk) - 64 * hf - 32 * sb;
          if (valid < 32) {  // only the last block of a ragged row
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              if (2 * i >= valid) x[i].x = -INFINITY;
              if (2 * i + 1 >= valid) x[i].y = -INFINITY;
            }
          }
          float mb = -INFINITY;
#pragma unroll
          for (int i = 0; i < 16; ++i) mb = fmaxf(mb, fmaxf(x[i].x, x[i].y));
          const bool move = mb > m + kLazyRescale;
          const float mn = move ? mb : m;
          const float corr = (mn == m) ? 1.f : ptx::ex2(m - mn);
          const float nmv = (mn == -INFINITY) ? 0.f : -mn;   // a half with no key yet
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
      float* xs = reinterpret_cast<float*>(sX + t * kXt);   // [m, l][half][128]
      xs[hf * kTile + r] = m;
      xs[2 * kTile + hf * kTile + r] = l;
      ptx::named_bar(1 + t, kTileThreads);
      if (hf == 0 && a1 < g.b1q) {
        const float mo = xs[kTile + r], lo = xs[3 * kTile + r];
        const float M = fmaxf(m, mo);
        const float L = (m == -INFINITY ? 0.f : l * ptx::ex2(m - M)) + (mo == -INFINITY ? 0.f : lo * ptx::ex2(mo - M));
        lse[(long long)zrow * g.b1q_pad + a1] = M + log2f(L);
      }
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 512);
}

// ===========================================================================
// Column pass for one (head, position a2, 256 key tiles), 128 queries per block:
//   q~[c1,a2] = sum_a1 L q / sum_a1 L,  L = 2^(s q.k~ + h - lse[a1]),
// with q, k~ and L in f16 and q~ stored as hi / lo planes of the input type TQ
// ([plane][BH][b2][b1k][d]), the A operand of the next R step.
// TMEM, tile t at column 256 t:  S^T [0, 128) for 128 queries; P^T is written
// over it per 32-query chunk c as [hi | lo] in columns [32 c, 32 c + 32)
// (16 columns each, two queries per column);  acc [128, 128 + D).
template <int D>
constexpr size_t col_smem() {
  constexpr int NH = D / 64;
  constexpr size_t need = (size_t)2 * 2 * NH * 2 * kBox /* k~ */ + (size_t)kQS * NH * 2 * kBox /* q */ +
                          kQS * kQBlk * 4 + 2 * 2 * xchg_tile_bytes<2>() + 32 * 8;
  return need > kExclusiveSmem ? need : kExclusiveSmem;
}

template <typename TQ, int D>
__global__ void __launch_bounds__(kThreads, 1)
l_col(const __grid_constant__ Maps maps, const float* __restrict__ hbuf, TQ* __restrict__ qt, Geo g) {
  constexpr int NH = D / 64;
  constexpr uint32_t kKt = 2 * NH * 2 * kBox;   // k~ hi+lo of one tile: [plane][d half][128 rows]
  constexpr uint32_t kQst = NH * 2 * kBox;      // 128 query rows: [d half][128 rows]
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (smem_misaligned(smem_raw)) return;
  uint8_t* sK = smem_raw;                                    // [2 tiles]
  uint8_t* sQ = sK + 2 * kKt;                                // [kQS]
  float* sL = reinterpret_cast<float*>(sQ + kQS * kQst);     // [kQS][128]
  float* sX = sL + kQS * kQBlk;                              // [item parity][tile][half][128]
  uint64_t* bar = reinterpret_cast<uint64_t*>(sX + 2 * 2 * xchg_tile_bytes<2>() / 4);
  uint64_t* k_full = bar + 0;
  uint64_t* k_empty = bar + 1;   // the score MMAs of an item are done with sK
  uint64_t* q_full = bar + 2;    // [kQS]
  uint64_t* q_free = bar + 4;    // [kQS]
  uint64_t* s_full = bar + 6;    // [tile]
  uint64_t* p_full = bar + 8;    // [tile]
  uint64_t* o_done = bar + 10;   // [tile]
  uint64_t* acc_free = bar + 12; // [tile] the epilogue has read the accumulator
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bar + 14);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int plane_rows = g.BH * g.b2;
  const int nqb = (g.b1q + kQBlk - 1) / kQBlk;
  const int nchunk = (g.b1k + 2 * kTile - 1) / (2 * kTile);
  const int n_items = g.BH * g.b2 * nchunk;
  // item -> (row of the [BH][b2] planes, first key tile, tiles in it, first
  // query block: under a causal mask no earlier query sees these key tiles)
  auto item_of = [&](int it, int& zrow, int& kb, int& ntiles, int& qb0) {
    zrow = it / nchunk;
    kb = (it - zrow * nchunk) * 2 * kTile;
    ntiles = (g.b1k - kb > kTile) ? 2 : 1;
    qb0 = query_start(g, kb) / kQBlk;
  };

  if (tid == 0) {
    ptx::mbar_init(k_full, 1);
    ptx::mbar_init(k_empty, 1);
    for (int i = 0; i < kQS; ++i) {
      ptx::mbar_init(q_full + i, 1);
      ptx::mbar_init(q_free + i, 1);
    }
    for (int t = 0; t < 2; ++t) {
      ptx::mbar_init(s_full + t, 1);
      ptx::mbar_init(p_full + t, 8);
      ptx::mbar_init(o_done + t, 1);
      ptx::mbar_init(acc_free + t, 8);
    }
    ptx::fence_mbar_init();
  }
  if (warp == 0) {
    ptx::tmem_alloc(sTmem, 512);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // dependents may start once every CTA of this grid holds its TMEM, so none
  // of theirs can take the columns a CTA of this grid still has to allocate
  ptx::griddep_launch();
  ptx::griddep_wait();   // set-up done: global data of the previous kernel from here on
  const uint32_t tmem = *sTmem;
  auto tS = [&](int t) { return tmem + 256 * t; };
  auto tA = [&](int t) { return tmem + 256 * t + 128; };

  if (warp == kLoadWarp) {
    if (lane == 0) {
      // --------------------------------------------------------- TMA producer
      ptx::prefetch_tmap(&maps.kt);
      ptx::prefetch_tmap(&maps.qb);
      bool ok = true;
      int gq = 0, ni = 0;   // query blocks and items loaded so far
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++ni) {
        int zrow, kb, ntiles, qb0;
        item_of(it, zrow, kb, ntiles, qb0);
        if (ni > 0) ok = ptx::mbar_wait(k_empty, (ni - 1) & 1);
        if (!ok) break;
        ptx::mbar_expect_tx(k_full, 2 * kKt);
        for (int t = 0; t < 2; ++t)
          for (int p = 0; p < 2; ++p)
            for (int hf = 0; hf < NH; ++hf)
              for (int rh = 0; rh < 2; ++rh)
                ptx::tma_load_3d(sK + t * kKt + (p * NH + hf) * 2 * kBox + rh * kBox, &maps.kt, k_full, hf * 64,
                                 kb + t * kTile + rh * kBlk, p * plane_rows + zrow);
        for (int blk = qb0; blk < nqb && ok; ++blk, ++gq) {
          const int qs = gq % kQS;
          if (gq >= kQS) ok = ptx::mbar_wait(q_free + qs, ((gq / kQS) - 1) & 1);
          if (!ok) break;
          ptx::mbar_expect_tx(q_full + qs, kQst + kQBlk * 4);
          for (int hf = 0; hf < NH; ++hf)
            for (int rh = 0; rh < 2; ++rh)
              ptx::tma_load_3d(sQ + qs * kQst + hf * 2 * kBox + rh * kBox, &maps.qb, q_full + qs, hf * 64,
                               blk * kQBlk + rh * kBlk, zrow);
          for (int rh = 0; rh < 2; ++rh)
            tma_load_2d(sL + qs * kQBlk + rh * kBlk, &maps.lse, q_full + qs, blk * kQBlk + rh * kBlk, zrow);
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      // ----------------------------------------------------------- MMA issuer
      constexpr uint32_t idS = ptx::idesc_f16(128, kQBlk, 0, 0, 0);   // f16 operands
      constexpr uint32_t idPQ = ptx::idesc_f16(128, D, 0, 0, 1);
      const uint32_t aK = ptx::smem_u32(sK), aQ = ptx::smem_u32(sQ);
      auto issue_s = [&](int t, int gblk) {
        const uint64_t a0 = ptx::sw128_desc(aK + t * kKt, 16, 1024);
        const uint64_t b0 = ptx::sw128_desc(aQ + (gblk % kQS) * kQst, 16, 1024);
        const uint32_t td = tS(t);
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
          for (int hf = 0; hf < NH; ++hf)
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4)
              ptx::mma_f16_ss(td, a0 + (((p * NH + hf) * 2 * kBox + k4 * 32) >> 4),
                              b0 + ((hf * 2 * kBox + k4 * 32) >> 4), idS, (p | hf | k4) != 0);
        ptx::mma_commit(s_full + t);
      };
      bool ok = true;
      int gq = 0, ni = 0;
      int cnt0 = 0, cnt1 = 0, icnt0 = 0, icnt1 = 0;   // blocks / items processed per tile
      for (int it = blockIdx.x; it < n_items && ok; it += gridDim.x, ++ni) {
        int zrow, kb, ntiles, qb0;
        item_of(it, zrow, kb, ntiles, qb0);
        ok = ptx::mbar_wait(k_full, ni & 1) && ptx::mbar_wait(q_full + gq % kQS, (gq / kQS) & 1);
        ptx::tc_fence_after();
        if (!ok) break;
        for (int t = 0; t < ntiles; ++t) issue_s(t, gq);
        if (nqb - qb0 == 1) ptx::mma_commit(k_empty);
        for (int i = qb0; i < nqb && ok; ++i) {
          const int qs = (gq + i - qb0) % kQS;
          const uint64_t q0 = ptx::sw128_desc(aQ + qs * kQst, 2 * kBox, 1024);
          for (int t = 0; t < ntiles && ok; ++t) {
            const int ct = t ? cnt1 : cnt0, it_t = t ? icnt1 : icnt0;
            ok = ptx::mbar_wait(p_full + t, ct & 1);
            // the first product of an item overwrites the accumulator the
            // previous item's epilogue reads
            if (ok && i == qb0 && it_t > 0) ok = ptx::mbar_wait(acc_free + t, (it_t - 1) & 1);
            ptx::tc_fence_after();
            if (!ok) break;
            const uint32_t tp = tS(t);
#pragma unroll
            for (int p = 0; p < 2; ++p)
#pragma unroll
              for (int kk = 0; kk < kQBlk / 16; ++kk)
                ptx::mma_f16_ts(tA(t), tp + (kk >> 1) * 32 + p * 16 + (kk & 1) * 8, q0 + ((kk * 2048) >> 4), idPQ,
                                ((i - qb0) | p | kk) != 0);
            if (t == ntiles - 1) ptx::mma_commit(q_free + qs);
            if (i + 1 < nqb) {
              // S^T(t, i+1) overwrites P^T(t, i): the P^T q product above runs first
              const int gn = gq + i + 1 - qb0;   // ring index of block i + 1
              ok = ptx::mbar_wait(q_full + gn % kQS, (gn / kQS) & 1);
              ptx::tc_fence_after();
              if (ok) issue_s(t, gn);
            } else {
              ptx::mma_commit(o_done + t);
            }
            if (t) ++cnt1; else ++cnt0;
          }
          // after the item's last score MMA, sK may take the next item's tiles
          if (i + 2 == nqb) ptx::mma_commit(k_empty);
        }
        ++icnt0;
        if (ntiles > 1) ++icnt1;
        gq += nqb - qb0;
      }
    }
  } else {
    const int t = warp >> 3;                 // tile
    const int hf = (warp >> 2) & 1;          // column half: queries 64 hf .. 64 hf + 63 of a block
    const int r = 32 * (warp & 3) + lane;    // key tile row / TMEM lane
    const uint32_t lane_off = (uint32_t)(32 * (warp & 3)) << 16;
    const float2 sl2 = make_float2(g.sl2, g.sl2);
    const long long plane = (long long)g.BH * g.b2 * g.b1k * D;
    bool ok = true;
    int gq = 0, cnt = 0, icnt = 0;
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
      int zrow, kb, ntiles, qb0;
      item_of(it, zrow, kb, ntiles, qb0);
      if (t < ntiles) {
        const int c1 = kb + t * kTile + r;
        const int qstart = query_start(g, min(c1, g.b1k - 1));   // queries [qstart, b1q) see this tile
        const float hb = (c1 < g.b1k) ? hbuf[(long long)zrow * g.b1k_pad + c1] + kColShift : 0.f;
        const float2 hb2 = make_float2(hb, hb);
        float2 beta2 = make_float2(0.f, 0.f);
        for (int i = qb0; i < nqb; ++i, ++cnt) {
          const int gi = gq + i - qb0;   // ring index of block i
          const int qs = gi % kQS;
          ok = ok && ptx::mbar_wait(s_full + t, cnt & 1) && ptx::mbar_wait(q_full + qs, (gi / kQS) & 1);
          ptx::tc_fence_after();
          const int valid = min(kQBlk, g.b1q - i * kQBlk);
          const int vlo = qstart - i * kQBlk;   // queries of this block below it are masked
#pragma unroll
          for (int hh = 0; hh < 2; ++hh) {  // 32 queries at a time
            const int cb = 64 * hf + 32 * hh;   // first S^T column (query) of this chunk
            uint32_t sr[32];
            ptx::tmem_ld32(tS(t) + lane_off + cb, sr);
            const float4* lv = reinterpret_cast<const float4*>(sL + qs * kQBlk + cb);
            ptx::tmem_wait_ld();
#pragma unroll
            for (int q8 = 0; q8 < 2; ++q8) {   // 16 queries: 8 packed columns per plane
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
              if (valid < kQBlk || vlo > 0) {  // a ragged last block, or queries hidden by the mask
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
            // P^T of these queries over the chunk's own S^T columns (all read
            // already): hi in [cb, cb + 16), lo in [cb + 16, cb + 32)
            ptx::tmem_st8(tS(t) + lane_off + cb + 8 * q8, hi);
            ptx::tmem_st8(tS(t) + lane_off + cb + 16 + 8 * q8, lo);
            }
          }
          ptx::tmem_wait_st();
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(p_full + t);
        }
        // beta = the two halves' column sums (slots alternate between items)
        float* xs = sX + ((icnt & 1) * 2 + t) * 2 * kTile;
        xs[hf * kTile + r] = beta2.x + beta2.y;
        ptx::named_bar(1 + t, kTileThreads);
        const float beta = beta2.x + beta2.y + xs[(hf ^ 1) * kTile + r];
        ok = ok && ptx::mbar_wait(o_done + t, icnt & 1);
        ptx::tc_fence_after();
        // beta = 0: every query gives this key tile a weight below 2^-141, so
        // every 2^(x - lse + 15) flushed to zero; the accumulator is zero too,
        // and q~ = 0 replaces the 0/0 that would spread NaN to every row
        const float inv = beta > 0.f ? 1.f / beta : 0.f;
        const float2 inv2 = make_float2(inv, inv);
        // q~ as hi / lo planes of the input type: the A operand of the next R step
        TQ* dst = qt + ((long long)zrow * g.b1k + (c1 < g.b1k ? c1 : 0)) * D + hf * (D / 2);
#pragma unroll 1
        for (int cc = 0; cc < D / 32; ++cc) {   // 16 columns at a time
          uint32_t o[16];
          ptx::tmem_ld16(tA(t) + lane_off + hf * (D / 2) + cc * 16, o);
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
        // the accumulator is read: the next item may overwrite it
        ptx::tc_fence_before();
        __syncwarp();
        if (lane == 0) ptx::mbar_arrive(acc_free + t);
        ++icnt;
      }
      gq += nqb - qb0;
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 512);
}

}  // namespace tc
}  // namespace monarch
