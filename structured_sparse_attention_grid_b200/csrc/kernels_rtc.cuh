// R step on the tensor cores for bf16 / f16 inputs.
//
// A CTA takes a group of G <= floor(128 / r8) consecutive key tiles of one head
// (r8 = b2 rounded up to 8) and stacks their rows at a stride rs (32 when at
// most four tiles of at most 32 positions are stacked, else r8): row
// r = g rs + a2 holds
// position a2 of key tile c1_0 + g.  With A = the stacked q~ rows (hi and lo
// planes, or the exact query rows) and B = the stacked key rows, one
// 128 x 128 score block
//     S = A K^T                     (tcgen05, N = 128, fp32 in TMEM)
// holds every tile's b2 x b2 scores on its diagonal.  Thread r (TMEM lane r)
// masks its row to the columns of its own tile and takes the softmax over c2
// (R = softmax_c2(s q~ . k)) and its entropy h, then writes R back over S as
// the hi / lo planes of the A operand of
//     k~ = R K,   z = R V           (A from TMEM, B = keys / values in shared
//                                    memory, N = d)
// R is zero outside the diagonal blocks, so these are the per-tile products.
// The epilogue splits each row into hi / lo planes, stages them in shared
// memory in the swizzled box layout, the G tiles' rows packed (tile g at rows
// [g b2, (g + 1) b2)), and one thread stores each (plane, d half) with one
// TMA box of all G tiles into [plane][BH][b2][b1k][d] (position-major), the
// layout the L step reads: the store map walks positions before tiles, so
// the box lands tile by tile.  In the first step the exact query rows go out
// the same way as the block-major copy of q.
//
// Loads: keys, values and exact query rows come through the 4-D grid map
// (d, W, H, frames) with one tile per box, so the grid -> block permutation is
// done by the TMA unit; q~ planes come through a 3-D map with one tile per box.
// Shared memory: A (two planes) and K, [d half][128 rows][128 B] boxes with the
// 128-byte swizzle; V reuses the A hi plane once the score MMAs are complete.
// That is 96 KB for d = 128 and 256 TMEM columns, so two CTAs share an SM and
// one CTA's loads overlap the other's arithmetic.
//
// Threads: eight row warps and a control warp.  Row warps w and w + 4 share
// TMEM lane quadrant w (rows 32 w .. 32 w + 31) and split the columns: in the
// softmax each takes one 16-column half of every 32-column chunk of S (the
// two halves combine their row max and sums through shared memory), in the
// epilogues and the query conversion each takes one half of d.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "kernels_tc.cuh"
#include "tc_common.cuh"

namespace monarch {

struct RtcMaps {
  CUtensorMap q;    // queries    {d, W, H, BH*T},        box {64, tw, th, 1}
  CUtensorMap k;    // keys       {d, W, H, BH*Tk},       box {64, tw, th, 1}
  CUtensorMap v;    // values     {d, W, H, BH*Tk},       box {64, tw, th, 1}
  CUtensorMap qt;   // q~ planes  {d, b1k, 2*BH*b2},      box {64, 1, b2}
  CUtensorMap qm;   // mean-query planes (KV init) {d, 1, 2*BH*b2}, box {64, 1, b2}
  CUtensorMap qb;   // block-major q, f16 (store) {d, b1q, BH*b2},   box {64, 1, b2}
  // stores of G tiles at once, positions before tiles (strides b1k d, d):
  CUtensorMap qbg;  // block-major q, f16 {d, b2, b1q, BH},     box {64, b2, G, 1}
  CUtensorMap kt;   // k~ planes, f16     {d, b2, b1k, 2*BH},   box {64, b2, G, 1}
  CUtensorMap z;    // z planes, f16      {d, b2, b1k, 2*BH},   box {64, b2, G, 1}
};

// Planes written by the R step.
template <typename TQ>
struct TcPlanes {
  __half* kt_hi;    // [BH][b2][b1k][d], then the lo plane at kt_hi + plane
  __half* z_hi;     // [BH][b2][b1k][d], then the lo plane
  long long plane;  // elements per plane
};

constexpr int kRtcRowThreads = 256;   // 8 row warps: two per TMEM lane quadrant
constexpr int kRtcThreads = kRtcRowThreads + 32;   // + the control warp (warp 8)
constexpr int kRtcRows = 128;
constexpr uint32_t kRBox = 128 * 128; // one [128 rows][128 B] swizzled box
constexpr size_t kRtcAux = 16 * 8 + 6 * 128 * 4;   // barriers, TMEM slot, softmax exchange

// At least 80 KB so that at most two CTAs (2 x 256 TMEM columns) share an SM.
template <int D>
constexpr size_t rtc_smem() {
  constexpr size_t need = (size_t)3 * (D / 64) * kRBox + kRtcAux;
  return need > 80 * 1024 ? need : 80 * 1024;
}

// Bytes of shared memory one R-step item uses (operand boxes, barriers,
// softmax exchange), and where a kernel running one item per CTA keeps the
// TMEM address (inside the item's barrier area, in a slot the item leaves
// alone).
template <int D>
constexpr uint32_t rtc_item_bytes() { return (uint32_t)(3 * (D / 64) * kRBox + kRtcAux); }
template <int D>
constexpr uint32_t rtc_tmem_slot() { return (uint32_t)(3 * (D / 64) * kRBox + 8 * 8); }

// One R-step item: key tiles [c1_0, c1_0 + G) of head bh (fewer at the end of
// the head), run by 288 threads with item-local thread index tid (eight row
// warps, then the control warp) on `smem` (1024-byte aligned,
// rtc_item_bytes<D>()) and 256 TMEM columns at `tmem`.  bar_row and bar_all
// are the named barriers of the item's row warps and of all its threads;
// warp0 is the CTA warp index of the item's first warp (its row warps reach
// the TMEM lane quadrants (warp0 + w) mod 4, two warps each).
// ready != nullptr: the control thread waits (bounded, acquire) for
// *ready >= ready_need before its loads, and the item does not wait for the
// previous grid (the count stands for it).
// done != nullptr: once every output of the item (k~, z and the block-major q
// copy through TMA, h by the row threads) is written and visible at GPU
// scope, one thread adds 1 to *done (release), for consumers in other CTAs
// that read these outputs with TMA after an acquire of the count.
template <typename TQ, int D>
__device__ __forceinline__ void r_step_item(const RtcMaps& maps, const TQ* __restrict__ q, const Work& w,
                                            const TcPlanes<TQ>& out, const Geo& g, int mode, int final_step, int G,
                                            int c1_0, int bh, uint8_t* smem_raw, uint32_t tmem, int tid,
                                            int warp0, int bar_row, int bar_all, const int* ready, int ready_need,
                                            int* done) {
  constexpr int NH = D / 64;
  constexpr int bf16 = TcType<TQ>::kBf16;
  uint8_t* sA = smem_raw;                  // [plane][d half] boxes; V in plane 0 later
  uint8_t* sK = sA + 2 * NH * kRBox;       // [d half] boxes
  uint64_t* bar = reinterpret_cast<uint64_t*>(sK + NH * kRBox);
  uint64_t* bar_ld = bar + 0;    // TMA: keys and query rows
  // bar + 1: unused
  uint64_t* bar_s = bar + 2;     // MMA: S complete
  uint64_t* bar_r = bar + 3;     // row warps: R in TMEM
  uint64_t* bar_acc = bar + 4;   // MMA: k~ (phase 0), z (phase 1) complete
  uint64_t* bar_free = bar + 5;  // row warps: k~ read out of TMEM
  uint64_t* bar_v = bar + 6;     // TMA: values
  uint64_t* bar_q = bar + 7;     // row warps: query rows read (first step, bf16, before V lands)
  // bar + 8: the TMEM slot of a one-item kernel (rtc_tmem_slot)
  float* sRed = reinterpret_cast<float*>(bar + 16);   // [max | sum p | sum p s][half][row]

  const int warp = tid >> 5, lane = tid & 31;
  const int r8 = (g.b2 + 7) & ~7;   // G * r8 <= 128 (the host's choice of G)
  // rows per stacked tile: 32 when four tiles of at most 32 positions fit, so
  // that each row warp holds one tile and reads one 32-column chunk of S;
  // else b2 rounded up to 8
  const int rs = (g.b2 <= 32 && G * 32 <= kRtcRows) ? 32 : r8;
  const int Gn = min(G, g.b1k - c1_0);

  if (tid == kRtcRowThreads) {
    ptx::mbar_init(bar_ld, 1);
    ptx::mbar_init(bar_s, 1);
    ptx::mbar_init(bar_r, 8);
    ptx::mbar_init(bar_acc, 1);
    ptx::mbar_init(bar_free, 8);
    ptx::mbar_init(bar_v, 1);
    ptx::mbar_init(bar_q, 8);
    ptx::fence_mbar_init();
  }
  auto exact_q = [&](int c1) { return mode == QT_IDENTITY || (mode == QT_KVINIT && c1 >= g.off); };
  // Zero every row that no load writes (in-tile padding, tiles past the end):
  // K and V rows there meet zero R entries, and 0 * NaN would not be zero.
  // With a KV cache the score MMA reads the A lo plane, which the exact query
  // rows leave unwritten: zero it there too.
  for (int i = tid; i < kRtcRows * NH * 8; i += kRtcThreads) {
    const int row = i / (NH * 8), rem = i - row * (NH * 8), hf = rem >> 3, ch = rem & 7;
    const int gg = row / rs, a = row - gg * rs;
    const uint4 z4 = make_uint4(0u, 0u, 0u, 0u);
    const uint32_t o = hf * kRBox + row * 128 + ch * 16;
    if (gg >= Gn || a >= g.b2) {
      *reinterpret_cast<uint4*>(sK + o) = z4;
      *reinterpret_cast<uint4*>(sA + o) = z4;
      *reinterpret_cast<uint4*>(sA + NH * kRBox + o) = z4;
    } else if (mode == QT_KVINIT && exact_q(c1_0 + gg)) {
      *reinterpret_cast<uint4*>(sA + NH * kRBox + o) = z4;
    }
  }
  ptx::fence_proxy_async();
  ptx::tc_fence_before();
  ptx::named_bar(bar_all, kRtcThreads);
  ptx::tc_fence_after();
  // set-up done: from here on global memory of the previous kernel is used
  if (!ready) ptx::griddep_wait();
  const uint32_t tS = tmem, tAcc = tmem + 128;

  // tile c1 -> (frame, tile row, tile column) of its grid box
  auto tile_coords = [&](int c1, int& t, int& y0, int& x0) {
    t = c1 / g.P;
    const int rem = c1 - t * g.P, ty = rem / g.ntx;
    y0 = ty * g.th;
    x0 = (rem - ty * g.ntx) * g.tw;
  };

  if (warp == kRtcRowThreads / 32) {
    if (lane == 0) {
      // ------------------------------------------------ loads and MMA issue
      ptx::prefetch_tmap(&maps.k);
      if (ready) {
        // the items this one reads from are done (acquire), before the loads
        ptx::wait_count(ready, ready_need);
        ptx::fence_proxy_async_global();
      }
      bool ok = true;
      uint32_t bytes = 0;
      for (int gg = 0; gg < Gn; ++gg) {
        const int c1 = c1_0 + gg;
        // q~ planes, or the exact query rows, or (cached tiles) the mean-query planes
        const int planes = (mode == QT_BUFFER || !exact_q(c1)) ? 2 : 1;
        bytes += (uint32_t)(NH * g.b2 * 128 * (1 + planes));
      }
      ptx::mbar_expect_tx(bar_ld, bytes);
      for (int gg = 0; gg < Gn; ++gg) {
        const int c1 = c1_0 + gg;
        int t, y0, x0;
        tile_coords(c1, t, y0, x0);
        const uint32_t row0 = (uint32_t)(gg * rs) * 128;
        for (int hf = 0; hf < NH; ++hf)
          ptx::tma_load_4d(sK + hf * kRBox + row0, &maps.k, bar_ld, hf * 64, x0, y0, bh * g.Tk + t);
        if (mode == QT_BUFFER) {
          for (int p = 0; p < 2; ++p)
            for (int hf = 0; hf < NH; ++hf)
              ptx::tma_load_3d(sA + (p * NH + hf) * kRBox + row0, &maps.qt, bar_ld, hf * 64, c1,
                               (p * g.BH + bh) * g.b2);
        } else if (exact_q(c1)) {
          const int tq = t - (g.Tk - g.T);   // the aligned query frame (== t without a cache)
          for (int hf = 0; hf < NH; ++hf)
            ptx::tma_load_4d(sA + hf * kRBox + row0, &maps.q, bar_ld, hf * 64, x0, y0, bh * g.T + tq);
        } else {
          // a cached tile (KV init): the mean query of each position, hi and lo
          for (int p = 0; p < 2; ++p)
            for (int hf = 0; hf < NH; ++hf)
              ptx::tma_load_3d(sA + (p * NH + hf) * kRBox + row0, &maps.qm, bar_ld, hf * 64, 0,
                               (p * g.BH + bh) * g.b2);
        }
      }
      ok = ptx::mbar_wait(bar_ld, 0);
      ptx::tc_fence_after();
      // S = A K^T: both operands K-major (d along the 128-byte rows)
      if (ok) {
        constexpr uint32_t idS = ptx::idesc_f16(128, 128, bf16, 0, 0);
        const uint64_t dA = ptx::sw128_desc(ptx::smem_u32(sA), 16, 1024);
        const uint64_t dK = ptx::sw128_desc(ptx::smem_u32(sK), 16, 1024);
        const bool use_lo = mode != QT_IDENTITY;
#pragma unroll
        for (int hf = 0; hf < NH; ++hf)
#pragma unroll
          for (int k4 = 0; k4 < 4; ++k4) {
            const uint32_t off = (hf * kRBox + k4 * 32) >> 4;
            ptx::mma_f16_ss(tS, dA + off, dK + off, idS, (hf | k4) != 0);
            if (use_lo) ptx::mma_f16_ss(tS, dA + ((NH * kRBox) >> 4) + off, dK + off, idS, 1);
          }
        ptx::mma_commit(bar_s);
      }
      if (ok && mode != QT_BUFFER && !bf16) {
        // first step, f16 input: the exact query rows just loaded are also the
        // block-major copy of q that the L step reads (the store, like S,
        // only reads A, so it goes out after the score MMAs are issued)
        for (int gg = 0; gg < Gn; ++gg) {
          const int c1 = c1_0 + gg;
          if (!exact_q(c1)) continue;
          for (int hf = 0; hf < NH; ++hf)
            ptx::tma_store_3d(&maps.qb, sA + hf * kRBox + (uint32_t)(gg * rs) * 128, hf * 64, c1 - g.off,
                              bh * g.b2);
        }
        ptx::bulk_commit();
      }
      if (final_step) {
        // V lands in the A hi plane once the score MMAs and the q copy (its
        // readers) are done
        ok = ok && ptx::mbar_wait(bar_s, 0);
        if (bf16 && mode != QT_BUFFER) ok = ok && ptx::mbar_wait(bar_q, 0);
        ptx::bulk_wait_read();
        if (ok) {
          ptx::mbar_expect_tx(bar_v, (uint32_t)(Gn * NH * g.b2 * 128));
          for (int gg = 0; gg < Gn; ++gg) {
            int t, y0, x0;
            tile_coords(c1_0 + gg, t, y0, x0);
            for (int hf = 0; hf < NH; ++hf)
              ptx::tma_load_4d(sA + hf * kRBox + (uint32_t)(gg * rs) * 128, &maps.v, bar_v, hf * 64, x0, y0,
                               bh * g.Tk + t);
          }
        }
      }
      // k~ = R K and z = R V: A = R in TMEM as 32-key chunks [hi 16 | lo 16]
      // columns, B MN-major (d along the 128-byte rows, keys down the rows)
      auto issue_rb = [&](const uint8_t* sB) {
        constexpr uint32_t idV = ptx::idesc_f16(128, D, bf16, 0, 1);
        const uint64_t dB = ptx::sw128_desc(ptx::smem_u32(sB), kRBox, 1024);
#pragma unroll
        for (int kk = 0; kk < kRtcRows / 16; ++kk)
#pragma unroll
          for (int p = 0; p < 2; ++p)
            ptx::mma_f16_ts(tAcc, tS + (kk >> 1) * 32 + p * 16 + (kk & 1) * 8, dB + ((kk * 2048) >> 4), idV,
                            (kk | p) != 0);
        ptx::mma_commit(bar_acc);
      };
      ok = ok && ptx::mbar_wait(bar_r, 0);
      ptx::tc_fence_after();
      if (ok) issue_rb(sK);
      if (final_step) {
        ok = ok && ptx::mbar_wait(bar_free, 0) && ptx::mbar_wait(bar_v, 0);
        ptx::tc_fence_after();
        if (ok) issue_rb(sA);
      }
      if (done) ptx::bulk_wait_all(); else ptx::bulk_wait_read();
    }
  } else {
    // ------------------------------------------------------------- row warps
    // lane quadrant: a warp reaches the TMEM lanes of its CTA warp index mod 4
    const int qw = (warp + warp0) & 3, half = warp >> 2;   // lane quadrant, column half
    const int r = 32 * qw + lane;               // stacked row = TMEM lane
    const int gg = r / rs, a2 = r - gg * rs;
    const int c1 = c1_0 + gg;
    const bool valid = gg < Gn && a2 < g.b2;
    // staging row of this TMEM lane: the G tiles packed at b2 rows, the
    // shared-memory order of one store box of all of them
    const bool staged = gg < G && a2 < g.b2;
    const int srow = gg * g.b2 + a2;
    const uint32_t lane_off = (uint32_t)(32 * qw) << 16;
    constexpr int kSeg = NH * 4;                // 16-byte chunks of a row per half
    bool ok = true;


    // First step, bf16 input: the L step reads q in f16 (exact for |q| <
    // 65504; larger finite magnitudes set kErrRange).  The loaded rows are
    // converted into the A lo plane and stored from there as the block-major
    // copy of q: without a KV cache in the packed staging order, one box of
    // all G tiles per d half; with one per exact tile, as loaded (a group may
    // also hold cached tiles, which have no copy).
    const bool packed_q = mode == QT_IDENTITY;
    auto convert_and_store_q = [&]() {
      if (valid && exact_q(c1)) {
        bool over = false;
        const int wrow = packed_q ? srow : r;   // row of the converted copy in the A lo plane
#pragma unroll
        for (int k = 0; k < kSeg; ++k) {
          const int i = half * kSeg + k, hf = i >> 3, ch = i & 7;
          const uint32_t o = hf * kRBox + r * 128 + ((ch ^ (r & 7)) << 4);
          const uint32_t ow = hf * kRBox + wrow * 128 + ((ch ^ (wrow & 7)) << 4);
          uint4 u = *reinterpret_cast<const uint4*>(sA + o);
          uint32_t* wv = reinterpret_cast<uint32_t*>(&u);
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            // a finite bf16 of magnitude >= 2^16 (exponent field >= 143) has no f16 value
            const uint32_t a0 = wv[e] & 0x7FFFu, a1 = (wv[e] >> 16) & 0x7FFFu;
            over |= (a0 >= 0x4780u && a0 < 0x7F80u) || (a1 >= 0x4780u && a1 < 0x7F80u);
            const __half2 hv = __floats2half2_rn(__uint_as_float(wv[e] << 16), __uint_as_float(wv[e] & 0xFFFF0000u));
            wv[e] = *reinterpret_cast<const uint32_t*>(&hv);
          }
          *reinterpret_cast<uint4*>(sA + NH * kRBox + ow) = u;
        }
        if (over) atomicExch(&ptx::g_device_error, ptx::kErrRange);
      }
      ptx::fence_proxy_async();
      __syncwarp();
      if (final_step && lane == 0) ptx::mbar_arrive(bar_q);
      ptx::named_bar(bar_row, kRtcRowThreads);
      if (tid == 0 && ok) {
        if (packed_q) {
          for (int hf = 0; hf < NH; ++hf)
            ptx::tma_store_4d(&maps.qbg, sA + (NH + hf) * kRBox, hf * 64, 0, c1_0, bh);
        } else {
          for (int t = 0; t < Gn; ++t) {
            if (!exact_q(c1_0 + t)) continue;
            for (int hf = 0; hf < NH; ++hf)
              ptx::tma_store_3d(&maps.qb, sA + (NH + hf) * kRBox + (uint32_t)(t * rs) * 128, hf * 64,
                                c1_0 + t - g.off, bh * g.b2);
          }
        }
        ptx::bulk_commit();
      }
    };
    // Without a KV cache the score MMA does not read the A lo plane: convert
    // while it runs.  With one, after the score MMA (below).
    if (bf16 && mode == QT_IDENTITY) {
      ok = ptx::mbar_wait(bar_ld, 0);
      convert_and_store_q();
    }

    // ---- R = softmax over this row's tile columns [cb, cb + b2) of S.  The
    // rows of a quadrant need at most three 32-column chunks, from ch_lo on;
    // this warp reads the 16-column half c0 of each into registers.
    ok = ptx::mbar_wait(bar_s, 0) && ok;
    ptx::tc_fence_after();
    const int cb = gg * rs;
    const int wg0 = (32 * qw) / rs, wg1 = min((32 * qw + 31) / rs, G - 1);
    const int ch_lo = (wg0 * rs) >> 5, ch_hi = min((wg1 * rs + g.b2 - 1) >> 5, 3);
    const int c0 = 16 * half;
    auto in_tile = [&](int c) { return (unsigned)(c - cb) < (unsigned)g.b2; };
    uint32_t sv[3][16];
#pragma unroll
    for (int j = 0; j < 3; ++j)
      if (ch_lo + j <= ch_hi) ptx::tmem_ld16(tS + lane_off + 32 * (ch_lo + j) + c0, sv[j]);
    ptx::tmem_wait_ld();
    // Branch-free: columns outside this row's tile become -inf (p = 0).  The
    // entropy uses sum p s (raw scores, finite everywhere) so that masked
    // terms are exactly zero; four partial sums shorten the dependency chains.
    // (chunks past ch_hi are skipped: ch_hi - ch_lo is the same for the whole warp)
    float mq[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      if (ch_lo + j > ch_hi) break;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const bool in = in_tile(32 * (ch_lo + j) + c0 + i);
        const float x = in ? __uint_as_float(sv[j][i]) : -INFINITY;
        sv[j][i] = __float_as_uint(x);
        mq[i & 3] = fmaxf(mq[i & 3], x);
      }
    }
    // the two halves' maxima; every S read of the quadrant completes before
    // either warp writes R over S
    sRed[half * 128 + r] = fmaxf(fmaxf(mq[0], mq[1]), fmaxf(mq[2], mq[3]));
    ptx::tc_fence_before();
    ptx::named_bar(bar_row, kRtcRowThreads);
    ptx::tc_fence_after();
    const float m = fmaxf(sRed[r], sRed[128 + r]);
    const float ms = (m == -INFINITY) ? 0.f : m * g.sl2;   // base-2 units; a row with no column stays 0
    float lq[4] = {0.f, 0.f, 0.f, 0.f}, pq[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      if (ch_lo + j > ch_hi) break;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const float x = __uint_as_float(sv[j][i]);
        const float p = ptx::ex2(fmaf(x, g.sl2, -ms));
        lq[i & 3] += p;
        pq[i & 3] = (p > 0.f) ? fmaf(p, x, pq[i & 3]) : pq[i & 3];
        sv[j][i] = __float_as_uint(p);
      }
    }
    sRed[256 + half * 128 + r] = (lq[0] + lq[1]) + (lq[2] + lq[3]);
    sRed[512 + half * 128 + r] = (pq[0] + pq[1]) + (pq[2] + pq[3]);
    ptx::named_bar(bar_row, kRtcRowThreads);
    const float l = sRed[256 + r] + sRed[384 + r];
    // sum p (x s2 - ms) with x the raw score
    const float xe = g.sl2 * (sRed[512 + r] + sRed[640 + r]) - ms * l;
    const float inv = 1.f / l;
    const float2 inv2 = make_float2(inv, inv);
    // R over S: chunk ch -> columns [32 ch, 32 ch + 16) hi, [32 ch + 16, 32 ch + 32) lo;
    // this warp's 16 keys are the 8 hi and 8 lo columns at offset c0 / 2
#pragma unroll
    for (int j = 0; j < 3; ++j) {
      if (ch_lo + j > ch_hi) continue;
      uint32_t hi[8], lo[8];
#pragma unroll
      for (int i = 0; i < 8; ++i)
        tc::split2<TQ>(tc::mul2(make_float2(__uint_as_float(sv[j][2 * i]), __uint_as_float(sv[j][2 * i + 1])), inv2),
                       hi[i], lo[i]);
      ptx::tmem_st8(tS + lane_off + 32 * (ch_lo + j) + c0 / 2, hi);
      ptx::tmem_st8(tS + lane_off + 32 * (ch_lo + j) + 16 + c0 / 2, lo);
    }
    {
      // chunks no row of the quadrant uses: this warp zeroes 16 of their 32 columns
      uint32_t zero[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) zero[i] = 0u;
      for (int ch = 0; ch < 4; ++ch)
        if (ch < ch_lo || ch > ch_hi) ptx::tmem_st16(tS + lane_off + 32 * ch + c0, zero);
    }
    ptx::tmem_wait_st();
    ptx::tc_fence_before();
    __syncwarp();
    if (lane == 0) ptx::mbar_arrive(bar_r);
    // h in bits: -sum R log2 R = log2 l - sum R (x - m)
    if (half == 0 && valid && ok) w.h[((long long)bh * g.b2 + a2) * g.b1k_pad + c1] = log2f(l) - xe * inv;
    if (bf16 && mode == QT_KVINIT) convert_and_store_q();
    // ---- epilogue: this warp's half of a row of k~ (or z) from TMEM, split
    // into hi / lo planes, staged in two swizzled [d half][128 rows][128 B]
    // regions.  The next 16-column group is read while the current one is
    // converted; with release set, the warp hands the accumulator back to the
    // MMA warp (bar_free) once its last read has landed.
    auto stage_row = [&](uint8_t* shi, uint8_t* slo, bool release) {
      constexpr int NG = D / 32;   // 16-column groups per half
      uint32_t a[2][16];
      ptx::tmem_ld16(tAcc + lane_off + 16 * (half * NG), a[0]);
#pragma unroll
      for (int k = 0; k < NG; ++k) {
        const int cc = half * NG + k;   // 16-column group of the accumulator
        ptx::tmem_wait_ld();
        if (k + 1 < NG) {
          ptx::tmem_ld16(tAcc + lane_off + 16 * (cc + 1), a[(k + 1) & 1]);
        } else if (release) {
          ptx::tc_fence_before();
          __syncwarp();
          if (lane == 0) ptx::mbar_arrive(bar_free);
        }
        uint32_t hi[8], lo[8];
#pragma unroll
        for (int i = 0; i < 8; ++i)
          tc::split2<__half>(make_float2(__uint_as_float(a[k & 1][2 * i]), __uint_as_float(a[k & 1][2 * i + 1])),
                             hi[i], lo[i]);
        if (staged) {
#pragma unroll
          for (int v = 0; v < 2; ++v) {
            const int ch8 = (cc & 3) * 2 + v;
            const uint32_t o = (cc >> 2) * kRBox + srow * 128 + ((ch8 ^ (srow & 7)) << 4);
            *reinterpret_cast<uint4*>(shi + o) = make_uint4(hi[4 * v], hi[4 * v + 1], hi[4 * v + 2], hi[4 * v + 3]);
            *reinterpret_cast<uint4*>(slo + o) = make_uint4(lo[4 * v], lo[4 * v + 1], lo[4 * v + 2], lo[4 * v + 3]);
          }
        }
      }
      ptx::fence_proxy_async();
    };
    // one thread: one box of all G tiles per (plane, d half); tiles past the
    // end of the head fall outside the tensor and are not written
    auto store_tiles = [&](const CUtensorMap* map, const uint8_t* shi, const uint8_t* slo) {
      for (int p = 0; p < 2; ++p)
        for (int hf = 0; hf < NH; ++hf)
          ptx::tma_store_4d(map, (p ? slo : shi) + hf * kRBox, hf * 64, 0, c1_0, p * g.BH + bh);
      ptx::bulk_commit();
    };
    ok = ok && ptx::mbar_wait(bar_acc, 0);
    ptx::tc_fence_after();
    if (bf16 && mode != QT_BUFFER) {
      if (tid == 0) ptx::bulk_wait_read();   // the q copy has read the A lo plane
      ptx::named_bar(bar_row, kRtcRowThreads);
    }
    // k~ (f16 planes): hi plane staged over the A lo plane, lo plane over K
    // (both read by now: S and k~ are complete)
    stage_row(sA + NH * kRBox, sK, final_step != 0);
    ptx::named_bar(bar_row, kRtcRowThreads);
    if (tid == 0 && ok) store_tiles(&maps.kt, sA + NH * kRBox, sK);
    if (final_step) {
      ok = ok && ptx::mbar_wait(bar_acc, 1);
      ptx::tc_fence_after();
      if (tid == 0) ptx::bulk_wait_read();   // the k~ stores have read their staging
      ptx::named_bar(bar_row, kRtcRowThreads);
      // z: hi plane over the A hi plane (V is consumed), lo over the A lo plane
      stage_row(sA, sA + NH * kRBox, false);
      ptx::named_bar(bar_row, kRtcRowThreads);
      if (tid == 0 && ok) store_tiles(&maps.z, sA, sA + NH * kRBox);
    }
    if (tid == 0) {
      if (done) ptx::bulk_wait_all(); else ptx::bulk_wait_read();
    }
    if (done) __threadfence();   // this thread's h store, before the count below
  }
  ptx::tc_fence_before();
  ptx::named_bar(bar_all, kRtcThreads);
  if (done && tid == 0) {
    // the TMA stores are complete (waited above by the threads that issued
    // them); order them and the h stores before the release of the count
    ptx::fence_proxy_async_global();
    __threadfence();
    ptx::red_release_add(done, 1);
  }
}

// grid (ceil(b1k / G), BH), block kRtcThreads; 1 <= G <= floor(128 / r8).
// Two CTAs (18 warps, five on some SM sub-partition) leave 96 registers a thread.
template <typename TQ, int D>
__global__ void __launch_bounds__(kRtcThreads, 2)
r_step_tc5(const __grid_constant__ RtcMaps maps, const TQ* __restrict__ q, Work w, TcPlanes<TQ> out, Geo g,
           int mode, int final_step, int G) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (tc::smem_misaligned(smem_raw)) return;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(smem_raw + rtc_tmem_slot<D>());
  if (threadIdx.x < 32) {
    ptx::tmem_alloc(sTmem, 256);
    ptx::tmem_relinquish();
  }
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  // dependents may start once every CTA of this grid holds its TMEM, so none
  // of theirs can take the columns a CTA of this grid still has to allocate
  ptx::griddep_launch();
  const uint32_t tmem = *sTmem;
  r_step_item<TQ, D>(maps, q, w, out, g, mode, final_step, G, blockIdx.x * G, blockIdx.y, smem_raw, tmem,
                     threadIdx.x, 0, 1, 2, nullptr, 0, nullptr);
  ptx::tc_fence_before();
  __syncthreads();
  if (threadIdx.x < 32) ptx::tmem_dealloc(tmem, 256);
}

}  // namespace monarch
