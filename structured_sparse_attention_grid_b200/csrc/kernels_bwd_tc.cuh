// tcgen05 kernels of the L-step backward for bf16 / f16 inputs (one-step
// forward, self-attention, optional frame-chunk causal mask).  Per position
// a2 the L step is a softmax attention of the queries q over the key tiles k~
// with values z and a per-key bias h, so its backward is
//   P = 2^(s log2(e) q.k~ + h - lse),  dS = P (dy.z - D),  D = dy.y,
//   dq = s dS k~,  dk~ = s dS^T q,  dz = P^T dy,  dh = colsum(dS).
//
// Two kernels, each with 128 rows on the TMEM lanes and 128-wide blocks of
// the other side streamed through shared memory:
//   l_bwd_kv: rows = key tiles c1, blocks of queries.
//     X = S^T = k~ q^T,  Y = dP^T = z dy^T        (shared-memory operands)
//     P^T, dS^T written over X, Y as f16 hi/lo    (A operands in TMEM)
//     dz += P^T dy,  dk~ += dS^T q                (accumulators in TMEM)
//   l_bwd_q:  rows = queries a1, blocks of key tiles.
//     X = S = q k~^T,  Y = dP = dy z^T;  dS over Y;  dq += dS k~.
//
// Precision: dS = P (dP - D) cancels where P is peaked, so a relative error e
// of dP becomes e |z| / |z - y| in dS.  Every operand of every product is
// therefore carried as f16 hi + lo planes where it is not exact: k~, z (from
// the R step), dy (scaled by a power of two sigma per head so that
// max |sigma dy| lies in [1/2, 1)), P and dS; q is exact in f16.  A product
// of two split operands takes three MMAs (hi hi, lo hi, hi lo).  dS is scaled
// by kDsShift = 16 before its split; fp32 accumulation throughout.
//
// TMEM (512 columns): X [0, 128), Y [128, 256), accumulators from 256.  A
// 16-column group of X or Y that held 16 scores holds, after the softmax, the
// hi values of those 16 entries in its first 8 columns and the lo values in
// the last 8 (two f16 per column): per 16 entries of K, the A operand of one
// MMA for each plane.
//
// Warps 0-15 run the softmax: warp w owns TMEM lanes 32 (w mod 4) .. + 31 and
// the 32 columns 32 (w / 4) .. + 31 of each block (later a quarter of d in the
// epilogue).  Warp 16 issues the MMAs, warp 17 the TMA loads.
// Each block's products that read P or dS are issued before the next block's
// score products, and one thread's MMAs run in issue order, so the next
// scores never overwrite an operand still in use.
//
// Overlap: the streamed operands have their own refill barriers, released in
// the order their last readers finish (l_bwd_kv: q after dk~, dy after dz;
// l_bwd_q: z right after dP, k~ after dq), so the next block's loads run under
// the current block's products.  The score and dP products commit separately
// and the softmax computes P while dP is still being formed.
#pragma once

#include "tc_common.cuh"
#include "kernels_bwd.cuh"

namespace monarch {
namespace tcb {

using tc::kBox;
constexpr int kSoftWarps = 16;                 // 4 lane quadrants x 4 column quarters
constexpr int kThreads = 32 * (kSoftWarps + 2);
constexpr int kMmaWarp = kSoftWarps;
constexpr int kLoadWarp = kSoftWarps + 1;
constexpr int kSoftThreads = 32 * kSoftWarps;
constexpr int kBlk = 128;                      // rows per tile and columns per streamed block
constexpr float kDsShift = 16.f;               // dS is split as 16 dS (range and subnormals)

struct BwdMaps {
  CUtensorMap dy;   // sigma dy planes  {d, b1q, 2*BH*b2}  box {64, 64, 1}  (f16)
  CUtensorMap dd;   // sigma D          {b1q_pad, BH*b2}   box {64, 1}      (f32)
};

// Power-of-two scale that maps the largest |dy| of a head into [1/2, 1).
__device__ __forceinline__ float dy_sigma(float amax) {
  if (!(amax > 0.f) || !(amax < INFINITY)) return 1.f;
  int e;
  frexpf(amax, &e);
  e = max(-120, min(120, e));
  return ldexpf(1.f, -e);
}

template <int D>
constexpr size_t kv_smem() {
  constexpr int NH = D / 64;
  return (size_t)2 * (2 * NH * 2 * kBox) /* k~, z planes */ + (size_t)NH * 2 * kBox /* q */ +
         (size_t)2 * NH * 2 * kBox /* dy planes */ + 2 * kBlk * 4 /* lse, D */ + 2 * kBlk * 4 /* dh partial sums */ +
         16 * 8 /* 9 barriers, TMEM address */;
}

template <int D>
constexpr size_t q_smem() {
  constexpr int NH = D / 64;
  return (size_t)NH * 2 * kBox /* q */ + (size_t)2 * NH * 2 * kBox /* dy planes */ +
         (size_t)2 * (2 * NH * 2 * kBox) /* k~, z planes */ + kBlk * 4 /* h */ + 16 * 8;
}

// The softmax of one 16-column group, in two phases so that the first runs
// while the dP products are still being computed:
//   softmax_p:  reads 16 scores X of this thread's row, forms P = 2^(x sl2 +
//               off(j)) (0 where keep(j) is false) and writes its f16 hi/lo
//               planes over the group (hi in the first 8 columns, lo in the
//               last 8);
//   softmax_ds: reads P back (hi + lo, about 22 bits) and 16 values Y, forms
//               dS = P (y - dd(j)) and writes the hi/lo planes of kDsShift dS
//               over the group of Y.  Accumulates dS into dsum; tracks
//               max |kDsShift dS|.
template <typename Off, typename Keep>
__device__ __forceinline__ void softmax_p(uint32_t tx, float sl2, Off off, Keep keep) {
  uint32_t xr[16];
  ptx::tmem_ld16(tx, xr);
  ptx::tmem_wait_ld();
  uint32_t phi[8], plo[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int j = 2 * e;
    float p0 = ptx::ex2(fmaf(__uint_as_float(xr[j]), sl2, off(j)));
    float p1 = ptx::ex2(fmaf(__uint_as_float(xr[j + 1]), sl2, off(j + 1)));
    if (!keep(j)) p0 = 0.f;
    if (!keep(j + 1)) p1 = 0.f;
    tc::split2<__half>(make_float2(p0, p1), phi[e], plo[e]);
  }
  ptx::tmem_st8(tx, phi);
  ptx::tmem_st8(tx + 8, plo);
}

template <typename Dv>
__device__ __forceinline__ void softmax_ds(uint32_t tx, uint32_t ty, Dv dd, float& dsum, float& dmax) {
  uint32_t pr[16], yr[16];
  ptx::tmem_ld16(tx, pr);
  ptx::tmem_ld16(ty, yr);
  ptx::tmem_wait_ld();
  uint32_t shi[8], slo[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int j = 2 * e;
    const float2 ph = __half22float2(*reinterpret_cast<const __half2*>(&pr[e]));
    const float2 pl = __half22float2(*reinterpret_cast<const __half2*>(&pr[8 + e]));
    const float d0 = (ph.x + pl.x) * (__uint_as_float(yr[j]) - dd(j));
    const float d1 = (ph.y + pl.y) * (__uint_as_float(yr[j + 1]) - dd(j + 1));
    dsum += d0 + d1;
    const float2 ds = make_float2(d0 * kDsShift, d1 * kDsShift);
    dmax = fmaxf(dmax, fmaxf(fabsf(ds.x), fabsf(ds.y)));
    tc::split2<__half>(ds, shi[e], slo[e]);
  }
  ptx::tmem_st8(ty, shi);
  ptx::tmem_st8(ty + 8, slo);
}

// Two-phase variant for the dq kernel, where only dS is an MMA operand:
//   softmax_p_regs: P of 16 columns from X, kept in registers as 8 packed f16
//                   pairs (P only scales dP - D, so one f16 rounding of P is a
//                   2^-11 relative error of dS, with no cancellation);
//   softmax_ds_regs: dS = P (y - dd) from those registers and 16 values Y,
//                   written over the group of Y as hi/lo planes of kDsShift dS.
template <typename Off, typename Keep>
__device__ __forceinline__ void softmax_p_regs(uint32_t tx, float sl2, Off off, Keep keep, uint32_t (&ph)[8]) {
  uint32_t xr[16];
  ptx::tmem_ld16(tx, xr);
  ptx::tmem_wait_ld();
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int j = 2 * e;
    float p0 = ptx::ex2(fmaf(__uint_as_float(xr[j]), sl2, off(j)));
    float p1 = ptx::ex2(fmaf(__uint_as_float(xr[j + 1]), sl2, off(j + 1)));
    if (!keep(j)) p0 = 0.f;
    if (!keep(j + 1)) p1 = 0.f;
    const __half2 h = __floats2half2_rn(p0, p1);
    ph[e] = *reinterpret_cast<const uint32_t*>(&h);
  }
}

__device__ __forceinline__ void softmax_ds_regs(uint32_t ty, const uint32_t (&ph)[8], float dd, float& dmax) {
  uint32_t yr[16];
  ptx::tmem_ld16(ty, yr);
  ptx::tmem_wait_ld();
  uint32_t shi[8], slo[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float2 p = __half22float2(*reinterpret_cast<const __half2*>(&ph[e]));
    const float2 ds = make_float2(p.x * (__uint_as_float(yr[2 * e]) - dd) * kDsShift,
                                  p.y * (__uint_as_float(yr[2 * e + 1]) - dd) * kDsShift);
    dmax = fmaxf(dmax, fmaxf(fabsf(ds.x), fabsf(ds.y)));
    tc::split2<__half>(ds, shi[e], slo[e]);
  }
  ptx::tmem_st8(ty, shi);
  ptx::tmem_st8(ty + 8, slo);
}

// The two MMA shapes of both kernels, issued by one thread (f16 operands,
// f32 accumulation in TMEM):
//   mma_scores: D[128 x 128] (+)= A[128 x d] B[128 x d]^T, both K-major
//               (d along the 128-byte swizzled rows): scores and dP;
//   mma_accum:  D[128 x d] += A[128 x 128] B[128 x d], A in TMEM (plane pa of
//               the [hi 8 | lo 8] groups), B MN-major: the accumulations.
template <int D>
__device__ __forceinline__ void mma_scores(uint32_t td, uint32_t a, uint32_t b, bool first) {
  constexpr int NH = D / 64;
  constexpr uint32_t idS = ptx::idesc_f16(128, kBlk, 0, 0, 0);
  const uint64_t da = ptx::sw128_desc(a, 16, 1024), db = ptx::sw128_desc(b, 16, 1024);
#pragma unroll
  for (int hf = 0; hf < NH; ++hf)
#pragma unroll
    for (int k4 = 0; k4 < 4; ++k4)
      ptx::mma_f16_ss(td, da + ((hf * 2 * kBox + k4 * 32) >> 4), db + ((hf * 2 * kBox + k4 * 32) >> 4), idS,
                      !(first && hf == 0 && k4 == 0));
}

template <int D>
__device__ __forceinline__ void mma_accum(uint32_t tacc, uint32_t ta, int pa, uint32_t b, bool first) {
  constexpr uint32_t idA = ptx::idesc_f16(128, D, 0, 0, 1);
  const uint64_t db = ptx::sw128_desc(b, 2 * kBox, 1024);
#pragma unroll
  for (int kk = 0; kk < kBlk / 16; ++kk)
    ptx::mma_f16_ts(tacc, ta + kk * 16 + pa * 8, db + ((kk * 2048) >> 4), idA, !(first && kk == 0));
}

// Writes 16 accumulator columns of this thread's row, times `scale`, as f32
// with two 32-byte stores (dst is a workspace row: 32-byte aligned).
__device__ __forceinline__ void store_acc16(uint32_t taddr, float scale, float* dst, bool ok) {
  uint32_t o[16];
  ptx::tmem_ld16(taddr, o);
  ptx::tmem_wait_ld();
  if (!ok) return;
  uint32_t a[8], b[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    a[i] = __float_as_uint(__uint_as_float(o[i]) * scale);
    b[i] = __float_as_uint(__uint_as_float(o[8 + i]) * scale);
  }
  ptx::st_global_v8(dst, a);
  ptx::st_global_v8(dst + 8, b);
}

// ===========================================================================
// dk~, dz, dh for 128 key tiles of one (head, position a2).
// grid (ceil(b1k/128), b2, BH), block kThreads, dynamic smem kv_smem<D>().
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
l_bwd_kv(const __grid_constant__ tc::Maps maps, const __grid_constant__ BwdMaps bmaps, const float* __restrict__ hbuf,
         const unsigned* __restrict__ amax, float* __restrict__ dkt, float* __restrict__ dz, float* __restrict__ dh,
         Geo g) {
  constexpr int NH = D / 64;
  constexpr uint32_t kPl = NH * 2 * kBox;   // one 128-row operand plane: [d half][row half][64 rows][128 B]
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (tc::smem_misaligned(smem_raw)) return;
  uint8_t* sK = smem_raw;               // k~ [plane]
  uint8_t* sZ = sK + 2 * kPl;           // z  [plane]
  uint8_t* sQ = sZ + 2 * kPl;           // q
  uint8_t* sY = sQ + kPl;               // sigma dy [plane]
  float* sL = reinterpret_cast<float*>(sY + 2 * kPl);   // lse of the block's queries
  float* sD = sL + kBlk;                                // sigma D
  float* sX = sD + kBlk;                                // dh partial sums of the column quarters
  uint64_t* bar = reinterpret_cast<uint64_t*>(sX + 2 * kBlk);
  uint64_t* k_full = bar + 0;
  uint64_t* q_full = bar + 1;    // q, lse, D of a query block
  uint64_t* q_free = bar + 2;
  uint64_t* s_full = bar + 3;    // X = S^T complete
  uint64_t* p_full = bar + 4;    // the softmax wrote P^T and dS^T
  uint64_t* o_done = bar + 5;
  uint64_t* y_full = bar + 6;    // dy planes of a query block
  uint64_t* y_free = bar + 7;
  uint64_t* d_full = bar + 8;    // Y = dP^T complete
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bar + 9);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int a2 = blockIdx.y, bh = blockIdx.z;
  const int kb = blockIdx.x * kBlk;
  const int zrow = bh * g.b2 + a2;
  const int rows = g.BH * g.b2;
  const int nqb = (g.b1q + kBlk - 1) / kBlk;
  const int qb0 = query_start(g, kb) / kBlk;   // earlier query blocks see none of these key tiles
  const int nblk = nqb - qb0;

  if (tid == 0) {
    ptx::mbar_init(k_full, 1);
    ptx::mbar_init(q_full, 1);
    ptx::mbar_init(q_free, 1);
    ptx::mbar_init(s_full, 1);
    ptx::mbar_init(p_full, kSoftWarps);
    ptx::mbar_init(o_done, 1);
    ptx::mbar_init(y_full, 1);
    ptx::mbar_init(y_free, 1);
    ptx::mbar_init(d_full, 1);
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
  ptx::griddep_wait();
  const uint32_t tmem = *sTmem;
  const uint32_t tX = tmem, tY = tmem + 128, tZ = tmem + 256, tK = tmem + 256 + D;

  if (warp == kLoadWarp) {
    if (lane == 0) {
      ptx::mbar_expect_tx(k_full, 4 * kPl);
      for (int p = 0; p < 2; ++p)
        for (int hf = 0; hf < NH; ++hf)
          for (int rh = 0; rh < 2; ++rh) {
            const int off = p * kPl + hf * 2 * kBox + rh * kBox;
            ptx::tma_load_3d(sK + off, &maps.kt, k_full, hf * 64, kb + rh * 64, p * rows + zrow);
            ptx::tma_load_3d(sZ + off, &maps.z, k_full, hf * 64, kb + rh * 64, p * rows + zrow);
          }
      // q (with lse, D) and dy are refilled separately: the products of a
      // block release q before dy, so the next q arrives while dz is summed
      bool ok = true;
      for (int j = 0; j < nblk && ok; ++j) {
        const int q0 = (qb0 + j) * kBlk;
        if (j > 0) ok = ptx::mbar_wait(q_free, (j - 1) & 1);
        if (!ok) break;
        ptx::mbar_expect_tx(q_full, kPl + 2 * kBlk * 4);
        for (int hf = 0; hf < NH; ++hf)
          for (int rh = 0; rh < 2; ++rh)
            ptx::tma_load_3d(sQ + hf * 2 * kBox + rh * kBox, &maps.qb, q_full, hf * 64, q0 + rh * 64, zrow);
        for (int rh = 0; rh < 2; ++rh) {
          tc::tma_load_2d(sL + rh * 64, &maps.lse, q_full, q0 + rh * 64, zrow);
          tc::tma_load_2d(sD + rh * 64, &bmaps.dd, q_full, q0 + rh * 64, zrow);
        }
        if (j > 0) ok = ptx::mbar_wait(y_free, (j - 1) & 1);
        if (!ok) break;
        ptx::mbar_expect_tx(y_full, 2 * kPl);
        for (int p = 0; p < 2; ++p)
          for (int hf = 0; hf < NH; ++hf)
            for (int rh = 0; rh < 2; ++rh)
              ptx::tma_load_3d(sY + p * kPl + hf * 2 * kBox + rh * kBox, &bmaps.dy, y_full, hf * 64, q0 + rh * 64,
                               p * rows + zrow);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t aK = ptx::smem_u32(sK), aZ = ptx::smem_u32(sZ), aQ = ptx::smem_u32(sQ), aY = ptx::smem_u32(sY);
      // score-like product: rows x 128 columns over K = d
      auto scores = [&](uint32_t td, uint32_t a, uint32_t b, bool first) { mma_scores<D>(td, a, b, first); };
      auto accum = [&](uint32_t tacc, uint32_t ta, int pa, uint32_t b, bool first) {
        mma_accum<D>(tacc, ta, pa, b, first);
      };
      bool ok = ptx::mbar_wait(k_full, 0);
      for (int j = 0; j < nblk && ok; ++j) {
        ok = ptx::mbar_wait(q_full, j & 1);
        ptx::tc_fence_after();
        if (!ok) break;
        scores(tX, aK, aQ, true);              // S^T = k~_hi q^T + k~_lo q^T
        scores(tX, aK + kPl, aQ, false);
        ptx::mma_commit(s_full);
        ok = ptx::mbar_wait(y_full, j & 1);
        ptx::tc_fence_after();
        if (!ok) break;
        scores(tY, aZ, aY, true);              // dP^T = z dy^T (hi hi, lo hi, hi lo)
        scores(tY, aZ + kPl, aY, false);
        scores(tY, aZ, aY + kPl, false);
        ptx::mma_commit(d_full);
        ok = ptx::mbar_wait(p_full, j & 1);
        ptx::tc_fence_after();
        if (!ok) break;
        accum(tK, tY, 0, aQ, j == 0);          // dk~ += dS^T q
        accum(tK, tY, 1, aQ, false);
        ptx::mma_commit(q_free);
        accum(tZ, tX, 0, aY, j == 0);          // dz += P^T dy
        accum(tZ, tX, 1, aY, false);
        accum(tZ, tX, 0, aY + kPl, false);
        ptx::mma_commit(y_free);
      }
      ptx::mma_commit(o_done);
    }
  } else {
    const int qd = warp & 3, cq = warp >> 2;   // lane quadrant, column quarter
    const int r = 32 * qd + lane;
    const int c1 = kb + r;
    const bool row_ok = c1 < g.b1k;
    const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
    const int qstart = query_start(g, row_ok ? c1 : g.b1k - 1);
    const float hb = row_ok ? hbuf[(long long)zrow * g.b1k_pad + c1] : 0.f;
    float dsum = 0.f, dmax = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      const int q0 = (qb0 + j) * kBlk;
      ok = ok && ptx::mbar_wait(s_full, j & 1) && ptx::mbar_wait(q_full, j & 1);
      ptx::tc_fence_after();
      const int lim = min(kBlk, g.b1q - q0);   // valid queries of the block
      const int lo = qstart - q0;              // queries below this one do not see the key tile
#pragma unroll
      for (int g16 = 0; g16 < 2; ++g16) {      // P^T while dP^T is computed
        const int cb = 32 * cq + 16 * g16;
        const float* l = sL + cb;
        softmax_p(tX + lane_off + cb, g.sl2, [&](int jj) { return hb - l[jj]; },
                  [&](int jj) { return cb + jj < lim && cb + jj >= lo; });
      }
      ptx::tmem_wait_st();   // P is read back below
      ok = ok && ptx::mbar_wait(d_full, j & 1);
      ptx::tc_fence_after();
#pragma unroll
      for (int g16 = 0; g16 < 2; ++g16) {
        const int cb = 32 * cq + 16 * g16;
        const float* dv = sD + cb;
        softmax_ds(tX + lane_off + cb, tY + lane_off + cb, [&](int jj) { return dv[jj]; }, dsum, dmax);
      }
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(p_full);
    }
    if (dmax >= 65504.f) atomicExch(&ptx::g_device_error, ptx::kErrRange);
    // dh = the four quarters' sums: 1 -> 0 and 3 -> 2, then 2 -> 0
    if (cq & 1) sX[(cq >> 1) * kBlk + r] = dsum;
    ptx::named_bar(1, kSoftThreads);
    if (!(cq & 1)) dsum += sX[(cq >> 1) * kBlk + r];
    ptx::named_bar(1, kSoftThreads);
    if (cq == 2) sX[r] = dsum;
    ptx::named_bar(1, kSoftThreads);
    ok = ok && ptx::mbar_wait(o_done, 0);
    ptx::tc_fence_after();
    const float inv = 1.f / dy_sigma(__uint_as_float(amax[bh]));
    const float s = g.sl2 * (1.f / kLog2e);
    const long long o = ((long long)zrow * g.b1k + (row_ok ? c1 : 0)) * D + cq * (D / 4);
#pragma unroll 1
    for (int cc = 0; cc < D / 64; ++cc) {
      store_acc16(tZ + lane_off + cq * (D / 4) + 16 * cc, inv, dz + o + 16 * cc, row_ok && ok);
      store_acc16(tK + lane_off + cq * (D / 4) + 16 * cc, inv * s / kDsShift, dkt + o + 16 * cc, row_ok && ok);
    }
    if (cq == 0 && row_ok && ok) dh[(long long)zrow * g.b1k_pad + c1] = (dsum + sX[r]) * inv;
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 512);
}

// ===========================================================================
// L-step dq for 128 queries of one (head, position a2).
// grid (ceil(b1q/128), b2, BH), block kThreads, dynamic smem q_smem<D>().
template <int D>
__global__ void __launch_bounds__(kThreads, 1)
l_bwd_q(const __grid_constant__ tc::Maps maps, const __grid_constant__ BwdMaps bmaps, const float* __restrict__ lse,
        const float* __restrict__ ddv, const unsigned* __restrict__ amax, float* __restrict__ dq, Geo g) {
  constexpr int NH = D / 64;
  constexpr uint32_t kPl = NH * 2 * kBox;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  if (tc::smem_misaligned(smem_raw)) return;
  uint8_t* sQ = smem_raw;               // q
  uint8_t* sY = sQ + kPl;               // sigma dy [plane]
  uint8_t* sK = sY + 2 * kPl;           // k~ [plane]
  uint8_t* sZ = sK + 2 * kPl;           // z  [plane]
  float* sH = reinterpret_cast<float*>(sZ + 2 * kPl);   // h of the block's key tiles (bits)
  uint64_t* bar = reinterpret_cast<uint64_t*>(sH + kBlk);
  uint64_t* c_full = bar + 0;
  uint64_t* k_full = bar + 1;    // k~ planes and h of a key block
  uint64_t* k_free = bar + 2;
  uint64_t* s_full = bar + 3;    // X = S complete
  uint64_t* p_full = bar + 4;    // the softmax wrote dS
  uint64_t* o_done = bar + 5;
  uint64_t* z_full = bar + 6;    // z planes of a key block
  uint64_t* z_free = bar + 7;
  uint64_t* d_full = bar + 8;    // Y = dP complete
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bar + 9);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int a2 = blockIdx.y, bh = blockIdx.z;
  const int ab = blockIdx.x * kBlk;
  const int zrow = bh * g.b2 + a2;
  const int rows = g.BH * g.b2;
  const int kmax = key_limit(g, min(ab + kBlk, g.b1q) - 1);   // key tiles any row of this CTA sees
  const int nblk = (kmax + kBlk - 1) / kBlk;

  if (tid == 0) {
    ptx::mbar_init(c_full, 1);
    ptx::mbar_init(k_full, 1);
    ptx::mbar_init(k_free, 1);
    ptx::mbar_init(s_full, 1);
    ptx::mbar_init(p_full, kSoftWarps);
    ptx::mbar_init(o_done, 1);
    ptx::mbar_init(z_full, 1);
    ptx::mbar_init(z_free, 1);
    ptx::mbar_init(d_full, 1);
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
  ptx::griddep_wait();
  const uint32_t tmem = *sTmem;
  const uint32_t tX = tmem, tY = tmem + 128, tA = tmem + 256;

  if (warp == kLoadWarp) {
    if (lane == 0) {
      ptx::mbar_expect_tx(c_full, 3 * kPl);
      for (int hf = 0; hf < NH; ++hf)
        for (int rh = 0; rh < 2; ++rh) {
          ptx::tma_load_3d(sQ + hf * 2 * kBox + rh * kBox, &maps.qb, c_full, hf * 64, ab + rh * 64, zrow);
          for (int p = 0; p < 2; ++p)
            ptx::tma_load_3d(sY + p * kPl + hf * 2 * kBox + rh * kBox, &bmaps.dy, c_full, hf * 64, ab + rh * 64,
                             p * rows + zrow);
        }
      // z is released right after the dP products, k~ (with h) after the dq
      // products: the next z arrives during the softmax
      bool ok = true;
      for (int j = 0; j < nblk && ok; ++j) {
        if (j > 0) ok = ptx::mbar_wait(z_free, (j - 1) & 1);
        if (!ok) break;
        ptx::mbar_expect_tx(z_full, 2 * kPl);
        for (int p = 0; p < 2; ++p)
          for (int hf = 0; hf < NH; ++hf)
            for (int rh = 0; rh < 2; ++rh)
              ptx::tma_load_3d(sZ + p * kPl + hf * 2 * kBox + rh * kBox, &maps.z, z_full, hf * 64, j * kBlk + rh * 64,
                               p * rows + zrow);
        if (j > 0) ok = ptx::mbar_wait(k_free, (j - 1) & 1);
        if (!ok) break;
        ptx::mbar_expect_tx(k_full, 2 * kPl + kBlk * 4);
        for (int p = 0; p < 2; ++p)
          for (int hf = 0; hf < NH; ++hf)
            for (int rh = 0; rh < 2; ++rh)
              ptx::tma_load_3d(sK + p * kPl + hf * 2 * kBox + rh * kBox, &maps.kt, k_full, hf * 64, j * kBlk + rh * 64,
                               p * rows + zrow);
        for (int rh = 0; rh < 2; ++rh) tc::tma_load_2d(sH + rh * 64, &maps.h, k_full, j * kBlk + rh * 64, zrow);
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      const uint32_t aK = ptx::smem_u32(sK), aZ = ptx::smem_u32(sZ), aQ = ptx::smem_u32(sQ), aY = ptx::smem_u32(sY);
      auto scores = [&](uint32_t td, uint32_t a, uint32_t b, bool first) { mma_scores<D>(td, a, b, first); };
      auto accum = [&](uint32_t tacc, uint32_t ta, int pa, uint32_t b, bool first) {
        mma_accum<D>(tacc, ta, pa, b, first);
      };
      bool ok = ptx::mbar_wait(c_full, 0);
      for (int j = 0; j < nblk && ok; ++j) {
        ok = ptx::mbar_wait(k_full, j & 1);
        ptx::tc_fence_after();
        if (!ok) break;
        scores(tX, aQ, aK, true);              // S = q k~_hi^T + q k~_lo^T
        scores(tX, aQ, aK + kPl, false);
        ptx::mma_commit(s_full);
        ok = ptx::mbar_wait(z_full, j & 1);
        ptx::tc_fence_after();
        if (!ok) break;
        scores(tY, aY, aZ, true);              // dP = dy z^T (hi hi, lo hi, hi lo)
        scores(tY, aY + kPl, aZ, false);
        scores(tY, aY, aZ + kPl, false);
        ptx::mma_commit(d_full);
        ptx::mma_commit(z_free);
        ok = ptx::mbar_wait(p_full, j & 1);
        ptx::tc_fence_after();
        if (!ok) break;
        accum(tA, tY, 0, aK, j == 0);          // dq += dS k~ (hi hi, lo hi, hi lo)
        accum(tA, tY, 1, aK, false);
        accum(tA, tY, 0, aK + kPl, false);
        ptx::mma_commit(k_free);
      }
      ptx::mma_commit(o_done);
    }
  } else {
    const int qd = warp & 3, cq = warp >> 2;   // lane quadrant, column quarter
    const int r = 32 * qd + lane;
    const int a1 = ab + r;
    const bool row_ok = a1 < g.b1q;
    const uint32_t lane_off = (uint32_t)(32 * qd) << 16;
    const long long lr = (long long)zrow * g.b1q_pad + (row_ok ? a1 : 0);
    const float l = lse[lr], dd = ddv[lr];
    const int climit = key_limit(g, row_ok ? a1 : g.b1q - 1);   // visible key tiles [0, climit)
    float dmax = 0.f;
    bool ok = true;
    for (int j = 0; j < nblk; ++j) {
      const int k0 = j * kBlk;
      ok = ok && ptx::mbar_wait(s_full, j & 1) && ptx::mbar_wait(k_full, j & 1);
      ptx::tc_fence_after();
      const int lim = climit - k0;
      uint32_t ph[2][8];   // P of the two 16-column groups (f16 pairs), formed while dP is computed
#pragma unroll
      for (int g16 = 0; g16 < 2; ++g16) {
        const int cb = 32 * cq + 16 * g16;
        const float* hv = sH + cb;
        softmax_p_regs(tX + lane_off + cb, g.sl2, [&](int jj) { return hv[jj] - l; },
                       [&](int jj) { return cb + jj < lim; }, ph[g16]);
      }
      ok = ok && ptx::mbar_wait(d_full, j & 1);
      ptx::tc_fence_after();
#pragma unroll
      for (int g16 = 0; g16 < 2; ++g16)
        softmax_ds_regs(tY + lane_off + 32 * cq + 16 * g16, ph[g16], dd, dmax);
      ptx::tmem_wait_st();
      ptx::tc_fence_before();
      __syncwarp();
      if (lane == 0) ptx::mbar_arrive(p_full);
    }
    if (dmax >= 65504.f) atomicExch(&ptx::g_device_error, ptx::kErrRange);
    ok = ok && ptx::mbar_wait(o_done, 0);
    ptx::tc_fence_after();
    const float scale = g.sl2 * (1.f / kLog2e) / (kDsShift * dy_sigma(__uint_as_float(amax[bh])));
    const long long o = ((long long)zrow * g.b1q + (row_ok ? a1 : 0)) * D + cq * (D / 4);
#pragma unroll 1
    for (int cc = 0; cc < D / 64; ++cc)
      store_acc16(tA + lane_off + cq * (D / 4) + 16 * cc, scale, dq + o + 16 * cc, row_ok && ok);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 512);
}

// ===========================================================================
// Largest |dy| per head (as the bits of a non-negative float, which order like
// unsigned integers).  Grid-stride over the head: each thread takes 16
// consecutive elements per step (four 16-byte or 8-byte loads in flight).
// grid (blocks per head, BH), block 256.
template <typename TG>
__global__ void __launch_bounds__(256) dy_amax(const TG* __restrict__ dy, unsigned* __restrict__ amax, Geo g) {
  const long long n = g.Nq * g.d;   // a multiple of 64
  const TG* p = dy + (long long)blockIdx.y * n;
  float m = 0.f;
  for (long long base = ((long long)blockIdx.x * 256 + threadIdx.x) * 16; base < n;
       base += (long long)gridDim.x * 256 * 16) {
    float4 v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = load4(p + base + 4 * i);
#pragma unroll
    for (int i = 0; i < 4; ++i) m = fmaxf(m, fmaxf(fmaxf(fabsf(v[i].x), fabsf(v[i].y)), fmaxf(fabsf(v[i].z), fabsf(v[i].w))));
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0 && m > 0.f) atomicMax(amax + blockIdx.y, __float_as_uint(m));
}

// One warp per query token: sigma dy as f16 hi/lo planes in block order
// ([plane][BH*b2][b1q][d]) and sigma D = sigma dy . y, y the forward output
// (f32, grid order).  grid (ceil(Nq/8), BH), block 256.
template <typename TG, int D>
__global__ void __launch_bounds__(256)
dy_planes(const TG* __restrict__ dy, const float* __restrict__ y, const unsigned* __restrict__ amax,
          __half* __restrict__ dyp, float* __restrict__ ddv, Geo g) {
  constexpr int PER = D / 32;
  const int bh = blockIdx.y;
  const long long n = (long long)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (n >= g.Nq) return;
  const float sig = dy_sigma(__uint_as_float(amax[bh]));
  // grid token -> (tile a1, position a2)
  const int hw = g.H * g.W;
  const int t = (int)(n / hw), rem = (int)(n - (long long)t * hw);
  const int yy = rem / g.W, xx = rem - yy * g.W;
  const int a1 = (t * (g.H / g.th) + yy / g.th) * g.ntx + xx / g.tw;
  const int a2 = (yy % g.th) * g.tw + xx % g.tw;
  const long long src = ((long long)bh * g.Nq + n) * D;
  const long long zrow = (long long)bh * g.b2 + a2;
  const long long plane = (long long)g.BH * g.b2 * g.b1q * D;
  __half* hi = dyp + (zrow * g.b1q + a1) * D;
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int c = lane + 32 * i;
    const float v = to_f(dy[src + c]) * sig;
    dot = fmaf(v, y[src + c], dot);
    const __half h = __float2half_rn(v);
    hi[c] = h;
    hi[plane + c] = __float2half_rn(v - __half2float(h));
  }
  dot = warp_sum(dot);
  if (lane == 0) ddv[zrow * g.b1q_pad + a1] = dot;
}

}  // namespace tcb
}  // namespace monarch
