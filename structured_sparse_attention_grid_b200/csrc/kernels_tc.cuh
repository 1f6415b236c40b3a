// Tensor-core (tcgen05 + TMA) kernels of the L step for bf16 / f16 inputs.
//
// Precision scheme (fp32 statistics and accumulation everywhere):
//   * s q.k~    : q is exact in its input type; k~ is stored as two planes
//                 hi = round(k~), lo = round(k~ - hi) of that type and both
//                 products accumulate into one TMEM tile (16 significant bits).
//   * L z       : P = 2^(x - m) rounded to f16 (the row sum adds the rounded
//                 values, so the weights stay exactly normalised); z is two
//                 f16 planes (hi, lo).
//   * L^T q     : L is split into hi / lo planes of the input type.
//
// Layout of every shared-memory operand tile: 64-element (128-byte) column
// halves, each [rows][128 B] with the 128-byte swizzle, 1024-byte aligned.
// This serves as a K-major operand (K = the 128-byte direction) and as an
// MN-major operand (MN = the 128-byte direction, K = rows).
#pragma once

#include "common.cuh"
#include "ptx.cuh"

namespace monarch {

template <typename T> struct TcType;
template <> struct TcType<__nv_bfloat16> {
  static constexpr int kBf16 = 1;
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  static __device__ __forceinline__ float round(float a) { return __bfloat162float(__float2bfloat16_rn(a)); }
};
template <> struct TcType<__half> {
  static constexpr int kBf16 = 0;
  static __device__ __forceinline__ uint32_t pack(float a, float b) {
    __half2 v = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&v);
  }
  static __device__ __forceinline__ float round(float a) { return __half2float(__float2half_rn(a)); }
};

constexpr int kTile = 128;          // rows of every tensor-core tile
constexpr int kHalfBytes = 16384;   // one [128 rows][128 B] swizzled half
constexpr float kColShift = 15.f;   // L^T q: L scaled by 2^15 (the ratio is unchanged)
constexpr float kLazyRescale = 8.f; // row pass: shift moves only when the max grows by > 2^8

// Gathers the 128 query rows (a1 = blk*128 + r) of position a2 into a
// swizzled operand tile with cp.async; thread r copies row r.  Rows past b1q
// are zero-filled.  The grid -> (tile, position) permutation happens here.
template <typename TQ, int D>
__device__ __forceinline__ void gather_q_rows(uint8_t* sQ, const TQ* qh, const Geo& g, int a1_base, int a2,
                                              int r) {
  const int a1 = a1_base + r;
  const bool valid = a1 < g.b1q;
  const TQ* src = qh + (valid ? token_of(g, a1, a2) * D : 0);
  const uint32_t dst = ptx::smem_u32(sQ);
#pragma unroll
  for (int c = 0; c < D / 8; ++c) {
    const int half = c >> 3, ch = c & 7;
    ptx::cp_async_16(dst + half * kHalfBytes + ptx::sw128_offset(r, ch), src + c * 8, valid ? 16u : 0u);
  }
}

// ---------------------------------------------------------------------------
// L step row pass over key tiles for one (head, position a2, 128 query rows).
//   S = s q.k~ + h  (base 2), online softmax over all key tiles c1.
//   OUT:  out[token(a1,a2)] = sum_c1 L z  (inverse permutation fused into the store)
//   !OUT: lse[a1] = log2 sum_c1 2^S
// grid (ceil(b1q/128), b2, BH), block 128 (thread r owns row r / TMEM lane r).
template <typename TQ, typename TO, int D, bool OUT>
__global__ void __launch_bounds__(128, 1)
l_row_tc(const TQ* __restrict__ q, TO* __restrict__ out, const __grid_constant__ CUtensorMap tm_kt,
         const __grid_constant__ CUtensorMap tm_z, const float* __restrict__ hbuf, float* __restrict__ lse, Geo g) {
  constexpr int NH = D / 64;                        // 128-byte halves per row
  constexpr uint32_t kQBytes = NH * kHalfBytes;
  constexpr uint32_t kPlane = NH * kHalfBytes;      // one k~ or z plane tile
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sQ = base;
  uint8_t* sK = sQ + kQBytes;                        // hi plane, lo plane
  uint8_t* sZ = sK + 2 * kPlane;                     // hi plane, lo plane (OUT)
  uint8_t* sP = sZ + (OUT ? 2 * kPlane : 0);         // 2 halves of 128 keys (OUT)
  float* sH = reinterpret_cast<float*>(sP + (OUT ? 2 * kHalfBytes : 0));
  uint64_t* bars = reinterpret_cast<uint64_t*>(sH + kTile);
  uint64_t* bar_k = bars + 0;
  uint64_t* bar_z = bars + 1;
  uint64_t* bar_s = bars + 2;
  uint64_t* bar_o = bars + 3;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 4);
  int* sFail = reinterpret_cast<int*>(sTmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int a2 = blockIdx.y, bh = blockIdx.z;
  const int a1_base = blockIdx.x * kTile;
  const int zrow = bh * g.b2 + a2;                  // row of (bh, a2) in a plane
  const int plane_rows = g.BH * g.b2;
  const int nkb = (g.b1k + kTile - 1) / kTile;

  if (tid == 0) {
    ptx::mbar_init(bar_k, 1);
    ptx::mbar_init(bar_z, 1);
    ptx::mbar_init(bar_s, 1);
    ptx::mbar_init(bar_o, 1);
    ptx::fence_mbar_init();
    *sFail = 0;
    ptx::prefetch_tmap(&tm_kt);
    if (OUT) ptx::prefetch_tmap(&tm_z);
  }
  if (warp == 0) {
    ptx::tmem_alloc(sTmem, 256);
    ptx::tmem_relinquish();
  }
  gather_q_rows<TQ, D>(sQ, q + (long long)bh * g.Nq * D, g, a1_base, a2, tid);
  ptx::cp_async_commit();
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t tS = tmem, tO = tmem + 128;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;

  if (tid == 0) {
    ptx::mbar_expect_tx(bar_k, 2 * kPlane);
    for (int p = 0; p < 2; ++p)
      for (int hf = 0; hf < NH; ++hf)
        ptx::tma_load_3d(sK + p * kPlane + hf * kHalfBytes, &tm_kt, bar_k, hf * 64, 0, p * plane_rows + zrow);
    if (OUT) {
      ptx::mbar_expect_tx(bar_z, 2 * kPlane);
      for (int p = 0; p < 2; ++p)
        for (int hf = 0; hf < NH; ++hf)
          ptx::tma_load_3d(sZ + p * kPlane + hf * kHalfBytes, &tm_z, bar_z, hf * 64, 0, p * plane_rows + zrow);
    }
  }
  ptx::cp_async_wait<0>();
  ptx::fence_proxy_async();
  __syncthreads();

  constexpr uint32_t idS = ptx::idesc_f16(128, 128, TcType<TQ>::kBf16, 0, 0);
  constexpr uint32_t idPV = ptx::idesc_f16(128, D, 0, 0, 1);
  const uint32_t aQ = ptx::smem_u32(sQ), aK = ptx::smem_u32(sK), aZ = ptx::smem_u32(sZ), aP = ptx::smem_u32(sP);
  const float* hrow = hbuf + (long long)zrow * g.b1k;

  float m = -INFINITY, l = 0.f;
  bool ok = true;
  for (int j = 0; j < nkb; ++j) {
    const int kb = j * kTile;
    sH[tid] = (kb + tid < g.b1k) ? hrow[kb + tid] * kLog2e : -INFINITY;  // -inf masks ragged keys
    if (tid == 0) {
      // S = q k~_hi^T + q k~_lo^T  (A: q, K-major; B: k~, K-major)
      if (!ptx::mbar_wait(bar_k, j & 1)) *sFail = 1;
      ptx::tc_fence_after();
#pragma unroll
      for (int p = 0; p < 2; ++p)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          ptx::mma_f16_ss(tS, ptx::sw128_desc(aQ + off, 16, 1024),
                          ptx::sw128_desc(aK + p * kPlane + off, 16, 1024), idS, (p | kk) != 0);
        }
      ptx::mma_commit(bar_s);
    }
    ok = ptx::mbar_wait(bar_s, j & 1);
    ptx::tc_fence_after();
    __syncthreads();  // sH visible
    if (tid == 0 && j + 1 < nkb) {
      // k~ tile consumed: fetch the next one while the softmax runs
      ptx::mbar_expect_tx(bar_k, 2 * kPlane);
      for (int p = 0; p < 2; ++p)
        for (int hf = 0; hf < NH; ++hf)
          ptx::tma_load_3d(sK + p * kPlane + hf * kHalfBytes, &tm_kt, bar_k, hf * 64, kb + kTile,
                           p * plane_rows + zrow);
    }
    if (OUT && tid == 0 && j > 0) {
      // the previous L z product finished with S: z buffer is free
      ptx::mbar_expect_tx(bar_z, 2 * kPlane);
      for (int p = 0; p < 2; ++p)
        for (int hf = 0; hf < NH; ++hf)
          ptx::tma_load_3d(sZ + p * kPlane + hf * kHalfBytes, &tm_z, bar_z, hf * 64, kb, p * plane_rows + zrow);
    }

    // ---- softmax of row `tid` over this key tile
    float x[kTile];
#pragma unroll
    for (int cc = 0; cc < kTile / 32; ++cc) {
      uint32_t r[32];
      ptx::tmem_ld32(tS + lane_off + cc * 32, r);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 32; ++i) x[cc * 32 + i] = fmaf(__uint_as_float(r[i]), g.sl2, sH[cc * 32 + i]);
    }
    float mb = -INFINITY;
#pragma unroll
    for (int i = 0; i < kTile; ++i) mb = fmaxf(mb, x[i]);
    // The running shift m moves only when the tile max exceeds it by more than
    // 2^8 (P <= 256 stays exact-range in f16); the accumulator is rescaled then.
    const bool move = mb > m + kLazyRescale;
    const float mn = move ? mb : m;
    const float corr = ptx::ex2(m - mn);  // 0 on the first tile, 1 when m stays
    float sum = 0.f;
    if (OUT) {
      // tcgen05.ld / st are warp-collective: rescale when any lane moved
      if (j > 0 && __any_sync(0xffffffffu, move)) {
#pragma unroll
        for (int cc = 0; cc < D / 32; ++cc) {
          uint32_t r[32];
          ptx::tmem_ld32(tO + lane_off + cc * 32, r);
          ptx::tmem_wait_ld();
#pragma unroll
          for (int i = 0; i < 32; ++i) r[i] = __float_as_uint(__uint_as_float(r[i]) * corr);
          ptx::tmem_st32(tO + lane_off + cc * 32, r);
        }
        ptx::tmem_wait_st();
      }
      // P row (f16) into the swizzled K-major A tile
#pragma unroll
      for (int c = 0; c < kTile / 8; ++c) {
        uint32_t pk[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const __half2 hp = __floats2half2_rn(ptx::ex2(x[c * 8 + 2 * e] - mn), ptx::ex2(x[c * 8 + 2 * e + 1] - mn));
          const float2 f = __half22float2(hp);
          sum += f.x + f.y;
          pk[e] = *reinterpret_cast<const uint32_t*>(&hp);
        }
        const uint32_t dst = aP + (c >> 3) * kHalfBytes + ptx::sw128_offset(tid, c & 7);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(dst), "r"(pk[0]), "r"(pk[1]), "r"(pk[2]),
                     "r"(pk[3])
                     : "memory");
      }
    } else {
#pragma unroll
      for (int i = 0; i < kTile; ++i) sum += ptx::ex2(x[i] - mn);
    }
    l = fmaf(l, corr, sum);
    m = mn;

    if (OUT) {
      ptx::fence_proxy_async();
      ptx::tc_fence_before();
      __syncthreads();
      if (tid == 0) {
        ptx::tc_fence_after();
        if (!ptx::mbar_wait(bar_z, j & 1)) *sFail = 1;
        // O += P z_hi + P z_lo  (A: P, K-major; B: z [keys][d], MN-major)
#pragma unroll
        for (int p = 0; p < 2; ++p)
#pragma unroll
          for (int kk = 0; kk < kTile / 16; ++kk) {
            const uint32_t aoff = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
            ptx::mma_f16_ss(tO, ptx::sw128_desc(aP + aoff, 16, 1024),
                            ptx::sw128_desc(aZ + p * kPlane + kk * 2048, kHalfBytes, 1024), idPV,
                            (j | p | kk) != 0);
          }
        if (j + 1 == nkb) ptx::mma_commit(bar_o);
      }
    } else {
      ptx::tc_fence_before();
      __syncthreads();
    }
    if (__syncthreads_or(!ok || *sFail)) break;
  }

  const int a1 = a1_base + tid;
  if (OUT) {
    ok = ok && ptx::mbar_wait(bar_o, 0);
    ptx::tc_fence_after();
    const float inv = 1.f / l;
    TO* orow = out + ((long long)bh * g.Nq + (a1 < g.b1q ? token_of(g, a1, a2) : 0)) * D;
#pragma unroll
    for (int cc = 0; cc < D / 32; ++cc) {
      uint32_t r[32];
      ptx::tmem_ld32(tO + lane_off + cc * 32, r);
      ptx::tmem_wait_ld();
      if (a1 < g.b1q && ok) {
#pragma unroll
        for (int i = 0; i < 32; i += 4) {
          if constexpr (sizeof(TO) == 4) {
            float4 v = make_float4(__uint_as_float(r[i]) * inv, __uint_as_float(r[i + 1]) * inv,
                                   __uint_as_float(r[i + 2]) * inv, __uint_as_float(r[i + 3]) * inv);
            *reinterpret_cast<float4*>(orow + cc * 32 + i) = v;
          } else {
            TO v[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) v[e] = from_f<TO>(__uint_as_float(r[i + e]) * inv);
            *reinterpret_cast<uint2*>(orow + cc * 32 + i) = *reinterpret_cast<uint2*>(v);
          }
        }
      }
    }
  } else if (a1 < g.b1q) {
    lse[(long long)zrow * g.b1q + a1] = m + log2f(l);
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 256);
}

// ---------------------------------------------------------------------------
// Column pass for one (head, position a2, 128 key tiles c1): with
// L[a1,c1] = 2^(S[a1,c1] - lse[a1]) (the row pass's normalisation),
//   q~[c1,a2] = sum_a1 L q[a1,a2] / sum_a1 L.
// S^T = k~ q^T is recomputed per 128-query block (A: k~, B: q, both K-major);
// the aggregate accumulates P^T_hi q + P^T_lo q in TMEM (A: P^T, K-major;
// B: q [queries][d], MN-major).  L is scaled by 2^15 (both sums, so q~ is
// unchanged) to keep small weights clear of the f16 subnormal range.
// grid (ceil(b1k/128), b2, BH), block 128 (thread r owns key row r).
template <typename TQ, int D>
__global__ void __launch_bounds__(128, 1)
l_col_tc(const TQ* __restrict__ q, const __grid_constant__ CUtensorMap tm_kt, const float* __restrict__ hbuf,
         const float* __restrict__ lse, float* __restrict__ qt, Geo g) {
  constexpr int NH = D / 64;
  constexpr uint32_t kPlane = NH * kHalfBytes;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sK = base;                     // k~ hi plane, lo plane
  uint8_t* sQ = sK + 2 * kPlane;          // two query-block buffers
  uint8_t* sP = sQ + 2 * kPlane;          // P^T hi, P^T lo: 2 halves of 128 queries each
  float* sL = reinterpret_cast<float*>(sP + 4 * kHalfBytes);  // two buffers of 128 lse values
  uint64_t* bars = reinterpret_cast<uint64_t*>(sL + 2 * kTile);
  uint64_t* bar_k = bars + 0;
  uint64_t* bar_s = bars + 1;
  uint64_t* bar_o = bars + 2;
  uint32_t* sTmem = reinterpret_cast<uint32_t*>(bars + 3);
  int* sFail = reinterpret_cast<int*>(sTmem + 1);

  const int tid = threadIdx.x, warp = tid >> 5;
  const int a2 = blockIdx.y, bh = blockIdx.z;
  const int kb = blockIdx.x * kTile;
  const int zrow = bh * g.b2 + a2;
  const int nqb = (g.b1q + kTile - 1) / kTile;
  const TQ* qh = q + (long long)bh * g.Nq * D;
  const float* lrow = lse + (long long)zrow * g.b1q;

  if (tid == 0) {
    ptx::mbar_init(bar_k, 1);
    ptx::mbar_init(bar_s, 1);
    ptx::mbar_init(bar_o, 1);
    ptx::fence_mbar_init();
    *sFail = 0;
    ptx::prefetch_tmap(&tm_kt);
  }
  if (warp == 0) {
    ptx::tmem_alloc(sTmem, 256);
    ptx::tmem_relinquish();
  }
  gather_q_rows<TQ, D>(sQ, qh, g, 0, a2, tid);
  ptx::cp_async_commit();
  sL[tid] = (tid < g.b1q) ? lrow[tid] : INFINITY;  // +inf: a ragged query contributes 2^-inf = 0
  const int c1 = kb + tid;
  const float hb = (c1 < g.b1k) ? hbuf[(long long)zrow * g.b1k + c1] * kLog2e + kColShift : 0.f;
  ptx::tc_fence_before();
  __syncthreads();
  ptx::tc_fence_after();
  const uint32_t tmem = *sTmem;
  const uint32_t tS = tmem, tA = tmem + 128;
  const uint32_t lane_off = (uint32_t)(warp * 32) << 16;
  if (tid == 0) {
    const int plane_rows = g.BH * g.b2;
    ptx::mbar_expect_tx(bar_k, 2 * kPlane);
    for (int p = 0; p < 2; ++p)
      for (int hf = 0; hf < NH; ++hf)
        ptx::tma_load_3d(sK + p * kPlane + hf * kHalfBytes, &tm_kt, bar_k, hf * 64, kb, p * plane_rows + zrow);
  }
  constexpr uint32_t idS = ptx::idesc_f16(128, 128, TcType<TQ>::kBf16, 0, 0);
  constexpr uint32_t idPQ = ptx::idesc_f16(128, D, TcType<TQ>::kBf16, 0, 1);
  const uint32_t aK = ptx::smem_u32(sK), aQ0 = ptx::smem_u32(sQ), aP = ptx::smem_u32(sP);

  float beta = 0.f;
  bool ok = true;
  for (int i = 0; i < nqb; ++i) {
    const int buf = i & 1;
    const uint32_t aQ = aQ0 + buf * kPlane;
    ptx::cp_async_wait<0>();
    ptx::fence_proxy_async();
    __syncthreads();  // query block i and its lse are in shared memory
    if (tid == 0) {
      if (i == 0 && !ptx::mbar_wait(bar_k, 0)) *sFail = 1;
      ptx::tc_fence_after();
#pragma unroll
      for (int p = 0; p < 2; ++p)
#pragma unroll
        for (int kk = 0; kk < D / 16; ++kk) {
          const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          ptx::mma_f16_ss(tS, ptx::sw128_desc(aK + p * kPlane + off, 16, 1024), ptx::sw128_desc(aQ + off, 16, 1024),
                          idS, (p | kk) != 0);
        }
      ptx::mma_commit(bar_s);
    }
    ok = ptx::mbar_wait(bar_s, i & 1);  // also: the previous P^T q products are done
    ptx::tc_fence_after();
    if (i + 1 < nqb) {
      // prefetch the next query block and its lse into the other buffers
      gather_q_rows<TQ, D>(sQ + (buf ^ 1) * kPlane, qh, g, (i + 1) * kTile, a2, tid);
      ptx::cp_async_commit();
      const int a1n = (i + 1) * kTile + tid;
      sL[(buf ^ 1) * kTile + tid] = (a1n < g.b1q) ? lrow[a1n] : INFINITY;
    }
    const float* lb = sL + buf * kTile;
    uint32_t aProw = aP;
#pragma unroll
    for (int cc = 0; cc < kTile / 32; ++cc) {
      uint32_t r[32];
      ptx::tmem_ld32(tS + lane_off + cc * 32, r);
      ptx::tmem_wait_ld();
#pragma unroll
      for (int c8 = 0; c8 < 4; ++c8) {
        uint32_t hi[4], lo[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int col = cc * 32 + c8 * 8 + 2 * e;
          const float p0 = ptx::ex2(fmaf(__uint_as_float(r[c8 * 8 + 2 * e]), g.sl2, hb) - lb[col]);
          const float p1 = ptx::ex2(fmaf(__uint_as_float(r[c8 * 8 + 2 * e + 1]), g.sl2, hb) - lb[col + 1]);
          const float h0 = TcType<TQ>::round(p0), h1 = TcType<TQ>::round(p1);
          const float l0 = TcType<TQ>::round(p0 - h0), l1 = TcType<TQ>::round(p1 - h1);
          beta += (h0 + l0) + (h1 + l1);
          hi[e] = TcType<TQ>::pack(h0, h1);
          lo[e] = TcType<TQ>::pack(l0, l1);
        }
        const int chunk = cc * 4 + c8;  // 16-byte chunk of the 128-query row
        const uint32_t off = (chunk >> 3) * kHalfBytes + ptx::sw128_offset(tid, chunk & 7);
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(aProw + off), "r"(hi[0]), "r"(hi[1]),
                     "r"(hi[2]), "r"(hi[3])
                     : "memory");
        asm volatile("st.shared.v4.b32 [%0], {%1,%2,%3,%4};" ::"r"(aProw + 2 * kHalfBytes + off), "r"(lo[0]),
                     "r"(lo[1]), "r"(lo[2]), "r"(lo[3])
                     : "memory");
      }
    }
    ptx::fence_proxy_async();
    ptx::tc_fence_before();
    __syncthreads();
    if (tid == 0) {
      ptx::tc_fence_after();
      // acc += P^T_hi q + P^T_lo q   (K = 128 queries)
#pragma unroll
      for (int p = 0; p < 2; ++p)
#pragma unroll
        for (int kk = 0; kk < kTile / 16; ++kk) {
          const uint32_t aoff = p * 2 * kHalfBytes + (kk >> 2) * kHalfBytes + (kk & 3) * 32;
          ptx::mma_f16_ss(tA, ptx::sw128_desc(aP + aoff, 16, 1024),
                          ptx::sw128_desc(aQ + kk * 2048, kHalfBytes, 1024), idPQ, (i | p | kk) != 0);
        }
      if (i + 1 == nqb) ptx::mma_commit(bar_o);
    }
    if (__syncthreads_or(!ok || *sFail)) break;
  }
  ok = ok && ptx::mbar_wait(bar_o, 0);
  ptx::tc_fence_after();
  const float inv = 1.f / beta;
  float* dst = qt + ((long long)zrow * g.b1k + (c1 < g.b1k ? c1 : 0)) * D;
#pragma unroll
  for (int cc = 0; cc < D / 32; ++cc) {
    uint32_t r[32];
    ptx::tmem_ld32(tA + lane_off + cc * 32, r);
    ptx::tmem_wait_ld();
    if (c1 < g.b1k && ok) {
#pragma unroll
      for (int e = 0; e < 32; e += 4)
        *reinterpret_cast<float4*>(dst + cc * 32 + e) =
            make_float4(__uint_as_float(r[e]) * inv, __uint_as_float(r[e + 1]) * inv,
                        __uint_as_float(r[e + 2]) * inv, __uint_as_float(r[e + 3]) * inv);
    }
  }
  ptx::tc_fence_before();
  __syncthreads();
  if (warp == 0) ptx::tmem_dealloc(tmem, 256);
}

template <int D>
constexpr size_t l_col_tc_smem() {
  return 1024 + (D / 64) * kHalfBytes * 4 + 4 * kHalfBytes + 2 * kTile * 4 + 64;
}

template <typename TQ, int D, bool OUT>
constexpr size_t l_row_tc_smem() {
  return 1024 + (D / 64) * kHalfBytes * (1 + 2 + (OUT ? 2 : 0)) + (OUT ? 2 * kHalfBytes : 0) + kTile * 4 + 64;
}

}  // namespace monarch
