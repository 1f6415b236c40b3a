// Helpers shared by the tcgen05 L-step kernels: packed fp32 pair arithmetic
// (sm_100 f32x2), hi/lo splitting, named barriers, 2-D TMA loads, row
// transfers into tensor memory and the tensor maps of one call.
#pragma once

#include "common.cuh"
#include "ptx.cuh"
#include "kernels_tc.cuh"

namespace monarch {
namespace tc {

constexpr int kBlk = 64;            // keys (row pass) / queries (column pass) per block
constexpr int kBox = 8192;          // one [64 rows][128 B] swizzled box
constexpr int kMaxSmem = 232448;    // opt-in shared memory per CTA

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


}  // namespace tc
}  // namespace monarch
