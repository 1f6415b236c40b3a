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
__device__ __forceinline__ float2 mul2(float2 a, float2 b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2u(a)), "l"(f2u(b)));
  return u2f(d);
}
__device__ __forceinline__ float2 sub2(float2 a, float2 b) {
  uint64_t d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(f2u(a)), "l"(f2u(b)));
  return u2f(d);
}

// 2^x of a pair on the FMA pipe (the MUFU unit is the other source of 2^x;
// the row pass sends part of its exponentials here to balance the two).
// x = n + f with n = rint(x) (the 1.5 * 2^23 rounding constant) and f in
// [-1/2, 1/2]; 2^f by the degree-5 equal-ripple polynomial of gen_exp2_poly.py
// (relative error 1.6e-7 in float32); 2^n is added to the exponent field.
// Inputs are clamped to -127, so -inf and anything below -127 give 0 or a
// value below 2^-126.  Inputs must be at most 127.
__device__ __forceinline__ float2 ex2_fma2(float2 x) {
  x.x = fmaxf(x.x, -127.f);
  x.y = fmaxf(x.y, -127.f);
  const float2 rc = make_float2(12582912.f, 12582912.f);
  const float2 t = add2(x, rc);
  const float2 f = sub2(x, sub2(t, rc));
  float2 p = fma2(make_float2(1.326821395e-03f, 1.326821395e-03f), f,
                  make_float2(9.671511129e-03f, 9.671511129e-03f));
  p = fma2(p, f, make_float2(5.550721660e-02f, 5.550721660e-02f));
  p = fma2(p, f, make_float2(2.402224243e-01f, 2.402224243e-01f));
  p = fma2(p, f, make_float2(6.931470037e-01f, 6.931470037e-01f));
  p = fma2(p, f, make_float2(1.f, 1.f));
  // the low bits of t hold n: (bits(t) << 23) is n in the exponent field
  return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                     __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
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

// Dynamic shared memory starts 1024-byte aligned (no static shared memory in
// these kernels); the 128-byte swizzle of the TMA boxes needs that.  A kernel
// that finds otherwise records kErrSmemAlign and returns before any TMA.
__device__ __forceinline__ bool smem_misaligned(const void* p) {
  if ((ptx::smem_u32(p) & 1023u) == 0) return false;
  if (threadIdx.x == 0) atomicExch(&ptx::g_device_error, ptx::kErrSmemAlign);
  return true;
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
