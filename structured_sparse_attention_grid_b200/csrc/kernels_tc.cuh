// Operand types and constants shared by the tensor-core kernels (bf16 / f16
// inputs).
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
constexpr float kColShift = 15.f;   // L^T q: L scaled by 2^15 (the ratio is unchanged)
constexpr float kLazyRescale = 8.f; // row pass: shift moves only when the max grows by > 2^8

}  // namespace monarch
