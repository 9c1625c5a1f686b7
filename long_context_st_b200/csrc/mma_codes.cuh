// Packed residual codes as tensor-core operands: b-bit code fields widened to exact f16 values in
// registers, and the warp-level m16n8k16 f16 MMA that consumes them (fp32 accumulation).
//
// The mask-and-or puts each field into the mantissa of 1024 (f16 0x6400), scaled by 2^shift; one
// f16x2 add or fused multiply-add with constant pairs then removes the offset and the scale. Every
// intermediate is a small integer or a power of two, so the result is exact.
//
// Fragment layouts of mma.sync.m16n8k16.row.col (lane = 4 * g + m, g = lane / 4, m = lane % 4):
//   A (16 x 16, row-major): a0 = (row g, cols 2m, 2m+1), a1 = (row g+8, cols 2m, 2m+1),
//                           a2 = (row g, cols 2m+8, 2m+9), a3 = (row g+8, cols 2m+8, 2m+9)
//   B (16 x 8, col-major):  b0 = (rows 2m, 2m+1, col g), b1 = (rows 2m+8, 2m+9, col g)
//   C/D (16 x 8):           c0 = (row g, col 2m), c1 = (row g, col 2m+1), c2 / c3 the same for row g+8
// (the lower column or row index sits in the lower half of each f16 pair).
#pragma once
#include <stdint.h>

namespace jolt {

__device__ __forceinline__ void mma_f16_16816(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t h2_add(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("add.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}
__device__ __forceinline__ uint32_t h2_fma(uint32_t a, uint32_t b, uint32_t c) {
  uint32_t d;
  asm("fma.rn.f16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
  return d;
}
constexpr uint32_t kH2M1024 = 0xE400E400u;  // (-1024, -1024)
__device__ __forceinline__ uint32_t field_or(uint32_t x, uint32_t mask) { return (x & mask) | 0x64006400u; }
// 4-bit fields at bits 0-3 / 16-19 (lo) or 4-7 / 20-23 (hi)
__device__ __forceinline__ uint32_t nib_lo(uint32_t x) { return h2_add(field_or(x, 0x000F000Fu), kH2M1024); }
__device__ __forceinline__ uint32_t nib_hi(uint32_t x) { return h2_fma(field_or(x, 0x00F000F0u), 0x2C002C00u, 0xD400D400u); }
// 2-bit fields at bits 2s / 16 + 2s: (1024 + 4^s c) * 4^-s - 1024 * 4^-s
__device__ __forceinline__ uint32_t crumb(uint32_t x, int s) {
  switch (s) {
    case 0: return h2_add(field_or(x, 0x00030003u), kH2M1024);
    case 1: return h2_fma(field_or(x, 0x000C000Cu), 0x34003400u, 0xDC00DC00u);
    case 2: return h2_fma(field_or(x, 0x00300030u), 0x2C002C00u, 0xD400D400u);
    default: return h2_fma(field_or(x, 0x00C000C0u), 0x24002400u, 0xCC00CC00u);
  }
}
// 8-bit fields at bits 0-7 / 16-23
__device__ __forceinline__ uint32_t byte_lo(uint32_t x) { return h2_add(field_or(x, 0x00FF00FFu), kH2M1024); }
// bytes of x chosen by sel next to 0x64 -> f16 pair (byte, byte)
__device__ __forceinline__ uint32_t byte_pair(uint32_t x, uint32_t sel) {
  return h2_add(__byte_perm(x, 0x64646464u, sel), kH2M1024);
}
// byte k (0..3) of x at bits 0-7 and byte k of y at bits 16-23 (the other bytes are don't-care)
__device__ __forceinline__ uint32_t bytes_xy(uint32_t x, uint32_t y, int k) {
  return __byte_perm(x, y, uint32_t(k) | (uint32_t(k) << 4) | (uint32_t(4 + k) << 8) | (uint32_t(4 + k) << 12));
}

}  // namespace jolt
