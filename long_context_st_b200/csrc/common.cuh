// Device-side helpers shared by the JoLT kernels.
#pragma once
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <cstdio>
#include <cstdlib>

#include "jolt_internal.h"

namespace jolt {

// ---- error reporting ------------------------------------------------------------------------
// The first 256 bytes of every workspace hold a small header; word 0 is the device error word.
struct WsHeader {
  int32_t err;          // first jolt_status a kernel reported (0 = none)
  int32_t where;        // kernel-specific detail (e.g. which wait gave up)
  uint64_t analyze_tag; // identifies the analyze call whose bases the workspace holds
  uint64_t pad[30];
};
static_assert(sizeof(WsHeader) == 256, "header must be 256 bytes");

__device__ __forceinline__ void report_error(int32_t* err, int32_t code) {
  if (err) atomicCAS(err, 0, code);
}

// Diagnostic printing to stderr: compiled in by a debug build (-DJOLT_DEBUG), never switched at
// run time.
#ifdef JOLT_DEBUG
constexpr bool kDebug = true;
#else
constexpr bool kDebug = false;
#endif

// In a debug build a failing CUDA call is printed with its location.
inline void jolt_note_cuda_error(cudaError_t e, const char* what, const char* file, int line) {
  if (kDebug) std::fprintf(stderr, "jolt: %s:%d: %s -> %s\n", file, line, what, cudaGetErrorString(e));
}

#define JOLT_CUDA_TRY(expr)                                       \
  do {                                                            \
    cudaError_t e_ = (expr);                                      \
    if (e_ != cudaSuccess) {                                      \
      jolt_note_cuda_error(e_, #expr, __FILE__, __LINE__);        \
      return JOLT_ERR_CUDA;                                       \
    }                                                             \
  } while (0)

// ---- counter-based randomness (SplitMix64 as a hash of a 64-bit counter) --------------------
__host__ __device__ __forceinline__ uint64_t mix64(uint64_t x) {
  uint64_t z = x + 0x9E3779B97F4A7C15ull;
  z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
  z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
  return z ^ (z >> 31);
}

// Sign s_j of the residual rotation: +1 when bit 63 of mix64(seed * 2^32 + j) is clear.
__host__ __device__ __forceinline__ float rot_sign(uint64_t seed, int j) {
  return (mix64((seed << 32) + uint64_t(j)) >> 63) ? -1.f : 1.f;
}

// ---- dtype helpers --------------------------------------------------------------------------
__device__ __forceinline__ float ld_as_float(const float* p, int64_t i) { return p[i]; }
__device__ __forceinline__ float ld_as_float(const __nv_bfloat16* p, int64_t i) {
  return __bfloat162float(p[i]);
}
__device__ __forceinline__ void st_from_float(float* p, int64_t i, float v) { p[i] = v; }
__device__ __forceinline__ void st_from_float(__nv_bfloat16* p, int64_t i, float v) {
  p[i] = __float2bfloat16_rn(v);
}

// ---- warp-level fast Walsh-Hadamard transform -----------------------------------------------
// A row of D values is spread over one warp: lane l holds elements [l*E, l*E + E), E = D/32.
// The transform is the Sylvester ordering: butterflies (a, b) -> (a + b, a - b) over strides
// 1, 2, 4, ..., D/2; strides below E are inside a lane, the rest cross lanes by shuffles.
template <int E>
__device__ __forceinline__ void warp_fwht(float (&v)[E]) {
#pragma unroll
  for (int s = 1; s < E; s <<= 1) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      if ((i & s) == 0) {
        float a = v[i], b = v[i + s];
        v[i] = a + b;
        v[i + s] = a - b;
      }
    }
  }
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int m = 1; m < 32; m <<= 1) {
#pragma unroll
    for (int i = 0; i < E; ++i) {
      float o = __shfl_xor_sync(0xffffffffu, v[i], m);
      v[i] = (lane & m) ? (o - v[i]) : (v[i] + o);
    }
  }
}

// Forward rotation (1/sqrt(D)) H diag(s) applied in place to a warp-distributed row.
template <int E>
__device__ __forceinline__ void warp_rotate(float (&v)[E], uint64_t seed, float inv_sqrt_d) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < E; ++i) v[i] *= rot_sign(seed, lane * E + i);
  warp_fwht<E>(v);
#pragma unroll
  for (int i = 0; i < E; ++i) v[i] *= inv_sqrt_d;
}

// Inverse rotation diag(s) H (1/sqrt(D)).
template <int E>
__device__ __forceinline__ void warp_unrotate(float (&v)[E], uint64_t seed, float inv_sqrt_d) {
  const int lane = threadIdx.x & 31;
  warp_fwht<E>(v);
#pragma unroll
  for (int i = 0; i < E; ++i) v[i] *= inv_sqrt_d * rot_sign(seed, lane * E + i);
}

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int m = 16; m; m >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int m = 16; m; m >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, m));
  return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int m = 16; m; m >>= 1) v += __shfl_xor_sync(0xffffffffu, v, m);
  return v;
}

// ---- per-row uniform quantiser ------------------------------------------------------------------
// Row of D = 32*E fp32 values held by one warp. Every operation is IEEE-rounded once:
//   scale = fp16((mx - mn) / (2^b - 1)), zero = fp16(mn),
//   code  = clip(rint((x - zero) / scale), 0, 2^b - 1)   (0 when scale == 0).
// Writes E codes per lane into `code`; returns false (numeric error) when scale or zero are not
// finite fp16 values.
template <int E>
__device__ __forceinline__ bool warp_quantize(const float (&x)[E], int b, uint8_t (&code)[E],
                                              __half* scale_out, __half* zero_out) {
  float mn = x[0], mx = x[0];
#pragma unroll
  for (int i = 1; i < E; ++i) {
    mn = fminf(mn, x[i]);
    mx = fmaxf(mx, x[i]);
  }
  mn = warp_min(mn);
  mx = warp_max(mx);
  const float levels = float((1 << b) - 1);
  const float step = __fdiv_rn(__fsub_rn(mx, mn), levels);
  const __half hs = __float2half_rn(step);
  const __half hz = __float2half_rn(mn);
  const float s = __half2float(hs), z = __half2float(hz);
  const bool ok = isfinite(s) && isfinite(z);
#pragma unroll
  for (int i = 0; i < E; ++i) {
    float c = 0.f;
    if (s != 0.f) {
      c = rintf(__fdiv_rn(__fsub_rn(x[i], z), s));
      c = fminf(fmaxf(c, 0.f), levels);
    }
    code[i] = uint8_t(c);
  }
  *scale_out = hs;
  *zero_out = hz;
  return ok;
}

// deq = fp32(code * scale + zero) with one rounding (the product is exact in fp32).
__device__ __forceinline__ float dequant(uint32_t code, float scale, float zero) {
  return __fmaf_rn(float(code), scale, zero);
}

}  // namespace jolt
