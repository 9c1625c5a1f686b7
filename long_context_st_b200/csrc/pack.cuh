// Bit packing of b-bit residual codes: code j of a row sits at bits [(j*b) mod 8, +b) of byte
// floor(j*b/8) (little-endian inside a byte).
#pragma once
#include "common.cuh"

namespace jolt {

// A warp holds a row's codes (lane l: codes [l*E, l*E+E)); stage them in shared memory, then
// each lane assembles and stores whole bytes (byte-coalesced across the warp).
template <int E>
__device__ __forceinline__ void warp_pack_store(const uint8_t (&c)[E], int b, uint8_t* stage,
                                                uint8_t* __restrict__ dst) {
  constexpr int D = 32 * E;
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int i = 0; i < E; ++i) stage[lane * E + i] = c[i];
  __syncwarp();
  const int nbytes = D * b / 8;
  const int per = 8 / b;
  for (int by = lane; by < nbytes; by += 32) {
    uint32_t v = 0;
    for (int k = 0; k < per; ++k) v |= uint32_t(stage[by * per + k]) << (k * b);
    dst[by] = uint8_t(v);
  }
  __syncwarp();
}

__device__ __forceinline__ uint32_t unpack_code(const uint8_t* __restrict__ row, int j, int b) {
  const int bit = j * b;
  return (uint32_t(row[bit >> 3]) >> (bit & 7)) & ((1u << b) - 1u);
}

}  // namespace jolt
