// Residual rotation, per-row quantise + pack and unpack + dequantise as standalone kernels.
// The same device functions run inside the fused residual kernel of the compressor; these
// entry points expose them for bit-exact testing and for callers that quantise their own rows.
#include "common.cuh"
#include "pack.cuh"

namespace jolt {

template <int E>
__global__ void k_rotate_rows(const float* __restrict__ in, float* __restrict__ out, int64_t n_rows,
                              uint64_t seed, int inverse) {
  constexpr int D = 32 * E;
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  const float isd = rsqrtf(float(D));
  for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n_rows; r += warps) {
    float v[E];
#pragma unroll
    for (int i = 0; i < E; ++i) v[i] = in[r * D + lane * E + i];
    if (inverse) warp_unrotate<E>(v, seed, isd);
    else warp_rotate<E>(v, seed, isd);
#pragma unroll
    for (int i = 0; i < E; ++i) out[r * D + lane * E + i] = v[i];
  }
}

template <int E>
__global__ void k_quantize_pack(const float* __restrict__ rows, int64_t n_rows, int b,
                                uint8_t* __restrict__ codes, __half2* __restrict__ sz,
                                int32_t* __restrict__ err) {
  constexpr int D = 32 * E;
  __shared__ uint8_t stage[8][D];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  const int nbytes = D * b / 8;
  for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + w; r < n_rows; r += warps) {
    float x[E];
#pragma unroll
    for (int i = 0; i < E; ++i) x[i] = rows[r * D + lane * E + i];
    uint8_t c[E];
    __half hs, hz;
    if (!warp_quantize<E>(x, b, c, &hs, &hz) && lane == 0) report_error(err, JOLT_ERR_NUMERIC);
    warp_pack_store<E>(c, b, stage[w], codes + r * nbytes);
    if (lane == 0) sz[r] = __halves2half2(hs, hz);
  }
}

template <int E>
__global__ void k_unpack_dequant(const uint8_t* __restrict__ codes, const __half2* __restrict__ sz,
                                 int64_t n_rows, int b, float* __restrict__ out) {
  constexpr int D = 32 * E;
  const int lane = threadIdx.x & 31;
  const int64_t warps = int64_t(gridDim.x) * (blockDim.x >> 5);
  const int nbytes = D * b / 8;
  for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < n_rows; r += warps) {
    const __half2 p = sz[r];
    const float s = __low2float(p), z = __high2float(p);
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const int j = lane * E + i;
      out[r * D + j] = dequant(unpack_code(codes + r * nbytes, j, b), s, z);
    }
  }
}

static int grid_for(int64_t rows) {
  int64_t g = (rows + 7) / 8;
  return int(g < 148 * 16 ? (g < 1 ? 1 : g) : 148 * 16);
}

}  // namespace jolt

using namespace jolt;

extern "C" jolt_status jolt_rotate_rows(const float* in, float* out, int64_t n_rows, int32_t d,
                                        uint64_t seed, int32_t inverse, void* stream) {
  if (n_rows < 0 || (d != 64 && d != 128)) return JOLT_ERR_INVALID_ARG;
  if (n_rows == 0) return JOLT_OK;
  if (!in || !out) return JOLT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (d == 64) k_rotate_rows<2><<<grid_for(n_rows), 256, 0, st>>>(in, out, n_rows, seed, inverse);
  else k_rotate_rows<4><<<grid_for(n_rows), 256, 0, st>>>(in, out, n_rows, seed, inverse);
  JOLT_CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

extern "C" jolt_status jolt_quantize_pack(const float* rows, int64_t n_rows, int32_t d, int32_t b,
                                          uint8_t* codes, void* sz, int32_t* err, void* stream) {
  if (n_rows < 0 || (d != 64 && d != 128) || !(b == 2 || b == 4 || b == 8))
    return JOLT_ERR_INVALID_ARG;
  if (n_rows == 0) return JOLT_OK;
  if (!rows || !codes || !sz || !err) return JOLT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (d == 64)
    k_quantize_pack<2><<<grid_for(n_rows), 256, 0, st>>>(rows, n_rows, b, codes, (__half2*)sz, err);
  else
    k_quantize_pack<4><<<grid_for(n_rows), 256, 0, st>>>(rows, n_rows, b, codes, (__half2*)sz, err);
  JOLT_CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

extern "C" jolt_status jolt_unpack_dequant(const uint8_t* codes, const void* sz, int64_t n_rows,
                                           int32_t d, int32_t b, float* out, void* stream) {
  if (n_rows < 0 || (d != 64 && d != 128) || !(b == 2 || b == 4 || b == 8))
    return JOLT_ERR_INVALID_ARG;
  if (n_rows == 0) return JOLT_OK;
  if (!codes || !sz || !out) return JOLT_ERR_INVALID_ARG;
  cudaStream_t st = (cudaStream_t)stream;
  if (d == 64)
    k_unpack_dequant<2><<<grid_for(n_rows), 256, 0, st>>>(codes, (const __half2*)sz, n_rows, b, out);
  else
    k_unpack_dequant<4><<<grid_for(n_rows), 256, 0, st>>>(codes, (const __half2*)sz, n_rows, b, out);
  JOLT_CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}
