// Host blob of a stored cache: a checked header (shape, choices, sizes) and the cache bytes.
#include <cuda_runtime.h>

#include <cstring>
#include <vector>

#include "jolt_internal.h"

namespace jolt {
namespace {

constexpr char kMagic[8] = {'J', 'O', 'L', 'T', 'C', 'A', 'C', 'H'};
constexpr uint32_t kVersion = 2;

uint64_t header_bytes(int n_cells) {
  const uint64_t raw = 16 + sizeof(jolt_shape) + 4 + uint64_t(n_cells) * sizeof(jolt_cell_choice) + 8;
  return (raw + 255) / 256 * 256;
}

// Parses and checks a header; on success fills the outputs (choices only when requested).
jolt_status parse(const uint8_t* b, uint64_t n, jolt_shape* shape, int32_t* nc_out, uint64_t* cache_bytes,
                  std::vector<jolt_cell_choice>* choices) {
  if (!b || n < 16 + sizeof(jolt_shape) + 4) return JOLT_ERR_INVALID_ARG;
  if (std::memcmp(b, kMagic, 8) != 0) return JOLT_ERR_INVALID_ARG;
  uint32_t ver = 0, hb = 0;
  std::memcpy(&ver, b + 8, 4);
  std::memcpy(&hb, b + 12, 4);
  if (ver != kVersion || hb % 256 || hb > n) return JOLT_ERR_INVALID_ARG;
  jolt_shape s;
  std::memcpy(&s, b + 16, sizeof(s));
  if (!shape_ok(&s)) return JOLT_ERR_INVALID_ARG;
  int32_t nc = 0;
  std::memcpy(&nc, b + 16 + sizeof(s), 4);
  if (nc != n_cells(s) || header_bytes(nc) != hb) return JOLT_ERR_INVALID_ARG;
  std::vector<jolt_cell_choice> ch(static_cast<size_t>(nc));
  std::memcpy(ch.data(), b + 16 + sizeof(s) + 4, ch.size() * sizeof(jolt_cell_choice));
  uint64_t cb = 0;
  std::memcpy(&cb, b + 16 + sizeof(s) + 4 + ch.size() * sizeof(jolt_cell_choice), 8);
  uint64_t need = 0;
  if (jolt_cache_layout(&s, ch.data(), nullptr, &need) != JOLT_OK || cb != need) return JOLT_ERR_INVALID_ARG;
  if (n < hb || n - hb < cb) return JOLT_ERR_INVALID_ARG;
  if (shape) *shape = s;
  if (nc_out) *nc_out = nc;
  if (cache_bytes) *cache_bytes = cb;
  if (choices) *choices = std::move(ch);
  return JOLT_OK;
}

}  // namespace
}  // namespace jolt

using namespace jolt;

extern "C" uint64_t jolt_cache_blob_bytes(const jolt_shape* shape, const jolt_cell_choice* choices) {
  if (!shape_ok(shape) || !choices) return 0;
  uint64_t total = 0;
  if (jolt_cache_layout(shape, choices, nullptr, &total) != JOLT_OK) return 0;
  return header_bytes(n_cells(*shape)) + total;
}

extern "C" jolt_status jolt_cache_serialize(const jolt_shape* shape, const jolt_cell_choice* choices,
                                            const void* cache, void* blob, uint64_t blob_bytes, void* stream) {
  if (!shape_ok(shape) || !choices || !cache || !blob) return JOLT_ERR_INVALID_ARG;
  uint64_t total = 0;
  if (jolt_cache_layout(shape, choices, nullptr, &total) != JOLT_OK) return JOLT_ERR_INVALID_ARG;
  const int32_t nc = n_cells(*shape);
  const uint64_t hb = header_bytes(nc);
  if (blob_bytes < hb + total) return JOLT_ERR_INVALID_ARG;
  uint8_t* b = static_cast<uint8_t*>(blob);
  std::memset(b, 0, hb);
  std::memcpy(b, kMagic, 8);
  std::memcpy(b + 8, &kVersion, 4);
  const uint32_t hb32 = uint32_t(hb);
  std::memcpy(b + 12, &hb32, 4);
  std::memcpy(b + 16, shape, sizeof(jolt_shape));
  std::memcpy(b + 16 + sizeof(jolt_shape), &nc, 4);
  std::memcpy(b + 16 + sizeof(jolt_shape) + 4, choices, size_t(nc) * sizeof(jolt_cell_choice));
  std::memcpy(b + 16 + sizeof(jolt_shape) + 4 + size_t(nc) * sizeof(jolt_cell_choice), &total, 8);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (total) {
    if (cudaMemcpyAsync(b + hb, cache, total, cudaMemcpyDeviceToHost, st) != cudaSuccess) return JOLT_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) return JOLT_ERR_CUDA;
  return JOLT_OK;
}

extern "C" jolt_status jolt_cache_blob_info(const void* blob, uint64_t blob_bytes, jolt_shape* shape_out,
                                            int32_t* n_cells_out, uint64_t* cache_bytes_out) {
  return parse(static_cast<const uint8_t*>(blob), blob_bytes, shape_out, n_cells_out, cache_bytes_out, nullptr);
}

extern "C" jolt_status jolt_cache_deserialize(const void* blob, uint64_t blob_bytes, jolt_cell_choice* choices_out,
                                              int32_t n_cells, void* cache, uint64_t cache_bytes, void* stream) {
  if (!choices_out || !cache) return JOLT_ERR_INVALID_ARG;
  jolt_shape s;
  int32_t nc = 0;
  uint64_t cb = 0;
  std::vector<jolt_cell_choice> ch;
  const uint8_t* b = static_cast<const uint8_t*>(blob);
  const jolt_status r = parse(b, blob_bytes, &s, &nc, &cb, &ch);
  if (r != JOLT_OK) return r;
  if (n_cells != nc || cache_bytes < cb) return JOLT_ERR_INVALID_ARG;
  std::memcpy(choices_out, ch.data(), ch.size() * sizeof(jolt_cell_choice));
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (cb) {
    if (cudaMemcpyAsync(cache, b + header_bytes(nc), cb, cudaMemcpyHostToDevice, st) != cudaSuccess)
      return JOLT_ERR_CUDA;
  }
  if (cudaStreamSynchronize(st) != cudaSuccess) return JOLT_ERR_CUDA;
  return JOLT_OK;
}
