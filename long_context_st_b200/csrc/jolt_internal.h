// Internal helpers shared by the host library and the CUDA translation units.
#pragma once
#include <cstddef>
#include <cstdint>

#include "../../include/jolt.h"

namespace jolt {

constexpr int kRankStep = 16;        // rank grid granularity (MMA K/N granularity)
constexpr uint64_t kSegAlign = 256;  // alignment of every stored-cache segment

inline uint64_t align_up(uint64_t x, uint64_t a) { return (x + a - 1) / a * a; }

inline int dtype_bytes(int32_t dt) { return dt == JOLT_F32 ? 4 : 2; }
inline int n_groups(const jolt_shape& s) { return s.n_layers / s.layers_per_group; }
inline int n_cells(const jolt_shape& s) { return 2 * s.batch * n_groups(s); }
inline int64_t n_cols(const jolt_shape& s) {
  return int64_t(s.layers_per_group) * s.n_kv * s.d_h;
}
inline int n_rt(const jolt_shape& s) { return s.q_cap / kRankStep + 1; }
inline int n_rd(const jolt_shape& s) { return s.d_h / kRankStep + 1; }

bool shape_ok(const jolt_shape* s);
bool choice_ok(const jolt_shape& s, const jolt_cell_choice& c);

// Byte offsets of one cell's segments relative to the cell start, and the cell's padded size.
struct CellSegs {
  uint64_t ut, ud, g, codes, sz, size;
};
CellSegs cell_segments(const jolt_shape& s, const jolt_cell_choice& c);

// Defined in the CUDA translation units.
size_t compress_workspace_bytes(const jolt_shape& s);
size_t decode_workspace_bytes(const jolt_shape& s);

}  // namespace jolt

namespace jolt {

// Per-cell descriptor handed to kernels: where the cell starts in the cache and its choice.
struct CellRef {
  uint64_t offset;
  int32_t r_T, r_d, b, pad;
};

#if defined(__CUDACC__)
#define JOLT_HD __host__ __device__
#else
#define JOLT_HD
#endif

// Segment offsets of a cell, relative to the cell start (same arithmetic as cell_segments).
struct SegOffsets {
  uint64_t ut, ud, g, codes, sz;
};
JOLT_HD inline SegOffsets seg_offsets(int T, int d_h, int L_g, int n_kv, int sf, int r_T, int r_d, int b) {
  auto al = [](uint64_t x) { return (x + 255) / 256 * 256; };
  SegOffsets o;
  const uint64_t rows = uint64_t(L_g) * n_kv * T;
  uint64_t off = 0;
  o.ut = off; off = al(off + uint64_t(sf) * T * r_T);
  o.ud = off; off = al(off + uint64_t(sf) * d_h * r_d);
  o.g = off;  off = al(off + uint64_t(sf) * L_g * n_kv * r_T * r_d);
  o.codes = off; off = al(off + (b ? rows * (uint64_t(d_h) * b / 8) : 0));
  o.sz = off;
  return o;
}

}  // namespace jolt
