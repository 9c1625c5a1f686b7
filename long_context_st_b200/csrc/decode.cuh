// Parameters shared by the decode-attention kernels.
#pragma once
#include "common.cuh"

namespace jolt {

constexpr int kMaxCallCells = 128;  // cells one launch can reference (kernel-parameter table)

struct DecodeParams {
  const uint8_t* cache;
  const void* q;
  void* out;
  float* lse;
  const float* inv_freq;
  float* ws_qrot;   // [B][Lc][n_q][d_h]
  float* ws_qsum;   // [B][Lc][n_q]
  float* ws_P;      // [B][Lc][n_q][q_cap]          non-RoPE keys
  float* ws_Bh;     // [B][Lc][n_kv][q_cap][d_h]    pre-RoPE keys
  float* ws_part;   // [B][Lc][n_q][S][2 + q_cap + d_h]
  int32_t* err;
  uint64_t rot_seed;
  float attn_scale, rope_scaling;
  int B, Lg, n_kv, n_q, gq, T, d_h, Lc, layer_begin, S, q_cap, pos_offset;
  int io_f32, fac_f32, pre_rope;
  int g_first, Gc;  // first group of the call and number of groups it touches
  double alg_bytes; // algorithmic bytes the main kernel must read (stats only)
  CellRef cells[kMaxCallCells];  // (b * Gc + (g - g_first)) * 2 + kv
};

jolt_status launch_decode_simt(const DecodeParams& p, cudaStream_t st);

}  // namespace jolt
