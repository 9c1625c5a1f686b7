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
  int skip_p;       // the query prologue leaves P to the caller (the fused path forms it itself)
  double alg_bytes; // algorithmic bytes the main kernel must read (stats only)
  CellRef cells[kMaxCallCells];  // (b * Gc + (g - g_first)) * 2 + kv
};

jolt_status launch_decode_simt(const DecodeParams& p, cudaStream_t st);
// First prologue kernel of both paths: q_rot = R q, qsum = sum(q_rot) and (non-RoPE keys) P.
jolt_status launch_decode_prologue_q(const DecodeParams& p, cudaStream_t st);
// Log-sum-exp merge of p.S split partials (p.ws_part) and the output projection.
jolt_status launch_decode_merge(const DecodeParams& p, cudaStream_t st);

// One stored cell as device pointers (bf16 factors), for the tensor-core path.
struct TcCellView {
  const __nv_bfloat16* Ut;  // [T][r_T]
  const __nv_bfloat16* Ud;  // [d_h][r_d]
  const __nv_bfloat16* G;   // [L_g][n_kv][r_T][r_d]
  const uint8_t* codes;     // [L_g][n_kv][T][d_h * b / 8]
  const __half2* sz;        // [L_g][n_kv][T] (scale, zero)
  int r_T, r_d, bits;
};

// Tensor-core decode (bf16 I/O and factors, d_h = 128, g_q <= 16).
bool decode_tc_supported(const jolt_shape& s);
size_t decode_tc_ws_bytes(const jolt_shape& s, int Lc);
// views: (b * Gc + (g - g_first)) * 2 + kv for the call's batch range; tcws: the path's workspace.
jolt_status launch_decode_tc(const DecodeParams& p, const TcCellView* views, uint8_t* tcws,
                             const jolt_shape& s, cudaStream_t st);

// Fused split-T decode for bf16 caches with non-RoPE keys (n_q = 32, n_kv = 4 or 8): one kernel
// for scores, online softmax and values per (sequence, layer, split), then the split merge.
bool decode_fused_supported(const jolt_shape& s);
size_t decode_fused_ws_bytes(const jolt_shape& s, int Lc);
int decode_fused_max_cells();
jolt_status launch_decode_fused(const DecodeParams& p, const TcCellView* views, uint8_t* ws,
                                const jolt_shape& s, cudaStream_t st);

}  // namespace jolt
