// jolt_decode_attn: argument checks, workspace carving, split choice and kernel dispatch.
#include <cuda.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "common.cuh"
#include "decode.cuh"

namespace jolt {

namespace {

constexpr int kSMs = 148;

int choose_splits(const jolt_shape& s, int Lc) {
  const int64_t units = int64_t(s.batch) * Lc * s.n_kv;
  int S = int((2 * kSMs + units - 1) / units);
  S = std::max(1, std::min(S, std::min(64, (s.T + 63) / 64)));
  return S;
}

// Workspace of one call: header, prologue outputs, then either the CUDA-core path's split
// partials (ws_Bh, part) or the tensor-core path's buffers (tc).
struct DecodeWs {
  size_t qrot, qsum, P, Bh, part, tc, total;
};

DecodeWs decode_ws_layout(const jolt_shape& s, int Lc, int S) {
  DecodeWs w{};
  const size_t B = s.batch, nq = s.n_q, d = s.d_h, qc = std::max(s.q_cap, 16);
  const bool tc = decode_tc_supported(s);
  size_t off = sizeof(WsHeader);
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  w.qrot = take(B * Lc * nq * d * 4);
  w.qsum = take(B * Lc * nq * 4);
  w.P = take(s.keys_pre_rope ? 0 : B * Lc * nq * qc * 4);
  w.Bh = take(s.keys_pre_rope && !tc ? B * Lc * s.n_kv * qc * d * 4 : 0);
  w.part = take(tc ? 0 : B * Lc * nq * size_t(S) * (2 + qc + d) * 4);
  w.tc = take(decode_fused_supported(s) ? decode_fused_ws_bytes(s, Lc) : tc ? decode_tc_ws_bytes(s, Lc) : 0);
  w.total = off;
  return w;
}

}  // namespace

size_t decode_workspace_bytes(const jolt_shape& s) {
  size_t mx = 0;
  for (int Lc = 1; Lc <= s.n_layers; ++Lc) mx = std::max(mx, decode_ws_layout(s, Lc, choose_splits(s, Lc)).total);
  return mx;
}

}  // namespace jolt

using namespace jolt;

namespace {

// The argument checks every decode entry makes before it looks at workspaces.
bool decode_args_ok(const jolt_shape* shape, const jolt_cell_choice* choices, const void* cache, int32_t layer_begin,
                    int32_t n_layers_call, const void* q, const void* out, const float* inv_freq, int32_t pos_offset) {
  if (!shape_ok(shape) || !choices || !cache || !q || !out) return false;
  const jolt_shape& s = *shape;
  if (layer_begin < 0 || n_layers_call < 1 || layer_begin + n_layers_call > s.n_layers) return false;
  if (s.keys_pre_rope && !inv_freq) return false;
  if (pos_offset < 0 || int64_t(pos_offset) + s.T > (int64_t(1) << 24)) return false;
  const int nc = n_cells(s);
  for (int c = 0; c < nc; ++c)
    if (!choice_ok(s, choices[c])) return false;
  // the tensor-core paths read the cache with 16-byte vector loads and TMA
  if (decode_tc_supported(s) && reinterpret_cast<uintptr_t>(cache) % 16) return false;
  return true;
}

}  // namespace

extern "C" jolt_status jolt_decode_attn(const jolt_shape* shape, const jolt_cell_choice* choices,
                                        const void* cache, int32_t layer_begin, int32_t n_layers_call,
                                        const void* q, void* out, float* lse, const float* inv_freq,
                                        int32_t pos_offset, void* ws, size_t ws_bytes, void* stream) {
  if (!ws || !decode_args_ok(shape, choices, cache, layer_begin, n_layers_call, q, out, inv_freq, pos_offset))
    return JOLT_ERR_INVALID_ARG;
  const jolt_shape& s = *shape;
  const int nc = n_cells(s);
  const int Lc = n_layers_call;
  const int S = choose_splits(s, Lc);
  const DecodeWs wl = decode_ws_layout(s, Lc, S);
  if (ws_bytes < wl.total) return JOLT_ERR_WORKSPACE;

  // cell offsets of the whole cache (host arithmetic, same layout as jolt_cache_layout)
  std::vector<uint64_t> cell_off(nc);
  {
    uint64_t off = 0;
    for (int c = 0; c < nc; ++c) {
      cell_off[c] = off;
      off += cell_segments(s, choices[c]).size;
    }
  }
  const int G = n_groups(s);
  const int g_first = layer_begin / s.layers_per_group;
  const int g_last = (layer_begin + Lc - 1) / s.layers_per_group;
  const int Gc = g_last - g_first + 1;

  DecodeParams p{};
  p.cache = static_cast<const uint8_t*>(cache);
  p.q = q;
  p.out = out;
  p.lse = lse;
  p.inv_freq = inv_freq;
  uint8_t* wsb = static_cast<uint8_t*>(ws);
  p.err = reinterpret_cast<int32_t*>(wsb);
  p.ws_qrot = reinterpret_cast<float*>(wsb + wl.qrot);
  p.ws_qsum = reinterpret_cast<float*>(wsb + wl.qsum);
  p.ws_P = reinterpret_cast<float*>(wsb + wl.P);
  p.ws_Bh = reinterpret_cast<float*>(wsb + wl.Bh);
  p.ws_part = reinterpret_cast<float*>(wsb + wl.part);
  p.rot_seed = s.rot_seed;
  p.attn_scale = s.attn_scale;
  p.rope_scaling = s.rope_attention_scaling;
  p.Lg = s.layers_per_group;
  p.n_kv = s.n_kv;
  p.n_q = s.n_q;
  p.gq = s.n_q / s.n_kv;
  p.T = s.T;
  p.d_h = s.d_h;
  p.Lc = Lc;
  p.layer_begin = layer_begin;
  p.S = S;
  p.q_cap = std::max(s.q_cap, 16);
  p.pos_offset = pos_offset;
  p.io_f32 = s.io_dtype == JOLT_F32;
  p.fac_f32 = s.factor_dtype == JOLT_F32;
  p.pre_rope = s.keys_pre_rope;
  p.g_first = g_first;
  p.Gc = Gc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);

  // one launch set per batch range whose cells fit the parameter table
  const bool fused = decode_fused_supported(s);
  const int bchunk = fused ? std::max(1, std::min(decode_fused_max_cells() / (2 * Gc), 512 / Lc))
                           : std::max(1, kMaxCallCells / (2 * Gc));
  for (int b0 = 0; b0 < s.batch; b0 += bchunk) {
    const int nb = std::min(bchunk, s.batch - b0);
    DecodeParams pc = p;
    pc.B = nb;
    for (int bi = 0; bi < nb; ++bi)
      for (int gi = 0; gi < Gc; ++gi)
        for (int kv = 0; kv < 2; ++kv) {
          const int c = ((b0 + bi) * G + g_first + gi) * 2 + kv;
          CellRef r;
          r.offset = cell_off[c];
          r.r_T = choices[c].r_T;
          r.r_d = choices[c].r_d;
          r.b = choices[c].b;
          r.pad = 0;
          pc.cells[(bi * Gc + gi) * 2 + kv] = r;
        }
    // shift the batch-major tensors to this batch range
    const size_t row = size_t(Lc) * s.n_q;
    const int iob = s.io_dtype == JOLT_F32 ? 4 : 2;
    pc.q = static_cast<const uint8_t*>(q) + size_t(b0) * row * s.d_h * iob;
    pc.out = static_cast<uint8_t*>(out) + size_t(b0) * row * s.d_h * iob;
    pc.lse = lse ? lse + size_t(b0) * row : nullptr;
    // algorithmic bytes of this launch set: per (b, layer) the U_T rows of K and V (per-layer
    // re-read), and per KV head the packed codes and scale/zero pairs, plus U_d, G, q and out
    double ab = 0.0;
    const int sf = s.factor_dtype == JOLT_F32 ? 4 : 2;
    for (int bi = 0; bi < nb; ++bi)
      for (int li = 0; li < Lc; ++li) {
        const int gi = (layer_begin + li) / s.layers_per_group - g_first;
        for (int kv = 0; kv < 2; ++kv) {
          const CellRef& c = pc.cells[(bi * Gc + gi) * 2 + kv];
          ab += double(sf) * s.T * c.r_T + double(sf) * s.d_h * c.r_d + double(sf) * s.n_kv * c.r_T * c.r_d;
          if (c.b) ab += double(s.n_kv) * s.T * (double(s.d_h) * c.b / 8 + 4);
        }
        ab += 2.0 * s.n_q * s.d_h * iob;
      }
    pc.alg_bytes = ab;
    jolt_status st_;
    if (decode_tc_supported(s)) {
      TcCellView views[kMaxCallCells];
      const uint8_t* cb = static_cast<const uint8_t*>(cache);
      for (int i = 0; i < 2 * nb * Gc; ++i) {
        const CellRef& c = pc.cells[i];
        const SegOffsets so = seg_offsets(s.T, s.d_h, s.layers_per_group, s.n_kv, 2, c.r_T, c.r_d, c.b);
        const uint8_t* base = cb + c.offset;
        views[i].Ut = reinterpret_cast<const __nv_bfloat16*>(base + so.ut);
        views[i].Ud = reinterpret_cast<const __nv_bfloat16*>(base + so.ud);
        views[i].G = reinterpret_cast<const __nv_bfloat16*>(base + so.g);
        views[i].codes = base + so.codes;
        views[i].sz = reinterpret_cast<const __half2*>(base + so.sz);
        views[i].r_T = c.r_T;
        views[i].r_d = c.r_d;
        views[i].bits = c.b;
      }
      st_ = fused ? launch_decode_fused(pc, views, wsb + wl.tc, s, st) : launch_decode_tc(pc, views, wsb + wl.tc, s, st);
    } else {
      st_ = launch_decode_simt(pc, st);
    }
    if (st_ != JOLT_OK) return st_;
  }
  return JOLT_OK;
}

extern "C" jolt_status jolt_check(void* ws, void* stream) {
  if (!ws) return JOLT_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  JOLT_CUDA_TRY(cudaStreamSynchronize(st));
  int32_t err = 0;
  JOLT_CUDA_TRY(cudaMemcpy(&err, ws, sizeof(int32_t), cudaMemcpyDeviceToHost));
  if (err) {
    const int32_t zero = 0;
    JOLT_CUDA_TRY(cudaMemcpy(ws, &zero, sizeof(int32_t), cudaMemcpyHostToDevice));
  }
  return static_cast<jolt_status>(err);
}

// ---- decode without a caller-provided workspace ------------------------------------------------
// Scratch of jolt_decode_attn_noalloc: a file-scope device array that every GPU loading this
// library holds until the process exits. Host code must not pass the array's name to a kernel (on
// the host it is only a stand-in symbol); its device address is looked up once per device.
namespace {
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr int kMaxDevices = 64;
std::mutex g_noalloc_mu;
void* g_noalloc_ptr[kMaxDevices] = {};
CUcontext g_noalloc_ctx[kMaxDevices] = {};  // the context the address was looked up in

typedef CUresult (*CtxGetCurrentFn)(CUcontext*);
CtxGetCurrentFn ctx_get_current_fn() {
  static CtxGetCurrentFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<CtxGetCurrentFn>(f);
  });
  return fn;
}
}  // namespace

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

extern "C" jolt_status jolt_decode_attn_noalloc(const jolt_shape* shape, const jolt_cell_choice* choices,
                                                const void* cache, int32_t layer_begin, int32_t n_layers_call,
                                                const void* q, void* out, float* lse, const float* inv_freq,
                                                int32_t pos_offset, void* stream) {
  if (!decode_args_ok(shape, choices, cache, layer_begin, n_layers_call, q, out, inv_freq, pos_offset))
    return JOLT_ERR_INVALID_ARG;
  // the scratch this call needs must fit the static array
  if (decode_ws_layout(*shape, n_layers_call, choose_splits(*shape, n_layers_call)).total > kNoAllocScratchBytes)
    return JOLT_ERR_WORKSPACE;
  int dev = 0;
  JOLT_CUDA_TRY(cudaGetDevice(&dev));
  if (dev < 0 || dev >= kMaxDevices) return JOLT_ERR_INVALID_ARG;
  void* ws = nullptr;
  {
    // the address is looked up once per device and context: a context the device got since (after
    // cudaDeviceReset, say) holds the array at a new address
    CUcontext ctx = nullptr;
    if (CtxGetCurrentFn get = ctx_get_current_fn()) get(&ctx);
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev] || g_noalloc_ctx[dev] != ctx) {
      void* ptr = nullptr;
      const cudaError_t e = cudaGetSymbolAddress(&ptr, g_noalloc_scratch);
      if (e != cudaSuccess || !ptr) return JOLT_ERR_CUDA;
      g_noalloc_ptr[dev] = ptr;
      g_noalloc_ctx[dev] = ctx;
    }
    ws = g_noalloc_ptr[dev];
  }
  // every call shares the array: the error word must start at zero; everything else the decode
  // kernels read is written earlier in the same call
  JOLT_CUDA_TRY(cudaMemsetAsync(ws, 0, sizeof(WsHeader), static_cast<cudaStream_t>(stream)));
  return jolt_decode_attn(shape, choices, cache, layer_begin, n_layers_call, q, out, lse, inv_freq, pos_offset, ws,
                          kNoAllocScratchBytes, stream);
}
