// Fused split-T decode attention over the stored factors: bf16 caches, keys stored after RoPE
// (no per-token rotation), d_h = 128, 32 query heads over 4 or 8 KV heads.
//
// One CTA per (sequence, layer, token split) walks its 128-token tiles once and reads every byte
// of the layer's compressed cache it needs exactly once from HBM (the group's U_T tiles are shared
// through L2 by the CTAs of the group's layers, which run side by side):
//   scores   s[t][j] = U_T^K[t] . P[:, j] + scale_t (codes^K_t . R q_j) + zero_t sum(R q_j), with
//            P = G^K (U_d^K^T q) ("A JoLT for the KV cache", §4.5: attention evaluated directly
//            over the stored factors; §3: the residual stored after a seeded rotation R)
//   softmax  online, per query head, in registers (exp2 domain; the reference maximum moves only
//            when a tile exceeds it by more than 2^8, so rescaling the accumulators is rare)
//   values   W[r][j] += sum_t U_T^V[t][r] p~[t][j] and acc[d][j] += sum_t p~[t][j] deq(codes^V_t)[d]
//   partials (m, l, W, acc) per split go to the workspace; k_decode_merge combines the splits and
//            applies U_d^V G^V^T and the inverse rotation.
// Where each contraction runs:
//   * U_T^K P (M = 128 tokens, N = 64: the 32 query heads' P as bf16 hi and lo columns, K = r_T)
//     and W (M = 128 rank rows per chunk, N = 32 heads, K = tokens; U_T^V
//     read MN-major, P~ K-major) on tcgen05 with TMEM accumulators, operands staged by TMA;
//   * both residual contractions (codes . R q and P~-weighted codes) on mma.sync m16n8k16 with
//     the f16 operands built in registers straight from the packed codes in shared memory (each
//     b-bit field becomes an exact f16 integer with one mask-and-or and one add): the codes are
//     never expanded to 16 bits in memory, which would cost four times their size in shared-memory
//     traffic per contraction. The key residual is stored into the tile's TMEM score buffer first
//     and the factor products accumulate on top of it, so the scores arrive complete.
// Warp roles (640 threads, five warpgroups whose register budgets are re-split with setmaxnreg):
//   0: warp 0 TMA producers (one lane per operand ring), warp 1 score-product issuer (owns TMEM),
//      warp 2 value-product issuer;
//   1, 2: key-residual warps, two per TMEM lane quarter (16 tokens each; the first stores the
//      quarter's 32 rows into TMEM);
//   3: softmax warps (thread = token of the tile: scores from TMEM, online softmax, P~);
//   4: value warps (value-residual MMAs, 32 features each).
// TMEM: two score buffers of 64 columns, W (32 columns per 128-rank chunk) from column 128, the
// value-residual accumulators (8 columns per KV head) from column 384.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <type_traits>
#include <vector>

#include "common.cuh"
#include "decode.cuh"
#include "gemm_tc.cuh"
#include "mma_codes.cuh"
#include "sm100.cuh"
#include "stats.h"

namespace jolt {

namespace {

constexpr int kD = 128;           // head dimension
constexpr int kBM = 128;          // tokens per tile
constexpr int kBK = 64;           // rank chunk of the score MMA
constexpr int kNQ = 32;           // query heads per layer this kernel serves
constexpr int kMaxFusedCells = 64;   // cells one launch references (tensor-map table)
constexpr int kMaxFusedRows = 512;   // (sequence, layer) rows one launch serves
constexpr int kKStages = 2, kVStages = 3, kCStages = 2;
constexpr int kKStageBytes = kBM * kBK * 2 + 2 * kNQ * kBK * 2;  // U_T^K chunk + P hi/lo chunk
constexpr int kVStageBytes = 2 * 64 * 64 * 2;                    // U_T^V: 128 ranks x 64 tokens
constexpr int kCStageBytes = 16384;                              // codes of 8/b heads x 128 tokens
constexpr int kPtBytes = kNQ * kBM * 2;                          // P~ (bf16, K-major, 32 rows)
constexpr int kWbBytes = kNQ * 256;                              // value weights (f16 fragments)
constexpr int kScrStride = kNQ + 1;                              // floats per token row of the exchange (odd: no bank conflicts)
constexpr int kScrBytes = 4 * 32 * kScrStride * 4;
constexpr int kQfBytes = kNQ * 256;                              // query fragments (f16)

constexpr int kOffK = 0;
constexpr int kOffV = kOffK + kKStages * kKStageBytes;
constexpr int kOffPt = kOffV + kVStages * kVStageBytes;
constexpr int kOffCK = kOffPt + 2 * kPtBytes;
constexpr int kOffCV = kOffCK + kCStages * kCStageBytes;
constexpr int kOffWb = kOffCV + kCStages * kCStageBytes;
constexpr int kOffScr = kOffWb + 2 * kWbBytes;
constexpr int kOffQf = kOffScr + kScrBytes;
constexpr int kOffRed = kOffQf + kQfBytes;          // [2][4][32] floats
constexpr int kOffAlpha = kOffRed + 2 * 4 * 32 * 4; // [2][64] floats: alpha[32], flag
constexpr int kOffFin = kOffAlpha + 2 * 64 * 4;     // [4][32] float2
constexpr int kOffZf = kOffFin + 4 * 32 * 8;        // [32]
constexpr int kOffQs = kOffZf + 32 * 4;             // [32]
constexpr int kOffZk = kOffQs + 32 * 4;             // [4 warps][8 heads][32 tokens] key scale/zero pairs
constexpr int kOffBars = kOffZk + 4 * 8 * 32 * 4;
constexpr int kNumBars = 32;
constexpr int kSmemUsed = kOffBars + kNumBars * 8 + 16;
constexpr int kSmem = kSmemUsed + 1024;             // 1024-byte alignment of the swizzled tiles
static_assert(kSmem <= 232448, "fused decode shared memory");
static_assert(kOffV % 1024 == 0 && kOffPt % 1024 == 0, "swizzled tiles need 1024-byte alignment");
static_assert(kOffCK % 16 == 0 && kOffCV % 16 == 0 && kOffBars % 8 == 0, "bulk-copy and mbarrier alignment");

constexpr int kThreads = 640;  // five warpgroups: control, key residual (two), softmax, value residual
// registers a thread after the warpgroups' re-split (launch: 128 each, 65536 in all)
constexpr int kRegCtl = 40, kRegKres = 96, kRegSoft = 168, kRegVres = 80;
constexpr uint32_t kTmemCols = 512;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.f;  // log2 units: p~ <= 2^8 between rescales

struct FusedCell {
  const uint8_t* codes;  // [L_g][n_kv][T][16 b] or null
  const __half2* sz;     // [L_g][n_kv][T] or null
  int r_T, b;
};

struct FusedMaps {
  CUtensorMap p;                      // P hi/lo [B*Lc][2*32][q_cap] bf16, K-major, box 64 x 64
  CUtensorMap ut[kMaxFusedCells];     // key cells: U_T [T][r_T] K-major box 64 x 128; value cells: MN-major box 64 x 64
};

struct FusedArgs {
  int T, nt, tps, S, Lc, Lg, layer_begin, g_first, Gc, n_kv, gq, q_cap;
  float attn_scale;
  const float* qrot;   // [B][Lc][32][128] of this launch set
  const float* qsum;   // [B][Lc][32]
  float* part;         // [B][Lc][32][S][2 + q_cap + 128]
  int32_t* err;
  FusedCell cells[kMaxFusedCells];  // (b * Gc + g - g_first) * 2 + kv
};

__device__ __forceinline__ void named_bar(int id, int n) { asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory"); }

// Within a lane's 32-code segment of a key-residual row, pair p (16 pairs, in the order the
// conversion produces them) holds the codes at offsets (lo, lo + gap).
__device__ __forceinline__ int pair_lo(int bits, int p) {
  return bits == 4 ? 8 * (p >> 2) + (p & 3) : bits == 2 ? 16 * (p >> 3) + (p & 7) : 4 * (p >> 1) + (p & 1);
}
__device__ __forceinline__ int pair_gap(int bits) { return bits == 4 ? 4 : bits == 2 ? 8 : 2; }

// Warp reduce-scatter over 32 values: afterwards v[0] of lane l combines value index l of all lanes.
template <bool MAX>
__device__ __forceinline__ float reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int w = 16; w >= 1; w >>= 1) {
    const bool up = (lane & w) != 0;
#pragma unroll
    for (int i = 0; i < w; ++i) {
      const float keep = up ? v[i + w] : v[i];
      const float send = up ? v[i] : v[i + w];
      const float got = __shfl_xor_sync(0xffffffffu, send, w);
      v[i] = MAX ? fmaxf(keep, got) : keep + got;
    }
  }
  return v[0];
}

// Key residual of KV head h (codes in slot k of the stage at cs) for the 16 tokens 32 q + 16 mb ..
// of quarter q: scr[token][h g_q + j] = scale (codes . R q_j) + zero sum(R q_j). zrow[i]: the
// (scale, zero) pair of token 32 q + 16 mb + i for this head.
template <int BITS, int GQ>
__device__ __forceinline__ void kres_head(const uint8_t* cs, int k, int h, int q, int mb, int lane, const uint2* qf,
                                          const float* qs, float* scr, const uint32_t* zrow) {
  constexpr int RB = 16 * BITS;
  const int gr = lane >> 2, m4 = lane & 3;
  uint2 bqs[8];  // the head's query fragments
#pragma unroll
  for (int kc = 0; kc < 8; ++kc) bqs[kc] = gr < GQ ? qf[((h * 8 + kc) * GQ + gr) * 4 + m4] : make_uint2(0u, 0u);
  {
    const int rA = 32 * q + 16 * mb + gr;  // tile rows of fragment rows g and g + 8
    const uint8_t* rowA = cs + (k * kBM + rA) * RB;
    const uint8_t* rowB = rowA + 8 * RB;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    uint32_t xa[8], xb[8];
    if (BITS == 4) {
      const uint4 u = *reinterpret_cast<const uint4*>(rowA + 16 * m4), v = *reinterpret_cast<const uint4*>(rowB + 16 * m4);
      xa[0] = u.x; xa[1] = u.y; xa[2] = u.z; xa[3] = u.w;
      xb[0] = v.x; xb[1] = v.y; xb[2] = v.z; xb[3] = v.w;
    } else if (BITS == 2) {
      const uint2 u = *reinterpret_cast<const uint2*>(rowA + 8 * m4), v = *reinterpret_cast<const uint2*>(rowB + 8 * m4);
      xa[0] = u.x; xa[1] = u.y;
      xb[0] = v.x; xb[1] = v.y;
    } else {
      const uint4 u0 = *reinterpret_cast<const uint4*>(rowA + 32 * m4), u1 = *reinterpret_cast<const uint4*>(rowA + 32 * m4 + 16);
      const uint4 v0 = *reinterpret_cast<const uint4*>(rowB + 32 * m4), v1 = *reinterpret_cast<const uint4*>(rowB + 32 * m4 + 16);
      xa[0] = u0.x; xa[1] = u0.y; xa[2] = u0.z; xa[3] = u0.w; xa[4] = u1.x; xa[5] = u1.y; xa[6] = u1.z; xa[7] = u1.w;
      xb[0] = v0.x; xb[1] = v0.y; xb[2] = v0.z; xb[3] = v0.w; xb[4] = v1.x; xb[5] = v1.y; xb[6] = v1.z; xb[7] = v1.w;
    }
#pragma unroll
    for (int kc = 0; kc < 8; ++kc) {
      uint32_t af[4];
      if (BITS == 4) {
        const uint32_t wa = xa[kc >> 1] >> ((kc & 1) * 8), wb = xb[kc >> 1] >> ((kc & 1) * 8);
        af[0] = nib_lo(wa); af[2] = nib_hi(wa);
        af[1] = nib_lo(wb); af[3] = nib_hi(wb);
      } else if (BITS == 2) {
        const int sft = ((kc & 3) >= 2) ? 8 : 0, s0 = (2 * (kc & 3)) & 3;
        const uint32_t wa = xa[kc >> 2] >> sft, wb = xb[kc >> 2] >> sft;
        af[0] = crumb(wa, s0); af[2] = crumb(wa, s0 + 1);
        af[1] = crumb(wb, s0); af[3] = crumb(wb, s0 + 1);
      } else {
        af[0] = byte_pair(xa[kc], 0x4240); af[2] = byte_pair(xa[kc], 0x4341);
        af[1] = byte_pair(xb[kc], 0x4240); af[3] = byte_pair(xb[kc], 0x4341);
      }
      mma_f16_16816(acc, af, bqs[kc].x, bqs[kc].y);
    }
    // rows g (tile row rA) and g + 8, query heads 2 m4, 2 m4 + 1 of KV head h
    const uint32_t zA = zrow[gr];
    const uint32_t zB = zrow[gr + 8];
    const float2 fA = __half22float2(*reinterpret_cast<const __half2*>(&zA));
    const float2 fB = __half22float2(*reinterpret_cast<const __half2*>(&zB));
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = 2 * m4 + e;
      if (j < GQ) {
        const float qsj = qs[h * GQ + j];
        scr[(16 * mb + gr) * kScrStride + h * GQ + j] = fA.x * acc[e] + fA.y * qsj;
        scr[(16 * mb + gr + 8) * kScrStride + h * GQ + j] = fB.x * acc[2 + e] + fB.y * qsj;
      }
    }
  }
}

// Value residual of KV head h (codes in slot k of the stage at cs) for one tile: eight chunks of 16
// tokens, feature pairs (d, d+1) and (d+2, d+3) with d = 16 g + 4 vw; ac[0], ac[1] the fragments.
template <int BITS, int GQ>
__device__ __forceinline__ void vres_head(float (&ac)[2][4], const uint8_t* cs, int k, const uint2* wbp, int h,
                                          int vw, int lane) {
  constexpr int RB = 16 * BITS;
  const int gr = lane >> 2, m4 = lane & 3;
  const uint8_t* base = cs + k * kBM * RB;
#pragma unroll
  for (int kc = 0; kc < 8; ++kc) {
    const int r0 = 16 * kc + m4;  // tile rows of tokens e = 0..3: r0 + 4 e
    uint32_t f0[4], f1[4];
    if (BITS == 4) {
      const uint8_t* p = base + 8 * gr + 2 * vw;
      const uint32_t xA = *reinterpret_cast<const uint16_t*>(p + (r0 + 0) * RB);
      const uint32_t xB = *reinterpret_cast<const uint16_t*>(p + (r0 + 4) * RB);
      const uint32_t xC = *reinterpret_cast<const uint16_t*>(p + (r0 + 8) * RB);
      const uint32_t xD = *reinterpret_cast<const uint16_t*>(p + (r0 + 12) * RB);
      const uint32_t u = xA | (xB << 16), w = xC | (xD << 16);
      f0[0] = nib_lo(u); f0[1] = nib_hi(u); f0[2] = nib_lo(w); f0[3] = nib_hi(w);
      f1[0] = nib_lo(u >> 8); f1[1] = nib_hi(u >> 8); f1[2] = nib_lo(w >> 8); f1[3] = nib_hi(w >> 8);
    } else if (BITS == 2) {
      const uint8_t* p = base + 4 * gr + vw;
      const uint32_t xA = p[(r0 + 0) * RB], xB = p[(r0 + 4) * RB];
      const uint32_t xC = p[(r0 + 8) * RB], xD = p[(r0 + 12) * RB];
      const uint32_t u = xA | (xB << 16), w = xC | (xD << 16);
      f0[0] = crumb(u, 0); f0[1] = crumb(u, 1); f0[2] = crumb(w, 0); f0[3] = crumb(w, 1);
      f1[0] = crumb(u, 2); f1[1] = crumb(u, 3); f1[2] = crumb(w, 2); f1[3] = crumb(w, 3);
    } else {
      const uint8_t* p = base + 16 * gr + 4 * vw;
      const uint32_t xA = *reinterpret_cast<const uint32_t*>(p + (r0 + 0) * RB);
      const uint32_t xB = *reinterpret_cast<const uint32_t*>(p + (r0 + 4) * RB);
      const uint32_t xC = *reinterpret_cast<const uint32_t*>(p + (r0 + 8) * RB);
      const uint32_t xD = *reinterpret_cast<const uint32_t*>(p + (r0 + 12) * RB);
      const uint32_t u0 = __byte_perm(xA, xB, 0x5140), u1 = __byte_perm(xA, xB, 0x7362);
      const uint32_t w0 = __byte_perm(xC, xD, 0x5140), w1 = __byte_perm(xC, xD, 0x7362);
      f0[0] = byte_pair(u0, 0x4140); f0[1] = byte_pair(u0, 0x4342);
      f0[2] = byte_pair(w0, 0x4140); f0[3] = byte_pair(w0, 0x4342);
      f1[0] = byte_pair(u1, 0x4140); f1[1] = byte_pair(u1, 0x4342);
      f1[2] = byte_pair(w1, 0x4140); f1[3] = byte_pair(w1, 0x4342);
    }
    uint2 bw = make_uint2(0u, 0u);
    if (gr < GQ) bw = wbp[((h * 8 + kc) * 4 + m4) * GQ + gr];
    mma_f16_16816(ac[0], f0, bw.x, bw.y);
    mma_f16_16816(ac[1], f1, bw.x, bw.y);
  }
}

// The key residual of one tile for this warp's 32 tokens, head after head (a runtime loop: one
// copy of the head's code per code width keeps the hot loop small), releasing each code stage.
template <int BITS, int GQ>
__device__ __forceinline__ bool kres_tile(const uint8_t* cbase, uint32_t full0, uint32_t empty0, int& ckit, int q,
                                       int mb, int lane, const uint2* qf, const float* qs, float* scr,
                                       const uint32_t* zks, int32_t* err, bool ok) {
  constexpr int NKV = kNQ / GQ, hps = 8 / BITS;
  int s = 0;
#pragma unroll 1
  for (int h = 0; h < NKV; ++h) {
    const int k = h % hps;
    if (k == 0) {
      s = ckit % kCStages;
      if (ok) ok = __all_sync(0xffffffffu, sm100::mbar_wait(full0 + 8u * s, (ckit / kCStages) & 1, err));
    }
    kres_head<BITS, GQ>(cbase + s * kCStageBytes, k, h, q, mb, lane, qf, qs, scr, zks + h * 16);
    if (k == hps - 1 || h == NKV - 1) {
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(empty0 + 8u * s);
      ++ckit;
    }
  }
  return ok;
}

// The value residual of one tile for this warp's features, head after head; the accumulators of
// head h live in TMEM columns tacc + 8 h of the warp's lane quarter (loaded, updated, stored back).
template <int BITS, int GQ>
__device__ __forceinline__ bool vres_tile(const uint8_t* cbase, uint32_t full0, uint32_t empty0, int& cvit,
                                       const uint2* wbp, uint32_t tacc, int vw, int lane, int32_t* err, bool ok) {
  constexpr int NKV = kNQ / GQ, hps = 8 / BITS;
  int s = 0;
#pragma unroll 1
  for (int h = 0; h < NKV; ++h) {
    const int k = h % hps;
    if (k == 0) {
      s = cvit % kCStages;
      if (ok) ok = __all_sync(0xffffffffu, sm100::mbar_wait(full0 + 8u * s, (cvit / kCStages) & 1, err));
    }
    uint32_t r[8];
    sm100::tmem_ld8(tacc + 8 * h, r);
    sm100::tmem_ld_wait();
    float ac[2][4];
#pragma unroll
    for (int e = 0; e < 8; ++e) ac[e >> 2][e & 3] = __uint_as_float(r[e]);
    vres_head<BITS, GQ>(ac, cbase + s * kCStageBytes, k, wbp, h, vw, lane);
#pragma unroll
    for (int e = 0; e < 8; ++e) r[e] = __float_as_uint(ac[e >> 2][e & 3]);
    sm100::tmem_st8(tacc + 8 * h, r);
    if (k == hps - 1 || h == NKV - 1) {
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(empty0 + 8u * s);
      ++cvit;
    }
  }
  sm100::tmem_st_wait();
  return ok;
}

template <int GQ>
__global__ void __launch_bounds__(kThreads, 1) k_decode_fused(const __grid_constant__ FusedMaps maps, const FusedArgs a) {
  constexpr int NKV = kNQ / GQ;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  const uint32_t sb = sm100::smem_u32(smem);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kOffBars);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);
  const uint32_t bar0 = sm100::smem_u32(bars);
  auto BK_FULL = [&](int s) { return bar0 + 8u * (0 + s); };
  auto BK_EMPTY = [&](int s) { return bar0 + 8u * (2 + s); };
  auto BV_FULL = [&](int s) { return bar0 + 8u * (4 + s); };
  auto BV_EMPTY = [&](int s) { return bar0 + 8u * (7 + s); };
  auto BCK_FULL = [&](int s) { return bar0 + 8u * (10 + s); };
  auto BCK_EMPTY = [&](int s) { return bar0 + 8u * (12 + s); };
  auto BCV_FULL = [&](int s) { return bar0 + 8u * (14 + s); };
  auto BCV_EMPTY = [&](int s) { return bar0 + 8u * (16 + s); };
  auto BS_FULL = [&](int s) { return bar0 + 8u * (18 + s); };   // score products done
  auto BS_EMPTY = [&](int s) { return bar0 + 8u * (20 + s); };  // softmax warps have read S
  auto BP_FULL = [&](int s) { return bar0 + 8u * (22 + s); };
  auto BP_EMPTY = [&](int s) { return bar0 + 8u * (24 + s); };
  auto BW_DONE = [&](int s) { return bar0 + 8u * (26 + s); };
  const uint32_t BDRAIN = bar0 + 8u * 28;
  auto BR_FULL = [&](int s) { return bar0 + 8u * (29 + s); };   // key residual stored into S

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int wg = warp >> 2;
  // this CTA's (sequence, split, layer): layers fastest, so the CTAs of one layer group that share
  // U_T tiles run side by side
  const int li = blockIdx.x % a.Lc;
  const int sp = (blockIdx.x / a.Lc) % a.S;
  const int bi = blockIdx.x / (a.Lc * a.S);
  const int layer = a.layer_begin + li, g = layer / a.Lg, ll = layer % a.Lg;
  const int ci = (bi * a.Gc + (g - a.g_first)) * 2;
  const FusedCell ck = a.cells[ci], cv = a.cells[ci + 1];
  const int tile0 = sp * a.tps;
  const int ntl = max(0, min(a.nt, tile0 + a.tps) - tile0);  // tiles of this CTA
  const int bl = bi * a.Lc + li;                              // (sequence, layer) row of the call
  const int nkb = ck.r_T > 0 ? (ck.r_T + kBK - 1) / kBK : 0;
  const int nmc = cv.r_T > 0 ? (cv.r_T + 127) / 128 : 0;
  const int bK = ck.b, bV = cv.b;
  const int rbK = 16 * bK, rbV = 16 * bV;                    // bytes per code row
  const int hpsK = bK ? 8 / bK : 1, hpsV = bV ? 8 / bV : 1;  // heads per code stage
  const int njK = bK ? (NKV + hpsK - 1) / hpsK : 0;
  const int njV = bV ? (NKV + hpsV - 1) / hpsV : 0;
  const size_t prow = size_t(2 + a.q_cap + kD);

  if (threadIdx.x == 0) {
    // arrival counts: TMA / MMA-commit barriers 1; code-stage releases, S releases, P~ hand-offs
    // and residual hand-offs 4 (one per consuming warp); a P~ buffer is free after the value
    // products (1 commit) and the four value warps
    for (int i = 0; i < 31; ++i) {
      uint32_t cnt = 1;
      if ((i >= 16 && i < 18) || (i >= 20 && i < 24) || i >= 29) cnt = 4;
      if (i >= 12 && i < 14) cnt = 8;  // key code stages: released by all eight key-residual warps
      if (i >= 24 && i < 26) cnt = 5;
      if (i == 28) cnt = 2;  // the drain: one commit per MMA-issuing thread
      sm100::mbar_init(bar0 + 8u * i, cnt);
    }
    sm100::fence_mbar_init();
    sm100::prefetch_tmap(&maps.p);
    if (nkb) sm100::prefetch_tmap(&maps.ut[ci]);
    if (nmc) sm100::prefetch_tmap(&maps.ut[ci + 1]);
  }
  if (warp == 1) sm100::tmem_alloc(sm100::smem_u32(tmem_slot), kTmemCols);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  // S: two buffers of 64 columns (hi and lo halves); W (up to 8 chunks of 32 columns) from column
  // 128; the value residual accumulators (8 columns per KV head) from column 384
  const uint32_t tS = tmem, tW = tmem + 128, tAcc = tmem + 384;

  if (wg == 0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegCtl));
    if (warp == 0 && lane < 4) {
      // ================= TMA producers: one lane per ring, each running ahead on its own =========
      // lane 0: U_T^K + P chunks, lane 1: key code stages, lane 2: U_T^V chunks, lane 3: value code
      // stages; a lane waits only for its own ring's free slots
      bool ok = true;
      int cnt = 0;
      const bool kside = lane < 2;
      const FusedCell& cell = kside ? ck : cv;
      const int rb = kside ? rbK : rbV, hps = kside ? hpsK : hpsV, nj = kside ? njK : njV;
      const uint8_t* codes = cell.codes ? cell.codes + int64_t(ll) * NKV * a.T * rb : nullptr;
      for (int it = 0; it < ntl && ok; ++it) {
        const int t0 = (tile0 + it) * kBM, nv = min(kBM, a.T - t0);
        if (lane == 0) {
          for (int kb = 0; kb < nkb && ok; ++kb, ++cnt) {
            const int s = cnt % kKStages;
            if (!(ok = sm100::mbar_wait(BK_EMPTY(s), ((cnt / kKStages) & 1) ^ 1, a.err))) break;
            sm100::mbar_expect_tx(BK_FULL(s), kKStageBytes);
            const uint32_t dst = sb + kOffK + s * kKStageBytes;
            sm100::tma_load_3d(dst, &maps.ut[ci], BK_FULL(s), kb * kBK, t0, 0);
            sm100::tma_load_3d(dst + kBM * kBK * 2, &maps.p, BK_FULL(s), kb * kBK, 0, bl);
          }
        } else if (lane == 2) {
          for (int mc = 0; mc < nmc && ok; ++mc)
            for (int h2 = 0; h2 < 2 && ok; ++h2, ++cnt) {
              const int s = cnt % kVStages;
              if (!(ok = sm100::mbar_wait(BV_EMPTY(s), ((cnt / kVStages) & 1) ^ 1, a.err))) break;
              sm100::mbar_expect_tx(BV_FULL(s), kVStageBytes);
              const uint32_t dst = sb + kOffV + s * kVStageBytes;
              sm100::tma_load_3d(dst, &maps.ut[ci + 1], BV_FULL(s), mc * 128, t0 + 64 * h2, 0);
              sm100::tma_load_3d(dst + 8192, &maps.ut[ci + 1], BV_FULL(s), mc * 128 + 64, t0 + 64 * h2, 0);
            }
        } else {
          for (int jb = 0; jb < nj && ok; ++jb, ++cnt) {
            const int s = cnt % kCStages;
            const uint32_t full = kside ? BCK_FULL(s) : BCV_FULL(s);
            const uint32_t empty = kside ? BCK_EMPTY(s) : BCV_EMPTY(s);
            if (!(ok = sm100::mbar_wait(empty, ((cnt / kCStages) & 1) ^ 1, a.err))) break;
            const int h0 = jb * hps, nh = min(hps, NKV - h0);
            sm100::mbar_expect_tx(full, uint32_t(nh * nv * rb));
            const uint32_t dst = sb + (kside ? kOffCK : kOffCV) + s * kCStageBytes;
            for (int k = 0; k < nh; ++k)
              sm100::bulk_load(dst + k * kBM * rb, codes + (int64_t(h0 + k) * a.T + t0) * rb, uint32_t(nv * rb), full);
          }
        }
      }
      // the copies still in flight complete before the block may exit
      const int depth = lane == 0 ? kKStages : lane == 2 ? kVStages : kCStages;
      for (int i = max(0, cnt - depth); i < cnt; ++i) {
        const int s = i % depth;
        const uint32_t full = lane == 0 ? BK_FULL(s) : lane == 2 ? BV_FULL(s) : lane == 1 ? BCK_FULL(s) : BCV_FULL(s);
        sm100::mbar_wait(full, (i / depth) & 1, a.err);
      }
    } else if (warp == 1 && lane == 0) {
      // ================= score-product issuer: S(it) += U_T^K (P_hi + P_lo) =================
      // on the buffer the key-residual warps have filled (or overwriting it when there is no key
      // residual); blocking waits, so the thread spends no issue slots while it waits
      constexpr uint32_t idK = sm100::idesc_bf16_f32(kBM, 2 * kNQ, 0, 0);
      bool ok = true;
      int kit = 0;
      for (int it = 0; it < ntl && ok && nkb > 0; ++it) {
        if (!(ok = sm100::mbar_wait(BR_FULL(it & 1), (it >> 1) & 1, a.err))) break;
        sm100::tc_fence_after();
        const uint32_t dt = tS + (it & 1) * 2 * kNQ;
        for (int kb = 0; kb < nkb; ++kb, ++kit) {
          const int s = kit % kKStages;
          if (!(ok = sm100::mbar_wait(BK_FULL(s), (kit / kKStages) & 1, a.err))) break;
          sm100::tc_fence_after();
          const uint32_t ka = sb + kOffK + s * kKStageBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {  // N = 64: P hi rows 0-31 and lo rows 32-63
            const uint64_t ad = sm100::smem_desc_sw128(ka + kk * 32, 16, 1024);
            const uint64_t bd = sm100::smem_desc_sw128(ka + kBM * kBK * 2 + kk * 32, 16, 1024);
            sm100::mma_bf16(dt, ad, bd, idK, (bK > 0 || kb > 0 || kk > 0) ? 1u : 0u);
          }
          sm100::mma_commit(BK_EMPTY(s));
        }
        if (ok) sm100::mma_commit(BS_FULL(it & 1));
      }
      sm100::mma_commit(BDRAIN);
      sm100::mbar_wait(BDRAIN, 0, a.err);
    } else if (warp == 2 && lane == 0) {
      // ================= value-product issuer: W += U_T^V^T P~(it) =================
      constexpr uint32_t idW = sm100::idesc_bf16_f32(128, kNQ, 1, 0);
      bool ok = true;
      int vit = 0;
      for (int it = 0; it < ntl && ok; ++it) {
        if (!(ok = sm100::mbar_wait(BP_FULL(it & 1), (it >> 1) & 1, a.err))) break;
        for (int wst = 0; wst < 2 * nmc; ++wst, ++vit) {
          const int s = vit % kVStages;
          if (!(ok = sm100::mbar_wait(BV_FULL(s), (vit / kVStages) & 1, a.err))) break;
          sm100::tc_fence_after();
          const int mc = wst >> 1, h2 = wst & 1;
          const uint32_t va = sb + kOffV + s * kVStageBytes;
          const uint32_t pt = sb + kOffPt + (it & 1) * kPtBytes;
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sm100::smem_desc_sw128(va + kk * 2048, 8192, 1024);
            const uint64_t bd = sm100::smem_desc_sw128(pt + h2 * (kNQ * 128) + kk * 32, 16, 1024);
            sm100::mma_bf16(tW + mc * kNQ, ad, bd, idW, (it > 0 || h2 > 0 || kk > 0) ? 1u : 0u);
          }
          sm100::mma_commit(BV_EMPTY(s));
        }
        if (!ok) break;
        sm100::mma_commit(BW_DONE(it & 1));
        sm100::mma_commit(BP_EMPTY(it & 1));
      }
      sm100::mma_commit(BDRAIN);
      sm100::mbar_wait(BDRAIN, 0, a.err);
    }
  } else if (wg <= 2) {
    // ================= key-residual warps: S(it) starts as scale (codes . R q) + zero sum(R q) ====
    // two warps per TMEM lane quarter: warpgroup 1 takes tokens 32q .. 32q+15 of the tile (mb = 0),
    // warpgroup 2 tokens 32q+16 .. 32q+31 (mb = 1); the mb = 0 warp stores the quarter's rows
    const int q = warp & 3;            // TMEM lane quarter = tokens 32q .. 32q+31 of the tile
    const int mb = wg - 1;
    const int tid = threadIdx.x - 128; // 0..255
    float* scr = reinterpret_cast<float*>(smem + kOffScr) + q * 32 * kScrStride;
    float* qs = reinterpret_cast<float*>(smem + kOffQs);
    uint2* qf = reinterpret_cast<uint2*>(smem + kOffQf);
    // query-side operands of the key residual: f16 fragments of R q in the pair order of this
    // cell's code width ([h][chunk][g < g_q][m]), and sum(R q)
    const float* qr = a.qrot + int64_t(bl) * kNQ * kD;
    if (bK) {
      const int gap = pair_gap(bK);
      for (int e = tid; e < NKV * 8 * GQ * 4; e += 256) {
        const int mm = e & 3, gg = (e >> 2) % GQ, kc = (e / (4 * GQ)) & 7, h = e / (32 * GQ);
        const float* qj = qr + (h * GQ + gg) * kD + 32 * mm;
        const int p0 = pair_lo(bK, 2 * kc), p1 = pair_lo(bK, 2 * kc + 1);
        const __half2 w0 = __floats2half2_rn(qj[p0], qj[p0 + gap]);
        const __half2 w1 = __floats2half2_rn(qj[p1], qj[p1 + gap]);
        qf[e] = make_uint2(*reinterpret_cast<const uint32_t*>(&w0), *reinterpret_cast<const uint32_t*>(&w1));
      }
    }
    if (tid < kNQ) qs[tid] = a.qsum[int64_t(bl) * kNQ + tid];
    named_bar(3, 256);
    int ckit = 0;
    bool ok = true;
    const __half2* szK = ck.sz ? ck.sz + int64_t(ll) * NKV * a.T : nullptr;
    // the key scale / zero pairs of this warp's 16 tokens (lane & 15), loaded one tile ahead into
    // registers, then into the warp's slab [head][16 tokens]
    uint32_t* zks = reinterpret_cast<uint32_t*>(smem + kOffZk) + (mb * 4 + q) * 8 * 16;
    uint32_t nzk[NKV];
    auto load_sz = [&](int it2, uint32_t (&k_)[NKV]) {
      const int t2 = (tile0 + it2) * kBM + 32 * q + 16 * mb + (lane & 15);
      const bool ok2 = it2 < ntl && t2 < a.T;
#pragma unroll
      for (int h = 0; h < NKV; ++h) k_[h] = (bK && ok2) ? sm100::ld_nc_early(szK + int64_t(h) * a.T + t2) : 0u;
    };
    load_sz(0, nzk);
    for (int it = 0; it < ntl; ++it) {
      __syncwarp();  // every lane has read the slab before it is rewritten
      if (lane < 16)
#pragma unroll
        for (int h = 0; h < NKV; ++h) zks[h * 16 + lane] = nzk[h];
      __syncwarp();
      load_sz(it + 1, nzk);
      if (bK) {
        const uint8_t* cbase = smem + kOffCK;
        if (bK == 4) ok = kres_tile<4, GQ>(cbase, BCK_FULL(0), BCK_EMPTY(0), ckit, q, mb, lane, qf, qs, scr, zks, a.err, ok);
        else if (bK == 2) ok = kres_tile<2, GQ>(cbase, BCK_FULL(0), BCK_EMPTY(0), ckit, q, mb, lane, qf, qs, scr, zks, a.err, ok);
        else ok = kres_tile<8, GQ>(cbase, BCK_FULL(0), BCK_EMPTY(0), ckit, q, mb, lane, qf, qs, scr, zks, a.err, ok);
      }
      named_bar(4 + q, 64);  // both halves of the quarter's rows are in the exchange buffer
      if (mb == 0) {
        // the S buffer is free once the softmax warps have read tile it - 2
        if (ok) ok = __all_sync(0xffffffffu, sm100::mbar_wait(BS_EMPTY(it & 1), ((it >> 1) & 1) ^ 1, a.err));
        sm100::tc_fence_after();
        if (bK || nkb == 0) {
          // the residual into the hi columns, zeros into the lo columns (the products accumulate)
          uint32_t r[kNQ];
          const uint32_t ta = tS + (it & 1) * 2 * kNQ + (uint32_t(32 * q) << 16);
#pragma unroll
          for (int j = 0; j < kNQ; ++j) r[j] = bK ? __float_as_uint(scr[lane * kScrStride + j]) : 0u;
          sm100::tmem_st32(ta, r);
#pragma unroll
          for (int j = 0; j < kNQ; ++j) r[j] = 0u;
          sm100::tmem_st32(ta + kNQ, r);
          sm100::tmem_st_wait();
        }
        sm100::tc_fence_before();
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(BR_FULL(it & 1));
      }
      named_bar(4 + q, 64);  // the rows have been read before the next tile rewrites them
    }
  } else if (wg == 3) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(kRegSoft));
    // ================= softmax warps: complete scores from TMEM, online softmax, P~ =================
    const int q = warp & 3;            // TMEM lane quarter = tokens 32q .. 32q+31 of the tile
    float* red = reinterpret_cast<float*>(smem + kOffRed);
    float* alph = reinterpret_cast<float*>(smem + kOffAlpha);
    float2* fin = reinterpret_cast<float2*>(smem + kOffFin);
    float* zf = reinterpret_cast<float*>(smem + kOffZf);
    // the reference maximum of query head `lane` (mref) and of every head (mr, the same in all
    // threads); this thread's partial sums of p~ (ell) and of p~ zero (zac) per head over its tokens
    float mref = -INFINITY;
    float mr[kNQ], ell[kNQ], zac[kNQ];
#pragma unroll
    for (int j = 0; j < kNQ; ++j) {
      mr[j] = -INFINITY;
      ell[j] = 0.f;
      zac[j] = 0.f;
    }
    bool ok = true;
    const __half2* szV = cv.sz ? cv.sz + int64_t(ll) * NKV * a.T : nullptr;
    uint32_t zv[NKV], nzv[NKV];
    auto load_sz = [&](int it2, uint32_t (&v_)[NKV]) {
      const int t2 = (tile0 + it2) * kBM + 32 * q + lane;
      const bool ok2 = it2 < ntl && t2 < a.T;
#pragma unroll
      for (int h = 0; h < NKV; ++h) v_[h] = (bV && ok2) ? sm100::ld_nc_early(szV + int64_t(h) * a.T + t2) : 0u;
    };
    load_sz(0, nzv);
    for (int it = 0; it < ntl; ++it) {
      const int t0 = (tile0 + it) * kBM;
      const int tl = 32 * q + lane, t = t0 + tl;
      const bool valid = t < a.T;
#pragma unroll
      for (int h = 0; h < NKV; ++h) zv[h] = nzv[h];
      load_sz(it + 1, nzv);
      // ---- scores of token t for the 32 query heads (factor part + key residual) ----
      float sv[kNQ];
      {
        const uint32_t ready = nkb ? BS_FULL(it & 1) : BR_FULL(it & 1);
        if (ok) ok = __all_sync(0xffffffffu, sm100::mbar_wait(ready, (it >> 1) & 1, a.err));
        sm100::tc_fence_after();
        uint32_t r[kNQ], r2[kNQ];
        const uint32_t ta = tS + (it & 1) * 2 * kNQ + (uint32_t(32 * q) << 16);
        sm100::tmem_ld32(ta, r);
        sm100::tmem_ld32(ta + kNQ, r2);
        sm100::tmem_ld_wait();
#pragma unroll
        for (int j = 0; j < kNQ; ++j) sv[j] = __uint_as_float(r[j]) + __uint_as_float(r2[j]);
        sm100::tc_fence_before();
        __syncwarp();
        if (lane == 0) sm100::mbar_arrive(BS_EMPTY(it & 1));
      }
      const float sc2 = a.attn_scale * kLog2e;
#pragma unroll
      for (int j = 0; j < kNQ; ++j) sv[j] = valid ? sv[j] * sc2 : -INFINITY;
      // ---- the reference maximum moves only when a tile exceeds it by more than 2^8: each thread
      // checks its token against every head's reference; only then is the tile maximum formed ----
      bool ex = false;
#pragma unroll
      for (int j = 0; j < kNQ; ++j) ex |= sv[j] > mr[j] + kRescaleThreshold;
      float* exf = alph + (it & 1) * 64 + 40;  // one flag per warp (alpha and rescale flag sit below)
      const bool wex = __any_sync(0xffffffffu, ex);  // every lane votes; lane 0 publishes
      if (lane == 0) exf[q] = wex ? 1.f : 0.f;
      named_bar(1, 128);
      const bool any_ex = (exf[0] + exf[1]) + (exf[2] + exf[3]) != 0.f;
      float al = 1.f;
      bool resc = false;
      if (any_ex) {
        float tmp[kNQ];
#pragma unroll
        for (int j = 0; j < kNQ; ++j) tmp[j] = sv[j];
        const float wmax = reduce_scatter32<true>(tmp, lane);
        float* rd = red + (it & 1) * 128;
        rd[q * 32 + lane] = wmax;
        named_bar(1, 128);
        const float tmax = fmaxf(fmaxf(rd[lane], rd[32 + lane]), fmaxf(rd[64 + lane], rd[96 + lane]));
        const float mnew = (tmax > mref + kRescaleThreshold || mref == -INFINITY) ? fmaxf(tmax, mref) : mref;
        al = (mnew == mref) ? 1.f : exp2f(mref - mnew);
        resc = __any_sync(0xffffffffu, mnew != mref);
        mref = mnew;
#pragma unroll
        for (int j = 0; j < kNQ; ++j) {
          const float alj = __shfl_sync(0xffffffffu, al, j);
          mr[j] = __shfl_sync(0xffffffffu, mnew, j);
          ell[j] *= alj;
          zac[j] *= alj;
        }
      }
      // the P~ / weight buffer of this tile is free once tile it - 2's value products are done
      if (it >= 2 && ok) ok = __all_sync(0xffffffffu, sm100::mbar_wait(BP_EMPTY(it & 1), ((it >> 1) & 1) ^ 1, a.err));
      if (resc && it > 0 && nmc > 0) {
        // W (TMEM) holds tiles 0 .. it-1 at the old reference: rescale its columns once the last of
        // those products is done
        if (ok) ok = __all_sync(0xffffffffu, sm100::mbar_wait(BW_DONE((it - 1) & 1), ((it - 1) >> 1) & 1, a.err));
        sm100::tc_fence_after();
        for (int mc = 0; mc < nmc; ++mc) {
          uint32_t w[32];
          const uint32_t ta = tW + mc * kNQ + (uint32_t(32 * q) << 16);
          sm100::tmem_ld32(ta, w);
          sm100::tmem_ld_wait();
#pragma unroll
          for (int j = 0; j < kNQ; ++j) w[j] = __float_as_uint(__uint_as_float(w[j]) * __shfl_sync(0xffffffffu, al, j));
          sm100::tmem_st32(ta, w);
        }
        sm100::tmem_st_wait();
        sm100::tc_fence_before();
      }
      // ---- probabilities: P~ (bf16) for the U_T^V product, f16 weights for the value residual ----
      uint8_t* pt = smem + kOffPt + (it & 1) * kPtBytes;
      uint8_t* wbp = smem + kOffWb + (it & 1) * kWbBytes;
      const int kcT = tl >> 4, rT = tl & 15, eT = rT >> 2, mT = rT & 3;
      const int pc = tl >> 6, pu = (tl & 63) >> 3;
#pragma unroll
      for (int j = 0; j < kNQ; ++j) {
        const __nv_bfloat16 pb = __float2bfloat16_rn(valid ? exp2f(sv[j] - mr[j]) : 0.f);
        const float pf = __bfloat162float(pb);
        ell[j] += pf;
        // K-major, 128-byte swizzle: row j, tokens in two 64-token chunks
        *reinterpret_cast<__nv_bfloat16*>(pt + pc * (kNQ * 128) + j * 128 + ((pu ^ (j & 7)) << 4) + (tl & 7) * 2) = pb;
        const int h = j / GQ, gg = j % GQ;
        if (bV) {
          const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&zv[h]));
          zac[j] += f.y * pf;
          const __half w = __float2half_rn(pf * f.x * 0.00390625f);
          *reinterpret_cast<__half*>(wbp + ((((h * 8 + kcT) * 4 + mT) * GQ + gg) * 2 + (eT >> 1)) * 4 + (eT & 1) * 2) = w;
        }
      }
      if (q == 0) {
        alph[(it & 1) * 64 + lane] = al;
        if (lane == 0) alph[(it & 1) * 64 + 32] = resc ? 1.f : 0.f;
      }
      sm100::fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(BP_FULL(it & 1));
    }
    // ---- partials of this split: m (natural log), l; W from TMEM ----
    {
      const float L = reduce_scatter32<false>(ell, lane), Z = reduce_scatter32<false>(zac, lane);
      fin[q * 32 + lane] = make_float2(L, Z);
    }
    named_bar(1, 128);
    if (q == 0) {
      float L = 0.f, Z = 0.f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        L += fin[w * 32 + lane].x;
        Z += fin[w * 32 + lane].y;
      }
      zf[lane] = Z;
      float* pr = a.part + ((size_t(bl) * kNQ + lane) * a.S + sp) * prow;
      pr[0] = mref == -INFINITY ? -INFINITY : mref * kLn2;
      pr[1] = L;
    }
    if (nmc > 0 && ntl > 0) {
      if (ok) ok = __all_sync(0xffffffffu, sm100::mbar_wait(BW_DONE((ntl - 1) & 1), ((ntl - 1) >> 1) & 1, a.err));
      sm100::tc_fence_after();
      for (int mc = 0; mc < nmc; ++mc) {
        uint32_t w[32];
        sm100::tmem_ld32(tW + mc * kNQ + (uint32_t(32 * q) << 16), w);
        sm100::tmem_ld_wait();
        const int r = mc * 128 + 32 * q + lane;
        if (r < cv.r_T)
#pragma unroll
          for (int j = 0; j < kNQ; ++j) a.part[((size_t(bl) * kNQ + j) * a.S + sp) * prow + 2 + r] = __uint_as_float(w[j]);
      }
      sm100::tc_fence_before();
    }
    named_bar(2, 256);  // zf ready for the value warps
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(kRegVres));
    // ================= value warps: acc[d][j] += sum_t weight[t][j] codes^V[t][d] =================
    const int vw = warp & 3;  // features 16 g + 4 vw .. + 3
    const int gr = lane >> 2, m4 = lane & 3;
    const float* alph = reinterpret_cast<const float*>(smem + kOffAlpha);
    const float* zf = reinterpret_cast<const float*>(smem + kOffZf);
    // accumulators of head h: TMEM columns tAcc + 8 h of this warp's lane quarter
    const uint32_t tacc = tAcc + (uint32_t(32 * vw) << 16);
    {
      const uint32_t z[8] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
      for (int h = 0; h < NKV; ++h) sm100::tmem_st8(tacc + 8 * h, z);
      sm100::tmem_st_wait();
    }
    int cvit = 0;
    bool ok = true;
    for (int it = 0; it < ntl; ++it) {
      if (ok) ok = __all_sync(0xffffffffu, sm100::mbar_wait(BP_FULL(it & 1), (it >> 1) & 1, a.err));
      if (bV) {
        if (alph[(it & 1) * 64 + 32] != 0.f) {
          const float* al = alph + (it & 1) * 64;
#pragma unroll 1
          for (int h = 0; h < NKV; ++h) {
            const int j0 = h * GQ + 2 * m4;
            const float a0 = (2 * m4 < GQ) ? al[j0] : 0.f;
            const float a1 = (2 * m4 + 1 < GQ) ? al[j0 + 1] : 0.f;
            uint32_t r[8];
            sm100::tmem_ld8(tacc + 8 * h, r);
            sm100::tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 8; ++e) r[e] = __float_as_uint(__uint_as_float(r[e]) * ((e & 1) ? a1 : a0));
            sm100::tmem_st8(tacc + 8 * h, r);
          }
          sm100::tmem_st_wait();
        }
        const uint2* wbp = reinterpret_cast<const uint2*>(smem + kOffWb + (it & 1) * kWbBytes);
        const uint8_t* cbase = smem + kOffCV;
        if (bV == 4) ok = vres_tile<4, GQ>(cbase, BCV_FULL(0), BCV_EMPTY(0), cvit, wbp, tacc, vw, lane, a.err, ok);
        else if (bV == 2) ok = vres_tile<2, GQ>(cbase, BCV_FULL(0), BCV_EMPTY(0), cvit, wbp, tacc, vw, lane, a.err, ok);
        else ok = vres_tile<8, GQ>(cbase, BCV_FULL(0), BCV_EMPTY(0), cvit, wbp, tacc, vw, lane, a.err, ok);
      }
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(BP_EMPTY(it & 1));
    }
    named_bar(2, 256);
    // acc entries: features d = 16 g + 4 vw + 2 mb + (0 | 1), query heads h g_q + 2 m4 + (0 | 1);
    // the stored value is 256 acc (the weights carry 2^-8) + sum_t p~ zero
#pragma unroll 1
    for (int h = 0; h < NKV; ++h) {
      uint32_t r[8];
      sm100::tmem_ld8(tacc + 8 * h, r);
      sm100::tmem_ld_wait();
      float acc[2][4];
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[e >> 2][e & 3] = __uint_as_float(r[e]);
#pragma unroll
      for (int e = 0; e < 2; ++e) {
        const int jj = 2 * m4 + e;
        if (jj >= GQ) continue;
        const int j = h * GQ + jj;
        float* pr = a.part + ((size_t(bl) * kNQ + j) * a.S + sp) * prow + 2 + a.q_cap;
        const float z = zf[j];
#pragma unroll
        for (int mb = 0; mb < 2; ++mb) {
          const int d = 16 * gr + 4 * vw + 2 * mb;
          pr[d] = 256.f * acc[mb][e] + z;
          pr[d + 1] = 256.f * acc[mb][2 + e] + z;
        }
      }
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) sm100::tmem_dealloc(tmem, kTmemCols);
}

// One key cell's stored factors for a (sequence, layer) row of a launch set.
struct PRow {
  const __nv_bfloat16* G;   // G^K of the row's layer: [n_kv][r_T][r_d]
  const __nv_bfloat16* Ud;  // U_d^K [128][r_d]
  int r_T, r_d;
};
struct PTab {
  PRow row[kMaxFusedRows];
};

// P = G^K_h (U_d^K^T q) for the g_q query heads of one KV head, written as bf16 hi rows then lo rows
// per (sequence, layer): out [B*Lc][64][q_cap], zero from r_T up to the 64-rank chunk boundary
// (those columns meet the zero fill of U_T's tensor map). grid (n_kv, B*Lc), 256 threads: q-hat =
// U_d^T q for the KV head's query heads in shared memory (thread c over the U_d rows, one load per
// row for all g_q heads), then a thread per row r of G_h (sixteen 16-byte loads in flight, q-hat
// read as broadcasts), no cross-lane reductions.
template <int GQ>
__global__ void __launch_bounds__(256) k_prologue_p(const __nv_bfloat16* __restrict__ q, int q_cap, const PTab tab,
                                                   __nv_bfloat16* __restrict__ out) {
  const int h = blockIdx.x, bl = blockIdx.y;
  const PRow pr = tab.row[bl];
  __shared__ float qs[GQ][kD];
  __shared__ __align__(16) float qh[kD][GQ];  // [feature][head]
  for (int e = threadIdx.x; e < GQ * kD; e += blockDim.x)
    qs[e / kD][e % kD] = __bfloat162float(q[(int64_t(bl) * kNQ + h * GQ) * kD + e]);
  __syncthreads();
  {
    // thread (c, half): rows i of U_d in one half of the features; halves added through shared memory
    const int c = threadIdx.x & (kD - 1), half = threadIdx.x >> 7;
    float acc[GQ];
#pragma unroll
    for (int j = 0; j < GQ; ++j) acc[j] = 0.f;
    if (c < pr.r_d && pr.r_T > 0) {
#pragma unroll 8
      for (int i = half * (kD / 2); i < (half + 1) * (kD / 2); ++i) {
        const float u = __bfloat162float(pr.Ud[int64_t(i) * pr.r_d + c]);
#pragma unroll
        for (int j = 0; j < GQ; ++j) acc[j] = fmaf(u, qs[j][i], acc[j]);
      }
    }
    if (half == 1)
#pragma unroll
      for (int j = 0; j < GQ; ++j) qh[c][j] = acc[j];
    __syncthreads();
    if (half == 0)
#pragma unroll
      for (int j = 0; j < GQ; ++j) qh[c][j] = c < pr.r_d ? acc[j] + qh[c][j] : 0.f;
  }
  __syncthreads();
  const int64_t n = int64_t(kNQ) * q_cap;
  __nv_bfloat16* hi = out + int64_t(bl) * 2 * n;
  __nv_bfloat16* lo = hi + n;
  const int rend = min(q_cap, (pr.r_T + 63) / 64 * 64);
  const __nv_bfloat16* Gh = pr.G + int64_t(h) * pr.r_T * pr.r_d;
  for (int r = threadIdx.x; r < rend; r += blockDim.x) {
    float acc[GQ];
#pragma unroll
    for (int j = 0; j < GQ; ++j) acc[j] = 0.f;
    if (r < pr.r_T) {
      const __nv_bfloat16* row = Gh + int64_t(r) * pr.r_d;
      if (pr.r_d == kD && (reinterpret_cast<uintptr_t>(row) & 15) == 0) {
        uint4 w[kD / 8];
#pragma unroll
        for (int k = 0; k < kD / 8; ++k) w[k] = __ldg(reinterpret_cast<const uint4*>(row) + k);
#pragma unroll
        for (int k = 0; k < kD / 8; ++k) {
          const uint32_t ww[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 g2 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&ww[u]));
            const int c = 8 * k + 2 * u;
#pragma unroll
            for (int j = 0; j < GQ; ++j) acc[j] = fmaf(g2.x, qh[c][j], fmaf(g2.y, qh[c + 1][j], acc[j]));
          }
        }
      } else {
        for (int c = 0; c < pr.r_d; ++c) {
          const float g1 = __bfloat162float(row[c]);
#pragma unroll
          for (int j = 0; j < GQ; ++j) acc[j] = fmaf(g1, qh[c][j], acc[j]);
        }
      }
    }
#pragma unroll
    for (int j = 0; j < GQ; ++j) {
      const __nv_bfloat16 hh = __float2bfloat16_rn(acc[j]);
      hi[int64_t(h * GQ + j) * q_cap + r] = hh;
      lo[int64_t(h * GQ + j) * q_cap + r] = __float2bfloat16_rn(acc[j] - __bfloat162float(hh));
    }
  }
}

// One value cell's stored factors and the output rows of a (sequence, layer) row of a launch set.
struct MRow {
  const __nv_bfloat16* G;   // G^V of the row's layer: [n_kv][r_T][r_d]
  const __nv_bfloat16* Ud;  // U_d^V [128][r_d]
  int r_T, r_d, bits;
};
struct MTab {
  MRow row[kMaxFusedRows];
};

// Merge of the split partials and the output projection for the g_q query heads of one KV head:
//   M = max_s m_s, c_s = exp(m_s - M), L = sum_s c_s l_s, w = sum_s c_s W_s, a = sum_s c_s acc_s,
//   out = (R^T a + U_d^V (G^V_h^T w)) / L, lse = M + log L.
// grid (n_kv, B*Lc), 512 threads; dynamic shared memory: c [g_q][S], w [g_q][r_T],
// v partials [4][g_q][128], v [g_q][128], a [g_q][128]. G^V_h is read once for all g_q heads.
template <int GQ>
__global__ void __launch_bounds__(512) k_merge_fused(const float* __restrict__ part, int S, int q_cap,
                                                    const __grid_constant__ MTab tab,
                                                    uint64_t rot_seed, __nv_bfloat16* __restrict__ out,
                                                    float* __restrict__ lse) {
  extern __shared__ float msm[];
  const int h = blockIdx.x, bl = blockIdx.y;
  const MRow mr = tab.row[bl];
  const int rT = mr.r_T, rd = mr.r_d;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const size_t prow = size_t(2 + q_cap + kD);
  float* cf = msm;                          // [GQ][S]
  float* w = cf + GQ * S;                   // [GQ][rT]
  float* vp = w + GQ * max(rT, 1);          // [4][GQ][128]
  float* v = vp + 4 * GQ * kD;              // [GQ][128]
  float* x = v + GQ * kD;                   // [GQ][128]
  __shared__ float sM[GQ], sL[GQ];
  auto prow_of = [&](int g, int sp) { return part + ((size_t(bl) * kNQ + h * GQ + g) * S + sp) * prow; };
  if (warp < GQ) {
    const int g = warp;
    float M = -INFINITY;
    for (int sp = lane; sp < S; sp += 32) M = fmaxf(M, prow_of(g, sp)[0]);
    M = warp_max(M);
    float L = 0.f;
    for (int sp = lane; sp < S; sp += 32) {
      const float* pr = prow_of(g, sp);
      const float c = pr[0] == -INFINITY ? 0.f : __expf(pr[0] - M);
      cf[g * S + sp] = c;
      L += c * pr[1];
    }
    L = warp_sum(L);
    if (lane == 0) {
      sM[g] = M;
      sL[g] = L;
    }
  }
  __syncthreads();
  for (int e = tid; e < GQ * rT; e += blockDim.x) {
    const int g = e / rT, r = e % rT;
    float a = 0.f;
    for (int sp = 0; sp < S; ++sp) a = fmaf(cf[g * S + sp], prow_of(g, sp)[2 + r], a);
    w[e] = a;
  }
  for (int e = tid; e < GQ * kD; e += blockDim.x) {
    const int g = e / kD, d = e % kD;
    float a = 0.f;
    if (mr.bits)
      for (int sp = 0; sp < S; ++sp) a = fmaf(cf[g * S + sp], prow_of(g, sp)[2 + q_cap + d], a);
    x[e] = a;
  }
  __syncthreads();
  {
    const int j = tid & (kD - 1), qt = tid >> 7;
    float sacc[GQ];
#pragma unroll
    for (int g = 0; g < GQ; ++g) sacc[g] = 0.f;
    if (j < rd && rT > 0) {
      const __nv_bfloat16* G = mr.G + int64_t(h) * rT * rd + j;
#pragma unroll 8
      for (int r = qt; r < rT; r += 4) {
        const float gv = __bfloat162float(G[int64_t(r) * rd]);
#pragma unroll
        for (int g = 0; g < GQ; ++g) sacc[g] = fmaf(gv, w[g * rT + r], sacc[g]);
      }
    }
#pragma unroll
    for (int g = 0; g < GQ; ++g) vp[(qt * GQ + g) * kD + j] = sacc[g];
  }
  __syncthreads();
  for (int e = tid; e < GQ * kD; e += blockDim.x) {
    const int j = e % kD;
    v[e] = j < rd ? (vp[e] + vp[GQ * kD + e]) + (vp[2 * GQ * kD + e] + vp[3 * GQ * kD + e]) : 0.f;
  }
  if (mr.bits && warp < GQ) {
    float xv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) xv[i] = x[warp * kD + lane * 4 + i];
    warp_unrotate<4>(xv, rot_seed, rsqrtf(float(kD)));
#pragma unroll
    for (int i = 0; i < 4; ++i) x[warp * kD + lane * 4 + i] = xv[i];
  }
  __syncthreads();
  // each warp's eight U_d rows are loaded before any is used
  float udr[kD / 16][4];
#pragma unroll
  for (int u = 0; u < kD / 16; ++u)
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = warp + 16 * u, j = lane * 4 + k;
      udr[u][k] = (rT > 0 && j < rd) ? __bfloat162float(mr.Ud[int64_t(i) * rd + j]) : 0.f;
    }
  const int64_t qr0 = int64_t(bl) * kNQ + h * GQ;
#pragma unroll
  for (int u = 0; u < kD / 16; ++u) {
    const int i = warp + 16 * u;
#pragma unroll
    for (int g = 0; g < GQ; ++g) {
      const float* vg = v + g * kD + lane * 4;
      float o = (udr[u][0] * vg[0] + udr[u][1] * vg[1]) + (udr[u][2] * vg[2] + udr[u][3] * vg[3]);
      o = warp_sum(o);
      if (lane == 0) out[(qr0 + g) * kD + i] = __float2bfloat16_rn((x[g * kD + i] + o) / sL[g]);
    }
  }
  if (tid < GQ && lse) lse[qr0 + tid] = sM[tid] + logf(sL[tid]);
}

size_t merge_fused_smem(int gq, int S, int r_T) {
  return (size_t(gq) * S + size_t(gq) * std::max(r_T, 1) + size_t(6) * gq * kD) * sizeof(float);
}

constexpr int kSMs = 148;

// Token tiles per split: the fewest whole-wave rounds of one CTA per SM times tiles per CTA, plus
// the partials each extra split writes and the merge reads (about 0.75 of a tile's bytes per layer).
int fused_tps(int units, int nt) {
  int best = nt;
  double best_c = 1e300;
  for (int tps = 1; tps <= nt; ++tps) {
    const int S = (nt + tps - 1) / tps;
    if (tps > 1 && (nt + tps - 2) / (tps - 1) == S) continue;  // the same split count with fewer tiles
    const double waves = double((int64_t(units) * S + kSMs - 1) / kSMs);
    const double c = waves * tps + 0.75 * double(units) * S / kSMs;
    if (c < best_c - 1e-9) {
      best_c = c;
      best = tps;
    }
  }
  return best;
}

struct FusedWs {
  size_t hl, part, total;
  int tps, S;
};

FusedWs fused_layout(const jolt_shape& s, int Lc) {
  FusedWs w{};
  const size_t BL = size_t(s.batch) * Lc, qc = std::max(s.q_cap, 16);
  const int nt = (s.T + kBM - 1) / kBM;
  w.tps = fused_tps(int(std::min<size_t>(BL, kMaxFusedRows)), nt);
  w.S = (nt + w.tps - 1) / w.tps;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  w.hl = take(BL * 2 * kNQ * qc * 2);
  w.part = take(BL * kNQ * size_t(w.S) * (2 + qc + kD) * 4);
  w.total = off;
  return w;
}

}  // namespace

bool decode_fused_supported(const jolt_shape& s) {
  return decode_tc_supported(s) && !s.keys_pre_rope && s.n_q == kNQ && (s.n_kv == 4 || s.n_kv == 8);
}

size_t decode_fused_ws_bytes(const jolt_shape& s, int Lc) { return fused_layout(s, Lc).total; }

int decode_fused_max_cells() { return kMaxFusedCells; }

jolt_status launch_decode_fused(const DecodeParams& p, const TcCellView* views, uint8_t* ws, const jolt_shape& s,
                                cudaStream_t st) {
  // the workspace is laid out for the whole call; this launch set's rows start at its first sequence
  const FusedWs wl = fused_layout(s, p.Lc);
  const int BL = p.B * p.Lc, qc = p.q_cap;
  const int ncell = 2 * p.B * p.Gc;
  if (ncell > kMaxFusedCells || BL > kMaxFusedRows) return JOLT_ERR_INVALID_ARG;
  __nv_bfloat16* hl = reinterpret_cast<__nv_bfloat16*>(ws + wl.hl);
  float* part = reinterpret_cast<float*>(ws + wl.part);
  jolt_status r;
  // ---- prologue: R q, sum(R q), P = G^K (U_d^K^T q); P as bf16 hi + lo rows ----
  {
    StatScope sc(JOLT_K_DECODE_AUX, st, 0.0, 0.0);
    DecodeParams pq = p;
    pq.skip_p = 1;
    if ((r = launch_decode_prologue_q(pq, st))) return r;
    static_assert(sizeof(PTab) <= 24 * 1024, "prologue parameter table");
    PTab tab;
    for (int b = 0; b < p.B; ++b)
      for (int li = 0; li < p.Lc; ++li) {
        const int layer = p.layer_begin + li, g = layer / p.Lg, ll = layer % p.Lg;
        const TcCellView& v = views[(b * p.Gc + (g - p.g_first)) * 2];
        PRow& r = tab.row[b * p.Lc + li];
        r.G = v.r_T ? v.G + int64_t(ll) * p.n_kv * v.r_T * v.r_d : nullptr;
        r.Ud = v.Ud;
        r.r_T = v.r_T;
        r.r_d = v.r_d;
      }
    const __nv_bfloat16* qb = static_cast<const __nv_bfloat16*>(p.q);
    if (p.gq == 4) k_prologue_p<4><<<dim3(p.n_kv, BL), 256, 0, st>>>(qb, qc, tab, hl);
    else k_prologue_p<8><<<dim3(p.n_kv, BL), 256, 0, st>>>(qb, qc, tab, hl);
    JOLT_CUDA_TRY(cudaGetLastError());
  }
  // ---- tensor maps and per-cell arguments ----
  FusedMaps maps;
  std::memset(&maps, 0, sizeof(maps));
  FusedArgs fa{};
  {
    Operand o;
    o.ptr = hl; o.major = kMajorK; o.inner = qc; o.outer = 2 * kNQ; o.outer_stride = qc;
    o.batch = BL; o.batch_stride = int64_t(2) * kNQ * qc;
    if (!make_tensor_map(&maps.p, o, 2 * kNQ)) return JOLT_ERR_INVALID_ARG;
  }
  for (int c = 0; c < ncell; ++c) {
    const TcCellView& v = views[c];
    const bool is_k = (c & 1) == 0;
    fa.cells[c].codes = v.bits ? v.codes : nullptr;
    fa.cells[c].sz = v.bits ? v.sz : nullptr;
    fa.cells[c].r_T = v.r_T;
    fa.cells[c].b = v.bits;
    if (v.r_T > 0) {
      Operand o;
      o.ptr = v.Ut; o.major = is_k ? kMajorK : kMajorMN; o.inner = v.r_T; o.outer = p.T; o.outer_stride = v.r_T;
      if (!make_tensor_map(&maps.ut[c], o, is_k ? kBM : 64)) return JOLT_ERR_INVALID_ARG;
    }
  }
  fa.T = p.T; fa.nt = (p.T + kBM - 1) / kBM; fa.tps = wl.tps; fa.S = wl.S;
  fa.Lc = p.Lc; fa.Lg = p.Lg; fa.layer_begin = p.layer_begin; fa.g_first = p.g_first; fa.Gc = p.Gc;
  fa.n_kv = p.n_kv; fa.gq = p.gq; fa.q_cap = qc; fa.attn_scale = p.attn_scale;
  fa.qrot = p.ws_qrot; fa.qsum = p.ws_qsum; fa.part = part; fa.err = p.err;
  // algorithmic work of the launch: the compressed bytes the call must read (p.alg_bytes) and each
  // contraction once: 2 T r_T per query head for the key and value factors, 2 T d_h per query head
  // for each residual
  double flops = 0.0;
  for (int b = 0; b < p.B; ++b)
    for (int li = 0; li < p.Lc; ++li) {
      const int g = (p.layer_begin + li) / p.Lg;
      const TcCellView& k = views[(b * p.Gc + (g - p.g_first)) * 2];
      const TcCellView& v = views[(b * p.Gc + (g - p.g_first)) * 2 + 1];
      flops += 2.0 * p.T * kNQ * (double(k.r_T) + v.r_T) + 2.0 * p.T * kNQ * kD * ((k.bits ? 1 : 0) + (v.bits ? 1 : 0));
    }
  {
    StatScope sc(JOLT_K_DECODE_MAIN, st, flops, p.alg_bytes);
    const int grid = BL * wl.S;
    // the warpgroups re-split the block's registers (setmaxnreg): decreases must not exceed and
    // increases must not fall below the launch count, and the new shares must fit what the block
    // was launched with, or an increasing warpgroup would wait for registers that never come
    cudaFuncAttributes fat;
    JOLT_CUDA_TRY(cudaFuncGetAttributes(&fat, p.gq == 4 ? k_decode_fused<4> : k_decode_fused<8>));
    // (the key-residual warpgroups keep the launch count: they do not re-split)
    if (fat.numRegs != kRegKres || fat.numRegs < kRegCtl || fat.numRegs > kRegSoft || fat.numRegs < kRegVres ||
        128 * (kRegCtl + 2 * kRegKres + kRegSoft + kRegVres) > kThreads * fat.numRegs)
      return JOLT_ERR_CUDA;
    if (p.gq == 4) {
      JOLT_CUDA_TRY(cudaFuncSetAttribute(k_decode_fused<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem));
      k_decode_fused<4><<<grid, kThreads, kSmem, st>>>(maps, fa);
    } else {
      JOLT_CUDA_TRY(cudaFuncSetAttribute(k_decode_fused<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmem));
      k_decode_fused<8><<<grid, kThreads, kSmem, st>>>(maps, fa);
    }
    JOLT_CUDA_TRY(cudaGetLastError());
  }
  // ---- merge of the splits and the output projection ----
  StatScope sc2(JOLT_K_DECODE_AUX, st, 0.0, 0.0);
  static_assert(sizeof(MTab) <= 24 * 1024, "merge parameter table");
  MTab mt;
  int rmax = 1;
  for (int b = 0; b < p.B; ++b)
    for (int li = 0; li < p.Lc; ++li) {
      const int layer = p.layer_begin + li, g = layer / p.Lg, ll = layer % p.Lg;
      const TcCellView& v = views[(b * p.Gc + (g - p.g_first)) * 2 + 1];
      MRow& r = mt.row[b * p.Lc + li];
      r.G = v.r_T ? v.G + int64_t(ll) * p.n_kv * v.r_T * v.r_d : nullptr;
      r.Ud = v.Ud;
      r.r_T = v.r_T;
      r.r_d = v.r_d;
      r.bits = v.bits;
      rmax = std::max(rmax, v.r_T);
    }
  const size_t msm = merge_fused_smem(p.gq, wl.S, rmax);
  __nv_bfloat16* ob = static_cast<__nv_bfloat16*>(p.out);
  if (p.gq == 4) {
    if (msm > 48 * 1024)
      JOLT_CUDA_TRY(cudaFuncSetAttribute(k_merge_fused<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(msm)));
    k_merge_fused<4><<<dim3(p.n_kv, BL), 512, msm, st>>>(part, wl.S, qc, mt, p.rot_seed, ob, p.lse);
  } else {
    if (msm > 48 * 1024)
      JOLT_CUDA_TRY(cudaFuncSetAttribute(k_merge_fused<8>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(msm)));
    k_merge_fused<8><<<dim3(p.n_kv, BL), 512, msm, st>>>(part, wl.S, qc, mt, p.rot_seed, ob, p.lse);
  }
  JOLT_CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

}  // namespace jolt
