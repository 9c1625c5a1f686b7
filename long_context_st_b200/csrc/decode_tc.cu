// Decode attention over the stored factors with tensor cores (bf16 caches, d_h = 128).
//
// The attention of one (sequence, layer group) runs as a short pipeline over the group's layers:
//   keys     : pre-RoPE keys — k_keys_tc rebuilds each 128-token tile's keys K = U_T^K B_h for every
//              (layer, KV head) of the group on tcgen05 (B_h = G^K_h U_d^K^T as fp32 split into
//              bf16 hi + lo terms, fp32 accumulation in TMEM); its epilogue (one thread per token)
//              adds the inverse-rotated dequantised residual, applies RoPE at the token's position
//              and writes q . k for the KV head's query heads.
//              Non-RoPE keys — S = P U_T^K^T on the tcgen05 GEMM (P = G^K U_d^K^T q, hi + lo), then
//              k_scores_res adds scale * (codes . R q) + zero * sum(R q) per (token, query head).
//   softmax  : per (layer, query head) row: m = max s, P~ = bf16(exp(s - m)), l = sum P~
//   values   : W = P~ U_T^V on the tcgen05 GEMM (split-K, atomic fp32) and, on CUDA cores,
//              acc = sum_t P~_t deq(codes^V_t) in the rotated domain
//   finalize : out = (U_d^V (G^V_h^T W) + R^T acc) / l,  lse = m + log l
// Rows of scores and probabilities go through the workspace (n_q * T * 6 bytes per layer, written
// once and read twice); everything else the attention reads is the compressed cache itself.
// Method: the JoLT pages' decode-time attention over the stored factors (scores from G q-hat and
// the U_T rows plus the rotated-query residual term; values from the softmax-weighted U_T, the
// core and U_d plus the inverse-rotated residual; RoPE re-applied per token for pre-RoPE keys).
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>

#include "common.cuh"
#include "decode.cuh"
#include "gemm_tc.cuh"
#include "mma_codes.cuh"
#include "pack.cuh"
#include "sm100.cuh"
#include "stats.h"

namespace jolt {

namespace {

constexpr int kD = 128;              // head dimension this path serves
constexpr int kBM = 128, kBK = 64;   // token tile, rank chunk
constexpr int kMaxG = 16;            // query heads per KV head
constexpr int kABytes = kBM * kBK * 2;
constexpr int kBBytes = kBK * kD * 2;

template <int NT>
struct KeysCfg {
  static constexpr int kStages = NT == 1 ? 4 : 3;
  static constexpr int kStageBytes = kABytes + NT * kBBytes;
  static constexpr int kQbBytes = 16 * kD * 2;             // a score group's queries: B of q . k (16 x 128 bf16)
  static constexpr int kRopeBytes = kD / 4 * kBM * 16;     // (cos, cos, sin, sin) of frequency pairs
  static constexpr int kSmem = 1024 + kStages * kStageBytes + 2 * kQbBytes + kRopeBytes + kD * 4 + 256;
  static constexpr int kThreads = 512;                     // four warpgroups: control, residual, 2 x score
  static constexpr int kNB = 3;                            // TMEM key buffers of 128 columns
  static constexpr int kScoreCol = kNB * 128;              // q . k accumulators: 16 columns per score group
  // registers a thread after the warpgroups' re-split (launch: 128 each, 65536 in all)
  static constexpr int kRegCtl = 40, kRegRes = 200, kRegScore = 120;
};
struct KeysMaps {
  CUtensorMap a;       // U_T^K [T][r_T], K-major, box 64 x 128
  CUtensorMap b[2];    // B_h hi / lo [pairs][r_T][128], MN-major, box 64 x 64
};

struct KeysArgs {
  int T, nkb, n_kv, gq, n_q, nl;
  int b_one;               // maps.b[0] loads both chunks of every term at once (5-D map)
  uint64_t rot_seed;
  float attn_scale;
  int pos0;
  float rope_scaling;
  const uint8_t* codes;    // residual codes of layer ll0, head 0: rows (li * n_kv + h) * T + t
  const __half2* sz;       // scale/zero pairs, same rows
  const __nv_bfloat16* q;  // queries of (b, li0): [nl][n_q][128]
  const float* inv_freq;   // [64]
  float* scores;           // [nl][n_q][T]
  int32_t* err;
};


// Residual row of one token: 128 codes of BITS bits (little-endian bit stream) as floats.
template <int BITS>
__device__ __forceinline__ void load_codes(const uint8_t* row, float (&v)[kD]) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
  uint32_t w[4 * BITS + 1];
  const uint4* r4 = reinterpret_cast<const uint4*>(row);
#pragma unroll
  for (int i = 0; i < BITS; ++i) {
    const uint4 x = __ldg(r4 + i);
    w[4 * i + 0] = x.x;
    w[4 * i + 1] = x.y;
    w[4 * i + 2] = x.z;
    w[4 * i + 3] = x.w;
  }
#pragma unroll
  for (int j = 0; j < kD; ++j) v[j] = float((w[(j * BITS) >> 5] >> ((j * BITS) & 31)) & mask);
}

// The same row's packed code words (issued early: the loads are consumed later by dequant2).
template <int BITS>
__device__ __forceinline__ void load_codes_raw(const uint8_t* row, uint32_t (&w)[4 * BITS + 1]) {
  const uint4* r4 = reinterpret_cast<const uint4*>(row);
#pragma unroll
  for (int i = 0; i < BITS; ++i) {
    const uint4 x = __ldg(r4 + i);
    w[4 * i + 0] = x.x;
    w[4 * i + 1] = x.y;
    w[4 * i + 2] = x.z;
    w[4 * i + 3] = x.w;
  }
  w[4 * BITS] = 0u;
}

// The row dequantised (code * scale + zero, one fp32 fused multiply-add per code), as 64 packed
// pairs of consecutive features. Each code becomes an exact float by placing it in the mantissa of
// 2^23 and subtracting 2^23 (no integer-to-float conversion).
template <int BITS>
__device__ __forceinline__ void dequant2(const uint32_t (&w)[4 * BITS + 1], float sc, float zr, float2 (&v)[kD / 2]) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
  const float2 sc2 = make_float2(sc, sc), zr2 = make_float2(zr, zr);
  const float2 m23 = make_float2(-8388608.f, -8388608.f);
#pragma unroll
  for (int m = 0; m < kD / 2; ++m) {
    const int j0 = 2 * m, j1 = 2 * m + 1;
    const uint32_t f0 = ((w[(j0 * BITS) >> 5] >> ((j0 * BITS) & 31)) & mask) | 0x4B000000u;
    const uint32_t f1 = ((w[(j1 * BITS) >> 5] >> ((j1 * BITS) & 31)) & mask) | 0x4B000000u;
    const float2 c = __fadd2_rn(make_float2(__uint_as_float(f0), __uint_as_float(f1)), m23);
    v[m] = __ffma2_rn(c, sc2, zr2);
  }
}

// Unnormalised Walsh-Hadamard transform of 128 values held as 64 packed pairs: the stride-1
// butterflies inside each pair, the wider strides pair-wise (a - b computed as b * -1 + a, exact
// in both forms), stages in increasing stride as in the scalar form.
__device__ __forceinline__ void fwht128x2(float2 (&v)[kD / 2]) {
#pragma unroll
  for (int m = 0; m < kD / 2; ++m) {
    const float a = v[m].x, c = v[m].y;
    v[m] = make_float2(a + c, a - c);
  }
  const float2 neg1 = make_float2(-1.f, -1.f);
#pragma unroll
  for (int sm = 1; sm < kD / 2; sm <<= 1) {
#pragma unroll
    for (int m = 0; m < kD / 2; ++m) {
      if ((m & sm) == 0) {
        const float2 a = v[m], c = v[m + sm];
        v[m] = __fadd2_rn(a, c);
        v[m + sm] = __ffma2_rn(c, neg1, a);
      }
    }
  }
}

// grid.x = token tiles; 512 threads in four warpgroups with re-split register budgets:
//   warpgroup 0: warp 0 TMA producer, warp 1 key-MMA issuer (+ TMEM owner), warp 2 score-MMA
//                issuer, warp 3 idle after setup;
//   warpgroup 1: residual warps — thread = token row of the tile (warp w: TMEM lanes 32 (w % 4) ..
//                +31); per (layer, KV head) pair they dequantise the residual row, undo the
//                rotation (FWHT and signs) and store it into the pair's TMEM key buffer, on which
//                the key MMAs then accumulate U_T B_h (so the key arrives complete in TMEM);
//   warpgroups 2, 3: two score groups taking alternate pairs: they read the key in 16-column
//                pieces, apply RoPE at the token's position and write the rotated key back in place
//                as bf16 hi and lo halves (columns 0-63 and 64-127 of the buffer); a tensor-core
//                product with the pair's queries (A = the rotated key in TMEM, B = the g_q query
//                rows in shared memory, N = 16) then forms q . k, which the group reads back.
// Three TMEM key buffers of 128 columns rotate over the pairs: residual -> key MMA -> RoPE ->
// score MMA -> free; each score group has its own 16 accumulator columns.
// The queries' features are ordered to match the rotated key's column layout: K index 32 c + r is
// feature 16 c + r for r < 16 and feature 64 + 16 c + (r - 16) otherwise (c = 0 .. 3).
template <int BITS, int NT>
__global__ void __launch_bounds__(512, 1) k_keys_tc(const __grid_constant__ KeysMaps maps, const KeysArgs p) {
  using C = KeysCfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  uint8_t* qb_all = smem + C::kStages * C::kStageBytes;                      // [2 groups][16][128] bf16, SW128
  float4* rope = reinterpret_cast<float4*>(qb_all + 2 * C::kQbBytes);        // [32][kBM]
  float2* sgn = reinterpret_cast<float2*>(rope + kD / 4 * kBM);               // [64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sgn + kD / 2);
  constexpr int kNumBars = 2 * C::kStages + 4 * C::kNB + 2 + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + kNumBars);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kBM;
  const int npairs = p.nl * p.n_kv;
  const bool fac = p.nkb > 0;

  const uint32_t bar0 = sm100::smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
  auto rfull_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + b); };               // residual stored
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + C::kNB + b); };      // key MMAs done
  auto afull_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + 2 * C::kNB + b); };  // rotated key stored
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + 3 * C::kNB + b); }; // score MMAs done
  auto sfull_bar = [&](int g) { return bar0 + 8u * (2 * C::kStages + 4 * C::kNB + g); };  // q . k ready
  const uint32_t drain_bar = bar0 + 8u * (2 * C::kStages + 4 * C::kNB + 2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      sm100::mbar_init(full_bar(s), 1);
      sm100::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < C::kNB; ++b) {
      sm100::mbar_init(rfull_bar(b), 4);  // one arrival per residual warp
      sm100::mbar_init(tfull_bar(b), 1);
      sm100::mbar_init(afull_bar(b), 4);  // one arrival per warp of the score group
      sm100::mbar_init(tempty_bar(b), 1);
    }
    for (int g = 0; g < 2; ++g) sm100::mbar_init(sfull_bar(g), 1);
    sm100::mbar_init(drain_bar, 2);  // one commit per MMA-issuing thread
    sm100::fence_mbar_init();
    if (fac) {
      sm100::prefetch_tmap(&maps.a);
      for (int t = 0; t < NT; ++t) sm100::prefetch_tmap(&maps.b[t]);
    }
  }
  if (threadIdx.x < kD / 2) {
    const float isd = rsqrtf(float(kD));
    sgn[threadIdx.x] = make_float2(isd * rot_sign(p.rot_seed, 2 * threadIdx.x), isd * rot_sign(p.rot_seed, 2 * threadIdx.x + 1));
  }
  // RoPE of the tile's tokens: cos / sin of (pos0 + t) * inv_freq[f], angle reduced mod 2 pi in
  // fp64, times the attention scaling; frequencies 2m and 2m + 1 side by side
  for (int e = threadIdx.x; e < kD / 4 * kBM; e += blockDim.x) {
    const int m = e / kBM, tt = e % kBM;
    float cs[2], sn[2];
#pragma unroll
    for (int u = 0; u < 2; ++u) {
      const double ang = double(p.pos0 + t0 + tt) * double(p.inv_freq[2 * m + u]);
      const double red = ang - 6.283185307179586 * rint(ang * 0.15915494309189535);
      sincosf(float(red), &sn[u], &cs[u]);
    }
    rope[e] = make_float4(cs[0] * p.rope_scaling, cs[1] * p.rope_scaling, sn[0] * p.rope_scaling, sn[1] * p.rope_scaling);
  }
  // the query tiles start as zeros: rows g_q .. 15 stay zero
  for (int e = threadIdx.x; e < 2 * C::kQbBytes / 16; e += blockDim.x)
    reinterpret_cast<uint4*>(qb_all)[e] = make_uint4(0u, 0u, 0u, 0u);
  if (warp == 1) sm100::tmem_alloc(sm100::smem_u32(tmem_slot), 512);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = sm100::smem_u32(smem);
  const int wg = warp >> 2;

  if (wg == 0) {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegCtl));
    if (warp == 0 && lane == 0 && fac) {
      // ---- TMA producer: per (layer, head) pair, the U_T tile chunk and the B_h chunk(s) ----
      int it = 0;
      bool ok = true;
      for (int pr = 0; pr < npairs && ok; ++pr) {
        for (int kb = 0; kb < p.nkb; ++kb) {
          const int s = it % C::kStages;
          const uint32_t ph = (it / C::kStages) & 1;
          if (!sm100::mbar_wait(empty_bar(s), ph ^ 1, p.err)) {
            ok = false;
            break;
          }
          const uint32_t sa = sbase + s * C::kStageBytes;
          sm100::mbar_expect_tx(full_bar(s), C::kStageBytes);
          sm100::tma_load_3d(sa, &maps.a, full_bar(s), kb * kBK, t0, 0);
          if (p.b_one) {
            sm100::tma_load_5d(sa + kABytes, &maps.b[0], full_bar(s), 0, kb * kBK, 0, pr, 0);
          } else {
#pragma unroll
            for (int t = 0; t < NT; ++t)
#pragma unroll
              for (int c = 0; c < 2; ++c)
                sm100::tma_load_3d(sa + kABytes + t * kBBytes + c * 8192, &maps.b[t], full_bar(s), c * 64, kb * kBK, pr);
          }
          ++it;
        }
      }
      // wait (bounded) for the copies still in flight before the block may exit
      for (int i = max(0, it - C::kStages); i < it; ++i)
        sm100::mbar_wait(full_bar(i % C::kStages), (i / C::kStages) & 1, p.err);
    } else if (warp == 1 && lane == 0) {
      // ---- key MMAs: D[pr % kNB] (= residual, or nothing for b = 0) += sum_k U_T (B_hi + B_lo) ----
      constexpr uint32_t idesc = sm100::idesc_bf16_f32(kBM, kD, 0, 1);
      int it = 0;
      bool ok = true;
      for (int pr = 0; pr < npairs && ok && fac; ++pr) {
        const int bi = pr % C::kNB;
        if (!sm100::mbar_wait(rfull_bar(bi), (pr / C::kNB) & 1, p.err)) break;
        sm100::tc_fence_after();
        const uint32_t dt = tmem + bi * kD;
        for (int kb = 0; kb < p.nkb; ++kb, ++it) {
          const int s = it % C::kStages;
          if (!sm100::mbar_wait(full_bar(s), (it / C::kStages) & 1, p.err)) {
            ok = false;
            break;
          }
          sm100::tc_fence_after();
          const uint32_t sa = sbase + s * C::kStageBytes;
#pragma unroll
          for (int kk = 0; kk < kBK / 16; ++kk) {
            const uint64_t ad = sm100::smem_desc_sw128(sa + kk * 32, 16, 1024);
#pragma unroll
            for (int t = 0; t < NT; ++t) {
              const uint64_t bd = sm100::smem_desc_sw128(sa + kABytes + t * kBBytes + kk * 2048, 8192, 1024);
              sm100::mma_bf16(dt, ad, bd, idesc, (BITS > 0 || kb > 0 || kk > 0 || t > 0) ? 1u : 0u);
            }
          }
          sm100::mma_commit(empty_bar(s));
        }
        if (ok) sm100::mma_commit(tfull_bar(bi));
      }
      // every MMA this thread issued has completed before TMEM is released
      sm100::mma_commit(drain_bar);
      sm100::mbar_wait(drain_bar, 0, p.err);
    } else if (warp == 2 && lane == 0) {
      // ---- score MMAs: q . k[g] = (rotated key hi + lo, in TMEM) x (queries of the pair) ----
      constexpr uint32_t idesc = sm100::idesc_bf16_f32(kBM, 16, 0, 0);
      for (int pr = 0; pr < npairs; ++pr) {
        const int bi = pr % C::kNB, g = pr & 1;
        if (!sm100::mbar_wait(afull_bar(bi), (pr / C::kNB) & 1, p.err)) break;
        sm100::tc_fence_after();
        const uint32_t qb = sbase + uint32_t(qb_all - smem) + g * C::kQbBytes;
        const uint32_t dt = tmem + C::kScoreCol + 16 * g;
#pragma unroll
        for (int term = 0; term < 2; ++term)
#pragma unroll
          for (int kk = 0; kk < kD / 16; ++kk) {
            const uint64_t bd = sm100::smem_desc_sw128(qb + (kk >> 2) * (16 * 128) + (kk & 3) * 32, 16, 1024);
            sm100::mma_bf16_tmem_a(dt, tmem + bi * kD + term * (kD / 2) + kk * 8, bd, idesc, (term > 0 || kk > 0) ? 1u : 0u);
          }
        sm100::mma_commit(sfull_bar(g));
        sm100::mma_commit(tempty_bar(bi));
      }
      sm100::mma_commit(drain_bar);
      sm100::mbar_wait(drain_bar, 0, p.err);
    }
  } else if (wg == 1) {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(C::kRegRes));
    // ---- residual warps: the inverse-rotated residual row of each pair into its TMEM buffer ----
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int t = t0 + row;
    const bool valid = t < p.T;
    bool live = true;
    uint32_t cw[4 * BITS + 1];
    float scv = 0.f, zrv = 0.f;
    auto load_res = [&](int prr) {
      const int li = prr / p.n_kv, h = prr % p.n_kv;
      const int64_t rr = (int64_t(li) * p.n_kv + h) * p.T + t;
      const __half2 szv = p.sz[rr];
      load_codes_raw<BITS>(p.codes + rr * (kD * BITS / 8), cw);
      scv = __low2float(szv);
      zrv = __high2float(szv);
    };
    if (BITS > 0 && valid) load_res(0);
    // without a factor part (r_T = 0) the buffer starts as the residual alone, or as zeros
    const bool store = BITS > 0 || !fac;
    for (int pr = 0; pr < npairs; ++pr) {
      const int bi = pr % C::kNB;
      float2 v[kD / 2];
      if (store) {
        if (BITS > 0 && valid) {
          dequant2<BITS>(cw, scv, zrv, v);
          if (pr + 1 < npairs) load_res(pr + 1);  // the next pair's row is in flight meanwhile
          fwht128x2(v);
#pragma unroll
          for (int m = 0; m < kD / 2; ++m) v[m] = __fmul2_rn(v[m], sgn[m]);
        } else {
#pragma unroll
          for (int m = 0; m < kD / 2; ++m) v[m] = make_float2(0.f, 0.f);
        }
      }
      // the buffer is free once the score MMAs of the pair kNB earlier have completed
      if (live) live = __all_sync(0xffffffffu, sm100::mbar_wait(tempty_bar(bi), ((pr / C::kNB) & 1) ^ 1, p.err));
      sm100::tc_fence_after();
      if (store) {
        const uint32_t ta = tmem + bi * kD + (uint32_t(quarter * 32) << 16);
#pragma unroll
        for (int c = 0; c < kD / 32; ++c) {
          uint32_t r[32];
#pragma unroll
          for (int k = 0; k < 16; ++k) {
            r[2 * k] = __float_as_uint(v[16 * c + k].x);
            r[2 * k + 1] = __float_as_uint(v[16 * c + k].y);
          }
          sm100::tmem_st32(ta + 32 * c, r);
        }
        sm100::tmem_st_wait();
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(rfull_bar(bi));
    }
  } else {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(C::kRegScore));
    // ---- score groups: group g takes pairs g, g + 2, ...; thread = token row ----
    const int g = wg - 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int et = threadIdx.x - 256 - 128 * g;
    const int t = t0 + row;
    const bool valid = t < p.T;
    uint8_t* qb = qb_all + g * C::kQbBytes;
    bool live = true;
    // a pair's g_q query rows (g_q * 128 bf16): thread et holds 8 consecutive values of each 1024,
    // loaded one pair ahead of their use
    const int nq8 = p.gq * kD / 8;
    uint4 qn[kMaxG * kD / 1024];
    auto q_issue = [&](int prq) {
      const uint4* src = reinterpret_cast<const uint4*>(
          p.q + (int64_t(prq / p.n_kv) * p.n_q + int64_t(prq % p.n_kv) * p.gq) * kD);
#pragma unroll
      for (int j = 0; j < kMaxG * kD / 1024; ++j)
        qn[j] = et + 128 * j < nq8 ? __ldg(src + et + 128 * j) : make_uint4(0u, 0u, 0u, 0u);
    };
    if (g < npairs) q_issue(g);
    int use = 0;  // pairs this group has taken
    for (int pr = g; pr < npairs; pr += 2, ++use) {
      const int li = pr / p.n_kv, h = pr % p.n_kv;
      const int bi = pr % C::kNB;
      // the pair's queries as B (16 x 128 bf16, K-major, 128-byte swizzle) in the key's column order;
      // the previous pair's score MMAs, which read this tile, completed before its scores were read
#pragma unroll
      for (int j = 0; j < kMaxG * kD / 1024; ++j) {
        const int e0 = (et + 128 * j) * 8;  // query row e0 / 128, features d0 .. d0 + 7
        if (e0 < p.gq * kD) {
          const int n = e0 / kD, d0 = e0 % kD;
          const int k0 = d0 < kD / 2 ? 32 * (d0 / 16) + d0 % 16 : 32 * ((d0 - kD / 2) / 16) + 16 + (d0 - kD / 2) % 16;
          const int chunk = k0 / 64, within = k0 % 64;  // 8 bf16 = one 16-byte unit of the row
          *reinterpret_cast<uint4*>(qb + chunk * (16 * 128) + n * 128 + (((within / 8) ^ (n & 7)) << 4)) = qn[j];
        }
      }
      sm100::fence_proxy_async_smem();
      if (pr + 2 < npairs) q_issue(pr + 2);
      const uint32_t ready = fac ? tfull_bar(bi) : rfull_bar(bi);
      if (live) live = __all_sync(0xffffffffu, sm100::mbar_wait(ready, (pr / C::kNB) & 1, p.err));
      sm100::tc_fence_after();
      const uint32_t ta = tmem + bi * kD + (uint32_t(quarter * 32) << 16);
#pragma unroll
      for (int c = 0; c < kD / 32; ++c) {
        uint32_t r1[16], r2[16];
        sm100::tmem_ld16(ta + 16 * c, r1);           // features 16c .. 16c + 15
        sm100::tmem_ld16(ta + kD / 2 + 16 * c, r2);  // their RoPE partners, + 64
        sm100::tmem_ld_wait();
        uint32_t hi[16], lo[16];  // hi: columns 16c .. 16c + 15, lo: the same + 64
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int m = 8 * c + k;  // features (2m, 2m+1) with (2m+64, 2m+65)
          const float4 r4 = rope[m * kBM + row];
          const float2 cs = make_float2(r4.x, r4.y), sn = make_float2(r4.z, r4.w);
          const float2 x1 = make_float2(__uint_as_float(r1[2 * k]), __uint_as_float(r1[2 * k + 1]));
          const float2 x2 = make_float2(__uint_as_float(r2[2 * k]), __uint_as_float(r2[2 * k + 1]));
          const float2 a = __fmul2_rn(x2, sn), bb = __fmul2_rn(x1, sn);
          const float2 y1 = __ffma2_rn(x1, cs, make_float2(-a.x, -a.y));
          const float2 y2 = __ffma2_rn(x2, cs, bb);
          const __nv_bfloat162 h1 = __floats2bfloat162_rn(y1.x, y1.y), h2 = __floats2bfloat162_rn(y2.x, y2.y);
          const float2 f1 = __bfloat1622float2(h1), f2 = __bfloat1622float2(h2);
          const __nv_bfloat162 l1 = __floats2bfloat162_rn(y1.x - f1.x, y1.y - f1.y);
          const __nv_bfloat162 l2 = __floats2bfloat162_rn(y2.x - f2.x, y2.y - f2.y);
          hi[k] = *reinterpret_cast<const uint32_t*>(&h1);
          hi[8 + k] = *reinterpret_cast<const uint32_t*>(&h2);
          lo[k] = *reinterpret_cast<const uint32_t*>(&l1);
          lo[8 + k] = *reinterpret_cast<const uint32_t*>(&l2);
        }
        sm100::tmem_st16(ta + 16 * c, hi);
        sm100::tmem_st16(ta + kD / 2 + 16 * c, lo);
      }
      sm100::tmem_st_wait();
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) sm100::mbar_arrive(afull_bar(bi));
      if (live) live = __all_sync(0xffffffffu, sm100::mbar_wait(sfull_bar(g), use & 1, p.err));
      sm100::tc_fence_after();
      uint32_t sc[16];
      sm100::tmem_ld16(tmem + C::kScoreCol + 16 * g + (uint32_t(quarter * 32) << 16), sc);
      sm100::tmem_ld_wait();
      sm100::tc_fence_before();
      if (valid && live) {
        float* out = p.scores + (int64_t(li) * p.n_q + int64_t(h) * p.gq) * p.T + t;
#pragma unroll
        for (int gg = 0; gg < kMaxG; ++gg)
          if (gg < p.gq) out[int64_t(gg) * p.T] = __uint_as_float(sc[gg]) * p.attn_scale;
      }
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) sm100::tmem_dealloc(tmem, 512);
}

// ---- CUDA-core stages -------------------------------------------------------------------------

// fp32 -> bf16 hi + lo parts (hi = rn(x), lo = rn(x - hi)).
__global__ void k_split_hilo(const float* __restrict__ x, int64_t n, __nv_bfloat16* __restrict__ hi,
                             __nv_bfloat16* __restrict__ lo) {
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x) {
    const float v = x[e];
    const __nv_bfloat16 hh = __float2bfloat16_rn(v);
    hi[e] = hh;
    lo[e] = __float2bfloat16_rn(v - __bfloat162float(hh));
  }
}

struct ResArgs {
  int T, n_kv, gq, n_q, has_fac;
  float attn_scale;
  const uint8_t* codes;   // rows (li * n_kv + h) * T + t
  const __half2* sz;
  const float* qrot;      // [nl][n_q][128]
  const float* qsum;      // [nl][n_q]
  float* scores;          // [nl][n_q][T]
};

// Non-RoPE keys: s = (s_fac + scale * (codes . q_rot) + zero * qsum) * attn_scale.
// grid (token tiles, n_kv, nl), thread = token.
template <int BITS>
__global__ void __launch_bounds__(128) k_scores_res(const ResArgs a) {
  __shared__ float qr[kMaxG][kD];
  __shared__ float qsm[kMaxG];
  const int h = blockIdx.y, li = blockIdx.z;
  const int64_t qrow0 = int64_t(li) * a.n_q + int64_t(h) * a.gq;
  for (int e = threadIdx.x; e < a.gq * kD; e += blockDim.x) qr[e / kD][e % kD] = a.qrot[qrow0 * kD + e];
  if (threadIdx.x < a.gq) qsm[threadIdx.x] = a.qsum[qrow0 + threadIdx.x];
  __syncthreads();
  const int t = blockIdx.x * 128 + threadIdx.x;
  if (t >= a.T) return;
  float c[kD];
  float sc = 0.f, zr = 0.f;
  if (BITS > 0) {
    const int64_t rr = (int64_t(li) * a.n_kv + h) * a.T + t;
    load_codes<BITS>(a.codes + rr * (kD * BITS / 8), c);
    const __half2 szv = a.sz[rr];
    sc = __low2float(szv);
    zr = __high2float(szv);
  }
  float* s = a.scores + qrow0 * a.T + t;
#pragma unroll 1
  for (int g = 0; g < a.gq; ++g) {
    float res = 0.f;
    if (BITS > 0) {
      float a0 = 0.f, a1 = 0.f, a2 = 0.f, a3 = 0.f;
#pragma unroll
      for (int j = 0; j < kD; j += 4) {
        a0 = fmaf(c[j], qr[g][j], a0);
        a1 = fmaf(c[j + 1], qr[g][j + 1], a1);
        a2 = fmaf(c[j + 2], qr[g][j + 2], a2);
        a3 = fmaf(c[j + 3], qr[g][j + 3], a3);
      }
      res = sc * ((a0 + a1) + (a2 + a3)) + zr * qsm[g];
    }
    const float f = a.has_fac ? s[int64_t(g) * a.T] : 0.f;
    s[int64_t(g) * a.T] = (f + res) * a.attn_scale;
  }
}

// Per row: m = max s, P~ = bf16(exp(s - m)) (row stride ldp), l = sum of the rounded P~. Rows of a
// multiple of 4 scores are read as float4 and written as four bf16 at a time.
__global__ void __launch_bounds__(512) k_softmax_rows(const float* __restrict__ scores, int T, int64_t ldp,
                                                      float* __restrict__ mrow, float* __restrict__ lrow,
                                                      __nv_bfloat16* __restrict__ ptil) {
  const int64_t r = blockIdx.x;
  const float* s = scores + r * T;
  __nv_bfloat16* pr = ptil + r * ldp;
  __shared__ float red[32];
  const int nw = blockDim.x >> 5, wid = threadIdx.x >> 5, ln = threadIdx.x & 31;
  const bool vec = (T % 4) == 0 && (ldp % 4) == 0;
  float m = -INFINITY;
  if (vec) {
    const float4* s4 = reinterpret_cast<const float4*>(s);
    for (int t = threadIdx.x; t < T / 4; t += blockDim.x) {
      const float4 x = s4[t];
      m = fmaxf(m, fmaxf(fmaxf(x.x, x.y), fmaxf(x.z, x.w)));
    }
  } else {
    for (int t = threadIdx.x; t < T; t += blockDim.x) m = fmaxf(m, s[t]);
  }
  m = warp_max(m);
  if (ln == 0) red[wid] = m;
  __syncthreads();
  if (wid == 0) {
    float x = ln < nw ? red[ln] : -INFINITY;
    x = warp_max(x);
    if (ln == 0) red[0] = x;
  }
  __syncthreads();
  m = red[0];
  __syncthreads();
  float l = 0.f;
  if (vec) {
    const float4* s4 = reinterpret_cast<const float4*>(s);
    uint2* p4 = reinterpret_cast<uint2*>(pr);
    for (int t = threadIdx.x; t < T / 4; t += blockDim.x) {
      const float4 x = s4[t];
      const __nv_bfloat162 e01 = __floats2bfloat162_rn(__expf(x.x - m), __expf(x.y - m));
      const __nv_bfloat162 e23 = __floats2bfloat162_rn(__expf(x.z - m), __expf(x.w - m));
      p4[t] = make_uint2(*reinterpret_cast<const uint32_t*>(&e01), *reinterpret_cast<const uint32_t*>(&e23));
      const float2 f01 = __bfloat1622float2(e01), f23 = __bfloat1622float2(e23);
      l += (f01.x + f01.y) + (f23.x + f23.y);
    }
  } else {
    for (int t = threadIdx.x; t < T; t += blockDim.x) {
      const __nv_bfloat16 e = __float2bfloat16_rn(__expf(s[t] - m));
      pr[t] = e;
      l += __bfloat162float(e);
    }
  }
  l = warp_sum(l);
  if (ln == 0) red[wid] = l;
  __syncthreads();
  if (threadIdx.x == 0) {
    float x = 0.f;
    for (int i = 0; i < nw; ++i) x += red[i];
    mrow[r] = m;
    lrow[r] = x;
  }
}

struct ValArgs {
  int T, n_kv, gq, n_q, bits, chunk;
  int64_t ldp;
  const uint8_t* codes;       // value residual rows (li * n_kv + h) * T + t
  const __half2* sz;
  const __nv_bfloat16* ptil;  // [nl][n_q][ldp]
  float* acc;                 // [nl][n_q][128], rotated domain
};

// acc[j][d] += sum_t P~[j][t] (scale_t code_t[d] + zero_t) for the query heads j of one KV head, in
// the rotated domain, on mma.sync: per 16-token step D[d][j] += sum_t code[t][d] (P~[j][t] scale_t)
// (M = 16 features per m-tile, eight m-tiles; N = 8 query heads per n-tile; K = 16 tokens), the codes
// widened to exact f16 in registers and the weights P~ scale rounded to f16; sum_t P~ zero_t is
// accumulated per query head on the side. grid (token chunks, n_kv, nl), 256 threads: warp w takes
// the steps w, w + 8, ... of the chunk; lane (g, m) loads features 16 g .. 16 g + 15 of its four
// tokens 2m, 2m+1, 2m+8, 2m+9 (one 4 / 8 / 16-byte load per code row for b = 2 / 4 / 8) and the
// weights of query head 8 n + g; the warps' partials meet in shared memory, one atomic add per
// (query head, feature) and CTA goes to the workspace accumulator.
template <int BITS>
__device__ __forceinline__ int vres_feature(int mt, int hi, int g) {
  return BITS == 2 ? 16 * g + 4 * (mt >> 1) + 2 * (mt & 1) + hi : BITS == 4 ? 16 * g + 2 * mt + hi : 16 * g + mt + 8 * hi;
}

template <int BITS, int NT>
__global__ void __launch_bounds__(256) k_values_res_mma(const ValArgs a) {
  constexpr int RB = kD * BITS / 8;  // bytes of one code row
  constexpr int LW = BITS / 2;       // 32-bit words of a lane's 16 features
  __shared__ float red[8 * NT][kD];
  __shared__ float zsh[8 * NT];
  const int h = blockIdx.y, li = blockIdx.z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, gr = lane >> 2, m4 = lane & 3;
  const int64_t qrow0 = int64_t(li) * a.n_q + int64_t(h) * a.gq;
  const int64_t rbase = (int64_t(li) * a.n_kv + h) * a.T;
  for (int e = threadIdx.x; e < 8 * NT * kD; e += blockDim.x) (&red[0][0])[e] = 0.f;
  if (threadIdx.x < 8 * NT) zsh[threadIdx.x] = 0.f;
  __syncthreads();
  float acc[8][NT][4];
#pragma unroll
  for (int mt = 0; mt < 8; ++mt)
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
  float zacc[NT];
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) zacc[nt] = 0.f;
  const int t_beg = blockIdx.x * a.chunk, t_end = min(a.T, t_beg + a.chunk);
  // raw operands of one 16-token step (code words, scale/zero pairs, P~ pairs), loaded ahead of
  // their use
  struct Raw {
    uint32_t w[4][LW];
    uint32_t sz[4];
    uint32_t pp[NT][2];
  };
  auto load = [&](int tb, Raw& r) {
    const int tA = tb + 2 * m4;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int t = tA + (k & 1) + 8 * (k >> 1);
      const bool ok = t < t_end;
      const uint8_t* row = a.codes + (rbase + t) * RB + 4 * LW * gr;
      if (LW == 1) {
        r.w[k][0] = ok ? __ldg(reinterpret_cast<const uint32_t*>(row)) : 0u;
      } else if (LW == 2) {
        const uint2 u = ok ? __ldg(reinterpret_cast<const uint2*>(row)) : make_uint2(0u, 0u);
        r.w[k][0] = u.x; r.w[k][LW > 1 ? 1 : 0] = u.y;
      } else {
        const uint4 u = ok ? __ldg(reinterpret_cast<const uint4*>(row)) : make_uint4(0u, 0u, 0u, 0u);
        r.w[k][0] = u.x; r.w[k][LW > 1 ? 1 : 0] = u.y; r.w[k][LW > 2 ? 2 : 0] = u.z; r.w[k][LW > 3 ? 3 : 0] = u.w;
      }
      r.sz[k] = ok ? __ldg(reinterpret_cast<const uint32_t*>(a.sz + rbase + t)) : 0u;
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const int j = 8 * nt + gr;
      const __nv_bfloat16* pr = a.ptil + (qrow0 + j) * a.ldp;
#pragma unroll
      for (int k2 = 0; k2 < 2; ++k2) {
        const int t = tA + 8 * k2;  // even: the pair (t, t + 1) is one aligned 4-byte word
        uint32_t v = 0u;
        if (j < a.gq) {
          if (t + 1 < t_end) v = __ldg(reinterpret_cast<const uint32_t*>(pr + t));
          else if (t < t_end) v = uint32_t(__ldg(reinterpret_cast<const unsigned short*>(pr + t)));
        }
        r.pp[nt][k2] = v;
      }
    }
  };
  // steps in flight ahead of the one being computed: two for 2-bit codes (small rows), one for
  // wider codes (the extra register set would cost CTAs per SM)
  constexpr int kAhead = BITS == 2 ? 2 : 1;
  Raw n1, n2;
  int tb = t_beg + 16 * warp;
  if (tb < t_end) load(tb, n1);
  if (kAhead == 2 && tb + 16 * 8 < t_end) load(tb + 16 * 8, n2);
  for (; tb < t_end; tb += 16 * 8) {
    const Raw cur = n1;
    if (kAhead == 2) {
      n1 = n2;
      if (tb + 2 * 16 * 8 < t_end) load(tb + 2 * 16 * 8, n2);
    } else if (tb + 16 * 8 < t_end) {
      load(tb + 16 * 8, n1);
    }
    float sc[4], zr[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&cur.sz[k]));
      sc[k] = f.x;
      zr[k] = f.y;
    }
    // weights of query heads 8 nt + g: B fragments (tokens 2m, 2m+1 | 2m+8, 2m+9)
    uint32_t bw[NT][2];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
      const float2 p01 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cur.pp[nt][0]));
      const float2 p23 = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&cur.pp[nt][1]));
      zacc[nt] += (p01.x * zr[0] + p01.y * zr[1]) + (p23.x * zr[2] + p23.y * zr[3]);
      const __half2 b0 = __floats2half2_rn(p01.x * sc[0], p01.y * sc[1]);
      const __half2 b1 = __floats2half2_rn(p23.x * sc[2], p23.y * sc[3]);
      bw[nt][0] = *reinterpret_cast<const uint32_t*>(&b0);
      bw[nt][1] = *reinterpret_cast<const uint32_t*>(&b1);
    }
    const uint32_t(&w)[4][LW] = cur.w;
    // A fragments straight from the code words, eight m-tiles
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      uint32_t af[4];
      if (BITS == 2) {
        const int bb = mt >> 1, s0 = 2 * (mt & 1);
        const uint32_t xab = bytes_xy(w[0][0], w[1][0], bb), xcd = bytes_xy(w[2][0], w[3][0], bb);
        af[0] = crumb(xab, s0); af[1] = crumb(xab, s0 + 1);
        af[2] = crumb(xcd, s0); af[3] = crumb(xcd, s0 + 1);
      } else if (BITS == 4) {
        const int wi = (mt >> 2) & (LW - 1), bb = mt & 3;
        const uint32_t xab = bytes_xy(w[0][wi], w[1][wi], bb), xcd = bytes_xy(w[2][wi], w[3][wi], bb);
        af[0] = nib_lo(xab); af[1] = nib_hi(xab);
        af[2] = nib_lo(xcd); af[3] = nib_hi(xcd);
      } else {
        const int wl = (mt >> 2) & (LW - 1), wh = (2 + (mt >> 2)) & (LW - 1), bb = mt & 3;
        af[0] = byte_lo(bytes_xy(w[0][wl], w[1][wl], bb)); af[1] = byte_lo(bytes_xy(w[0][wh], w[1][wh], bb));
        af[2] = byte_lo(bytes_xy(w[2][wl], w[3][wl], bb)); af[3] = byte_lo(bytes_xy(w[2][wh], w[3][wh], bb));
      }
#pragma unroll
      for (int nt = 0; nt < NT; ++nt) mma_f16_16816(acc[mt][nt], af, bw[nt][0], bw[nt][1]);
    }
  }
  // the warps' partials in shared memory, then one global add per (query head, feature)
#pragma unroll
  for (int nt = 0; nt < NT; ++nt) {
#pragma unroll
    for (int mt = 0; mt < 8; ++mt) {
      const int f0 = vres_feature<BITS>(mt, 0, gr), f1 = vres_feature<BITS>(mt, 1, gr);
      const int j = 8 * nt + 2 * m4;
      atomicAdd(&red[j][f0], acc[mt][nt][0]);
      atomicAdd(&red[j + 1][f0], acc[mt][nt][1]);
      atomicAdd(&red[j][f1], acc[mt][nt][2]);
      atomicAdd(&red[j + 1][f1], acc[mt][nt][3]);
    }
    float z = zacc[nt];
    z += __shfl_xor_sync(0xffffffffu, z, 1);
    z += __shfl_xor_sync(0xffffffffu, z, 2);
    if (m4 == 0) atomicAdd(&zsh[8 * nt + gr], z);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < a.gq * kD; e += blockDim.x) {
    const int j = e / kD, d = e % kD;
    atomicAdd(&a.acc[(qrow0 + j) * kD + d], red[j][d] + zsh[j]);
  }
}

struct FinArgs {
  int n_kv, gq, n_q, q_cap, row_base;
  uint64_t rot_seed;
  const float* W;            // [rows][n_q][q_cap], rows = (b, layer) of the call
  const float* acc;          // [rows][n_q][128]
  const float* mrow;         // [rows][n_q]
  const float* lrow;
  __nv_bfloat16* out;        // [rows][n_q][128]
  float* lse;                // [rows][n_q] or null
};

// The value cell of one (sequence, layer) row: the layer's core, the group's U_d and the sizes.
struct FinRow {
  const __nv_bfloat16* G;    // [n_kv][r_T][r_d] of the row's layer
  const __nv_bfloat16* Ud;   // [128][r_d]
  int r_T, r_d, bits;
};
constexpr int kMaxFinRows = 512;
struct FinTab {
  FinRow row[kMaxFinRows];
};

// out = (U_d^V (G_h^V^T w) + R^T acc) / l, lse = m + log l for the g_q query heads of one KV head.
// One launch for the whole call after every group's values: grid (n_kv, rows of this launch),
// 512 threads; dynamic shared memory: w [g_q][r_T], v partials [4][g_q][128],
// v [g_q][128], x [g_q][128]. G_h^V is read once for all g_q heads: thread (j, quarter) takes rows
// r = quarter, quarter + 4, ... of column j; the U_d^V rows are read by one warp each (lanes over
// the r_d columns) and reduced per query head.
__global__ void __launch_bounds__(512) k_finalize(const FinArgs a, const __grid_constant__ FinTab tab) {
  extern __shared__ float fsm[];
  const FinRow fr = tab.row[blockIdx.y];
  const int gq = a.gq, rT = fr.r_T, rd = fr.r_d;
  float* w = fsm;                          // [gq][rT]
  float* vp = w + gq * max(rT, 1);         // [4][gq][128]
  float* v = vp + 4 * gq * kD;             // [gq][128]
  float* x = v + gq * kD;                  // [gq][128]
  const int h = blockIdx.x, tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t qr0 = int64_t(a.row_base + blockIdx.y) * a.n_q + int64_t(h) * gq;
  for (int e = tid; e < gq * rT; e += blockDim.x) w[e] = a.W[(qr0 + e / rT) * a.q_cap + e % rT];
  for (int e = tid; e < gq * kD; e += blockDim.x) x[e] = fr.bits ? a.acc[qr0 * kD + e] : 0.f;
  __syncthreads();
  {
    const int j = tid & (kD - 1), qt = tid >> 7;
    float s[kMaxG];
#pragma unroll
    for (int g = 0; g < kMaxG; ++g) s[g] = 0.f;
    if (j < rd && rT > 0) {
      const __nv_bfloat16* G = fr.G + int64_t(h) * rT * rd + j;
#pragma unroll 8
      for (int r = qt; r < rT; r += 4) {
        const float gv = __bfloat162float(G[int64_t(r) * rd]);
#pragma unroll
        for (int g = 0; g < kMaxG; ++g)
          if (g < gq) s[g] = fmaf(gv, w[g * rT + r], s[g]);
      }
    }
#pragma unroll
    for (int g = 0; g < kMaxG; ++g)
      if (g < gq) vp[(qt * gq + g) * kD + j] = s[g];
  }
  __syncthreads();
  for (int e = tid; e < gq * kD; e += blockDim.x) {
    const int j = e % kD;
    v[e] = j < rd ? (vp[e] + vp[gq * kD + e]) + (vp[2 * gq * kD + e] + vp[3 * gq * kD + e]) : 0.f;
  }
  // inverse rotation of each head's residual accumulator (one warp per head)
  if (fr.bits && warp < gq) {
    float xv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) xv[i] = x[warp * kD + lane * 4 + i];
    warp_unrotate<4>(xv, a.rot_seed, rsqrtf(float(kD)));
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
      udr[u][k] = (rT > 0 && j < rd) ? __bfloat162float(fr.Ud[int64_t(i) * rd + j]) : 0.f;
    }
#pragma unroll
  for (int u = 0; u < kD / 16; ++u) {
    const int i = warp + 16 * u;
    const float(&ud)[4] = udr[u];
    for (int g = 0; g < gq; ++g) {
      const float* vg = v + g * kD + lane * 4;
      float o = (ud[0] * vg[0] + ud[1] * vg[1]) + (ud[2] * vg[2] + ud[3] * vg[3]);
      o = warp_sum(o);
      if (lane == 0) {
        const int64_t qr = qr0 + g;
        a.out[qr * kD + i] = __float2bfloat16_rn((x[g * kD + i] + o) / a.lrow[qr]);
      }
    }
  }
  if (tid < gq && a.lse) a.lse[qr0 + tid] = a.mrow[qr0 + tid] + logf(a.lrow[qr0 + tid]);
}

size_t finalize_smem(int gq, int r_T) { return (size_t(gq) * std::max(r_T, 1) + size_t(6) * gq * kD) * sizeof(float); }

int grid1(int64_t n) { return int(std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 148 * 16))); }

Operand op(const void* ptr, int major, int64_t inner, int64_t outer, int64_t ld, int64_t batch = 1,
           int64_t bstride = 0) {
  Operand o;
  o.ptr = ptr;
  o.major = major;
  o.inner = inner;
  o.outer = outer;
  o.outer_stride = ld;
  o.batch = batch;
  o.batch_stride = bstride;
  return o;
}

// Workspace regions of the tensor-core path (per-group buffers are reused group after group).
struct TcWs {
  size_t hl, bh, scores, ptil, ml, W, acc, total;
};

TcWs tc_layout(const jolt_shape& s, int Lc) {
  const size_t B = s.batch, nq = s.n_q, T = s.T, qc = std::max(s.q_cap, 16);
  const size_t nl = std::min(Lc, s.layers_per_group);
  const size_t Tp = (T + 7) / 8 * 8;
  TcWs w{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  w.hl = take(s.keys_pre_rope ? 2 * nl * s.n_kv * qc * kD * 2 : 2 * B * Lc * nq * qc * 2);
  w.bh = take(s.keys_pre_rope ? nl * s.n_kv * qc * kD * 4 : 0);
  w.scores = take(nl * nq * T * 4);
  w.ptil = take(nl * nq * Tp * 2);
  w.ml = take(2 * B * Lc * nq * 4);
  w.W = take(B * Lc * nq * qc * 4);
  w.acc = take(B * Lc * nq * kD * 4);
  w.total = off;
  return w;
}

template <int BITS, int NT>
jolt_status launch_keys(const KeysMaps& maps, const KeysArgs& a, cudaStream_t st) {
  auto kern = k_keys_tc<BITS, NT>;
  cudaFuncAttributes fa;
  JOLT_CUDA_TRY(cudaFuncGetAttributes(&fa, kern));
  if (fa.maxThreadsPerBlock < KeysCfg<NT>::kThreads) {  // the block would not fit the register file
    if (kDebug)
      std::fprintf(stderr, "jolt: k_keys_tc needs %d threads, registers allow %d (%d per thread)\n",
                   KeysCfg<NT>::kThreads, fa.maxThreadsPerBlock, fa.numRegs);
    return JOLT_ERR_CUDA;
  }
  // the warpgroups re-split the block's registers (setmaxnreg): the decreases must not exceed and
  // the increase must not fall below the launch count, and the new shares must fit what the block
  // was launched with, or the increasing warpgroup would wait for registers that never come
  using C = KeysCfg<NT>;
  if (fa.numRegs < C::kRegCtl || fa.numRegs < C::kRegScore || fa.numRegs > C::kRegRes ||
      128 * (C::kRegCtl + C::kRegRes + 2 * C::kRegScore) > C::kThreads * fa.numRegs) {
    if (kDebug) std::fprintf(stderr, "jolt: k_keys_tc launched with %d registers a thread\n", fa.numRegs);
    return JOLT_ERR_CUDA;
  }
  JOLT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, KeysCfg<NT>::kSmem));
  const int ntiles = (a.T + kBM - 1) / kBM;
  kern<<<ntiles, KeysCfg<NT>::kThreads, KeysCfg<NT>::kSmem, st>>>(maps, a);
  const cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) {
    if (kDebug) std::fprintf(stderr, "jolt: k_keys_tc launch: %s\n", cudaGetErrorString(e));
    return JOLT_ERR_CUDA;
  }
  return JOLT_OK;
}

template <int NT>
jolt_status launch_keys_bits(int bits, const KeysMaps& maps, const KeysArgs& a, cudaStream_t st) {
  switch (bits) {
    case 0: return launch_keys<0, NT>(maps, a, st);
    case 2: return launch_keys<2, NT>(maps, a, st);
    case 4: return launch_keys<4, NT>(maps, a, st);
    default: return launch_keys<8, NT>(maps, a, st);
  }
}

jolt_status launch_scores_res(int bits, const ResArgs& a, int nl, cudaStream_t st) {
  const dim3 grid((a.T + 127) / 128, a.n_kv, nl);
  switch (bits) {
    case 0: k_scores_res<0><<<grid, 128, 0, st>>>(a); break;
    case 2: k_scores_res<2><<<grid, 128, 0, st>>>(a); break;
    case 4: k_scores_res<4><<<grid, 128, 0, st>>>(a); break;
    default: k_scores_res<8><<<grid, 128, 0, st>>>(a); break;
  }
  JOLT_CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

}  // namespace

bool decode_tc_supported(const jolt_shape& s) {
  return s.io_dtype == JOLT_BF16 && s.factor_dtype == JOLT_BF16 && s.d_h == kD && s.n_q % s.n_kv == 0 &&
         s.n_q / s.n_kv <= kMaxG;
}

size_t decode_tc_ws_bytes(const jolt_shape& s, int Lc) { return tc_layout(s, Lc).total; }

jolt_status launch_decode_tc(const DecodeParams& p, const TcCellView* views, uint8_t* tcws,
                             const jolt_shape& s, cudaStream_t st) {
  const TcWs wl = tc_layout(s, p.Lc);
  const int T = p.T, nq = p.n_q, qc = p.q_cap, n_kv = p.n_kv, gq = p.gq;
  const int64_t Tp = (int64_t(T) + 7) / 8 * 8;
  __nv_bfloat16* hl = reinterpret_cast<__nv_bfloat16*>(tcws + wl.hl);
  float* bh = reinterpret_cast<float*>(tcws + wl.bh);
  float* scores = reinterpret_cast<float*>(tcws + wl.scores);
  __nv_bfloat16* ptil = reinterpret_cast<__nv_bfloat16*>(tcws + wl.ptil);
  float* mrow = reinterpret_cast<float*>(tcws + wl.ml);
  float* W = reinterpret_cast<float*>(tcws + wl.W);
  float* acc = reinterpret_cast<float*>(tcws + wl.acc);
  const int nrows = p.B * p.Lc;  // (sequence, layer) rows of the call
  float* lrow = mrow + size_t(nrows) * nq;
  // the finalize table (passed by value at launch) holds rows fin_base .. fin_base + kMaxFinRows - 1
  FinTab ftab;
  int fin_base = 0, fin_rmax = 1;
  auto fin_flush = [&](int upto) -> jolt_status {
    if (upto <= fin_base) return JOLT_OK;
    FinArgs fa{};
    fa.n_kv = n_kv; fa.gq = gq; fa.n_q = nq; fa.q_cap = qc; fa.row_base = fin_base;
    fa.rot_seed = p.rot_seed;
    fa.W = reinterpret_cast<float*>(tcws + wl.W); fa.acc = reinterpret_cast<float*>(tcws + wl.acc);
    fa.mrow = mrow; fa.lrow = lrow;
    fa.out = static_cast<__nv_bfloat16*>(p.out);
    fa.lse = p.lse;
    const size_t fsm = finalize_smem(gq, fin_rmax);
    if (fsm > 48 * 1024) JOLT_CUDA_TRY(cudaFuncSetAttribute(k_finalize, cudaFuncAttributeMaxDynamicSharedMemorySize, int(fsm)));
    k_finalize<<<dim3(n_kv, upto - fin_base), 512, fsm, st>>>(fa, ftab);
    JOLT_CUDA_TRY(cudaGetLastError());
    fin_base = upto;
    fin_rmax = 1;
    return JOLT_OK;
  };
  jolt_status r;

  // ---- per-call prologue: R q, sum(R q), P (non-RoPE, as hi + lo) ----
  const size_t nP = size_t(p.B) * p.Lc * nq * qc;
  {
    StatScope sc(JOLT_K_DECODE_AUX, st, 0.0, 0.0);
    if ((r = launch_decode_prologue_q(p, st))) return r;  // records no scope of its own
    if (!p.pre_rope) {
      k_split_hilo<<<grid1(int64_t(nP)), 256, 0, st>>>(p.ws_P, int64_t(nP), hl, hl + nP);
      JOLT_CUDA_TRY(cudaGetLastError());
    }
  }
  const __nv_bfloat16* qall = static_cast<const __nv_bfloat16*>(p.q);

  for (int b = 0; b < p.B; ++b) {
    for (int gi = 0; gi < p.Gc; ++gi) {
      const int g = p.g_first + gi;
      const int l_lo = std::max(p.layer_begin, g * p.Lg), l_hi = std::min(p.layer_begin + p.Lc, (g + 1) * p.Lg);
      const int nl = l_hi - l_lo;
      if (nl <= 0) continue;
      const int li0 = l_lo - p.layer_begin, ll0 = l_lo - g * p.Lg;
      const TcCellView& ck = views[(b * p.Gc + gi) * 2 + 0];
      const TcCellView& cv = views[(b * p.Gc + gi) * 2 + 1];
      const int rows = nl * nq;
      const int64_t row0 = (int64_t(b) * p.Lc + li0) * nq;  // first (b, layer, head) row of the call
      const int64_t res_off = int64_t(ll0) * n_kv * T;       // first residual row of layer ll0

      // ---- scores ----
      if (p.pre_rope) {
        KeysMaps maps;
        std::memset(&maps, 0, sizeof(maps));
        KeysArgs ka{};
        ka.nkb = 0;
        if (ck.r_T > 0) {
          // B_h = G_h U_d^T for the group's (layer, head) pairs: exact bf16 products, fp32 sums
          GemmCall gc;
          gc.M = ck.r_T; gc.N = kD; gc.K = ck.r_d;
          gc.A[0] = op(ck.G + int64_t(ll0) * n_kv * ck.r_T * ck.r_d, kMajorK, ck.r_d, ck.r_T, ck.r_d, nl * n_kv,
                       int64_t(ck.r_T) * ck.r_d);
          gc.B[0] = op(ck.Ud, kMajorK, ck.r_d, kD, ck.r_d);
          gc.C = bh; gc.ldc = kD; gc.c_batch_stride = int64_t(qc) * kD; gc.batch = nl * n_kv; gc.err = p.err;
          gc.plan = s.gemm_plan;
          if ((r = gemm_tc(gc, st))) return r;
          const int64_t nb = int64_t(nl) * n_kv * qc * kD;
          {
            StatScope sc(JOLT_K_DECODE_AUX, st, 0.0, 0.0);
            k_split_hilo<<<grid1(nb), 256, 0, st>>>(bh, nb, hl, hl + nb);
            JOLT_CUDA_TRY(cudaGetLastError());
          }
          if (!make_tensor_map(&maps.a, op(ck.Ut, kMajorK, ck.r_T, T, ck.r_T), kBM)) return JOLT_ERR_INVALID_ARG;
          // both terms' two 64-wide chunks in one copy per k-block when the driver takes the
          // 5-D layout (hi and lo parts are nb elements apart); else four copies
          ka.b_one = make_tensor_map_mn_chunks(&maps.b[0], hl, ck.r_T, kD, 2, int64_t(nl) * n_kv, int64_t(qc) * kD, 2, nb)
                         ? 1 : 0;
          if (!ka.b_one &&
              (!make_tensor_map(&maps.b[0], op(hl, kMajorMN, kD, ck.r_T, kD, nl * n_kv, int64_t(qc) * kD), kD) ||
               !make_tensor_map(&maps.b[1], op(hl + nb, kMajorMN, kD, ck.r_T, kD, nl * n_kv, int64_t(qc) * kD), kD)))
            return JOLT_ERR_INVALID_ARG;
          ka.nkb = (ck.r_T + kBK - 1) / kBK;
        }
        ka.T = T; ka.n_kv = n_kv; ka.gq = gq; ka.n_q = nq; ka.nl = nl;
        ka.rot_seed = p.rot_seed; ka.attn_scale = p.attn_scale;
        ka.codes = ck.bits ? ck.codes + res_off * (kD * ck.bits / 8) : nullptr;
        ka.sz = ck.bits ? ck.sz + res_off : nullptr;
        ka.q = qall + row0 * kD;
        ka.pos0 = p.pos_offset; ka.rope_scaling = p.rope_scaling; ka.inv_freq = p.inv_freq;
        ka.scores = scores; ka.err = p.err;
        // algorithmic work of the launch: the U_T^K rows once, each pair's residual rows
        const double kbytes = 2.0 * T * ck.r_T + (ck.bits ? double(nl) * n_kv * T * (kD * ck.bits / 8 + 4) : 0.0);
        // the key rebuild once per (token, layer, KV head); issued: both bf16 terms of B_h
        StatScope sc(JOLT_K_DECODE_MAIN, st, 2.0 * T * ck.r_T * kD * nl * n_kv, kbytes, 2.0 * 2.0 * T * ck.r_T * kD * nl * n_kv);
        if ((r = launch_keys_bits<2>(ck.bits, maps, ka, st))) return r;
      } else {
        if (ck.r_T > 0) {
          GemmCall gc;
          gc.M = rows; gc.N = T; gc.K = ck.r_T; gc.n_terms = 2;
          gc.A[0] = op(hl + row0 * qc, kMajorK, ck.r_T, rows, qc);
          gc.A[1] = op(hl + nP + row0 * qc, kMajorK, ck.r_T, rows, qc);
          gc.B[0] = op(ck.Ut, kMajorK, ck.r_T, T, ck.r_T);
          gc.B[1] = gc.B[0];
          gc.C = scores; gc.ldc = T; gc.err = p.err;
          gc.plan = s.gemm_plan;
          if ((r = gemm_tc(gc, st))) return r;
        }
        ResArgs ra{};
        ra.T = T; ra.n_kv = n_kv; ra.gq = gq; ra.n_q = nq; ra.has_fac = ck.r_T > 0;
        ra.attn_scale = p.attn_scale;
        ra.codes = ck.bits ? ck.codes + res_off * (kD * ck.bits / 8) : nullptr;
        ra.sz = ck.bits ? ck.sz + res_off : nullptr;
        ra.qrot = p.ws_qrot + row0 * kD;
        ra.qsum = p.ws_qsum + row0;
        ra.scores = scores;
        const double rbytes = ck.bits ? double(nl) * n_kv * T * (kD * ck.bits / 8 + 4) : 0.0;
        StatScope sc(JOLT_K_DECODE_MAIN, st, 0.0, rbytes);
        if ((r = launch_scores_res(ck.bits, ra, nl, st))) return r;
      }

      // ---- softmax rows ----
      {
        StatScope sc(JOLT_K_DECODE_AUX, st, 0.0, 0.0);
        k_softmax_rows<<<rows, 512, 0, st>>>(scores, T, Tp, mrow + row0, lrow + row0, ptil);
        JOLT_CUDA_TRY(cudaGetLastError());
      }
      // ---- values ----
      float* Wg = W + row0 * qc;
      float* accg = acc + row0 * kD;
      JOLT_CUDA_TRY(cudaMemsetAsync(Wg, 0, size_t(rows) * qc * 4, st));
      if (cv.bits) JOLT_CUDA_TRY(cudaMemsetAsync(accg, 0, size_t(rows) * kD * 4, st));
      if (cv.r_T > 0) {
        GemmCall gc;
        gc.M = rows; gc.N = cv.r_T; gc.K = T;
        gc.A[0] = op(ptil, kMajorK, T, rows, Tp);
        gc.B[0] = op(cv.Ut, kMajorMN, cv.r_T, T, cv.r_T);
        gc.C = Wg; gc.ldc = qc; gc.err = p.err;
        gc.k_split = 0;  // split K to fill whole waves
        gc.accumulate = true;
        gc.plan = s.gemm_plan;
          if ((r = gemm_tc(gc, st))) return r;
      }
      StatScope sc(JOLT_K_DECODE_AUX, st, 0.0, 0.0);
      if (cv.bits) {
        ValArgs va{};
        va.T = T; va.n_kv = n_kv; va.gq = gq; va.n_q = nq; va.bits = cv.bits; va.ldp = Tp;
        // one wave: as many CTAs as fit on the device at once, spread over the group's (layer, KV
        // head) pairs (a second, partial wave would double the time of the last CTAs)
        const void* kv = gq <= 8 ? (cv.bits == 2 ? (const void*)k_values_res_mma<2, 1>
                                               : cv.bits == 4 ? (const void*)k_values_res_mma<4, 1>
                                                              : (const void*)k_values_res_mma<8, 1>)
                                 : (cv.bits == 2 ? (const void*)k_values_res_mma<2, 2>
                                               : cv.bits == 4 ? (const void*)k_values_res_mma<4, 2>
                                                              : (const void*)k_values_res_mma<8, 2>);
        int per_sm = 0, dev = 0, nsm = 0;
        JOLT_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kv, 256, 0));
        JOLT_CUDA_TRY(cudaGetDevice(&dev));
        JOLT_CUDA_TRY(cudaDeviceGetAttribute(&nsm, cudaDevAttrMultiProcessorCount, dev));
        const int nch = std::max(1, std::min(std::max(1, per_sm) * nsm / (n_kv * nl), (T + 1023) / 1024));
        va.chunk = ((T + nch - 1) / nch + 15) / 16 * 16;
        va.codes = cv.codes + res_off * (kD * cv.bits / 8);
        va.sz = cv.sz + res_off;
        va.ptil = ptil; va.acc = accg;
        const dim3 vg((T + va.chunk - 1) / va.chunk, n_kv, nl);
        if (gq <= 8) {
          if (cv.bits == 2) k_values_res_mma<2, 1><<<vg, 256, 0, st>>>(va);
          else if (cv.bits == 4) k_values_res_mma<4, 1><<<vg, 256, 0, st>>>(va);
          else k_values_res_mma<8, 1><<<vg, 256, 0, st>>>(va);
        } else {
          if (cv.bits == 2) k_values_res_mma<2, 2><<<vg, 256, 0, st>>>(va);
          else if (cv.bits == 4) k_values_res_mma<4, 2><<<vg, 256, 0, st>>>(va);
          else k_values_res_mma<8, 2><<<vg, 256, 0, st>>>(va);
        }
        JOLT_CUDA_TRY(cudaGetLastError());
      }
      // ---- the group's rows for the finalize launch (rows arrive in increasing order) ----
      for (int l = 0; l < nl; ++l) {
        const int row = b * p.Lc + li0 + l;
        if (row - fin_base >= kMaxFinRows && (r = fin_flush(row))) return r;
        FinRow& fr = ftab.row[row - fin_base];
        fr.G = cv.r_T ? cv.G + int64_t(ll0 + l) * n_kv * cv.r_T * cv.r_d : nullptr;
        fr.Ud = cv.Ud;
        fr.r_T = cv.r_T;
        fr.r_d = cv.r_d;
        fr.bits = cv.bits;
        fin_rmax = std::max(fin_rmax, cv.r_T);
      }
    }
  }
  {
    StatScope sc(JOLT_K_DECODE_AUX, st, 0.0, 0.0);
    if ((r = fin_flush(nrows))) return r;
  }
  return JOLT_OK;
}

}  // namespace jolt
