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
  static constexpr int kQsBytes = 2 * kMaxG * kD * 4;      // queries of each epilogue group's pair, fp32
  static constexpr int kRopeBytes = kD / 4 * kBM * 16;     // (cos, cos, sin, sin) of frequency pairs
  static constexpr int kSmem = 1024 + kStages * kStageBytes + kQsBytes + kRopeBytes + kD * 4 + 256;
  static constexpr int kThreads = 320;                     // producer, MMA, two groups of four epilogue warps
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

// Named barrier of one epilogue group (ids 1 and 2; 0 is __syncthreads).
__device__ __forceinline__ void group_bar(int g) { asm volatile("bar.sync %0, 128;" ::"r"(1 + g) : "memory"); }

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
// pairs of consecutive features.
template <int BITS>
__device__ __forceinline__ void dequant2(const uint32_t (&w)[4 * BITS + 1], float sc, float zr, float2 (&v)[kD / 2]) {
  constexpr uint32_t mask = (1u << BITS) - 1u;
  const float2 sc2 = make_float2(sc, sc), zr2 = make_float2(zr, zr);
#pragma unroll
  for (int m = 0; m < kD / 2; ++m) {
    const int j0 = 2 * m, j1 = 2 * m + 1;
    const float c0 = float((w[(j0 * BITS) >> 5] >> ((j0 * BITS) & 31)) & mask);
    const float c1 = float((w[(j1 * BITS) >> 5] >> ((j1 * BITS) & 31)) & mask);
    v[m] = __ffma2_rn(make_float2(c0, c1), sc2, zr2);
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

// grid.x = token tiles; 320 threads (three warps share some SM sub-partitions, whose register files
// hold 16384 registers each, so at most 168 registers a thread): warp 0 TMA producer, warp 1 MMA
// issuer (+ TMEM owner),
// warps 2..5 and 6..9 two epilogue groups taking alternate (layer, head) pairs and TMEM buffers
// (warp w reads TMEM lanes 32 * (w % 4) .. +31, i.e. token rows of the tile).
template <int BITS, int NT>
__global__ void __launch_bounds__(320, 1) k_keys_tc(const __grid_constant__ KeysMaps maps, const KeysArgs p) {
  using C = KeysCfg<NT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  float* qs = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes);  // [2 groups][kMaxG][kD]
  float4* rope = reinterpret_cast<float4*>(qs + 2 * kMaxG * kD);            // [32][kBM]
  float2* sgn = reinterpret_cast<float2*>(rope + kD / 4 * kBM);               // [64]
  uint64_t* bars = reinterpret_cast<uint64_t*>(sgn + kD / 2);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::kStages + 5);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int t0 = blockIdx.x * kBM;
  const int npairs = p.nl * p.n_kv;
  const bool fac = p.nkb > 0;

  const uint32_t bar0 = sm100::smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
  auto tfull_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + b); };
  auto tempty_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + 2 + b); };
  const uint32_t drain_bar = bar0 + 8u * (2 * C::kStages + 4);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      sm100::mbar_init(full_bar(s), 1);
      sm100::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      sm100::mbar_init(tfull_bar(b), 1);
      sm100::mbar_init(tempty_bar(b), 128);
    }
    sm100::mbar_init(drain_bar, 1);
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
  if (warp == 1) sm100::tmem_alloc(sm100::smem_u32(tmem_slot), 256);
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t sbase = sm100::smem_u32(smem);

  if (warp == 0) {
    if (lane == 0 && fac) {
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
    }
  } else if (warp == 1) {
    if (lane == 0 && fac) {
      // ---- MMA issuer: D[pr % 2] = sum_k U_T[t][k] (B_hi + B_lo)[k][:] ----
      constexpr uint32_t idesc = sm100::idesc_bf16_f32(kBM, kD, 0, 1);
      int it = 0;
      bool ok = true;
      for (int pr = 0; pr < npairs && ok; ++pr) {
        const int bi = pr & 1;
        if (!sm100::mbar_wait(tempty_bar(bi), ((pr >> 1) & 1) ^ 1, p.err)) break;
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
              sm100::mma_bf16(dt, ad, bd, idesc, (kb > 0 || kk > 0 || t > 0) ? 1u : 0u);
            }
          }
          sm100::mma_commit(empty_bar(s));
        }
        if (ok) sm100::mma_commit(tfull_bar(bi));
      }
      // every MMA this thread issued has completed before TMEM is released
      sm100::mma_commit(drain_bar);
      sm100::mbar_wait(drain_bar, 0, p.err);
    }
  } else {
    // ---- epilogue: group g takes pairs g, g + 2, ... (TMEM buffer g); thread = token row ----
    const int g = (warp - 2) >> 2;
    const int quarter = warp & 3;
    const int row = quarter * 32 + lane;
    const int et = threadIdx.x - 64 - 128 * g;
    const int t = t0 + row;
    const bool valid = t < p.T;
    float* qb = qs + g * kMaxG * kD;
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
    for (int pr = g; pr < npairs; pr += 2) {
      const int li = pr / p.n_kv, h = pr % p.n_kv;
      // this pair's residual row first: its loads overlap the query staging below
      uint32_t cw[4 * BITS + 1];
      float scv = 0.f, zrv = 0.f;
      if (BITS > 0 && valid) {
        const int64_t rr = (int64_t(li) * p.n_kv + h) * p.T + t;
        const __half2 szv = p.sz[rr];
        load_codes_raw<BITS>(p.codes + rr * (kD * BITS / 8), cw);
        scv = __low2float(szv);
        zrv = __high2float(szv);
      }
#pragma unroll
      for (int j = 0; j < kMaxG * kD / 1024; ++j) {
        const int e0 = (et + 128 * j) * 8;
        if (e0 < p.gq * kD) {
          const uint32_t wq[4] = {qn[j].x, qn[j].y, qn[j].z, qn[j].w};
          float f[8];
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const float2 ff = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&wq[u]));
            f[2 * u] = ff.x;
            f[2 * u + 1] = ff.y;
          }
          *reinterpret_cast<float4*>(qb + e0) = make_float4(f[0], f[1], f[2], f[3]);
          *reinterpret_cast<float4*>(qb + e0 + 4) = make_float4(f[4], f[5], f[6], f[7]);
        }
      }
      if (pr + 2 < npairs) q_issue(pr + 2);
      group_bar(g);
      float2 v[kD / 2];
      if (BITS > 0 && valid) {
        dequant2<BITS>(cw, scv, zrv, v);
        fwht128x2(v);
#pragma unroll
        for (int m = 0; m < kD / 2; ++m) v[m] = __fmul2_rn(v[m], sgn[m]);
      } else {
#pragma unroll
        for (int m = 0; m < kD / 2; ++m) v[m] = make_float2(0.f, 0.f);
      }
      if (fac) {
        // warp-uniform: the TMEM loads below are warp-collective
        if (live) live = __all_sync(0xffffffffu, sm100::mbar_wait(tfull_bar(g), (pr >> 1) & 1, p.err));
        sm100::tc_fence_after();
#pragma unroll
        for (int c = 0; c < kD / 16; ++c) {
          uint32_t r[16];
          sm100::tmem_ld16(tmem + g * kD + c * 16 + (uint32_t(quarter * 32) << 16), r);
          sm100::tmem_ld_wait();
#pragma unroll
          for (int k = 0; k < 8; ++k)
            v[c * 8 + k] = __fadd2_rn(v[c * 8 + k], make_float2(__uint_as_float(r[2 * k]), __uint_as_float(r[2 * k + 1])));
        }
        sm100::tc_fence_before();
        sm100::mbar_arrive(tempty_bar(g));
      }
      if (valid && live) {
#pragma unroll
        for (int m = 0; m < kD / 4; ++m) {  // features (2m, 2m+1) with (2m+64, 2m+65)
          const float4 r4 = rope[m * kBM + row];
          const float2 cs = make_float2(r4.x, r4.y), sn = make_float2(r4.z, r4.w);
          const float2 x1 = v[m], x2 = v[m + kD / 4];
          const float2 a = __fmul2_rn(x2, sn), b = __fmul2_rn(x1, sn);
          v[m] = __ffma2_rn(x1, cs, make_float2(-a.x, -a.y));
          v[m + kD / 4] = __ffma2_rn(x2, cs, b);
        }
        float* out = p.scores + (int64_t(li) * p.n_q + int64_t(h) * p.gq) * p.T + t;
#pragma unroll 1
        for (int gg = 0; gg < p.gq; ++gg) {
          const float4* qg = reinterpret_cast<const float4*>(qb + gg * kD);
          float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
          for (int k = 0; k < kD / 4; ++k) {
            const float4 qq = qg[k];
            a0 = __ffma2_rn(v[2 * k], make_float2(qq.x, qq.y), a0);
            a1 = __ffma2_rn(v[2 * k + 1], make_float2(qq.z, qq.w), a1);
          }
          out[int64_t(gg) * p.T] = ((a0.x + a0.y) + (a1.x + a1.y)) * p.attn_scale;
        }
      }
      group_bar(g);  // every thread is done with this pair's queries
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 1) sm100::tmem_dealloc(tmem, 256);
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

// acc[h'][j] += sum_t P~[h'][t] deq(code_t[j]) (rotated domain). grid (token chunks, n_kv, nl),
// 128 threads: lane l owns features 4l .. 4l+3 (one 4-code word per token), warp w the tokens
// w, w+4, ... of every 128-token sub-tile, whose code rows (16-byte loads), scale/zero pairs and
// probabilities are staged in shared memory first; the four warps' partial sums are added in
// shared memory before one atomic add per (query head, feature).
template <int BITS>
__global__ void __launch_bounds__(128) k_values_res(const ValArgs a) {
  constexpr int RB = kD * BITS / 8;        // bytes of one code row
  constexpr uint32_t mask = (1u << BITS) - 1u;
  __shared__ __align__(16) uint8_t cs[128][RB];
  __shared__ __align__(16) __nv_bfloat16 pr[128][kMaxG];  // P~ as stored (bf16): 8 heads per 16-byte load
  __shared__ float2 szs[128];
  __shared__ __align__(16) float red[2][kMaxG][kD];
  const int h = blockIdx.y, li = blockIdx.z, lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t qrow0 = int64_t(li) * a.n_q + int64_t(h) * a.gq;
  const int64_t rbase = (int64_t(li) * a.n_kv + h) * a.T;
  float acc[kMaxG][4];
#pragma unroll
  for (int g = 0; g < kMaxG; ++g)
#pragma unroll
    for (int f = 0; f < 4; ++f) acc[g][f] = 0.f;
  const int t_beg = blockIdx.x * a.chunk, t_end = min(a.T, t_beg + a.chunk);
  for (int tb = t_beg; tb < t_end; tb += 128) {
    const int nt = min(128, t_end - tb);
    __syncthreads();
    if (threadIdx.x < nt) {
      const int64_t rr = rbase + tb + threadIdx.x;
      const uint4* src = reinterpret_cast<const uint4*>(a.codes + rr * RB);
#pragma unroll
      for (int q = 0; q < RB / 16; ++q) reinterpret_cast<uint4*>(cs[threadIdx.x])[q] = __ldg(src + q);
      const __half2 szv = a.sz[rr];
      szs[threadIdx.x] = make_float2(__low2float(szv), __high2float(szv));
#pragma unroll
      for (int g = 0; g < kMaxG; ++g)
        pr[threadIdx.x][g] = g < a.gq ? a.ptil[(qrow0 + g) * a.ldp + tb + threadIdx.x] : __float2bfloat16_rn(0.f);
    }
    __syncthreads();
    for (int tt = w; tt < nt; tt += 4) {
      uint32_t word;
      if (BITS == 2) word = cs[tt][lane];
      else if (BITS == 4) word = reinterpret_cast<const uint16_t*>(cs[tt])[lane];
      else word = reinterpret_cast<const uint32_t*>(cs[tt])[lane];
      const float2 z = szs[tt];
      float dv[4];
#pragma unroll
      for (int f = 0; f < 4; ++f) dv[f] = dequant((word >> (f * BITS)) & mask, z.x, z.y);
      const uint4* p8 = reinterpret_cast<const uint4*>(pr[tt]);
#pragma unroll
      for (int g8 = 0; g8 < kMaxG / 8; ++g8) {
        if (8 * g8 < a.gq) {
          const uint4 pw = p8[g8];
          const uint32_t pb[4] = {pw.x, pw.y, pw.z, pw.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 pv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&pb[e]));
#pragma unroll
            for (int f = 0; f < 4; ++f) {
              acc[8 * g8 + 2 * e][f] = fmaf(pv.x, dv[f], acc[8 * g8 + 2 * e][f]);
              acc[8 * g8 + 2 * e + 1][f] = fmaf(pv.y, dv[f], acc[8 * g8 + 2 * e + 1][f]);
            }
          }
        }
      }
    }
  }
  // warps 2, 3 -> shared; warps 0, 1 add; warp 1 -> shared; warp 0 adds and commits
  __syncthreads();
  if (w >= 2)
#pragma unroll
    for (int g = 0; g < kMaxG; ++g)
      if (g < a.gq) *reinterpret_cast<float4*>(&red[w - 2][g][4 * lane]) = make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
  __syncthreads();
  if (w < 2)
#pragma unroll
    for (int g = 0; g < kMaxG; ++g)
      if (g < a.gq) {
        const float4 o = *reinterpret_cast<const float4*>(&red[w][g][4 * lane]);
        acc[g][0] += o.x; acc[g][1] += o.y; acc[g][2] += o.z; acc[g][3] += o.w;
      }
  __syncthreads();
  if (w == 1)
#pragma unroll
    for (int g = 0; g < kMaxG; ++g)
      if (g < a.gq) *reinterpret_cast<float4*>(&red[0][g][4 * lane]) = make_float4(acc[g][0], acc[g][1], acc[g][2], acc[g][3]);
  __syncthreads();
  if (w == 0)
#pragma unroll
    for (int g = 0; g < kMaxG; ++g)
      if (g < a.gq) {
        const float4 o = *reinterpret_cast<const float4*>(&red[0][g][4 * lane]);
        float* dst = &a.acc[(qrow0 + g) * kD + 4 * lane];
        atomicAdd(dst + 0, acc[g][0] + o.x);
        atomicAdd(dst + 1, acc[g][1] + o.y);
        atomicAdd(dst + 2, acc[g][2] + o.z);
        atomicAdd(dst + 3, acc[g][3] + o.w);
      }
}

struct FinArgs {
  int n_kv, gq, n_q, r_T, r_d, bits, q_cap;
  uint64_t rot_seed;
  const __nv_bfloat16* G;    // value core of layer ll0: [nl][n_kv][r_T][r_d]
  const __nv_bfloat16* Ud;   // [128][r_d]
  const float* W;            // [nl][n_q][q_cap]
  const float* acc;          // [nl][n_q][128]
  const float* mrow;         // [nl][n_q]
  const float* lrow;
  __nv_bfloat16* out;        // [nl][n_q][128] rows of (b, li0)
  float* lse;                // [nl][n_q] or null
};

// out = (U_d^V (G_h^V^T w) + R^T acc) / l, lse = m + log l for one query head.
// grid (n_kv, nl, g_q), 128 threads; dynamic smem: w [r_T] floats.
__global__ void __launch_bounds__(128) k_finalize(const FinArgs a) {
  extern __shared__ float w[];
  __shared__ float v[kD];
  __shared__ float x[kD];
  const int h = blockIdx.x, li = blockIdx.y, g = blockIdx.z, tid = threadIdx.x;
  const int64_t qr = int64_t(li) * a.n_q + int64_t(h) * a.gq + g;
  for (int r = tid; r < a.r_T; r += blockDim.x) w[r] = a.W[qr * a.q_cap + r];
  x[tid] = a.bits ? a.acc[qr * kD + tid] : 0.f;
  __syncthreads();
  // v[j] = sum_r G[r][j] w[r]
  if (tid < a.r_d) {
    const __nv_bfloat16* G = a.G + (int64_t(li) * a.n_kv + h) * a.r_T * a.r_d + tid;
    float s0 = 0.f, s1 = 0.f, s2 = 0.f, s3 = 0.f;
    int r = 0;
    for (; r + 4 <= a.r_T; r += 4) {
      s0 = fmaf(__bfloat162float(G[int64_t(r) * a.r_d]), w[r], s0);
      s1 = fmaf(__bfloat162float(G[int64_t(r + 1) * a.r_d]), w[r + 1], s1);
      s2 = fmaf(__bfloat162float(G[int64_t(r + 2) * a.r_d]), w[r + 2], s2);
      s3 = fmaf(__bfloat162float(G[int64_t(r + 3) * a.r_d]), w[r + 3], s3);
    }
    for (; r < a.r_T; ++r) s0 = fmaf(__bfloat162float(G[int64_t(r) * a.r_d]), w[r], s0);
    v[tid] = (s0 + s1) + (s2 + s3);
  }
  // inverse rotation of the residual accumulator (one warp)
  if (a.bits && tid < 32) {
    float xv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) xv[i] = x[tid * 4 + i];
    warp_unrotate<4>(xv, a.rot_seed, rsqrtf(float(kD)));
#pragma unroll
    for (int i = 0; i < 4; ++i) x[tid * 4 + i] = xv[i];
  }
  __syncthreads();
  float o = x[tid];
  if (a.r_T > 0) {
    const __nv_bfloat16* ud = a.Ud + int64_t(tid) * a.r_d;
    for (int jj = 0; jj < a.r_d; ++jj) o = fmaf(__bfloat162float(ud[jj]), v[jj], o);
  }
  a.out[qr * kD + tid] = __float2bfloat16_rn(o / a.lrow[qr]);
  if (tid == 0 && a.lse) a.lse[qr] = a.mrow[qr] + logf(a.lrow[qr]);
}

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
  w.ml = take(2 * nl * nq * 4);
  w.W = take(nl * nq * qc * 4);
  w.acc = take(nl * nq * kD * 4);
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
  const int nlmax = std::min(p.Lc, p.Lg);
  float* lrow = mrow + size_t(nlmax) * nq;
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
  __nv_bfloat16* oall = static_cast<__nv_bfloat16*>(p.out);

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
        k_softmax_rows<<<rows, 512, 0, st>>>(scores, T, Tp, mrow, lrow, ptil);
        JOLT_CUDA_TRY(cudaGetLastError());
      }
      // ---- values ----
      JOLT_CUDA_TRY(cudaMemsetAsync(W, 0, size_t(rows) * qc * 4, st));
      if (cv.bits) JOLT_CUDA_TRY(cudaMemsetAsync(acc, 0, size_t(rows) * kD * 4, st));
      if (cv.r_T > 0) {
        GemmCall gc;
        gc.M = rows; gc.N = cv.r_T; gc.K = T;
        gc.A[0] = op(ptil, kMajorK, T, rows, Tp);
        gc.B[0] = op(cv.Ut, kMajorMN, cv.r_T, T, cv.r_T);
        gc.C = W; gc.ldc = qc; gc.err = p.err;
        gc.k_split = 0;  // split K to fill whole waves
        gc.accumulate = true;
        gc.plan = s.gemm_plan;
          if ((r = gemm_tc(gc, st))) return r;
      }
      StatScope sc(JOLT_K_DECODE_AUX, st, 0.0, 0.0);
      if (cv.bits) {
        ValArgs va{};
        va.T = T; va.n_kv = n_kv; va.gq = gq; va.n_q = nq; va.bits = cv.bits; va.ldp = Tp;
        va.chunk = 512;
        va.codes = cv.codes + res_off * (kD * cv.bits / 8);
        va.sz = cv.sz + res_off;
        va.ptil = ptil; va.acc = acc;
        const dim3 vg((T + va.chunk - 1) / va.chunk, n_kv, nl);
        if (cv.bits == 2) k_values_res<2><<<vg, 128, 0, st>>>(va);
        else if (cv.bits == 4) k_values_res<4><<<vg, 128, 0, st>>>(va);
        else k_values_res<8><<<vg, 128, 0, st>>>(va);
        JOLT_CUDA_TRY(cudaGetLastError());
      }
      // ---- finalize ----
      FinArgs fa{};
      fa.n_kv = n_kv; fa.gq = gq; fa.n_q = nq; fa.r_T = cv.r_T; fa.r_d = cv.r_d; fa.bits = cv.bits; fa.q_cap = qc;
      fa.rot_seed = p.rot_seed;
      fa.G = cv.r_T ? cv.G + int64_t(ll0) * n_kv * cv.r_T * cv.r_d : nullptr;
      fa.Ud = cv.Ud;
      fa.W = W; fa.acc = acc; fa.mrow = mrow; fa.lrow = lrow;
      fa.out = oall + row0 * kD;
      fa.lse = p.lse ? p.lse + row0 : nullptr;
      k_finalize<<<dim3(n_kv, nl, gq), 128, size_t(std::max(cv.r_T, 1)) * 4, st>>>(fa);
      JOLT_CUDA_TRY(cudaGetLastError());
    }
  }
  return JOLT_OK;
}

}  // namespace jolt
