// tcgen05 GEMM for sm_100a: TMA (128-byte swizzle) streams bf16 A/B tiles into a ring of shared-
// memory stages; one thread issues tcgen05.mma into TMEM accumulators; epilogue warps drain TMEM
// with tcgen05.ld and store (or atomically add) fp32 C.
//
// Two kernels. k_gemm (the default): one output tile per CTA of 128 threads — lane 0 of warp 0
// streams A and lane 0 of warp 2 streams B by TMA, lane 0 of warp 1 issues the MMAs, warp 2 owns
// the TMEM allocation, all four warps run the epilogue (fp32 stores or atomics, the bf16 hi/lo
// split of the result, or the fused residual coder). k_gemm_p (selected with JOLT_GEMM_PLAN):
// persistent, as single CTAs or CTA pairs (cta_group::2, M = 256 per MMA, each SM stages half of
// B), with two TMEM accumulators so the epilogue of one tile overlaps the main loop of the next.
// Every mbarrier wait is bounded (2 s) and reports JOLT_ERR_TIMEOUT instead of hanging.
//
// Several (A_t, B_t) "terms" can accumulate into one tile: a fp32 operand split as hi + lo bf16
// parts gives x*y ~ hi*hi + hi*lo + lo*hi with ~2^-16 relative error at bf16 tensor-core speed.
#include <dlfcn.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "gemm_tc.cuh"
#include "sm100.cuh"
#include "stats.h"

namespace jolt {

namespace {

constexpr int BM = 128, BK = 64;

struct TmaPack {
  CUtensorMap a[kMaxTerms];
  CUtensorMap b[kMaxTerms];
};

struct GemmDev {
  int M, N, K, n_terms, nkb_split, k_split;
  int a_fold[kMaxTerms], b_fold[kMaxTerms];    // fold length (0 = plain)
  int a_chunk[kMaxTerms], b_chunk[kMaxTerms];  // MN-major operand loaded by one chunked copy
  int a_batch[kMaxTerms], b_batch[kMaxTerms];  // operand batch extents (coordinate = z % extent)
  float* C;
  int64_t ldc, c_bstride;
  int c_div, accumulate, c_upper, b_upper;
  int32_t* err;
  int ntile, mtiles, n_tiles;  // persistent kernels: tile grid (N tiles fastest, then M, then z)
  int c_vec;                   // output rows start 16-byte aligned (pointer, ldc, batch stride)
  __nv_bfloat16* Ch;           // bf16 hi (and lo) outputs instead of fp32 C
  __nv_bfloat16* Cl;
  ResidualEpi res;             // fused residual coding (k_gemm<..., EPI = 1>)
};

__device__ __forceinline__ uint32_t bf2_bits(__nv_bfloat162 h) { return *reinterpret_cast<uint32_t*>(&h); }

// bf16 hi / lo split of one fp32 value (lo = rounding of the exact remainder).
__device__ __forceinline__ void split_hl(float v, __nv_bfloat16& h, __nv_bfloat16& l) {
  h = __float2bfloat16_rn(v);
  l = __float2bfloat16_rn(v - __bfloat162float(h));
}

// Store one 32-row x 32-column slice of an accumulator: lane = row (row0 + lane), r[i] = column
// col0 + i. Plain stores of whole 32-column slices go straight from registers, 16 bytes at a
// time along each lane's row; atomic accumulation (and ragged or unaligned slices) is transposed
// through shared memory first, so that each instruction covers 32 consecutive columns of a row.
// zoff: element offset of this tile's batch entry in the output.
__device__ __forceinline__ void store_chunk(const GemmDev& p, int64_t zoff, const uint32_t (&r)[32],
                                            float* st, int row0, int col0, int lane) {
  if (p.Ch) {
    if (p.c_vec && col0 + 32 <= p.N) {
      const int row = row0 + lane;
      if (row < p.M) {
        const int64_t o = zoff + int64_t(row) * p.ldc + col0;
        uint4* dh = reinterpret_cast<uint4*>(p.Ch + o);
        uint4* dl = p.Cl ? reinterpret_cast<uint4*>(p.Cl + o) : nullptr;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          uint32_t hw[4], lw[4];
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            __nv_bfloat16 h0, l0, h1, l1;
            split_hl(__uint_as_float(r[8 * j + 2 * e]), h0, l0);
            split_hl(__uint_as_float(r[8 * j + 2 * e + 1]), h1, l1);
            hw[e] = bf2_bits(__halves2bfloat162(h0, h1));
            lw[e] = bf2_bits(__halves2bfloat162(l0, l1));
          }
          dh[j] = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          if (dl) dl[j] = make_uint4(lw[0], lw[1], lw[2], lw[3]);
        }
      }
      return;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) st[lane * 33 + i] = __uint_as_float(r[i]);
    __syncwarp();
    float v[32];
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = st[i * 33 + lane];
    __syncwarp();
    const int col = col0 + lane;
    const int nrow = min(32, p.M - row0);
    if (col < p.N && nrow > 0) {
      const int64_t o = zoff + int64_t(row0) * p.ldc + col;
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < nrow) {
          __nv_bfloat16 h, l;
          split_hl(v[i], h, l);
          p.Ch[o + int64_t(i) * p.ldc] = h;
          if (p.Cl) p.Cl[o + int64_t(i) * p.ldc] = l;
        }
    }
    return;
  }
  float* Cz = p.C + zoff;
  if (!p.accumulate && p.c_vec && col0 + 32 <= p.N) {
    const int row = row0 + lane;
    if (row < p.M) {
      float4* dst = reinterpret_cast<float4*>(Cz + int64_t(row) * p.ldc + col0);
#pragma unroll
      for (int j = 0; j < 8; ++j)
        dst[j] = make_float4(__uint_as_float(r[4 * j]), __uint_as_float(r[4 * j + 1]),
                             __uint_as_float(r[4 * j + 2]), __uint_as_float(r[4 * j + 3]));
    }
    return;
  }
#pragma unroll
  for (int i = 0; i < 32; ++i) st[lane * 33 + i] = __uint_as_float(r[i]);
  __syncwarp();
  float v[32];
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = st[i * 33 + lane];
  __syncwarp();
  const int col = col0 + lane;
  const int nrow = min(32, p.M - row0);
  if (col < p.N && nrow > 0) {
    float* base = Cz + int64_t(row0) * p.ldc + col;
    if (p.accumulate) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < nrow) atomicAdd(base + int64_t(i) * p.ldc, v[i]);
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if (i < nrow) base[int64_t(i) * p.ldc] = v[i];
    }
  }
}

// MT: 128-row M tiles per CTA; with MT = 2 two accumulators share every B tile (half the B
// bytes per flop, and each stage covers twice the MMA time).
// EPI = 1 (fused residual coding, compute-heavy epilogue): three stages and no transpose buffer,
// so that two CTAs fit on an SM and one's epilogue overlaps the other's main loop.
template <int BN, int MT, int EPI = 0>
struct Cfg {
  static constexpr int kABytes1 = BM * BK * 2;
  static constexpr int kABytes = MT * kABytes1;
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = EPI ? 3 : ((192 * 1024) / kStageBytes < 6 ? (192 * 1024) / kStageBytes : 6);
  static constexpr int kCols = MT * BN;
  static constexpr int kTmemCols = kCols <= 32 ? 32 : (kCols <= 64 ? 64 : (kCols <= 128 ? 128 : (kCols <= 256 ? 256 : 512)));
  static constexpr int kEpiBytes = EPI ? 0 : 4 * 32 * 33 * 4;
  static constexpr int kSmem = 1024 + kStages * kStageBytes + kEpiBytes + 256;
};

// TMA coordinates of one operand for one (tile, term), precomputed so that the producer's
// per-k-block work is a few adds (its scalar address arithmetic, not memory, otherwise bounds the
// stage rate). K-major: row mn0, k advanced by 64 per k-block (folded: k % fold, k / fold kept
// incrementally). MN-major: per 64-wide chunk the (mn % fold, mn / fold) pair, k as given.
struct OpCoord {
  int fold, zb, mn0, kf, kq;
  int c0[4], c2[4];
  int chunked, cs, cf;  // chunked MN-major map: sub-chunk and fold (or chunk) coordinates of the tile
};

template <int MAJ>
__device__ __forceinline__ void op_coord(OpCoord& o, int fold, int bext, int z, int mn0, int rows, int k0,
                                         int chunked = 0) {
  o.fold = fold;
  o.zb = bext > 1 ? z % bext : 0;
  o.mn0 = mn0;
  o.chunked = (MAJ == kMajorMN) ? chunked : 0;
  if (o.chunked) {
    // plain: chunk index mn0 / 64; folded: (sub-chunk within the fold, fold index)
    o.cs = fold ? (mn0 % fold) / 64 : mn0 / 64;
    o.cf = fold ? mn0 / fold : 0;
  }
  if (MAJ == kMajorK) {
    o.kf = fold ? k0 % fold : k0;
    o.kq = fold ? k0 / fold : 0;
  } else {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int mn = mn0 + 64 * i;
      o.c0[i] = (i < rows / 64) ? (fold ? mn % fold : mn) : 0;
      o.c2[i] = (i < rows / 64 && fold) ? mn / fold : 0;
    }
  }
}

template <int MAJ, int ROWS, bool PAIRLOAD>
__device__ __forceinline__ void op_issue(const CUtensorMap* map, OpCoord& o, uint32_t dst, uint32_t bar, int k0) {
  if (MAJ == kMajorK) {
    if (o.fold) {
      if (PAIRLOAD) sm100::tma_load_4d_pair(dst, map, bar, o.kf, o.mn0, o.kq, o.zb);
      else sm100::tma_load_4d(dst, map, bar, o.kf, o.mn0, o.kq, o.zb);
      o.kf += BK;
      if (o.kf >= o.fold) {
        o.kf -= o.fold;
        ++o.kq;
      }
    } else {
      if (PAIRLOAD) sm100::tma_load_3d_pair(dst, map, bar, k0, o.mn0, o.zb);
      else sm100::tma_load_3d(dst, map, bar, k0, o.mn0, o.zb);
    }
  } else if (!PAIRLOAD && o.chunked) {
    // every 64-wide chunk of the tile in one copy: [chunk][64 k rows][64]
    if (o.fold) sm100::tma_load_5d(dst, map, bar, 0, k0, o.cs, o.cf, o.zb);
    else sm100::tma_load_4d(dst, map, bar, 0, k0, o.cs, o.zb);
  } else {
#pragma unroll
    for (int i = 0; i < ROWS / 64; ++i) {
      const uint32_t d = dst + i * (64 * BK * 2);
      if (o.fold) {
        if (PAIRLOAD) sm100::tma_load_4d_pair(d, map, bar, o.c0[i], k0, o.c2[i], o.zb);
        else sm100::tma_load_4d(d, map, bar, o.c0[i], k0, o.c2[i], o.zb);
      } else {
        if (PAIRLOAD) sm100::tma_load_3d_pair(d, map, bar, o.c0[i], k0, o.zb);
        else sm100::tma_load_3d(d, map, bar, o.c0[i], k0, o.zb);
      }
    }
  }
}

// ---- fused residual coding epilogue (one thread per token row of 128 features) ---------------
// The arithmetic is the stand-alone coder's, operation for operation: x = X - x~ (fp32), signs,
// fast Walsh-Hadamard butterflies with strides 1, 2, ..., 64 ((lo, hi) -> (lo + hi, lo - hi)),
// x rsqrt(128); min / max; step = (max - min) / (2^b - 1) and zero = min rounded to fp16;
// code = clip(rint((x - zero) / scale)), packed little-endian.
// The code is clip(rint(fl((x - zero) / scale))). The quotient is first taken as fl(a * fl(1/scale)):
// two correctly rounded operations put it within 1.5 * 2^-23 |a / scale| of the exact quotient,
// and the correctly rounded fl(a / scale) within 2^-24 |a / scale| of it, so for |q| <= 512 they
// are within 2^-13 of each other and round to the same integer unless q lies within 2^-12 of a
// half-integer; only then is the division itself done (beyond 512 both clip alike).
template <int B>
__device__ __forceinline__ void res_pack_store(const float (&v)[128], float s, float zf, uint8_t* dst) {
  constexpr int kPer = 32 / B;
  const float levels = float((1 << B) - 1);
  const float rs = s != 0.f ? __frcp_rn(s) : 0.f;
#pragma unroll
  for (int q = 0; q < B; ++q) {
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      uint32_t acc = 0;
#pragma unroll
      for (int k = 0; k < kPer; ++k) {
        const int i = (q * 4 + e) * kPer + k;
        float c = 0.f;
        if (s != 0.f) {
          const float a = __fsub_rn(v[i], zf);
          const float qt = __fmul_rn(a, rs);
          c = rintf(qt);
          if (fabsf(qt) <= 512.f && fabsf(qt - c) >= 0.5f - 0.000244140625f) c = rintf(__fdiv_rn(a, s));
          c = fminf(fmaxf(c, 0.f), levels);
        }
        acc |= uint32_t(c) << (k * B);
      }
      w[e] = acc;
    }
    reinterpret_cast<uint4*>(dst)[q] = make_uint4(w[0], w[1], w[2], w[3]);
  }
}

template <int MT, int BN>
__device__ __forceinline__ void residual_epilogue(const GemmDev& p, uint32_t tmem, int warp, int lane, int m0, int z,
                                                  const uint32_t* smask) {
  const float isd = rsqrtf(128.f);
  for (int mt = 0; mt < MT; ++mt) {
    float v[128];
#pragma unroll
    for (int ch = 0; ch < 4; ++ch) {
      uint32_t r[32];
      sm100::tmem_ld32(tmem + (uint32_t(warp * 32) << 16) + uint32_t(mt * BN + ch * 32), r);
      sm100::tmem_ld_wait();
#pragma unroll
      for (int i = 0; i < 32; ++i) v[ch * 32 + i] = __uint_as_float(r[i]);
    }
    const int t = m0 + mt * BM + warp * 32 + lane;
    if (t >= p.M) continue;
    const int64_t rr = int64_t(z) * p.res.T + t;
    if (p.res.x_f32) {
      const float4* xr = reinterpret_cast<const float4*>(static_cast<const float*>(p.res.X) + rr * 128);
#pragma unroll
      for (int j = 0; j < 32; ++j) {
        const float4 x = xr[j];
        v[4 * j] = x.x - v[4 * j];
        v[4 * j + 1] = x.y - v[4 * j + 1];
        v[4 * j + 2] = x.z - v[4 * j + 2];
        v[4 * j + 3] = x.w - v[4 * j + 3];
      }
    } else {
      const uint4* xr = reinterpret_cast<const uint4*>(static_cast<const __nv_bfloat16*>(p.res.X) + rr * 128);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        const uint4 x = xr[j];
        const uint32_t w[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float2 f = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&w[e]));
          v[8 * j + 2 * e] = f.x - v[8 * j + 2 * e];
          v[8 * j + 2 * e + 1] = f.y - v[8 * j + 2 * e + 1];
        }
      }
    }
#pragma unroll
    for (int i = 0; i < 128; ++i)
      if ((smask[i >> 5] >> (i & 31)) & 1u) v[i] = -v[i];
#pragma unroll
    for (int st = 1; st < 128; st <<= 1) {
#pragma unroll
      for (int i = 0; i < 128; ++i) {
        if ((i & st) == 0) {
          const float a = v[i], b = v[i + st];
          v[i] = a + b;
          v[i + st] = a - b;
        }
      }
    }
    bool ok = true;
    float mn, mx;
#pragma unroll
    for (int i = 0; i < 128; ++i) {
      v[i] *= isd;
      ok &= isfinite(v[i]);
      mn = i ? fminf(mn, v[i]) : v[i];
      mx = i ? fmaxf(mx, v[i]) : v[i];
    }
    const float levels = float((1 << p.res.b) - 1);
    const float step = __fdiv_rn(__fsub_rn(mx, mn), levels);
    const __half hs = __float2half_rn(step);
    const __half hz = __float2half_rn(mn);
    const float sc = __half2float(hs), zf = __half2float(hz);
    if (!(ok && isfinite(sc) && isfinite(zf))) report_error(p.err, JOLT_ERR_NUMERIC);
    uint8_t* dst = p.res.codes + rr * (16 * p.res.b);
    if (p.res.b == 2) res_pack_store<2>(v, sc, zf, dst);
    else if (p.res.b == 4) res_pack_store<4>(v, sc, zf, dst);
    else res_pack_store<8>(v, sc, zf, dst);
    static_cast<__half2*>(p.res.sz)[rr] = __halves2half2(hs, hz);
  }
}

template <int BN, int AMAJ, int BMAJ, int MT, int EPI = 0>
__global__ void __launch_bounds__(128, EPI ? 2 : 1) k_gemm(const __grid_constant__ TmaPack maps, GemmDev p) {
  using C = Cfg<BN, MT, EPI>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  float* epi = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes + C::kEpiBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::kStages + 1);
  uint32_t* smask = tmem_slot + 1;  // EPI = 1: rotation signs of the 128 features, one bit each

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n0 = blockIdx.x * BN, m0 = blockIdx.y * BM * MT;
  if (p.c_upper && m0 >= n0 + BN) return;  // whole tile below the diagonal (uniform per CTA)
  const int z = blockIdx.z / p.k_split, kz = blockIdx.z % p.k_split;
  const int nkb_all = (p.K + BK - 1) / BK;
  const int nkb_total = p.b_upper ? min(nkb_all, (n0 + BN + BK - 1) / BK) : nkb_all;
  const int kb_begin = kz * p.nkb_split;
  const int nkb = max(0, min(p.nkb_split, nkb_total - kb_begin));
  const int n_iters = nkb * p.n_terms;

  const uint32_t bar0 = sm100::smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
  const uint32_t done_bar = bar0 + 8u * (2 * C::kStages);

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      sm100::mbar_init(full_bar(s), 1);
      sm100::mbar_init(empty_bar(s), 1);
    }
    sm100::mbar_init(done_bar, 1);
    sm100::fence_mbar_init();
    for (int t = 0; t < p.n_terms; ++t) {
      sm100::prefetch_tmap(&maps.a[t]);
      sm100::prefetch_tmap(&maps.b[t]);
    }
  }
  if (warp == 2) sm100::tmem_alloc(sm100::smem_u32(tmem_slot), C::kTmemCols);
  if (EPI == 1 && warp == 3) {
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t m = __ballot_sync(0xffffffffu, rot_sign(p.res.seed, w * 32 + lane) < 0.f);
      if (lane == 0) smask[w] = m;
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t smem_base = sm100::smem_u32(smem);

  if (n_iters > 0) {
    if ((warp == 0 || warp == 2) && lane == 0) {
      // ---- TMA producers: warp 0 streams A (and posts the stage's byte count), warp 2 streams
      // B; both wait for the same free stage ----
      const bool is_a = warp == 0;
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int t = 0; ok && t < p.n_terms; ++t) {
        int k0 = kb_begin * BK;
        OpCoord o[MT];
        // a chunked MN-major A covers all MT row tiles (consecutive in shared memory) in one copy
        const bool a_one = AMAJ == kMajorMN && p.a_chunk[t];
        if (is_a) {
#pragma unroll
          for (int mt = 0; mt < MT; ++mt)
            op_coord<AMAJ>(o[mt], p.a_fold[t], p.a_batch[t], z, m0 + mt * BM, BM, k0, p.a_chunk[t]);
        } else {
          op_coord<BMAJ>(o[0], p.b_fold[t], p.b_batch[t], z, n0, BN, k0, p.b_chunk[t]);
        }
        for (int kb = 0; kb < nkb; ++kb, k0 += BK) {
          if (!sm100::mbar_wait(empty_bar(stage), phase ^ 1, p.err)) { ok = false; break; }
          const uint32_t sa = smem_base + stage * C::kStageBytes;
          if (is_a) {
            sm100::mbar_expect_tx(full_bar(stage), C::kStageBytes);
            if (a_one) {
              op_issue<AMAJ, BM, false>(&maps.a[t], o[0], sa, full_bar(stage), k0);
            } else {
#pragma unroll
              for (int mt = 0; mt < MT; ++mt)
                op_issue<AMAJ, BM, false>(&maps.a[t], o[mt], sa + mt * C::kABytes1, full_bar(stage), k0);
            }
          } else {
            op_issue<BMAJ, BN, false>(&maps.b[t], o[0], sa + C::kABytes, full_bar(stage), k0);
          }
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
    } else if (warp == 1 && lane == 0) {
      // ---- MMA issuer ----
      constexpr uint32_t idesc = sm100::idesc_bf16_f32(BM, BN, AMAJ, BMAJ);
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1;
        if (!sm100::mbar_wait(full_bar(s), ph, p.err)) break;
        sm100::tc_fence_after();
        const uint32_t sa = smem_base + s * C::kStageBytes;
        const uint32_t sb = sa + C::kABytes;
#pragma unroll
        for (int kk = 0; kk < BK / 16; ++kk) {
          uint64_t bd;
          if (BMAJ == kMajorK) bd = sm100::smem_desc_sw128(sb + kk * 32, 16, 1024);
          else bd = sm100::smem_desc_sw128(sb + kk * 2048, 64 * BK * 2, 1024);
#pragma unroll
          for (int mt = 0; mt < MT; ++mt) {
            const uint32_t sam = sa + mt * C::kABytes1;
            uint64_t ad;
            if (AMAJ == kMajorK) ad = sm100::smem_desc_sw128(sam + kk * 32, 16, 1024);
            else ad = sm100::smem_desc_sw128(sam + kk * 2048, 64 * BK * 2, 1024);
            sm100::mma_bf16(tmem + mt * BN, ad, bd, idesc, (it > 0 || kk > 0) ? 1u : 0u);
          }
        }
        sm100::mma_commit(empty_bar(s));
      }
      sm100::mma_commit(done_bar);
    }
    __syncwarp();
    // ---- epilogue: TMEM -> registers -> smem transpose -> coalesced global ----
    // warp-uniform (the TMEM loads below are warp-collective)
    const bool ok = __all_sync(0xffffffffu, sm100::mbar_wait(done_bar, 0, p.err));
    sm100::tc_fence_after();
    if (ok && EPI == 1) {
      residual_epilogue<MT, BN>(p, tmem, warp, lane, m0, z, smask);
    } else if (ok) {
      float* st = epi + warp * 32 * 33;
      const int64_t zoff = int64_t(z / p.c_div) * p.c_bstride;
      for (int cc = 0; cc < MT * BN; cc += 32) {
        const int mt = cc / BN, c0 = cc % BN;
        uint32_t r[32];
        sm100::tmem_ld32(tmem + (uint32_t(warp * 32) << 16) + cc, r);
        sm100::tmem_ld_wait();
        store_chunk(p, zoff, r, st, m0 + mt * BM + warp * 32, n0 + c0, lane);
      }
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 2) sm100::tmem_dealloc(tmem, C::kTmemCols);
}

// ---- persistent variant: double-buffered accumulators -----------------------------------------
// Each CTA (or CTA pair) walks tiles t = cluster, cluster + clusters, ... with the N tile fastest
// (CTAs running at the same time share rows of A in L2). Two 128 x 256 fp32 accumulators live
// in TMEM (all 512 columns), so four epilogue warps drain tile i while the MMA warp fills tile
// i + 1 and two TMA warps stream its stages. 224 threads: warp 0 TMA for A, warp 6 TMA for B,
// warp 1 MMA (+ TMEM allocation), warps 2..5 epilogue (TMEM lane quarter = warp % 4).
// PAIR = 1 is the cta_group::2 form: a tile is 256 x 256, each CTA stages its 128 rows of A and
// 128 columns of B, the even CTA issues the MMAs and owns the stage "full" barriers and the
// accumulator "empty" barriers (the odd CTA's epilogue arrives there remotely).
template <int PAIR>
struct CfgP {
  static constexpr int BN = 256;
  static constexpr int kBCols = PAIR ? 128 : 256;
  static constexpr int kABytes = BM * BK * 2;
  static constexpr int kBBytes = kBCols * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (192 * 1024) / kStageBytes < 8 ? (192 * 1024) / kStageBytes : 8;
  static constexpr int kTmemCols = 512;
  static constexpr int kEpiBytes = 4 * 32 * 33 * 4;
  static constexpr int kThreads = 224;
  static constexpr int kSmem = 1024 + kStages * kStageBytes + kEpiBytes + 256;
};

struct TileP {
  int n0, m0, z, kb_begin, nkb;
};

// Tile t of the persistent walk; false if it has no work (below a c_upper diagonal, or a split-K
// slice past a b_upper triangle). Every role calls this with the same t and gets the same answer.
template <int ROWS>
__device__ __forceinline__ bool tile_p(const GemmDev& p, int t, TileP& ti) {
  constexpr int BN = 256;
  const int nt = t % p.ntile;
  const int r = t / p.ntile;
  const int mt = r % p.mtiles;
  const int zz = r / p.mtiles;
  ti.n0 = nt * BN;
  ti.m0 = mt * ROWS;
  ti.z = zz / p.k_split;
  const int kz = zz % p.k_split;
  if (p.c_upper && ti.m0 >= ti.n0 + BN) return false;
  const int nkb_all = (p.K + BK - 1) / BK;
  const int nkb_total = p.b_upper ? min(nkb_all, (ti.n0 + BN + BK - 1) / BK) : nkb_all;
  ti.kb_begin = kz * p.nkb_split;
  ti.nkb = max(0, min(p.nkb_split, nkb_total - ti.kb_begin));
  return ti.nkb > 0;
}

template <int PAIR, int AMAJ, int BMAJ>
__global__ void __launch_bounds__(224, 1) k_gemm_p(const __grid_constant__ TmaPack maps, GemmDev p) {
  using C = CfgP<PAIR>;
  constexpr int BN = C::BN;
  constexpr int ROWS = PAIR ? 2 * BM : BM;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = sm100::align_smem_1024(smem_raw);
  float* epi = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes + C::kEpiBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::kStages + 4);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = PAIR ? sm100::cluster_ctarank() : 0u;
  const int cluster = PAIR ? int(blockIdx.x >> 1) : int(blockIdx.x);
  const int n_clusters = PAIR ? int(gridDim.x >> 1) : int(gridDim.x);

  const uint32_t bar0 = sm100::smem_u32(bars);
  auto full_bar = [&](int s) { return bar0 + 8u * s; };
  auto empty_bar = [&](int s) { return bar0 + 8u * (C::kStages + s); };
  auto accf_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + b); };
  auto acce_bar = [&](int b) { return bar0 + 8u * (2 * C::kStages + 2 + b); };

  if (threadIdx.x == 0) {
    for (int s = 0; s < C::kStages; ++s) {
      sm100::mbar_init(full_bar(s), 1);
      sm100::mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      sm100::mbar_init(accf_bar(b), 1);
      sm100::mbar_init(acce_bar(b), PAIR ? 8 : 4);
    }
    *abort_flag = 0;
    sm100::fence_mbar_init();
    for (int t = 0; t < p.n_terms; ++t) {
      sm100::prefetch_tmap(&maps.a[t]);
      sm100::prefetch_tmap(&maps.b[t]);
    }
  }
  if (warp == 1) {
    if (PAIR) sm100::tmem_alloc_pair(sm100::smem_u32(tmem_slot), C::kTmemCols);
    else sm100::tmem_alloc(sm100::smem_u32(tmem_slot), C::kTmemCols);
  }
  sm100::tc_fence_before();
  if (PAIR) sm100::cluster_sync();
  else __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t smem_base = sm100::smem_u32(smem);
  auto aborted = [&]() { return *abort_flag != 0 || (p.err && *reinterpret_cast<volatile int32_t*>(p.err) != 0); };
  auto fail = [&]() { *abort_flag = 1; };

  if (warp == 0 || warp == 6) {
    if (lane == 0) {
      // ---- TMA producers: warp 0 streams A (and posts the stage's byte count), warp 6 streams
      // B; both wait for the same free stage ----
      const bool is_a = warp == 0;
      int stage = 0;
      uint32_t phase = 0;
      const uint32_t full_own = full_bar(0);
      const uint32_t full_lead = PAIR ? sm100::mapa_shared(full_bar(0), 0) : full_bar(0);
      const uint32_t tx = PAIR ? 2 * C::kStageBytes : C::kStageBytes;
      TileP ti;
      bool ok = true;
      for (int t = cluster; ok && t < p.n_tiles && !aborted(); t += n_clusters) {
        if (!tile_p<ROWS>(p, t, ti)) continue;
        const int arow = ti.m0 + int(rank) * BM;
        const int bcol = ti.n0 + int(rank) * C::kBCols;
        for (int term = 0; ok && term < p.n_terms; ++term) {
          int k0 = ti.kb_begin * BK;
          OpCoord o;
          if (is_a) op_coord<AMAJ>(o, p.a_fold[term], p.a_batch[term], ti.z, arow, BM, k0);
          else op_coord<BMAJ>(o, p.b_fold[term], p.b_batch[term], ti.z, bcol, C::kBCols, k0);
          const CUtensorMap* m = is_a ? &maps.a[term] : &maps.b[term];
          for (int kb = 0; kb < ti.nkb; ++kb, k0 += BK) {
            if (!sm100::mbar_wait(empty_bar(stage), phase ^ 1, p.err)) { ok = false; break; }
            const uint32_t sa = smem_base + stage * C::kStageBytes;
            const uint32_t fb = (PAIR ? full_lead : full_own) + 8u * stage;
            if (is_a) {
              if (rank == 0) sm100::mbar_expect_tx(full_bar(stage), tx);
              op_issue<AMAJ, BM, PAIR != 0>(m, o, sa, fb, k0);
            } else {
              op_issue<BMAJ, C::kBCols, PAIR != 0>(m, o, sa + C::kABytes, fb, k0);
            }
            if (++stage == C::kStages) {
              stage = 0;
              phase ^= 1;
            }
          }
        }
      }
      if (!ok) fail();
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---- MMA issuer ----
      constexpr uint32_t idesc = sm100::idesc_bf16_f32(ROWS, BN, AMAJ, BMAJ);
      // descriptor of stage 0's A / B tiles; per K16 step the start address advances by 32 bytes
      // (K-major) or 2048 bytes (MN-major), per stage by kStageBytes (encoded >> 4)
      const uint64_t a0 = AMAJ == kMajorK ? sm100::smem_desc_sw128(smem_base, 16, 1024)
                                          : sm100::smem_desc_sw128(smem_base, 64 * BK * 2, 1024);
      const uint64_t b0 = BMAJ == kMajorK ? sm100::smem_desc_sw128(smem_base + C::kABytes, 16, 1024)
                                          : sm100::smem_desc_sw128(smem_base + C::kABytes, 64 * BK * 2, 1024);
      constexpr uint32_t a_step = (AMAJ == kMajorK ? 32 : 2048) >> 4;
      constexpr uint32_t b_step = (BMAJ == kMajorK ? 32 : 2048) >> 4;
      int stage = 0, lt = 0;
      uint32_t phase = 0;
      TileP ti;
      for (int t = cluster; t < p.n_tiles && !aborted(); t += n_clusters) {
        if (!tile_p<ROWS>(p, t, ti)) continue;
        const int b = lt & 1;
        const uint32_t aph = (lt >> 1) & 1;
        ++lt;
        if (!sm100::mbar_wait(acce_bar(b), aph ^ 1, p.err)) { fail(); break; }
        sm100::tc_fence_after();
        const uint32_t dt = tmem + uint32_t(b * BN);
        const int n_it = ti.nkb * p.n_terms;
        bool ok = true;
        for (int it = 0; it < n_it; ++it) {
          if (!sm100::mbar_wait(full_bar(stage), phase, p.err)) { ok = false; break; }
          sm100::tc_fence_after();
          const uint64_t soff = uint64_t((uint32_t(stage) * C::kStageBytes) >> 4);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = a0 + soff + kk * a_step;
            const uint64_t bd = b0 + soff + kk * b_step;
            const uint32_t acc = (it > 0 || kk > 0) ? 1u : 0u;
            if (PAIR) sm100::mma_bf16_pair(dt, ad, bd, idesc, acc);
            else sm100::mma_bf16(dt, ad, bd, idesc, acc);
          }
          if (PAIR) sm100::mma_commit_pair(empty_bar(stage), 0x3);
          else sm100::mma_commit(empty_bar(stage));
          if (++stage == C::kStages) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (!ok) { fail(); break; }
        if (PAIR) sm100::mma_commit_pair(accf_bar(b), 0x3);
        else sm100::mma_commit(accf_bar(b));
      }
    }
  } else if (warp >= 2 && warp <= 5) {
    // ---- epilogue: TMEM -> registers -> smem transpose -> coalesced global ----
    const int q = warp & 3;  // TMEM lane quarter this warp may read
    float* st = epi + (warp - 2) * 32 * 33;
    const uint32_t acce_target = PAIR ? sm100::mapa_shared(acce_bar(0), 0) : acce_bar(0);
    int lt = 0;
    TileP ti;
    for (int t = cluster; t < p.n_tiles && !aborted(); t += n_clusters) {
      if (!tile_p<ROWS>(p, t, ti)) continue;
      const int b = lt & 1;
      const uint32_t aph = (lt >> 1) & 1;
      ++lt;
      if (!__all_sync(0xffffffffu, sm100::mbar_wait(accf_bar(b), aph, p.err))) { fail(); break; }
      sm100::tc_fence_after();
      const int64_t zoff = int64_t(ti.z / p.c_div) * p.c_bstride;
      const int rbase = ti.m0 + int(rank) * BM + q * 32;
      for (int cc = 0; cc < BN; cc += 32) {
        uint32_t r[32];
        sm100::tmem_ld32(tmem + (uint32_t(q * 32) << 16) + uint32_t(b * BN + cc), r);
        sm100::tmem_ld_wait();
        store_chunk(p, zoff, r, st, rbase, ti.n0 + cc, lane);
      }
      sm100::tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (PAIR) sm100::mbar_arrive_cluster(acce_target + 8u * b);
        else sm100::mbar_arrive(acce_bar(b));
      }
    }
  }
  __syncwarp();
  sm100::tc_fence_before();
  if (PAIR) sm100::cluster_sync();
  else __syncthreads();
  sm100::tc_fence_after();
  if (warp == 1) {
    if (PAIR) sm100::tmem_dealloc_pair(tmem, C::kTmemCols);
    else sm100::tmem_dealloc(tmem, C::kTmemCols);
  }
}

// ---- host: tensor maps ----------------------------------------------------------------------

template <int BN, int AM, int BMJ, int MT>
jolt_status launch(const TmaPack& maps, const GemmDev& d, dim3 grid, cudaStream_t st) {
  using C = Cfg<BN, MT>;
  auto kern = k_gemm<BN, AM, BMJ, MT>;
  JOLT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem));
  kern<<<grid, 128, C::kSmem, st>>>(maps, d);
  JOLT_CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

template <int PAIR, int AM, int BMJ>
jolt_status launch_p(const TmaPack& maps, const GemmDev& d, dim3 grid, cudaStream_t st) {
  using C = CfgP<PAIR>;
  auto kern = k_gemm_p<PAIR, AM, BMJ>;
  JOLT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = dim3(C::kThreads);
  cfg.dynamicSmemBytes = C::kSmem;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = PAIR ? 2 : 1;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  JOLT_CUDA_TRY(cudaLaunchKernelEx(&cfg, kern, maps, d));
  return JOLT_OK;
}

template <int PAIR>
jolt_status launch_pers(int am, int bm, const TmaPack& maps, const GemmDev& d, dim3 grid, cudaStream_t st) {
  if (am == kMajorK && bm == kMajorK) return launch_p<PAIR, kMajorK, kMajorK>(maps, d, grid, st);
  if (am == kMajorK && bm == kMajorMN) return launch_p<PAIR, kMajorK, kMajorMN>(maps, d, grid, st);
  if (am == kMajorMN && bm == kMajorK) return launch_p<PAIR, kMajorMN, kMajorK>(maps, d, grid, st);
  return launch_p<PAIR, kMajorMN, kMajorMN>(maps, d, grid, st);
}

template <int MT>
jolt_status launch_res(const TmaPack& maps, const GemmDev& d, dim3 grid, cudaStream_t st) {
  using C = Cfg<128, MT, 1>;
  auto kern = k_gemm<128, kMajorK, kMajorMN, MT, 1>;
  JOLT_CUDA_TRY(cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, C::kSmem));
  kern<<<grid, 128, C::kSmem, st>>>(maps, d);
  JOLT_CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

template <int BN, int MT>
jolt_status launch_bn(int am, int bm, const TmaPack& maps, const GemmDev& d, dim3 grid, cudaStream_t st) {
  if (am == kMajorK && bm == kMajorK) return launch<BN, kMajorK, kMajorK, MT>(maps, d, grid, st);
  if (am == kMajorK && bm == kMajorMN) return launch<BN, kMajorK, kMajorMN, MT>(maps, d, grid, st);
  if (am == kMajorMN && bm == kMajorK) return launch<BN, kMajorMN, kMajorK, MT>(maps, d, grid, st);
  return launch<BN, kMajorMN, kMajorMN, MT>(maps, d, grid, st);
}

}  // namespace

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(f);
  });
  return fn;
}

bool make_tensor_map(CUtensorMap* m, const Operand& o, int rows) {
  constexpr int BK = 64;
  EncodeTiledFn enc = encode_fn();
  if (!enc || !o.ptr) return false;
  if (reinterpret_cast<uintptr_t>(o.ptr) % 16) return false;
  cuuint64_t dims[4], strides[3];
  cuuint32_t box[4], estr[4] = {1, 1, 1, 1};
  const int64_t bext = std::max<int64_t>(1, o.batch_stride ? o.batch : 1);
  int rank;
  const uint32_t outer_box = (o.major == kMajorK) ? uint32_t(rows) : uint32_t(BK);
  if (o.fold) {
    rank = 4;
    dims[0] = o.fold; dims[1] = o.outer; dims[2] = o.nfold; dims[3] = bext;
    strides[0] = o.outer_stride * 2; strides[1] = o.fold_stride * 2;
    strides[2] = (o.batch_stride ? o.batch_stride : o.fold_stride * o.nfold) * 2;
    box[0] = 64; box[1] = outer_box; box[2] = 1; box[3] = 1;
  } else {
    rank = 3;
    dims[0] = o.inner; dims[1] = o.outer; dims[2] = bext;
    strides[0] = o.outer_stride * 2;
    strides[1] = (o.batch_stride ? o.batch_stride : o.outer_stride * o.outer) * 2;
    box[0] = 64; box[1] = outer_box; box[2] = 1;
  }
  for (int i = 0; i < rank - 1; ++i)
    if (strides[i] % 16 || strides[i] == 0) return false;
  CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(o.ptr), dims, strides,
                   box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && kDebug) {
    std::fprintf(stderr, "jolt: tensor map rejected (CUresult %d) rank %d dims", int(r), rank);
    for (int i = 0; i < rank; ++i) std::fprintf(stderr, " %llu", (unsigned long long)dims[i]);
    std::fprintf(stderr, " box");
    for (int i = 0; i < rank; ++i) std::fprintf(stderr, " %u", box[i]);
    std::fprintf(stderr, "\n");
  }
  return r == CUDA_SUCCESS;
}

// MN-major operand tile of `rows` MN elements (a multiple of 64, starting at a multiple of rows) in
// one copy: plain (64, K, inner/64, batch) with box (64, 64, rows/64, 1); folded (64, K, fold/64,
// nfold, batch) with box (64, 64, min(rows, fold)/64, max(1, rows/fold), 1). The chunk stride is
// 128 bytes (the next 64 elements of a row). False where the layout does not fit (the caller then
// copies chunk by chunk).
bool make_tensor_map_chunked(CUtensorMap* m, const Operand& o, int rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || !o.ptr || o.major != kMajorMN || rows % 64) return false;
  if (reinterpret_cast<uintptr_t>(o.ptr) % 16) return false;
  const int64_t bext = std::max<int64_t>(1, o.batch_stride ? o.batch : 1);
  cuuint64_t dims[5], strides[4];
  cuuint32_t box[5], estr[5] = {1, 1, 1, 1, 1};
  int rank;
  if (o.fold) {
    if (o.fold % 64) return false;
    if (o.fold >= rows ? (o.fold % rows) : (rows % o.fold)) return false;
    rank = 5;
    dims[0] = 64; dims[1] = o.outer; dims[2] = o.fold / 64; dims[3] = o.nfold; dims[4] = bext;
    strides[0] = o.outer_stride * 2; strides[1] = 128; strides[2] = o.fold_stride * 2;
    strides[3] = (o.batch_stride ? o.batch_stride : o.fold_stride * o.nfold) * 2;
    box[0] = 64; box[1] = 64; box[2] = uint32_t(std::min<int64_t>(rows, o.fold) / 64);
    box[3] = uint32_t(std::max<int64_t>(1, rows / o.fold)); box[4] = 1;
  } else {
    if (o.inner % 64) return false;  // the last chunk must end at the row's end
    rank = 4;
    dims[0] = 64; dims[1] = o.outer; dims[2] = o.inner / 64; dims[3] = bext;
    strides[0] = o.outer_stride * 2; strides[1] = 128;
    strides[2] = (o.batch_stride ? o.batch_stride : o.outer_stride * o.outer) * 2;
    box[0] = 64; box[1] = 64; box[2] = uint32_t(rows / 64); box[3] = 1;
  }
  for (int i = 0; i < rank - 1; ++i)
    if (strides[i] % 16 || strides[i] == 0) return false;
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, rank, const_cast<void*>(o.ptr), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool make_tensor_map_mn_chunks(CUtensorMap* m, const void* ptr, int64_t K, int64_t ld, int chunks, int64_t batch,
                               int64_t batch_stride, int terms, int64_t term_stride) {
  EncodeTiledFn enc = encode_fn();
  if (!enc || !ptr || reinterpret_cast<uintptr_t>(ptr) % 16) return false;
  cuuint64_t dims[5] = {64, cuuint64_t(K), cuuint64_t(chunks), cuuint64_t(std::max<int64_t>(1, batch)),
                        cuuint64_t(terms)};
  cuuint64_t strides[4] = {cuuint64_t(ld) * 2, 128, cuuint64_t(batch_stride) * 2, cuuint64_t(term_stride) * 2};
  cuuint32_t box[5] = {64, 64, cuuint32_t(chunks), 1, cuuint32_t(terms)};
  cuuint32_t estr[5] = {1, 1, 1, 1, 1};
  for (int i = 0; i < 4; ++i)
    if (strides[i] % 16 || strides[i] == 0) return false;
  const CUresult r = enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 5, const_cast<void*>(ptr), dims, strides, box, estr,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS && kDebug)
    std::fprintf(stderr, "jolt: chunked MN tensor map rejected (CUresult %d)\n", int(r));
  return r == CUDA_SUCCESS;
}

namespace {

// Tile plan: the one-tile-per-CTA kernel with MT 128-row accumulators and the split-K factor that
// minimise the estimated time, i.e. whole waves of one CTA per SM x (k-blocks per CTA + 1 for
// its epilogue) over the relative per-SM speed (two accumulators sharing B run ~1.2x the flops
// per cycle of one). Tiles a symmetric (c_upper) output skips are not counted.
// The persistent forms (JOLT_GEMM_PERSISTENT: single CTAs, JOLT_GEMM_PAIRS: CTA pairs; N > 128 and
// more than one 128-row tile) are faster in isolation at a fixed clock, but in a whole compression
// pass under the board's power cap they lower the clock the rest of the pass runs at by more than
// they gain, so the one-tile kernel is the default.
struct TilePlan {
  int kind, MT, k_split;  // kind: 0 one tile per CTA, 2 persistent single CTA, 3 persistent pair
};

TilePlan plan_tiles(const GemmCall& g, int BN) {
  constexpr int kSMs = 148;
  int only = g.plan == JOLT_GEMM_PERSISTENT ? 2 : g.plan == JOLT_GEMM_PAIRS ? 3 : 0;
  const bool pers_ok = BN == 256 && g.M > BM;
  if (only < 0 || !pers_ok) only = 0;
  const int64_t ntile = (g.N + BN - 1) / BN, kb = (g.K + BK - 1) / BK;
  // tiles with work when one CTA (or pair) covers `rows` rows
  auto active = [&](int rows) {
    const int64_t mt = (g.M + rows - 1) / rows;
    int64_t a = 0;
    for (int64_t i = 0; i < mt; ++i)
      for (int64_t j = 0; j < ntile; ++j) a += (g.c_upper && i * rows >= j * BN + BN) ? 0 : 1;
    return a * g.batch;
  };
  const int kmax = (g.Ch || g.res) ? 1 : (g.k_split == 0 ? int(std::max<int64_t>(1, std::min<int64_t>(64, kb / 2))) : g.k_split);
  const int kmin = g.k_split == 0 ? 1 : g.k_split;
  TilePlan best{only, 1, kmin};
  double best_t = 1e300;
  // the fused residual epilogue runs with one accumulator, two CTAs per SM
  for (int MT = (only == 0 && !g.res ? 2 : 1); MT >= 1; --MT) {
    if (MT == 2 && g.M <= BM) continue;
    const bool pair = only == 3;
    const int slots = pair ? kSMs / 2 : kSMs;  // tiles in flight at once
    const int64_t act = active((pair ? 2 : 1) * BM * MT);
    for (int k = kmin; k <= kmax; ++k) {
      const int64_t tiles = act * k;
      const double rounds = double((tiles + slots - 1) / slots);
      const double per = double((kb + k - 1) / k);
      // one-tile kernel: two accumulators sharing B run ~1.2x the flops per cycle of one
      const double t = only == 0 ? rounds * MT * (per + 1.0) / (MT == 2 ? 1.2 : 1.0) : rounds * (per + 2.0);
      if (t < best_t * 0.999) {
        best_t = t;
        best = TilePlan{only, MT, k};
      }
    }
  }
  return best;
}

}  // namespace

jolt_status gemm_tc(const GemmCall& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return JOLT_OK;
  if (g.n_terms < 1 || g.n_terms > kMaxTerms || (!g.C && !g.Ch && !g.res) || (g.C && g.Ch) || g.batch < 1 || g.k_split < 0 ||
      g.c_batch_div < 1)
    return JOLT_ERR_INVALID_ARG;
  if (g.Ch && (g.accumulate || g.k_split > 1 || g.c_batch_div > 1)) return JOLT_ERR_INVALID_ARG;
  if (g.Cl && !g.Ch) return JOLT_ERR_INVALID_ARG;
  if (g.res) {
    const ResidualEpi& e = *g.res;
    if (g.C || g.Ch || g.accumulate || g.k_split > 1 || g.c_batch_div > 1 || g.N != 128 || !e.X || !e.codes ||
        !e.sz || e.T != g.M || !(e.b == 2 || e.b == 4 || e.b == 8) ||
        reinterpret_cast<uintptr_t>(e.codes) % 16 || reinterpret_cast<uintptr_t>(e.X) % 16 ||
        reinterpret_cast<uintptr_t>(e.sz) % 4 || g.A[0].major != kMajorK || g.B[0].major != kMajorMN)
      return JOLT_ERR_INVALID_ARG;
  }
  if ((g.k_split != 1 || g.c_batch_div > 1) && !g.accumulate) return JOLT_ERR_INVALID_ARG;
  const int am = g.A[0].major, bm = g.B[0].major;
  for (int t = 0; t < g.n_terms; ++t)
    if (g.A[t].major != am || g.B[t].major != bm) return JOLT_ERR_INVALID_ARG;
  // BN: 256 whenever N exceeds one 128-wide tile — a 128 x 256 tile runs ~1.5x more flops per
  // cycle than 128 x 128 (half the operand bytes per flop), which outweighs the padding of N
  const int BN = g.N > 128 ? 256 : 128;
  const TilePlan tp = plan_tiles(g, BN);
  const int MT = tp.MT;
  TmaPack maps;
  memset(&maps, 0, sizeof(maps));
  GemmDev d{};
  // MN-major operands as one multi-chunk copy per stage unless the call asks for per-chunk copies
  const bool try_chunk = tp.kind == 0 && g.plan != JOLT_GEMM_PER_CHUNK;
  for (int t = 0; t < g.n_terms; ++t) {
    d.a_chunk[t] = try_chunk && g.A[t].major == kMajorMN && make_tensor_map_chunked(&maps.a[t], g.A[t], BM * tp.MT);
    d.b_chunk[t] = try_chunk && g.B[t].major == kMajorMN && make_tensor_map_chunked(&maps.b[t], g.B[t], BN);
    if (!d.a_chunk[t] && !make_tensor_map(&maps.a[t], g.A[t], BM)) return JOLT_ERR_INVALID_ARG;
    if (!d.b_chunk[t] && !make_tensor_map(&maps.b[t], g.B[t], tp.kind == 3 ? BN / 2 : BN)) return JOLT_ERR_INVALID_ARG;
    d.a_fold[t] = int(g.A[t].fold);
    d.b_fold[t] = int(g.B[t].fold);
    d.a_batch[t] = g.A[t].batch_stride ? int(g.A[t].batch) : 1;
    d.b_batch[t] = g.B[t].batch_stride ? int(g.B[t].batch) : 1;
    if ((g.A[t].fold && g.A[t].fold % 64) || (g.B[t].fold && g.B[t].fold % 64)) return JOLT_ERR_INVALID_ARG;
  }
  d.M = g.M; d.N = g.N; d.K = g.K; d.n_terms = g.n_terms; d.k_split = tp.k_split;
  const int nkb = (g.K + BK - 1) / BK;
  d.nkb_split = (nkb + tp.k_split - 1) / tp.k_split;
  d.C = g.C; d.ldc = g.ldc; d.c_bstride = g.c_batch_stride; d.c_div = g.c_batch_div;
  d.accumulate = g.accumulate ? 1 : 0;
  d.c_upper = g.c_upper ? 1 : 0;
  d.b_upper = g.b_upper ? 1 : 0;
  d.err = g.err;
  d.Ch = g.Ch;
  d.Cl = g.Cl;
  if (g.res) d.res = *g.res;
  if (g.Ch)
    d.c_vec = (reinterpret_cast<uintptr_t>(g.Ch) % 16 == 0 && reinterpret_cast<uintptr_t>(g.Cl) % 16 == 0 &&
               g.ldc % 8 == 0 && g.c_batch_stride % 8 == 0) ? 1 : 0;
  else
    d.c_vec = (reinterpret_cast<uintptr_t>(g.C) % 16 == 0 && g.ldc % 4 == 0 && g.c_batch_stride % 4 == 0) ? 1 : 0;
  const int64_t ntile = (g.N + BN - 1) / BN, zc = int64_t(g.batch) * tp.k_split;
  // single CTAs: (N tile, M tile); pairs: (2 x N tile + CTA of the pair, pair tile), so that
  // consecutive CTAs share the rows of A
  const bool pair = tp.kind == 3;
  const int64_t rows = int64_t(pair ? 2 : 1) * BM * MT;
  const int64_t gy = (g.M + rows - 1) / rows;
  dim3 grid{unsigned(ntile * (pair ? 2 : 1)), unsigned(gy), unsigned(zc)};
  if (tp.kind >= 2) {
    // persistent: one CTA (pair) per SM (pair of SMs), tiles walked in-kernel
    const int64_t n_tiles = ntile * gy * zc;
    if (n_tiles > INT32_MAX) return JOLT_ERR_INVALID_ARG;
    d.ntile = int(ntile);
    d.mtiles = int(gy);
    d.n_tiles = int(n_tiles);
    const int64_t slots = pair ? 74 : 148;
    grid = dim3{unsigned(std::min(n_tiles, slots) * (pair ? 2 : 1)), 1u, 1u};
  } else if (gy > 65535 || zc > 65535) {
    return JOLT_ERR_INVALID_ARG;
  }
  // algorithmic flops: the product once (its bf16 terms only restore fp32 precision of one
  // operand), halved for a triangular B or a wanted upper triangle of C; issued: once per term
  const double tri = (g.b_upper || g.c_upper) ? 0.5 : 1.0;
  const double prod = tri * 2.0 * g.M * double(g.N) * g.K * g.batch;
  StatScope sc(g.res ? -1 : JOLT_K_GEMM, st, prod, 0.0, prod * g.n_terms);
  if (g.res) return launch_res<1>(maps, d, grid, st);
  if (tp.kind == 3) return launch_pers<1>(am, bm, maps, d, grid, st);
  if (tp.kind == 2) return launch_pers<0>(am, bm, maps, d, grid, st);
  if (MT == 2) return BN == 256 ? launch_bn<256, 2>(am, bm, maps, d, grid, st) : launch_bn<128, 2>(am, bm, maps, d, grid, st);
  return BN == 256 ? launch_bn<256, 1>(am, bm, maps, d, grid, st) : launch_bn<128, 1>(am, bm, maps, d, grid, st);
}

}  // namespace jolt

using namespace jolt;

extern "C" jolt_status jolt_gemm_bf16(const void* A, int32_t a_mn_major, const void* B,
                                      int32_t b_mn_major, float* C, int32_t M, int32_t N, int32_t K,
                                      int64_t lda, int64_t ldb, int64_t ldc, int32_t batch,
                                      int64_t stride_a, int64_t stride_b, int64_t stride_c,
                                      int32_t k_split, int32_t accumulate, int32_t plan, void* stream) {
  if (M < 0 || N < 0 || K < 0 || batch < 1 || k_split < 1) return JOLT_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return JOLT_OK;
  if (!A || !B || !C || ldc < N) return JOLT_ERR_INVALID_ARG;
  if (K == 0) return JOLT_OK;
  GemmCall g;
  g.M = M; g.N = N; g.K = K;
  Operand& a = g.A[0];
  a.ptr = A; a.major = a_mn_major ? kMajorMN : kMajorK;
  a.inner = a_mn_major ? M : K; a.outer = a_mn_major ? K : M; a.outer_stride = lda;
  a.batch = batch; a.batch_stride = stride_a;
  Operand& b = g.B[0];
  b.ptr = B; b.major = b_mn_major ? kMajorMN : kMajorK;
  b.inner = b_mn_major ? N : K; b.outer = b_mn_major ? K : N; b.outer_stride = ldb;
  b.batch = batch; b.batch_stride = stride_b;
  if (lda < a.inner || ldb < b.inner) return JOLT_ERR_INVALID_ARG;
  g.C = C; g.ldc = ldc; g.c_batch_stride = stride_c; g.batch = batch;
  g.k_split = k_split; g.accumulate = accumulate != 0;
  if (plan < JOLT_GEMM_DEFAULT || plan > JOLT_GEMM_PAIRS) return JOLT_ERR_INVALID_ARG;
  g.plan = plan;
  if (k_split > 1 && !accumulate) return JOLT_ERR_INVALID_ARG;
  return gemm_tc(g, static_cast<cudaStream_t>(stream));
}

extern "C" jolt_status jolt_gemm_bf16_hilo(const void* A, int32_t a_mn_major, const void* B,
                                           int32_t b_mn_major, void* Ch, void* Cl, int32_t M, int32_t N,
                                           int32_t K, int64_t lda, int64_t ldb, int64_t ldc, int32_t batch,
                                           int64_t stride_a, int64_t stride_b, int64_t stride_c,
                                           void* stream) {
  if (M < 0 || N < 0 || K < 0 || batch < 1) return JOLT_ERR_INVALID_ARG;
  if (M == 0 || N == 0) return JOLT_OK;
  if (!A || !B || !Ch || ldc < N || K == 0) return JOLT_ERR_INVALID_ARG;
  GemmCall g;
  g.M = M; g.N = N; g.K = K;
  Operand& a = g.A[0];
  a.ptr = A; a.major = a_mn_major ? kMajorMN : kMajorK;
  a.inner = a_mn_major ? M : K; a.outer = a_mn_major ? K : M; a.outer_stride = lda;
  a.batch = batch; a.batch_stride = stride_a;
  Operand& b = g.B[0];
  b.ptr = B; b.major = b_mn_major ? kMajorMN : kMajorK;
  b.inner = b_mn_major ? N : K; b.outer = b_mn_major ? K : N; b.outer_stride = ldb;
  b.batch = batch; b.batch_stride = stride_b;
  if (lda < a.inner || ldb < b.inner) return JOLT_ERR_INVALID_ARG;
  g.Ch = static_cast<__nv_bfloat16*>(Ch);
  g.Cl = static_cast<__nv_bfloat16*>(Cl);
  g.ldc = ldc; g.c_batch_stride = stride_c; g.batch = batch;
  g.k_split = 1;
  return gemm_tc(g, static_cast<cudaStream_t>(stream));
}

extern "C" jolt_status jolt_gemm_bf16_residual(const void* A, const void* B, int32_t M, int32_t K, int64_t lda,
                                               int64_t ldb, int32_t batch, int64_t stride_a, int64_t stride_b,
                                               const void* X, int32_t x_f32, uint64_t seed, int32_t b,
                                               uint8_t* codes, void* sz, int32_t* err, void* stream) {
  if (M < 0 || K < 1 || batch < 1) return JOLT_ERR_INVALID_ARG;
  if (M == 0) return JOLT_OK;
  if (!A || !B || !X || !codes || !sz || lda < K || ldb < 128) return JOLT_ERR_INVALID_ARG;
  GemmCall g;
  g.M = M; g.N = 128; g.K = K;
  Operand& a = g.A[0];
  a.ptr = A; a.major = kMajorK; a.inner = K; a.outer = M; a.outer_stride = lda;
  a.batch = batch; a.batch_stride = stride_a;
  Operand& bo = g.B[0];
  bo.ptr = B; bo.major = kMajorMN; bo.inner = 128; bo.outer = K; bo.outer_stride = ldb;
  bo.batch = batch; bo.batch_stride = stride_b;
  ResidualEpi e;
  e.X = X; e.x_f32 = x_f32 ? 1 : 0; e.T = M; e.seed = seed; e.b = b; e.codes = codes; e.sz = sz;
  g.res = &e;
  g.batch = batch;
  g.err = err;
  return gemm_tc(g, static_cast<cudaStream_t>(stream));
}
