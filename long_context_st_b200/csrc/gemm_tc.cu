// tcgen05 GEMM for sm_100a: TMA (128-byte swizzle) streams bf16 A/B tiles into a ring of shared-
// memory stages; one thread issues tcgen05.mma (M=128, N=BN, K=16) into a TMEM accumulator; four
// warps drain TMEM with tcgen05.ld and store (or atomically add) fp32 C with coalesced writes.
//
// Warp roles (128 threads): warp 0 lane 0 = TMA producer, warp 1 lane 0 = MMA issuer, warp 2 =
// TMEM allocator; all four warps run the epilogue. Every mbarrier wait is bounded (2 s) and
// reports JOLT_ERR_TIMEOUT instead of hanging.
//
// Several (A_t, B_t) "terms" can accumulate into one tile: a fp32 operand split as hi + lo bf16
// parts gives x*y ~ hi*hi + hi*lo + lo*hi with ~2^-16 relative error at bf16 tensor-core speed.
#include <dlfcn.h>

#include <algorithm>
#include <cstdio>
#include <cstdlib>
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
  int a_batch[kMaxTerms], b_batch[kMaxTerms];  // operand batch extents (coordinate = z % extent)
  float* C;
  int64_t ldc, c_bstride;
  int c_div, accumulate, c_upper, b_upper;
  int32_t* err;
};

// MT: 128-row M tiles per CTA; with MT = 2 two accumulators share every B tile (half the B
// bytes per flop, and each stage covers twice the MMA time).
template <int BN, int MT>
struct Cfg {
  static constexpr int kABytes1 = BM * BK * 2;
  static constexpr int kABytes = MT * kABytes1;
  static constexpr int kBBytes = BN * BK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes;
  static constexpr int kStages = (192 * 1024) / kStageBytes < 6 ? (192 * 1024) / kStageBytes : 6;
  static constexpr int kCols = MT * BN;
  static constexpr int kTmemCols = kCols <= 32 ? 32 : (kCols <= 64 ? 64 : (kCols <= 128 ? 128 : (kCols <= 256 ? 256 : 512)));
  static constexpr int kEpiBytes = 4 * 32 * 33 * 4;
  static constexpr int kSmem = 1024 + kStages * kStageBytes + kEpiBytes + 256;
};

__device__ __forceinline__ void load_operand(const CUtensorMap* map, int major, int fold, int bext,
                                             uint32_t dst, uint32_t bar, int mn0, int rows, int k0,
                                             int z) {
  const int zb = bext > 1 ? z % bext : 0;
  if (major == kMajorK) {
    if (fold) sm100::tma_load_4d(dst, map, bar, k0 % fold, mn0, k0 / fold, zb);
    else sm100::tma_load_3d(dst, map, bar, k0, mn0, zb);
  } else {
    for (int i = 0; i < rows / 64; ++i) {
      const int mn = mn0 + 64 * i;
      const uint32_t d = dst + i * (64 * BK * 2);
      if (fold) sm100::tma_load_4d(d, map, bar, mn % fold, k0, mn / fold, zb);
      else sm100::tma_load_3d(d, map, bar, mn, k0, zb);
    }
  }
}

template <int BN, int AMAJ, int BMAJ, int MT>
__global__ void __launch_bounds__(128, 1) k_gemm(const __grid_constant__ TmaPack maps, GemmDev p) {
  using C = Cfg<BN, MT>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  float* epi = reinterpret_cast<float*>(smem + C::kStages * C::kStageBytes);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::kStages * C::kStageBytes + C::kEpiBytes);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * C::kStages + 1);

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
  sm100::tc_fence_before();
  __syncthreads();
  sm100::tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  const uint32_t smem_base = sm100::smem_u32(smem);

  if (n_iters > 0) {
    if (warp == 0 && lane == 0) {
      // ---- TMA producer ----
      for (int it = 0; it < n_iters; ++it) {
        const int s = it % C::kStages;
        const uint32_t ph = (it / C::kStages) & 1;
        if (!sm100::mbar_wait(empty_bar(s), ph ^ 1, p.err)) break;
        const int t = it / nkb, kb = it % nkb;
        const int k0 = (kb_begin + kb) * BK;
        const uint32_t sa = smem_base + s * C::kStageBytes;
        const uint32_t sb = sa + C::kABytes;
        sm100::mbar_expect_tx(full_bar(s), C::kStageBytes);
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
          load_operand(&maps.a[t], AMAJ, p.a_fold[t], p.a_batch[t], sa + mt * C::kABytes1, full_bar(s), m0 + mt * BM,
                       BM, k0, z);
        load_operand(&maps.b[t], BMAJ, p.b_fold[t], p.b_batch[t], sb, full_bar(s), n0, BN, k0, z);
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
    const bool ok = sm100::mbar_wait(done_bar, 0, p.err);
    sm100::tc_fence_after();
    if (ok) {
      float* st = epi + warp * 32 * 33;
      float* Cz = p.C + int64_t(z / p.c_div) * p.c_bstride;
      for (int cc = 0; cc < MT * BN; cc += 32) {
        const int mt = cc / BN, c0 = cc % BN;
        uint32_t r[32];
        sm100::tmem_ld32(tmem + (uint32_t(warp * 32) << 16) + cc, r);
        sm100::tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) st[lane * 33 + i] = __uint_as_float(r[i]);
        __syncwarp();
        const int col = n0 + c0 + lane;
#pragma unroll 4
        for (int i = 0; i < 32; ++i) {
          const int row = m0 + mt * BM + warp * 32 + i;
          if (row < p.M && col < p.N) {
            float* dst = Cz + int64_t(row) * p.ldc + col;
            const float v = st[i * 33 + lane];
            if (p.accumulate) atomicAdd(dst, v);
            else *dst = v;
          }
        }
        __syncwarp();
      }
    }
  }
  sm100::tc_fence_before();
  __syncthreads();
  if (warp == 2) sm100::tmem_dealloc(tmem, C::kTmemCols);
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
  if (r != CUDA_SUCCESS && std::getenv("JOLT_DEBUG")) {
    std::fprintf(stderr, "jolt: tensor map rejected (CUresult %d) rank %d dims", int(r), rank);
    for (int i = 0; i < rank; ++i) std::fprintf(stderr, " %llu", (unsigned long long)dims[i]);
    std::fprintf(stderr, " box");
    for (int i = 0; i < rank; ++i) std::fprintf(stderr, " %u", box[i]);
    std::fprintf(stderr, "\n");
  }
  return r == CUDA_SUCCESS;
}

namespace {

// Tile plan: 128-row tiles per CTA (MT) and split-K factor. Estimated time = whole waves of one
// CTA per SM x the k-blocks one CTA runs (+1 for its epilogue), with two-accumulator CTAs ~1.2x
// faster per flop (measured); tiles a symmetric (c_upper) output skips are not counted.
struct TilePlan {
  int MT, k_split;
};

TilePlan plan_tiles(const GemmCall& g, int BN) {
  constexpr int kSMs = 148;
  const int64_t ntile = (g.N + BN - 1) / BN, kb = (g.K + BK - 1) / BK;
  auto active = [&](int MT) {
    const int64_t mt = (g.M + BM * MT - 1) / (BM * MT);
    int64_t a = 0;
    for (int64_t i = 0; i < mt; ++i)
      for (int64_t j = 0; j < ntile; ++j) a += (g.c_upper && i * BM * MT >= j * BN + BN) ? 0 : 1;
    return a * g.batch;
  };
  const int kmax = g.k_split == 0 ? int(std::max<int64_t>(1, std::min<int64_t>(64, kb / 2))) : g.k_split;
  const int kmin = g.k_split == 0 ? 1 : g.k_split;
  TilePlan best{1, kmin};
  double best_t = 1e300;
  for (int MT = 2; MT >= 1; --MT) {
    if (MT == 2 && g.M <= BM) continue;
    const int64_t act = active(MT);
    for (int k = kmin; k <= kmax; ++k) {
      const int64_t ctas = act * k;
      const double waves = double((ctas + kSMs - 1) / kSMs);
      const double t = waves * MT * (double((kb + k - 1) / k) + 1.0) / (MT == 2 ? 1.2 : 1.0);
      if (t < best_t * 0.999) {
        best_t = t;
        best = TilePlan{MT, k};
      }
    }
  }
  return best;
}

}  // namespace

jolt_status gemm_tc(const GemmCall& g, cudaStream_t st) {
  if (g.M <= 0 || g.N <= 0 || g.K <= 0) return JOLT_OK;
  if (g.n_terms < 1 || g.n_terms > kMaxTerms || !g.C || g.batch < 1 || g.k_split < 0 || g.c_batch_div < 1)
    return JOLT_ERR_INVALID_ARG;
  if ((g.k_split != 1 || g.c_batch_div > 1) && !g.accumulate) return JOLT_ERR_INVALID_ARG;
  const int am = g.A[0].major, bm = g.B[0].major;
  for (int t = 0; t < g.n_terms; ++t)
    if (g.A[t].major != am || g.B[t].major != bm) return JOLT_ERR_INVALID_ARG;
  // BN: 256 whenever N exceeds one 128-wide tile — a 128 x 256 tile runs ~1.5x more flops per
  // cycle than 128 x 128 (half the operand bytes per flop), which outweighs the padding of N
  const int BN = g.N > 128 ? 256 : 128;
  TmaPack maps;
  memset(&maps, 0, sizeof(maps));
  GemmDev d{};
  for (int t = 0; t < g.n_terms; ++t) {
    if (!make_tensor_map(&maps.a[t], g.A[t], BM)) return JOLT_ERR_INVALID_ARG;
    if (!make_tensor_map(&maps.b[t], g.B[t], BN)) return JOLT_ERR_INVALID_ARG;
    d.a_fold[t] = int(g.A[t].fold);
    d.b_fold[t] = int(g.B[t].fold);
    d.a_batch[t] = g.A[t].batch_stride ? int(g.A[t].batch) : 1;
    d.b_batch[t] = g.B[t].batch_stride ? int(g.B[t].batch) : 1;
    if ((g.A[t].fold && g.A[t].fold % 64) || (g.B[t].fold && g.B[t].fold % 64)) return JOLT_ERR_INVALID_ARG;
  }
  const TilePlan tp = plan_tiles(g, BN);
  const int MT = tp.MT;
  d.M = g.M; d.N = g.N; d.K = g.K; d.n_terms = g.n_terms; d.k_split = tp.k_split;
  const int nkb = (g.K + BK - 1) / BK;
  d.nkb_split = (nkb + tp.k_split - 1) / tp.k_split;
  d.C = g.C; d.ldc = g.ldc; d.c_bstride = g.c_batch_stride; d.c_div = g.c_batch_div;
  d.accumulate = g.accumulate ? 1 : 0;
  d.c_upper = g.c_upper ? 1 : 0;
  d.b_upper = g.b_upper ? 1 : 0;
  d.err = g.err;
  const int64_t ntile = (g.N + BN - 1) / BN, zc = int64_t(g.batch) * tp.k_split;
  const dim3 grid(unsigned(ntile), unsigned((g.M + BM * MT - 1) / (BM * MT)), unsigned(zc));
  if (grid.y > 65535 || grid.z > 65535) return JOLT_ERR_INVALID_ARG;
  // algorithmic flops: a triangular B or a wanted upper triangle of C halves the product
  const double tri = (g.b_upper || g.c_upper) ? 0.5 : 1.0;
  StatScope sc(JOLT_K_GEMM, st, tri * 2.0 * g.M * double(g.N) * g.K * g.batch * g.n_terms, 0.0);
  if (MT == 2) return BN == 256 ? launch_bn<256, 2>(am, bm, maps, d, grid, st) : launch_bn<128, 2>(am, bm, maps, d, grid, st);
  return BN == 256 ? launch_bn<256, 1>(am, bm, maps, d, grid, st) : launch_bn<128, 1>(am, bm, maps, d, grid, st);
}

}  // namespace jolt

using namespace jolt;

extern "C" jolt_status jolt_gemm_bf16(const void* A, int32_t a_mn_major, const void* B,
                                      int32_t b_mn_major, float* C, int32_t M, int32_t N, int32_t K,
                                      int64_t lda, int64_t ldb, int64_t ldc, int32_t batch,
                                      int64_t stride_a, int64_t stride_b, int64_t stride_c,
                                      int32_t k_split, int32_t accumulate, void* stream) {
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
  if (k_split > 1 && !accumulate) return JOLT_ERR_INVALID_ARG;
  return gemm_tc(g, static_cast<cudaStream_t>(stream));
}
