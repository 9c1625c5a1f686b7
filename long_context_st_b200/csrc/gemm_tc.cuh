// Host interface of the tcgen05 GEMM: C[z] (+)= sum_t A_t[z] * B_t[z], bf16 operands in global
// memory described by TMA tensor maps, fp32 accumulation in TMEM, fp32 output.
#pragma once
#include <cuda.h>
#include <cuda_bf16.h>

#include "common.cuh"

namespace jolt {

enum Major { kMajorK = 0, kMajorMN = 1 };

// One bf16 operand. Logical matrix A[mn][k] (or B[k][mn]); `major` says which index is
// contiguous in memory. The contiguous ("inner") index may be folded: inner = fold_index * fold +
// r (0 <= r < fold), where consecutive folds are `fold_stride` elements apart — this is how the
// token unfolding X_(T)[t][(l,h,j)] of a [L_g*n_kv][T][d_h] cell is addressed without a copy.
struct Operand {
  const void* ptr = nullptr;  // bf16
  int major = kMajorK;
  int64_t inner = 0;          // extent of the contiguous index (fold length when folded)
  int64_t outer = 0;          // extent of the other index
  int64_t outer_stride = 0;   // elements between consecutive outer indices
  int64_t fold = 0;           // 0: not folded
  int64_t nfold = 1;          // number of folds
  int64_t fold_stride = 0;    // elements between folds
  int64_t batch = 1;
  int64_t batch_stride = 0;   // elements between batch entries
};

constexpr int kMaxTerms = 6;

// Fused residual coding: with N = 128 output columns (the features of one token row), each
// output row x~ = C[z][t][:] is not stored; the epilogue forms x = X[z*T + t][:] - x~, rotates it by
// (1/sqrt(128)) H diag(s) (s the seeded signs), quantises it per row to b bits (fp16 scale and
// zero) and packs the codes, exactly as the stand-alone residual coder does.
struct ResidualEpi {
  const void* X = nullptr;   // [batch][T][128] input rows (bf16, or fp32 when x_f32)
  int x_f32 = 0;
  int64_t T = 0;             // rows per batch entry (= M)
  uint64_t seed = 0;         // rotation sign seed
  int b = 0;                 // 2, 4 or 8
  uint8_t* codes = nullptr;  // [batch*T][128*b/8], 16-byte aligned
  void* sz = nullptr;        // __half2 [batch*T]: (scale, zero)
};

struct GemmCall {
  int M = 0, N = 0, K = 0;
  int n_terms = 1;
  Operand A[kMaxTerms], B[kMaxTerms];
  float* C = nullptr;
  // Instead of fp32 C (C = nullptr): the bf16 rounding of each result to Ch and, when Cl is given,
  // the bf16 rounding of the remainder to Cl (the hi/lo split of the fp32 result), with C's
  // ldc / batch layout. Requires accumulate = false and no split-K.
  __nv_bfloat16* Ch = nullptr;
  __nv_bfloat16* Cl = nullptr;
  int64_t ldc = 0;
  int64_t c_batch_stride = 0;  // elements between C batch entries
  int c_batch_div = 1;         // C entry of operand batch z is z / c_batch_div
  int batch = 1;               // operand batch entries (grid z)
  int k_split = 1;             // split-K factor; 0 = chosen to fill whole waves; != 1 (or
                               // c_batch_div > 1) requires accumulate
  bool accumulate = false;     // atomically add into C instead of storing
  bool c_upper = false;        // only C[m][n] with m <= n is wanted: skip tiles entirely below the diagonal
  bool b_upper = false;        // B[k][n] = 0 for k > n (upper triangular): K stops at the tile's last column
  const ResidualEpi* res = nullptr;  // fused residual coding instead of any C output (see above)
  int plan = 0;                // jolt_gemm_plan: kernel form (0 = the tile planner's default)
  int32_t* err = nullptr;
};

// TMA tensor map (bf16, 128-byte swizzle) for an operand: box = 64 contiguous elements x `rows`
// (K-major) or 64 x 64 (MN-major). False if the driver rejects it or the pointer is misaligned.
bool make_tensor_map(CUtensorMap* m, const Operand& o, int rows);

// TMA tensor map that loads `chunks` 64-wide MN chunks x 64 k rows of `terms` equally spaced
// MN-major bf16 operands in one copy: dims (64, K, chunks, batch, terms), element strides
// (ld, 64, batch_stride, term_stride), box (64, 64, chunks, 1, terms), 128-byte swizzle; the
// shared-memory tile is [term][chunk][64 k rows][64]. False if the driver rejects the layout.
bool make_tensor_map_mn_chunks(CUtensorMap* m, const void* ptr, int64_t K, int64_t ld, int chunks, int64_t batch,
                               int64_t batch_stride, int terms, int64_t term_stride);

// Launch; validates shapes and alignment (JOLT_ERR_INVALID_ARG) before any launch.
jolt_status gemm_tc(const GemmCall& g, cudaStream_t st);

}  // namespace jolt
