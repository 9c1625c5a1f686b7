// Batched small dense linear algebra used by the compressor (l x l and d_h x d_h problems).
#pragma once
#include "common.cuh"

namespace jolt {

// Blocked upper Cholesky of (G + shift*I) in fp64, G fp32 [nb][n][ld_g] symmetric, followed by the
// triangular inverse. shift = shift_rel * ||G||_F per matrix. Outputs R^{-1} split into bf16
// hi/lo parts [nb][n][n] (ready as a GEMM operand). Scratch: chol_scratch_bytes(nb, n).
// min_ratio (host, may be null; synchronises): the smallest pivot ratio R_jj^2 / (G_jj + shift)
// over the batch — 0 when a pivot was not positive (the factor is then unusable), near 1 for a
// well-conditioned G.
size_t chol_scratch_bytes(int nb, int n);
jolt_status chol_inverse(const float* G, int64_t ld_g, int nb, int n, double shift_rel,
                         __nv_bfloat16* rinv_hi, __nv_bfloat16* rinv_lo, void* scratch,
                         int32_t* err, cudaStream_t st, float* min_ratio = nullptr);

// Symmetric eigendecomposition by block Jacobi (fp32), nb matrices A fp32 [nb][n][ld_a].
// Outputs eigenvalues descending (fp32 [nb][n]) and eigenvectors as columns of V fp32 [nb][n][n]
// in the same order. Scratch: jacobi_scratch_bytes(nb, n).
size_t jacobi_scratch_bytes(int nb, int n);
jolt_status jacobi_eig(const float* A, int64_t ld_a, int nb, int n, float* evals, float* evecs,
                       void* scratch, int max_sweeps, double tol, int32_t* err, cudaStream_t st);

// Same solver with fp64 input and outputs (A [nb][n][ld_a] fp64).
jolt_status jacobi_eig64(const double* A, int64_t ld_a, int nb, int n, double* evals, double* evecs,
                         void* scratch, int max_sweeps, double tol, int32_t* err, cudaStream_t st);

// fp32 -> (hi, lo) bf16 with hi = bf16(x), lo = bf16(x - hi); rows x cols with leading dims.
jolt_status split_bf16(const float* x, int64_t ldx, int64_t rows, int64_t cols, int batch,
                       int64_t bstride_x, __nv_bfloat16* hi, __nv_bfloat16* lo, int64_t ldo,
                       int64_t bstride_o, cudaStream_t st);

// fp32 -> three bf16 parts x ~ hi + mid + lo (about 24 significant bits), same layout rules.
jolt_status split3_bf16(const float* x, int64_t n, __nv_bfloat16* hi, __nv_bfloat16* mid, __nv_bfloat16* lo,
                        cudaStream_t st);

}  // namespace jolt
