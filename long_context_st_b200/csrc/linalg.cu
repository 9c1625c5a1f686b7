// Batched small dense linear algebra for the compressor.
//
// chol_inverse: right-looking blocked Cholesky (64-wide blocks, fp64) of G + shift*I, G = R^T R
//   with R upper triangular, then the blocked triangular inverse R^{-1} by block diagonals (the
//   products of one diagonal spread over all CTAs, summed with fp64 atomics). One cooperative
//   launch; block steps are separated by bounded grid barriers, and every step's grid covers all
//   matrices of the batch and all independent blocks.
// jacobi_eig: two-sided block Jacobi (32-wide blocks, tournament ordering, fp64 working storage):
//   each round runs one cyclic sweep on every 64 x 64 pair subproblem in shared memory (writing
//   the rotated diagonal pair-block back), then, in one pass, applies Theta1^T . Theta2 to every
//   off-diagonal pair-block of A and Theta to the block columns of V; sweeps until the
//   off-diagonal norm is below tol.
#include <algorithm>
#include <cstdio>
#include <cstdlib>
#include <vector>

#include "linalg.cuh"
#include "sm100.cuh"
#include "stats.h"

namespace jolt {

namespace {

constexpr int NB = 64;     // Cholesky block
constexpr int JW = 32;     // Jacobi block width (sub-problem is 2*JW)
constexpr int JS = 2 * JW;

inline int rup(int x, int a) { return (x + a - 1) / a * a; }

// Grid-wide barrier for cooperative launches (all blocks co-resident), with a time limit: a block
// that waits more than ~2 s reports JOLT_ERR_TIMEOUT and stops waiting; once the error word is set,
// later barriers do not wait at all, so a failure never hangs the GPU.
struct GridBar {
  unsigned int* count;
  unsigned int* gen;
  int32_t* err;
};

__device__ __forceinline__ void grid_barrier(const GridBar& gb, uint64_t limit_ns = 2000000000ull) {
  __syncthreads();
  if (threadIdx.x == 0) {
    volatile unsigned int* vgen = gb.gen;
    const unsigned int g = *vgen;
    __threadfence();
    const unsigned int arrived = atomicAdd(gb.count, 1u);
    if (arrived == gridDim.x - 1) {
      *gb.count = 0;
      __threadfence();
      atomicAdd(gb.gen, 1u);
    } else {
      uint64_t t0;
      asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t0));
      while (*vgen == g) {
        if (*reinterpret_cast<volatile int32_t*>(gb.err) != 0) break;
        uint64_t t1;
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t1));
        if (t1 - t0 > limit_ns) {
          atomicCAS(gb.err, 0, int32_t(JOLT_ERR_TIMEOUT));
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
  }
  __syncthreads();
}

struct CholScratch {
  double* Gd;    // [nb][np][np]
  double* Xd;    // [nb][np][np]
  double* mdiag; // [nb]
  double* diag0; // [nb][np] diagonal of G + shift
  float* ratio;  // [nb] min pivot ratio
  unsigned int* bar;  // [2] grid barrier count, generation
};

CholScratch chol_carve(void* scratch, int nb, int n) {
  const int np = rup(n, NB);
  CholScratch s;
  uint8_t* p = static_cast<uint8_t*>(scratch);
  s.Gd = reinterpret_cast<double*>(p);
  p += align_up(size_t(nb) * np * np * 8, 256);
  s.Xd = reinterpret_cast<double*>(p);
  p += align_up(size_t(nb) * np * np * 8, 256);
  s.mdiag = reinterpret_cast<double*>(p);
  p += align_up(size_t(nb) * 8, 256);
  s.diag0 = reinterpret_cast<double*>(p);
  p += align_up(size_t(nb) * np * 8, 256);
  s.ratio = reinterpret_cast<float*>(p);
  p += align_up(size_t(nb) * 4, 256);
  s.bar = reinterpret_cast<unsigned int*>(p);
  return s;
}




// 64x64 fp64 tile load (row stride np) into shared memory; a warp reads half a row per access.
__device__ __forceinline__ void tile_load(double (*S)[NB + 1], const double* src, int np) {
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) S[e >> 6][e & 63] = src[int64_t(e >> 6) * np + (e & 63)];
}

// 64x64x64 tile product held in registers: thread (ty, tx) of a 16 x 16 grid owns the strided
// 4 x 4 set C[ty + 16u][tx + 16v] (a warp reads 16 consecutive B elements and broadcasts two A
// elements per step: no shared-memory bank conflicts). TA: C = A^T B when true, else C = A B.
template <bool TA, int LD>
__device__ __forceinline__ void tile_mm(double (&acc)[4][4], const double (*A)[LD], const double (*B)[LD]) {
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll 4
  for (int k = 0; k < NB; ++k) {
    double a[4], bb[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) a[u] = TA ? A[k][ty + 16 * u] : A[ty + 16 * u][k];
#pragma unroll
    for (int v = 0; v < 4; ++v) bb[v] = B[k][tx + 16 * v];
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) acc[u][v] = fma(a[u], bb[v], acc[u][v]);
  }
}

// Factor the diagonal block p of matrix b (right-looking; the trailing update uses the unscaled
// pivot row, S_ic -= S_ji S_jc / d_j, and rows are scaled by 1/sqrt(d_j) at the end), then invert
// the upper-triangular factor row by row from the bottom. Thread t: column t & 63 and row group
// t >> 6 in the factorisation; column t >> 2 and k-residue t & 3 in the inverse.
__device__ void dev_chol_diag(double* __restrict__ Gd, double* __restrict__ Xd, int np, int p,
                              const double* __restrict__ diag0, float* ratio, int b, double* sh) {
  double(*S)[NB + 1] = reinterpret_cast<double(*)[NB + 1]>(sh);
  double(*X)[NB + 1] = reinterpret_cast<double(*)[NB + 1]>(sh + NB * (NB + 1));
  __shared__ double dpiv[NB], pinv[NB], rs[NB];
  double* gd = Gd + int64_t(b) * np * np + int64_t(p) * NB * np + p * NB;
  double* xd = Xd + int64_t(b) * np * np + int64_t(p) * NB * np + p * NB;
  tile_load(S, gd, np);
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) X[e >> 6][e & 63] = 0.0;
  __syncthreads();
  if (threadIdx.x == 0) {
    const double d = S[0][0];
    dpiv[0] = d;
    pinv[0] = d > 0.0 ? 1.0 / d : 1.0;  // breakdown: recorded below, the caller retries with a shift
  }
  __syncthreads();
  {
    const int c = threadIdx.x & 63, rg = threadIdx.x >> 6;
    for (int j = 0; j < NB; ++j) {
      if (c > j) {
        const double f = S[j][c] * pinv[j];
        int i = j + 1 + rg;
        for (; i + 12 <= c; i += 16) {  // four independent read-modify-writes in flight
          const double s0 = S[j][i], s1 = S[j][i + 4], s2 = S[j][i + 8], s3 = S[j][i + 12];
          const double t0 = S[i][c], t1 = S[i + 4][c], t2 = S[i + 8][c], t3 = S[i + 12][c];
          S[i][c] = fma(-s0, f, t0);
          S[i + 4][c] = fma(-s1, f, t1);
          S[i + 8][c] = fma(-s2, f, t2);
          S[i + 12][c] = fma(-s3, f, t3);
        }
        for (; i <= c; i += 4) S[i][c] = fma(-S[j][i], f, S[i][c]);
        // the owner of the next pivot has just finalised it: publish its reciprocal
        if (c == j + 1 && rg == 0) {
          const double d = S[c][c];
          dpiv[c] = d;
          pinv[c] = d > 0.0 ? 1.0 / d : 1.0;
        }
      }
      __syncthreads();
    }
  }
  if (threadIdx.x < NB) {
    const double d = dpiv[threadIdx.x];
    rs[threadIdx.x] = d > 0.0 ? 1.0 / sqrt(d) : 1.0;  // a broken-down pivot becomes 1 (result discarded)
  }
  if (threadIdx.x == 0) {
    float rmin = 1.f;
    for (int j = 0; j < NB; ++j) {
      const double d = dpiv[j], d0 = diag0[int64_t(b) * np + p * NB + j];
      rmin = (d > 0.0 && d0 > 0.0) ? fminf(rmin, float(d / d0)) : 0.f;
    }
    atomicMin(reinterpret_cast<int*>(ratio + b), __float_as_int(rmin));
  }
  __syncthreads();
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    const int i = e >> 6, k = e & 63;
    S[i][k] = (i > k) ? 0.0 : (i == k ? (dpiv[i] > 0.0 ? dpiv[i] * rs[i] : 1.0) : S[i][k] * rs[i]);
  }
  __syncthreads();
  // X = R^-1: X_ic = (delta_ic - sum_{i<k<=c} R_ik X_kc) / R_ii, one barrier per row
  {
    const int c = threadIdx.x >> 2, q = threadIdx.x & 3;
    for (int i = NB - 1; i >= 0; --i) {
      double a0 = 0.0, a1 = 0.0;
      int k = i + 1 + q;
      for (; k + 4 <= c; k += 8) {
        a0 = fma(S[i][k], X[k][c], a0);
        a1 = fma(S[i][k + 4], X[k + 4][c], a1);
      }
      if (k <= c) a0 = fma(S[i][k], X[k][c], a0);
      double a = a0 + a1;
      a += __shfl_xor_sync(0xffffffffu, a, 1);
      a += __shfl_xor_sync(0xffffffffu, a, 2);
      // 1 / R_ii = rs[i] (R_ii = sqrt(d_i), or 1 after a breakdown)
      if (q == 0 && c >= i) X[i][c] = ((c == i ? 1.0 : 0.0) - a) * rs[i];
      __syncthreads();
    }
  }
  for (int e = threadIdx.x; e < NB * NB; e += blockDim.x) {
    gd[int64_t(e >> 6) * np + (e & 63)] = S[e >> 6][e & 63];
    xd[int64_t(e >> 6) * np + (e & 63)] = X[e >> 6][e & 63];
  }
  __syncthreads();
}

// Panel: R_pj = X_pp^T G_pj for j > p, and W_pj = X_pp R_pj (kept in the unused lower block
// (j, p) of Gd for the triangular inverse).
__device__ void dev_chol_panel(double* __restrict__ Gd, const double* __restrict__ Xd, int np, int p, int b,
                               int j, double* sh) {
  double(*A)[NB + 1] = reinterpret_cast<double(*)[NB + 1]>(sh);
  double(*B)[NB + 1] = reinterpret_cast<double(*)[NB + 1]>(sh + NB * (NB + 1));
  const double* xpp = Xd + int64_t(b) * np * np + int64_t(p) * NB * np + p * NB;
  double* gpj = Gd + int64_t(b) * np * np + int64_t(p) * NB * np + j * NB;
  double* wjp = Gd + int64_t(b) * np * np + int64_t(j) * NB * np + p * NB;
  tile_load(A, xpp, np);
  tile_load(B, gpj, np);
  __syncthreads();
  double acc[4][4] = {};
  tile_mm<true, NB + 1>(acc, A, B);
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
  __syncthreads();
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      gpj[int64_t(ty + 16 * u) * np + tx + 16 * v] = acc[u][v];
      B[ty + 16 * u][tx + 16 * v] = acc[u][v];
    }
  __syncthreads();
  double w[4][4] = {};
  tile_mm<false, NB + 1>(w, A, B);
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) wjp[int64_t(ty + 16 * u) * np + tx + 16 * v] = w[u][v];
  __syncthreads();
}

// Trailing update: G_ij -= R_pi^T R_pj for p < i <= j (pair number idx).
__device__ void dev_chol_update(double* __restrict__ Gd, int np, int P, int p, int b, int idx, double* sh) {
  double(*A)[NB + 1] = reinterpret_cast<double(*)[NB + 1]>(sh);
  double(*B)[NB + 1] = reinterpret_cast<double(*)[NB + 1]>(sh + NB * (NB + 1));
  int i = p + 1;
  while (idx >= P - i) {
    idx -= P - i;
    ++i;
  }
  const int j = i + idx;
  double* g = Gd + int64_t(b) * np * np;
  tile_load(A, g + int64_t(p) * NB * np + i * NB, np);
  tile_load(B, g + int64_t(p) * NB * np + j * NB, np);
  __syncthreads();
  double acc[4][4] = {};
  tile_mm<true, NB + 1>(acc, A, B);
  double* gij = g + int64_t(i) * NB * np + j * NB;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) gij[int64_t(ty + 16 * u) * np + tx + 16 * v] -= acc[u][v];
  __syncthreads();
}

// Triangular inverse, block diagonal d: X_ij -= W_ik X_kj for one k in (i, j], j = i + d, with
// W_ik = X_ii R_ik (so X_ij = -X_ii sum_k R_ik X_kj), accumulated with fp64 atomics into the
// still-zero block X_ij.
__device__ void dev_trinv(const double* __restrict__ Gd, double* __restrict__ Xd, int np, int i, int j, int k,
                          int b, double* sh) {
  double(*A)[NB + 1] = reinterpret_cast<double(*)[NB + 1]>(sh);
  double(*B)[NB + 1] = reinterpret_cast<double(*)[NB + 1]>(sh + NB * (NB + 1));
  const double* g = Gd + int64_t(b) * np * np;
  double* x = Xd + int64_t(b) * np * np;
  tile_load(A, g + int64_t(k) * NB * np + i * NB, np);  // W_ik, stored in block (k, i)
  tile_load(B, x + int64_t(k) * NB * np + j * NB, np);
  __syncthreads();
  double acc[4][4] = {};
  tile_mm<false, NB + 1>(acc, A, B);
  double* xij = x + int64_t(i) * NB * np + j * NB;
  const int ty = threadIdx.x >> 4, tx = threadIdx.x & 15;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) atomicAdd(&xij[int64_t(ty + 16 * u) * np + tx + 16 * v], -acc[u][v]);
  __syncthreads();
}

struct CholArgs {
  const float* G;
  int64_t ldg;
  int n, np, P, nb;
  double shift_rel;
  double *Gd, *Xd, *md, *diag0;  // md: sums of squares, zeroed before the launch
  float* ratio;
  __nv_bfloat16 *hi, *lo;
  GridBar bar;
  unsigned long long* stamps;  // optional (diagnostics): globaltimer after each phase, block 0
};

__device__ __forceinline__ void stamp(unsigned long long* st, int& k) {
  if (st && blockIdx.x == 0 && threadIdx.x == 0) {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    st[k] = t;
  }
  ++k;
}

// The whole blocked Cholesky + triangular inverse of nb matrices in one cooperative launch.
__global__ void __launch_bounds__(256) k_chol_coop(CholArgs a) {
  extern __shared__ double sh[];
  const int nbk = gridDim.x;
  int sk = 0;
  if (a.stamps) {  // diagnostics: cost of 100 empty grid barriers, in stamps[4000..4001]
    int s2 = 4000;
    stamp(a.stamps, s2);
    for (int i = 0; i < 100; ++i) grid_barrier(a.bar);
    stamp(a.stamps, s2);
  }
  stamp(a.stamps, sk);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const int64_t gw = int64_t(blockIdx.x) * nw + wid, nwt = int64_t(nbk) * nw;
  // Frobenius norms (a warp per row), pivot ratios reset
  for (int64_t row = gw; row < int64_t(a.nb) * a.n; row += nwt) {
    const int b = int(row / a.n), i = int(row % a.n);
    const float* g = a.G + int64_t(b) * a.n * a.ldg + int64_t(i) * a.ldg;
    double m = 0.0;
    for (int j = i + lane; j < a.n; j += 32) {  // upper triangle, off-diagonal entries twice
      const double v = g[j];
      m = fma(j > i ? 2.0 * v : v, v, m);
    }
    for (int o = 16; o; o >>= 1) m += __shfl_xor_sync(0xffffffffu, m, o);
    if (lane == 0) atomicAdd(a.md + b, m);
  }
  if (blockIdx.x == 0)
    for (int b = threadIdx.x; b < a.nb; b += blockDim.x) a.ratio[b] = 1.f;
  grid_barrier(a.bar);
  // shifted copy into fp64 working storage (padding: identity), X zeroed
  for (int64_t row = gw; row < int64_t(a.nb) * a.np; row += nwt) {
    const int b = int(row / a.np), i = int(row % a.np);
    const double shift = a.shift_rel * sqrt(a.md[b]);
    const float* g = a.G + int64_t(b) * a.n * a.ldg + int64_t(i) * a.ldg;
    double* gd = a.Gd + row * a.np;
    double* xd = a.Xd + row * a.np;
    for (int j = lane; j < a.np; j += 32) {
      double v;
      if (i < a.n && j < a.n)  // symmetric input: only its upper triangle is read
        v = double(j >= i ? g[j] : a.G[int64_t(b) * a.n * a.ldg + int64_t(j) * a.ldg + i]) + (i == j ? shift : 0.0);
      else v = (i == j) ? 1.0 : 0.0;
      gd[j] = v;
      xd[j] = 0.0;
      if (i == j) a.diag0[int64_t(b) * a.np + i] = v;
    }
  }
  grid_barrier(a.bar);
  stamp(a.stamps, sk);
  // block 0's diagonal factor, then per step: panel, and the trailing update in which the CTA that
  // updates block (p+1, p+1) (its last update) factors it right away
  for (int b = blockIdx.x; b < a.nb; b += nbk) dev_chol_diag(a.Gd, a.Xd, a.np, 0, a.diag0, a.ratio, b, sh);
  grid_barrier(a.bar);
  stamp(a.stamps, sk);
  for (int p = 0; p + 1 < a.P; ++p) {
    const int np1 = a.P - p - 1;
    for (int it = blockIdx.x; it < a.nb * np1; it += nbk) dev_chol_panel(a.Gd, a.Xd, a.np, p, it / np1, p + 1 + it % np1, sh);
    grid_barrier(a.bar);
    stamp(a.stamps, sk);
    const int npairs = np1 * (np1 + 1) / 2;
    for (int it = blockIdx.x; it < a.nb * npairs; it += nbk) {
      const int b = it / npairs, w = it % npairs;
      dev_chol_update(a.Gd, a.np, a.P, p, b, w, sh);
      if (w == 0) dev_chol_diag(a.Gd, a.Xd, a.np, p + 1, a.diag0, a.ratio, b, sh);
    }
    grid_barrier(a.bar);
    stamp(a.stamps, sk);
  }
  // X = R^-1 by block diagonals
  for (int d = 1; d < a.P; ++d) {
    const int cnt = a.P - d;  // blocks on the diagonal
    const int items = a.nb * cnt * d;
    for (int it = blockIdx.x; it < items; it += nbk) {
      const int b = it / (cnt * d), r = it % (cnt * d);
      const int i = r / d, k = i + 1 + r % d;
      dev_trinv(a.Gd, a.Xd, a.np, i, i + d, k, b, sh);
    }
    grid_barrier(a.bar);
    stamp(a.stamps, sk);
  }
  // R^-1 (upper triangle) as bf16 hi + lo, a warp per row
  for (int64_t row = gw; row < int64_t(a.nb) * a.n; row += nwt) {
    const int b = int(row / a.n), i = int(row % a.n);
    const double* x = a.Xd + (int64_t(b) * a.np + i) * a.np;
    for (int j = lane; j < a.n; j += 32) {
      const float v = (i <= j) ? float(x[j]) : 0.f;
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      a.hi[row * a.n + j] = h;
      a.lo[row * a.n + j] = __float2bfloat16_rn(v - __bfloat162float(h));
    }
  }
  stamp(a.stamps, sk);
}


// ---- block Jacobi (fp64 working precision) -----------------------------------------------------

constexpr int kJacMaxSweeps = 40;

struct JacScratch {
  double* A;     // [nb][np][np]
  double* V;     // [nb][np][np]
  double* Th;    // [nb][npair][JS][JS]
  double* norms; // [kJacMaxSweeps][nb][2] off^2, total^2
  int* perm;     // [nb][np]
  int* skip;     // [nb][npair] this round's pair was already diagonal (rotation = identity)
  unsigned int* bar;  // [2] grid barrier count, generation
  int* sweeps;   // [1]
};

JacScratch jac_carve(void* scratch, int nb, int n) {
  const int np = rup(n, JS);
  const int npair = np / JS;
  JacScratch s;
  uint8_t* p = static_cast<uint8_t*>(scratch);
  s.A = reinterpret_cast<double*>(p); p += align_up(size_t(nb) * np * np * 8, 256);
  s.V = reinterpret_cast<double*>(p); p += align_up(size_t(nb) * np * np * 8, 256);
  s.Th = reinterpret_cast<double*>(p); p += align_up(size_t(nb) * npair * JS * JS * 8, 256);
  s.norms = reinterpret_cast<double*>(p); p += align_up(size_t(kJacMaxSweeps) * nb * 16, 256);
  s.perm = reinterpret_cast<int*>(p); p += align_up(size_t(nb) * np * 4, 256);
  s.skip = reinterpret_cast<int*>(p); p += align_up(size_t(nb) * npair * 4, 256);
  s.bar = reinterpret_cast<unsigned int*>(p); p += 256;
  s.sweeps = reinterpret_cast<int*>(p);
  return s;
}

template <typename TA>
__global__ void k_jac_init(const TA* __restrict__ A, int64_t lda, int n, int np, double* __restrict__ Aw,
                           double* __restrict__ V) {
  const int b = blockIdx.y;
  const int64_t total = int64_t(np) * np;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += int64_t(gridDim.x) * blockDim.x) {
    const int i = int(e / np), j = int(e % np);
    double v;
    if (i < n && j < n)
      v = double(i <= j ? A[int64_t(b) * n * lda + int64_t(i) * lda + j] : A[int64_t(b) * n * lda + int64_t(j) * lda + i]);
    else v = (i == j) ? -1.0 : 0.0;
    Aw[int64_t(b) * total + e] = v;
    V[int64_t(b) * total + e] = (i == j) ? 1.0 : 0.0;
  }
}

// tournament (circle method) pairing of m players in round r: pair k -> (first, second)
__host__ __device__ __forceinline__ void tour_pair(int m, int r, int k, int* a, int* b) {
  auto pos = [&](int x) { return x == 0 ? 0 : ((x - 1 + r) % (m - 1)) + 1; };
  *a = pos(k);
  *b = pos(m - 1 - k);
}

typedef double Tile[JS][JS + 1];

// thr: off-diagonal mass of the 64 x 64 subproblem at or below which the pair is left as it is
// (its rotation recorded as the identity); negative in the first sweep.
__device__ void dev_jac_solve(double* __restrict__ Aw, int np, int nblk, int round, double* __restrict__ Th,
                              int* __restrict__ skip, double thr, int b, int k, double* jsm) {
  Tile& S = *reinterpret_cast<Tile*>(jsm);
  Tile& Q = *reinterpret_cast<Tile*>(jsm + JS * (JS + 1));
  __shared__ double cs[JW], sn[JW];
  __shared__ int pp[JW], qq[JW];
  __shared__ double red[8];
  __shared__ int s_skip;
  const int npair = nblk / 2;
  int I, J;
  tour_pair(nblk, round, k, &I, &J);
  double* a = Aw + int64_t(b) * np * np;
  for (int e = threadIdx.x; e < JS * JS; e += blockDim.x) {
    const int u = e / JS, v = e % JS;
    const int gu = (u < JW ? I * JW + u : J * JW + u - JW);
    const int gv = (v < JW ? I * JW + v : J * JW + v - JW);
    S[u][v] = a[int64_t(gu) * np + gv];
    Q[u][v] = (u == v) ? 1.0 : 0.0;
  }
  __syncthreads();
  {
    double off = 0.0;
    for (int e = threadIdx.x; e < JS * JS; e += blockDim.x)
      if (e / JS != e % JS) off = fma(S[e / JS][e % JS], S[e / JS][e % JS], off);
    for (int m = 16; m; m >>= 1) off += __shfl_xor_sync(0xffffffffu, off, m);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = off;
    __syncthreads();
    if (threadIdx.x == 0) {
      double t = 0.0;
      for (int w = 0; w < int(blockDim.x >> 5); ++w) t += red[w];
      s_skip = (thr >= 0.0 && t <= thr) ? 1 : 0;
    }
    __syncthreads();
  }
  double* th = Th + (int64_t(b) * npair + k) * JS * JS;
  if (s_skip) {
    for (int e = threadIdx.x; e < JS * JS; e += blockDim.x) th[e] = (e / JS == e % JS) ? 1.0 : 0.0;
    if (threadIdx.x == 0) skip[b * npair + k] = 1;
    __syncthreads();
    return;
  }
  if (threadIdx.x == 0) skip[b * npair + k] = 0;
  for (int r = 0; r < JS - 1; ++r) {
    if (threadIdx.x < JW) {
      int p, q;
      tour_pair(JS, r, threadIdx.x, &p, &q);
      if (p > q) { const int t = p; p = q; q = t; }
      const double apq = S[p][q], app = S[p][p], aqq = S[q][q];
      double c = 1.0, s = 0.0;
      // Rotation angle in fp32 (tan t of the annihilating angle, small-angle form for huge
      // cot 2phi), then (c, s) renormalised in fp64 by one Newton step of 1/sqrt(c^2 + s^2) so the
      // rotation is orthogonal to fp64 rounding; an fp32 angle only leaves ~1e-7 of a_pq behind,
      // which later rotations remove. (The fp64 divide/sqrt chain was the solve's critical path.)
      const float af = float(apq);
      if (af != 0.f) {
        const float th = float(aqq - app) / (2.f * af);
        const float at = fabsf(th);
        const float tt = at > 1e18f ? 0.5f / at : 1.f / (at + sqrtf(fmaf(at, at, 1.f)));
        const float t = th >= 0.f ? tt : -tt;
        const float c32 = rsqrtf(fmaf(t, t, 1.f));
        const double cd = c32, sd = double(t * c32);
        const double corr = 1.5 - 0.5 * fma(cd, cd, sd * sd);
        c = cd * corr;
        s = sd * corr;
      }
      cs[threadIdx.x] = c; sn[threadIdx.x] = s; pp[threadIdx.x] = p; qq[threadIdx.x] = q;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < JW * JS; e += blockDim.x) {  // rows p, q
      const int kk = e / JS, m = e % JS;
      const int p = pp[kk], q = qq[kk];
      const double c = cs[kk], s = sn[kk];
      const double xp = S[p][m], xq = S[q][m];
      S[p][m] = c * xp - s * xq;
      S[q][m] = s * xp + c * xq;
    }
    __syncthreads();
    for (int e = threadIdx.x; e < JW * JS; e += blockDim.x) {  // columns p, q of S and Q
      const int kk = e / JS, m = e % JS;
      const int p = pp[kk], q = qq[kk];
      const double c = cs[kk], s = sn[kk];
      const double xp = S[m][p], xq = S[m][q];
      S[m][p] = c * xp - s * xq;
      S[m][q] = s * xp + c * xq;
      const double yp = Q[m][p], yq = Q[m][q];
      Q[m][p] = c * yp - s * yq;
      Q[m][q] = s * yp + c * yq;
    }
    __syncthreads();
  }
  // the pair's diagonal block is now Theta^T S Theta: write it back (pairs of a round are disjoint)
  for (int e = threadIdx.x; e < JS * JS; e += blockDim.x) {
    const int u = e / JS, v = e % JS;
    const int gu = (u < JW ? I * JW + u : J * JW + u - JW);
    const int gv = (v < JW ? I * JW + v : J * JW + v - JW);
    th[e] = Q[u][v];
    a[int64_t(gu) * np + gv] = S[u][v];
  }
  __syncthreads();
}

// Off-diagonal pair-block (k1 < k2) of A: A[R1, C2] <- Theta1^T A[R1, C2] Theta2 and its mirror
// A[C2, R1] <- the transpose (R1, C2: the 64 indices of pairs k1 and k2 in this round).
__device__ void dev_jac_off(double* __restrict__ Aw, int np, int nblk, int round, const double* __restrict__ Th,
                            const int* __restrict__ skip, int b, int idx, double* jsm) {
  Tile& X = *reinterpret_cast<Tile*>(jsm);
  Tile& T1 = *reinterpret_cast<Tile*>(jsm + JS * (JS + 1));
  Tile& T2 = *reinterpret_cast<Tile*>(jsm + 2 * JS * (JS + 1));
  const int npair = nblk / 2;
  int k1 = 0;
  while (idx >= npair - 1 - k1) {
    idx -= npair - 1 - k1;
    ++k1;
  }
  const int k2 = k1 + 1 + idx;
  if (skip[b * npair + k1] && skip[b * npair + k2]) return;  // both rotations are the identity
  int I1, J1, I2, J2;
  tour_pair(nblk, round, k1, &I1, &J1);
  tour_pair(nblk, round, k2, &I2, &J2);
  double* a = Aw + int64_t(b) * np * np;
  const double* th1 = Th + (int64_t(b) * npair + k1) * JS * JS;
  const double* th2 = Th + (int64_t(b) * npair + k2) * JS * JS;
  for (int e = threadIdx.x; e < JS * JS; e += blockDim.x) {
    const int u = e / JS, v = e % JS;
    const int gu = (u < JW ? I1 * JW + u : J1 * JW + u - JW);
    const int gv = (v < JW ? I2 * JW + v : J2 * JW + v - JW);
    X[u][v] = a[int64_t(gu) * np + gv];
    T1[u][v] = th1[e];
    T2[u][v] = th2[e];
  }
  __syncthreads();
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[4][4] = {};
  tile_mm<true, JS + 1>(acc, T1, X);  // Z = Theta1^T X
  __syncthreads();
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) X[ty + 16 * u][tx + 16 * v] = acc[u][v];
  __syncthreads();
  double y[4][4] = {};
  tile_mm<false, JS + 1>(y, X, T2);   // Y = Z Theta2
  __syncthreads();
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int row = ty + 16 * u;
    const int gu = (row < JW ? I1 * JW + row : J1 * JW + row - JW);
#pragma unroll
    for (int v = 0; v < 4; ++v) {
      const int col = tx + 16 * v;
      const int gv = (col < JW ? I2 * JW + col : J2 * JW + col - JW);
      a[int64_t(gu) * np + gv] = y[u][v];
      X[row][col] = y[u][v];
    }
  }
  __syncthreads();
  for (int e = threadIdx.x; e < JS * JS; e += blockDim.x) {  // mirror, coalesced along R1
    const int r = e / JS, c = e % JS;
    const int gr = (r < JW ? I2 * JW + r : J2 * JW + r - JW);
    const int gc = (c < JW ? I1 * JW + c : J1 * JW + c - JW);
    a[int64_t(gr) * np + gc] = X[c][r];
  }
  __syncthreads();
}

// columns I u J of V (chunk of 64 rows per CTA): V[:, IJ] <- V[:, IJ] * Theta
__device__ void dev_jac_cols(double* __restrict__ V, int np, int nblk, int round,
                             const double* __restrict__ Th, int b, int k, int chunk, double* jsm) {
  Tile& T = *reinterpret_cast<Tile*>(jsm);
  Tile& X = *reinterpret_cast<Tile*>(jsm + JS * (JS + 1));
  const int r0 = chunk * JS, npair = nblk / 2;
  int I, J;
  tour_pair(nblk, round, k, &I, &J);
  const double* th = Th + (int64_t(b) * npair + k) * JS * JS;
  for (int e = threadIdx.x; e < JS * JS; e += blockDim.x) T[e / JS][e % JS] = th[e];
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  {
    double* M = V + int64_t(b) * np * np;
    __syncthreads();
    for (int e = threadIdx.x; e < JS * JS; e += blockDim.x) {
      const int u = e / JS, v = e % JS;
      const int gv = (v < JW ? I * JW + v : J * JW + v - JW);
      X[u][v] = M[int64_t(r0 + u) * np + gv];
    }
    __syncthreads();
    double acc[4][4] = {};
    tile_mm<false, JS + 1>(acc, X, T);
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        const int col = tx + 16 * v;
        const int gv = (col < JW ? I * JW + col : J * JW + col - JW);
        M[int64_t(r0 + ty + 16 * u) * np + gv] = acc[u][v];
      }
  }
  __syncthreads();
}

struct JacArgs {
  double *A, *V, *Th, *norms;  // norms [max_sweeps][nb][2], zeroed before launch
  int* skip;
  unsigned long long* stamps;  // optional (diagnostics): [0] solve ns, [1] update ns, [2] norm ns
  int np, nblk, npair, chunks, nb, max_sweeps;
  double tol;
  int* sweeps_done;
  GridBar bar;
};

// Block-Jacobi sweeps until the off-diagonal norm of every matrix is below tol (one launch).
__global__ void __launch_bounds__(256) k_jac_coop(JacArgs a) {
  extern __shared__ double jsm[];
  const int nbk = gridDim.x;
  __shared__ int s_done;
  for (int sweep = 0; sweep < a.max_sweeps; ++sweep) {
    for (int r = 0; r < a.nblk - 1; ++r) {
      unsigned long long tr0 = 0, tr1 = 0, tr2 = 0;
      if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(tr0));
      for (int it = blockIdx.x; it < a.nb * a.npair; it += nbk) {
        const int b = it / a.npair;
        // a subproblem whose off-diagonal mass is below tol^2 |A|^2 / nblk^2 is left alone: the
        // sum over all of them stays below the convergence bound tol^2 |A|^2
        const double thr = sweep > 0 ? a.tol * a.tol * a.norms[int64_t(sweep - 1) * a.nb * 2 + 2 * b + 1] /
                                           (double(a.nblk) * a.nblk)
                                     : -1.0;
        dev_jac_solve(a.A, a.np, a.nblk, r, a.Th, a.skip, thr, b, it % a.npair, jsm);
      }
      grid_barrier(a.bar);
      if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(tr1));
      // one pass over A (off-diagonal pair-blocks, two-sided) and V (block columns)
      const int noff = a.npair * (a.npair - 1) / 2;
      const int per = a.npair * a.chunks;
      for (int it = blockIdx.x; it < a.nb * (noff + per); it += nbk) {
        const int b = it / (noff + per), w = it % (noff + per);
        if (w < noff) dev_jac_off(a.A, a.np, a.nblk, r, a.Th, a.skip, b, w, jsm);
        else if (!a.skip[b * a.npair + (w - noff) / a.chunks])
          dev_jac_cols(a.V, a.np, a.nblk, r, a.Th, b, (w - noff) / a.chunks, (w - noff) % a.chunks, jsm);
      }
      grid_barrier(a.bar);
      if (a.stamps && blockIdx.x == 0 && threadIdx.x == 0) {
        asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(tr2));
        a.stamps[0] += tr1 - tr0;
        a.stamps[1] += tr2 - tr1;
      }
    }
    // off-diagonal and total Frobenius mass of every matrix
    double* nm = a.norms + int64_t(sweep) * a.nb * 2;
    {
      // a warp per row of every matrix
      const int lane = threadIdx.x & 31, nw = blockDim.x >> 5;
      for (int64_t row = int64_t(blockIdx.x) * nw + (threadIdx.x >> 5); row < int64_t(a.nb) * a.np;
           row += int64_t(nbk) * nw) {
        const int b = int(row / a.np), i = int(row % a.np);
        const double* ar = a.A + row * a.np;
        double off = 0.0, all = 0.0;
        for (int j = lane; j < a.np; j += 32) {
          const double v = ar[j];
          all = fma(v, v, all);
          if (j != i) off = fma(v, v, off);
        }
        for (int m = 16; m; m >>= 1) {
          off += __shfl_xor_sync(0xffffffffu, off, m);
          all += __shfl_xor_sync(0xffffffffu, all, m);
        }
        if (lane == 0 && (off != 0.0 || all != 0.0)) {
          atomicAdd(&nm[2 * b], off);
          atomicAdd(&nm[2 * b + 1], all);
        }
      }
    }
    grid_barrier(a.bar);
    if (threadIdx.x == 0) {
      int done = 1;
      for (int b = 0; b < a.nb; ++b) {
        const double off = *reinterpret_cast<volatile double*>(&nm[2 * b]);
        const double all = *reinterpret_cast<volatile double*>(&nm[2 * b + 1]);
        if (off > a.tol * a.tol * all) done = 0;
      }
      s_done = done;
    }
    __syncthreads();
    if (s_done) {
      if (blockIdx.x == 0 && threadIdx.x == 0) *a.sweeps_done = sweep + 1;
      break;
    }
    if (sweep + 1 == a.max_sweeps && blockIdx.x == 0 && threadIdx.x == 0) *a.sweeps_done = sweep + 1;
  }
}

template <typename TO>
__global__ void k_jac_sort(const double* __restrict__ Aw, int np, int n, TO* evals, int* perm) {
  const int b = blockIdx.y;
  const double* a = Aw + int64_t(b) * np * np;
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) {
    const double di = a[int64_t(i) * np + i];
    int rank = 0;
    for (int j = 0; j < n; ++j) {
      const double dj = a[int64_t(j) * np + j];
      rank += (dj > di) || (dj == di && j < i);
    }
    evals[int64_t(b) * n + rank] = TO(di);
    perm[int64_t(b) * np + rank] = i;
  }
}

template <typename TO>
__global__ void k_jac_out(const double* __restrict__ V, int np, int n, const int* __restrict__ perm, TO* evecs) {
  const int b = blockIdx.y;
  const int64_t total = int64_t(n) * n;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += int64_t(gridDim.x) * blockDim.x) {
    const int row = int(e / n), col = int(e % n);
    evecs[int64_t(b) * total + e] = TO(V[int64_t(b) * np * np + int64_t(row) * np + perm[int64_t(b) * np + col]]);
  }
}

// Strided rows: a warp per row.
__global__ void k_split(const float* __restrict__ x, int64_t ldx, int64_t rows, int64_t cols, int64_t bsx,
                        __nv_bfloat16* __restrict__ hi, __nv_bfloat16* __restrict__ lo, int64_t ldo, int64_t bso) {
  const int b = blockIdx.y, lane = threadIdx.x & 31;
  const int64_t nw = int64_t(gridDim.x) * (blockDim.x >> 5);
  for (int64_t r = int64_t(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); r < rows; r += nw) {
    const float* xr = x + b * bsx + r * ldx;
    __nv_bfloat16* hr = hi + b * bso + r * ldo;
    __nv_bfloat16* lr = lo ? lo + b * bso + r * ldo : nullptr;
    for (int64_t c = lane; c < cols; c += 32) {
      const float v = xr[c];
      const __nv_bfloat16 h = __float2bfloat16_rn(v);
      hr[c] = h;
      if (lr) lr[c] = __float2bfloat16_rn(v - __bfloat162float(h));
    }
  }
}

// Contiguous rows (ldx = ldo = cols), 4 values per thread: one 16-byte load, two 8-byte stores.
__global__ void k_split_vec(const float4* __restrict__ x, int64_t n4, int64_t bsx4, uint2* __restrict__ hi,
                            uint2* __restrict__ lo, int64_t bso4) {
  const int b = blockIdx.y;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < n4; e += int64_t(gridDim.x) * blockDim.x) {
    const float4 v = x[b * bsx4 + e];
    const __nv_bfloat162 h01 = __floats2bfloat162_rn(v.x, v.y), h23 = __floats2bfloat162_rn(v.z, v.w);
    hi[b * bso4 + e] = make_uint2(*reinterpret_cast<const uint32_t*>(&h01), *reinterpret_cast<const uint32_t*>(&h23));
    if (lo) {
      const float2 f01 = __bfloat1622float2(h01), f23 = __bfloat1622float2(h23);
      const __nv_bfloat162 l01 = __floats2bfloat162_rn(v.x - f01.x, v.y - f01.y);
      const __nv_bfloat162 l23 = __floats2bfloat162_rn(v.z - f23.x, v.w - f23.y);
      lo[b * bso4 + e] = make_uint2(*reinterpret_cast<const uint32_t*>(&l01), *reinterpret_cast<const uint32_t*>(&l23));
    }
  }
}

__global__ void k_split3(const float* __restrict__ x, int64_t n, __nv_bfloat16* __restrict__ hi,
                         __nv_bfloat16* __restrict__ mid, __nv_bfloat16* __restrict__ lo) {
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < n; e += int64_t(gridDim.x) * blockDim.x) {
    const float v = x[e];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(h);
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    const float r2 = r1 - __bfloat162float(m);
    hi[e] = h;
    mid[e] = m;
    lo[e] = __float2bfloat16_rn(r2);
  }
}

int grid_1d(int64_t n, int per = 256) {
  int64_t g = (n + per - 1) / per;
  return int(std::max<int64_t>(1, std::min<int64_t>(g, 148 * 8)));
}

}  // namespace

size_t chol_scratch_bytes(int nb, int n) {
  const int np = rup(n, NB);
  return 2 * align_up(size_t(nb) * np * np * 8, 256) + align_up(size_t(nb) * 8, 256) +
         align_up(size_t(nb) * np * 8, 256) + align_up(size_t(nb) * 4, 256) + 256;
}

// per_sm_cap: at most this many resident CTAs per SM (fewer CTAs make each grid barrier cheaper)
template <typename K, typename A>
jolt_status launch_coop(K kernel, const A& args, int smem, cudaStream_t st, int per_sm_cap = 64) {
  static_assert(sizeof(A) < 4000, "kernel arguments must fit the parameter space");
  int dev = 0, sms = 0, per = 0;
  JOLT_CUDA_TRY(cudaGetDevice(&dev));
  JOLT_CUDA_TRY(cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev));
  JOLT_CUDA_TRY(cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem));
  JOLT_CUDA_TRY(cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per, kernel, 256, smem));
  if (per < 1) return JOLT_ERR_CUDA;
  per = std::min(per, per_sm_cap);
  A local = args;
  void* params[] = {&local};
  JOLT_CUDA_TRY(cudaLaunchCooperativeKernel(reinterpret_cast<void*>(kernel), dim3(sms * per), dim3(256), params,
                                            size_t(smem), st));
  return JOLT_OK;
}

// ---- failure-detection self-tests: a wait that nothing will end must give up and report ----------

// An mbarrier no thread arrives on: the bounded wait (the one every TMA / MMA pipeline uses)
// returns false after limit_ns and sets JOLT_ERR_TIMEOUT in the error word.
__global__ void k_selftest_mbar(int32_t* err, uint64_t limit_ns) {
  __shared__ __align__(8) uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(sm100::smem_u32(&bar), 1);
    sm100::fence_mbar_init();
  }
  __syncthreads();
  sm100::mbar_wait(sm100::smem_u32(&bar), 0, err, limit_ns);
}

// A cooperative grid whose last CTA returns without arriving: the others' grid barrier (the one
// the Cholesky and Jacobi kernels use) gives up after limit_ns with JOLT_ERR_TIMEOUT.
struct SelftestGridArgs {
  GridBar bar;
  uint64_t limit_ns;
};
__global__ void k_selftest_grid(SelftestGridArgs a) {
  if (blockIdx.x == gridDim.x - 1) return;
  grid_barrier(a.bar, a.limit_ns);
}

jolt_status chol_inverse(const float* G, int64_t ld_g, int nb, int n, double shift_rel,
                         __nv_bfloat16* rinv_hi, __nv_bfloat16* rinv_lo, void* scratch, int32_t* err,
                         cudaStream_t st, float* min_ratio) {
  if (nb < 1 || n < 1) return JOLT_OK;
  const int np = rup(n, NB), P = np / NB;
  CholScratch s = chol_carve(scratch, nb, n);
  JOLT_CUDA_TRY(cudaMemsetAsync(s.bar, 0, 2 * sizeof(unsigned int), st));
  JOLT_CUDA_TRY(cudaMemsetAsync(s.mdiag, 0, size_t(nb) * sizeof(double), st));
  CholArgs a;
  a.G = G; a.ldg = ld_g; a.n = n; a.np = np; a.P = P; a.nb = nb; a.shift_rel = shift_rel;
  a.Gd = s.Gd; a.Xd = s.Xd; a.md = s.mdiag; a.diag0 = s.diag0; a.ratio = s.ratio;
  a.hi = rinv_hi; a.lo = rinv_lo;
  a.bar = GridBar{s.bar, s.bar + 1, err};
  a.stamps = nullptr;
  jolt_status r;
  {
    // fp64 work: factor n^3/3 plus triangular inverse n^3/3 per matrix
    StatScope sc(JOLT_K_CHOL, st, nb * 2.0 * double(n) * n * n / 3.0, 0.0);
    r = launch_coop(k_chol_coop, a, 2 * NB * (NB + 1) * 8, st);
  }
  if (r) return r;
  if (min_ratio) {
    std::vector<float> h(nb);
    JOLT_CUDA_TRY(cudaMemcpyAsync(h.data(), s.ratio, sizeof(float) * nb, cudaMemcpyDeviceToHost, st));
    JOLT_CUDA_TRY(cudaStreamSynchronize(st));
    float m = 1.f;
    for (float v : h) m = std::min(m, v);
    *min_ratio = m;
  }
  return JOLT_OK;
}

size_t jacobi_scratch_bytes(int nb, int n) {
  const int np = rup(n, JS), npair = np / JS;
  return 2 * align_up(size_t(nb) * np * np * 8, 256) + align_up(size_t(nb) * npair * JS * JS * 8, 256) +
         align_up(size_t(kJacMaxSweeps) * nb * 16, 256) + align_up(size_t(nb) * np * 4, 256) +
         align_up(size_t(nb) * npair * 4, 256) + 512;
}

template <typename TA, typename TO>
jolt_status jacobi_impl(const TA* A, int64_t ld_a, int nb, int n, TO* evals, TO* evecs, void* scratch,
                        int max_sweeps, double tol, int32_t* err, cudaStream_t st) {
  if (nb < 1 || n < 1) return JOLT_OK;
  const int np = rup(n, JS), nblk = np / JW, npair = nblk / 2, chunks = np / JS;
  JacScratch s = jac_carve(scratch, nb, n);
  k_jac_init<<<dim3(grid_1d(int64_t(np) * np), nb), 256, 0, st>>>(A, ld_a, n, np, s.A, s.V);
  JOLT_CUDA_TRY(cudaMemsetAsync(s.norms, 0, size_t(kJacMaxSweeps) * nb * 16, st));
  JOLT_CUDA_TRY(cudaMemsetAsync(s.bar, 0, 2 * sizeof(unsigned int), st));
  JacArgs a;
  a.A = s.A; a.V = s.V; a.Th = s.Th; a.norms = s.norms; a.skip = s.skip;
  a.np = np; a.nblk = nblk; a.npair = npair; a.chunks = chunks; a.nb = nb;
  a.max_sweeps = std::min(max_sweeps, kJacMaxSweeps);
  a.tol = tol;
  a.sweeps_done = s.sweeps;
  a.bar = GridBar{s.bar, s.bar + 1, err};
  a.stamps = nullptr;
  jolt_status r;
  {
    StatScope sc(JOLT_K_EIG, st, 0.0, 0.0);
    r = launch_coop(k_jac_coop, a, 3 * JS * (JS + 1) * 8, st);
  }
  if (r) return r;
  if (kDebug) {
    int sw = 0;
    JOLT_CUDA_TRY(cudaMemcpyAsync(&sw, s.sweeps, sizeof(int), cudaMemcpyDeviceToHost, st));
    JOLT_CUDA_TRY(cudaStreamSynchronize(st));
    std::fprintf(stderr, "jolt jacobi: n %d batch %d sweeps %d\n", n, nb, sw);
  }
  k_jac_sort<<<dim3((n + 255) / 256, nb), 256, 0, st>>>(s.A, np, n, evals, s.perm);
  k_jac_out<<<dim3(grid_1d(int64_t(n) * n), nb), 256, 0, st>>>(s.V, np, n, s.perm, evecs);
  JOLT_CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

jolt_status jacobi_eig(const float* A, int64_t ld_a, int nb, int n, float* evals, float* evecs, void* scratch,
                       int max_sweeps, double tol, int32_t* err, cudaStream_t st) {
  return jacobi_impl<float, float>(A, ld_a, nb, n, evals, evecs, scratch, max_sweeps, tol, err, st);
}

jolt_status jacobi_eig64(const double* A, int64_t ld_a, int nb, int n, double* evals, double* evecs, void* scratch,
                         int max_sweeps, double tol, int32_t* err, cudaStream_t st) {
  return jacobi_impl<double, double>(A, ld_a, nb, n, evals, evecs, scratch, max_sweeps, tol, err, st);
}

jolt_status split3_bf16(const float* x, int64_t n, __nv_bfloat16* hi, __nv_bfloat16* mid, __nv_bfloat16* lo,
                        cudaStream_t st) {
  if (n <= 0) return JOLT_OK;
  k_split3<<<grid_1d(n), 256, 0, st>>>(x, n, hi, mid, lo);
  JOLT_CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

jolt_status split_bf16(const float* x, int64_t ldx, int64_t rows, int64_t cols, int batch, int64_t bstride_x,
                       __nv_bfloat16* hi, __nv_bfloat16* lo, int64_t ldo, int64_t bstride_o, cudaStream_t st) {
  if (rows <= 0 || cols <= 0) return JOLT_OK;
  const int64_t n = rows * cols;
  const bool vec = ldx == cols && ldo == cols && n % 4 == 0 && bstride_x % 4 == 0 && bstride_o % 4 == 0 &&
                   reinterpret_cast<uintptr_t>(x) % 16 == 0 && reinterpret_cast<uintptr_t>(hi) % 8 == 0 &&
                   (!lo || reinterpret_cast<uintptr_t>(lo) % 8 == 0);
  if (vec) {
    const int gx = int(std::max<int64_t>(1, std::min<int64_t>((n / 4 + 255) / 256, 148 * 8 / std::max(1, batch) + 1)));
    k_split_vec<<<dim3(gx, batch), 256, 0, st>>>(reinterpret_cast<const float4*>(x), n / 4, bstride_x / 4,
                                                 reinterpret_cast<uint2*>(hi), reinterpret_cast<uint2*>(lo), bstride_o / 4);
  } else {
    const int gx = int(std::max<int64_t>(1, std::min<int64_t>((rows + 7) / 8, 148 * 8)));
    k_split<<<dim3(gx, batch), 256, 0, st>>>(x, ldx, rows, cols, bstride_x, hi, lo, ldo, bstride_o);
  }
  JOLT_CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

}  // namespace jolt

using namespace jolt;

extern "C" jolt_status jolt_selftest_timeout(int32_t which, uint64_t limit_ns, void* ws, size_t ws_bytes,
                                             void* stream) {
  if (!ws || ws_bytes < 512 || limit_ns == 0 || limit_ns > 2000000000ull || (which != 0 && which != 1))
    return JOLT_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  int32_t* err = static_cast<int32_t*>(ws);
  JOLT_CUDA_TRY(cudaMemsetAsync(ws, 0, 512, st));
  if (which == 0) {
    k_selftest_mbar<<<1, 32, 0, st>>>(err, limit_ns);
    JOLT_CUDA_TRY(cudaGetLastError());
    return JOLT_OK;
  }
  SelftestGridArgs a;
  unsigned int* bar = reinterpret_cast<unsigned int*>(static_cast<uint8_t*>(ws) + 256);
  a.bar.count = bar;
  a.bar.gen = bar + 1;
  a.bar.err = err;
  a.limit_ns = limit_ns;
  void* params[] = {&a};
  JOLT_CUDA_TRY(cudaLaunchCooperativeKernel(reinterpret_cast<void*>(k_selftest_grid), dim3(2), dim3(32), params, 0, st));
  return JOLT_OK;
}

extern "C" size_t jolt_sym_eig_workspace(int32_t n, int32_t batch) {
  if (n < 1 || batch < 1) return 0;
  return sizeof(WsHeader) + jacobi_scratch_bytes(batch, n);
}

extern "C" jolt_status jolt_sym_eig(const float* A, int32_t n, int32_t batch, float* evals, float* evecs,
                                    void* ws, size_t ws_bytes, void* stream) {
  if (n < 1 || batch < 1) return JOLT_ERR_INVALID_ARG;
  if (!A || !evals || !evecs || !ws) return JOLT_ERR_INVALID_ARG;
  if (ws_bytes < jolt_sym_eig_workspace(n, batch)) return JOLT_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  JOLT_CUDA_TRY(cudaMemsetAsync(ws, 0, sizeof(WsHeader), st));
  jolt_status r = jacobi_eig(A, n, batch, n, evals, evecs, static_cast<uint8_t*>(ws) + sizeof(WsHeader), 30,
                             1e-10, static_cast<int32_t*>(ws), st);
  if (r) return r;
  JOLT_CUDA_TRY(cudaStreamSynchronize(st));
  return JOLT_OK;
}
