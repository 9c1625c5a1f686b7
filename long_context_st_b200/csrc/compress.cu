// jolt_analyze and jolt_compress: the compressor half of the codec.
//
// analyze, per pass of up to cells_per_pass cells of one kind (K or V), all batched:
//   ||X||^2 (fp64), S_d = sum_lh X_lh^T X_lh (tcgen05), Y = X_(T) Omega (tcgen05, Rademacher Omega),
//   q power iterations Y <- X_(T) orth(X_(T)^T orth(Y)), Q = orth(Y), B^T = X_(T)^T Q (hi/lo terms),
//   W = B B^T, eig(W) (block Jacobi), U_T = Q V[:, :q_cap] (hi/lo terms) kept in the workspace.
//   orth() is shifted CholeskyQR: passes of Gram (hi/lo terms) -> fp64 Cholesky of G + s*I ->
//   Y R^{-1} (hi/lo terms) with s = 1e-4*||G||_F until the Gram is well conditioned, then s = 0.
// compress, per cell: U_T (first r_T columns) stored; Y_lh = U_T^T X_lh (tcgen05);
//   S_Y = sum Y_lh^T Y_lh; U_d = top-r_d eigenvectors (block Jacobi); G = Y U_d; X~ = U_T (G U_d^T)
//   from the stored (rounded) factors (tcgen05, hi/lo terms); residual X - X~ rotated by the
//   seeded randomized Hadamard, quantised per row and packed.
#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <cstring>
#include <vector>

#include "gemm_tc.cuh"
#include "linalg.cuh"
#include "pack.cuh"
#include "stats.h"

namespace jolt {

namespace {

constexpr uint64_t kAnalyzeMagic = 0x4A4F4C54414E4C5Aull;  // "JOLTANLZ"

uint64_t shape_tag(const jolt_shape& s) {
  uint64_t h = kAnalyzeMagic;
  const uint32_t* w = reinterpret_cast<const uint32_t*>(&s);
  for (size_t i = 0; i < sizeof(jolt_shape) / 4; ++i) h = mix64(h ^ w[i]);
  return h;
}

struct Plan {
  int C;          // cells per pass
  int cc;         // cells per compress chunk
  int T, d, LgH, n, l, qcap;
  int64_t cell_elems;
  size_t off_ut, off_pass, off_cmp, total;
  // pass scratch offsets (relative to off_pass)
  size_t om, Yh2, Yl2, Yh, Yl, Gm, Rh, Rl, Z, Zh, Zl, ev, evec, Vh, Vl, Sd, evd, evecd, nrm, chol, jac, xb;
  size_t g64, ev64, evec64, sd64, evd64, evecd64;  // exact path (sketch width == n)
  // compress scratch (relative to off_cmp)
  size_t uh, ul, um, ylh, sy, evy, evecy, ud, blh, bh, bm, bl, xt, jac2;
};

// jolt_compress handles cells in chunks of this many: per chunk one batched eigensolver launch for
// the feature-mode Grams S_Y of all its cells.
constexpr int kCmpChunk = 40;  // at most this many cells per chunk (one eigensolver launch each)

Plan make_plan(const jolt_shape& s) {
  Plan p{};
  p.T = s.T;
  p.d = s.d_h;
  p.LgH = s.layers_per_group * s.n_kv;
  p.n = p.LgH * p.d;
  p.l = s.sketch_cols;
  p.qcap = s.q_cap;
  p.cell_elems = int64_t(p.LgH) * s.T * s.d_h;
  const int per_kind = s.batch * n_groups(s);
  p.C = std::max(1, std::min(s.cells_per_pass, per_kind));
  const size_t C = p.C, T = p.T, l = std::max(p.l, 16), n = p.n, d = p.d, q = std::max(p.qcap, 16);
  size_t off = sizeof(WsHeader);
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  p.off_ut = take(size_t(n_cells(s)) * T * q * 4);
  const size_t pass0 = off;
  auto rel = [&](size_t bytes) { return take(bytes) - pass0; };
  p.off_pass = pass0;
  const size_t rowsmax = std::max(T, n);
  p.om = rel(l * n * 2);
  p.Yh2 = rel(C * rowsmax * l * 2);  // second hi / lo buffer: orthonormalisation passes ping-pong
  p.Yl2 = rel(C * rowsmax * l * 2);
  p.Yh = rel(C * rowsmax * l * 2);
  p.Yl = rel(C * rowsmax * l * 2);
  p.Gm = rel(C * l * l * 4);
  p.Rh = rel(C * l * l * 2);
  p.Rl = rel(C * l * l * 2);
  p.Z = rel(C * n * l * 4);
  p.Zh = rel(C * n * l * 2);
  p.Zl = rel(C * n * l * 2);
  p.ev = rel(C * l * 4);
  p.evec = rel(C * l * l * 4);
  p.Vh = rel(C * l * l * 2);
  p.Vl = rel(C * l * l * 2);
  p.Sd = rel(C * d * d * 4);
  p.evd = rel(C * d * 4);
  p.evecd = rel(C * d * d * 4);
  p.nrm = rel(C * 8);
  p.chol = rel(chol_scratch_bytes(int(C), int(l)));
  p.jac = rel(std::max(jacobi_scratch_bytes(int(C), int(l)), jacobi_scratch_bytes(int(C), int(d))));
  p.xb = rel(s.io_dtype == JOLT_F32 ? 2 * C * size_t(p.cell_elems) * 2 : 0);  // hi/lo bf16 of f32 inputs
  const bool exact = (p.l == p.n);
  p.g64 = rel(exact ? C * n * n * 8 : 0);
  p.ev64 = rel(exact ? C * n * 8 : 0);
  p.evec64 = rel(exact ? C * n * n * 8 : 0);
  p.sd64 = rel(C * d * d * 8);
  p.evd64 = rel(C * d * 8);
  p.evecd64 = rel(C * d * d * 8);
  if (exact) p.jac = rel(std::max(jacobi_scratch_bytes(int(C), int(n)), jacobi_scratch_bytes(int(C), int(d))));
  const size_t cmp0 = off;
  auto relc = [&](size_t bytes) { return take(bytes) - cmp0; };
  p.off_cmp = cmp0;
  p.uh = relc(T * q * 2);
  p.ul = relc(T * q * 2);
  p.um = relc(T * q * 2);
  p.cc = std::max(1, std::min(kCmpChunk, n_cells(s)));
  p.ylh = relc(size_t(p.cc) * p.LgH * q * d * 4);
  p.sy = relc(size_t(p.cc) * d * d * 4);
  p.evy = relc(size_t(p.cc) * d * 4);
  p.evecy = relc(size_t(p.cc) * d * d * 4);
  p.ud = relc(d * d * 4);
  p.blh = relc(size_t(p.LgH) * q * d * 4);
  p.bh = relc(size_t(p.LgH) * q * d * 2);
  p.bm = relc(size_t(p.LgH) * q * d * 2);
  p.bl = relc(size_t(p.LgH) * q * d * 2);
  p.xt = relc(size_t(p.LgH) * T * d * 4);
  p.jac2 = relc(jacobi_scratch_bytes(p.cc, int(d)));
  p.total = off;
  return p;
}

// ---- small kernels ------------------------------------------------------------------------------

__global__ void k_omega(__nv_bfloat16* om, int l, int n, uint64_t seed) {
  const int64_t total = int64_t(l) * n;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += int64_t(gridDim.x) * blockDim.x) {
    // om[j][i] = Omega[i][j]: the sketch matrix stored K-major (row j holds column j of Omega)
    const int64_t j = e / n, i = e % n;
    const uint64_t ctr = (seed << 32) + uint64_t(i) * uint64_t(l) + uint64_t(j);
    om[e] = __float2bfloat16_rn((mix64(ctr) >> 63) ? -1.f : 1.f);
  }
}

template <typename T>
__global__ void k_norm2(const T* __restrict__ X, int64_t cell_elems, double* out) {
  const int c = blockIdx.y;
  const T* x = X + int64_t(c) * cell_elems;
  double acc = 0.0;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < cell_elems; e += int64_t(gridDim.x) * blockDim.x) {
    const double v = ld_as_float(x, e);
    acc += v * v;
  }
  for (int m = 16; m; m >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, m);
  if ((threadIdx.x & 31) == 0) atomicAdd(&out[c], acc);
}

// Copy the first r columns of U [T][q] (fp32) to the stored cache (dtype) and to bf16 GEMM operands
// [T][r]: hi, mid, lo with U ~ hi + mid + lo (mid may be null). With bf16 storage the stored
// value is hi.
__global__ void k_store_ut(const float* __restrict__ U, int T, int q, int r, int fac_f32, uint8_t* cache_ut,
                           __nv_bfloat16* hi, __nv_bfloat16* mid, __nv_bfloat16* lo) {
  const int64_t total = int64_t(T) * r;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t t = e / r, c = e % r;
    const float v = U[t * q + c];
    const __nv_bfloat16 h = __float2bfloat16_rn(v);
    const float r1 = v - __bfloat162float(h);
    const __nv_bfloat16 m = __float2bfloat16_rn(r1);
    if (fac_f32) reinterpret_cast<float*>(cache_ut)[e] = v;
    else reinterpret_cast<__nv_bfloat16*>(cache_ut)[e] = h;
    if (hi) hi[e] = h;
    if (mid) {
      mid[e] = m;
      lo[e] = __float2bfloat16_rn(r1 - __bfloat162float(m));
    } else if (lo) {
      lo[e] = m;
    }
  }
}

// S = sum_b Y_b^T Y_b, Y [nb][r][d] fp32, S [d][d] fp32 (pre-zeroed), partial sums per CTA.
__global__ void __launch_bounds__(256) k_gram_small(const float* __restrict__ Y, int nrows, int d, float* S) {
  extern __shared__ float sy[];  // [32][d]
  const int i0 = blockIdx.y * 32, j0 = blockIdx.z * 32;
  const int ti = threadIdx.x / 32, tj = threadIdx.x % 32;  // 8 x 32 threads, 4 rows each
  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  for (int r0 = blockIdx.x * 32; r0 < nrows; r0 += gridDim.x * 32) {
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * 64; e += blockDim.x) {
      const int rr = e / 64, cc = e % 64;
      const int row = r0 + rr;
      const int col = cc < 32 ? i0 + cc : j0 + cc - 32;
      sy[rr * 64 + cc] = (row < nrows && col < d) ? Y[int64_t(row) * d + col] : 0.f;
    }
    __syncthreads();
    for (int rr = 0; rr < 32; ++rr) {
      const float bj = sy[rr * 64 + 32 + tj];
#pragma unroll
      for (int u = 0; u < 4; ++u) acc[u] += sy[rr * 64 + ti * 4 + u] * bj;
    }
  }
#pragma unroll
  for (int u = 0; u < 4; ++u) {
    const int i = i0 + ti * 4 + u, j = j0 + tj;
    if (i < d && j < d) atomicAdd(&S[i * d + j], acc[u]);
  }
}

// out[b][r][j] = sum_i Y[b][r][i] * M[i][j]  (Y [nb][r][d], M [d][ldm] first m columns)
// optionally rounded to the factor dtype and written to the cache.
__global__ void k_proj_small(const float* __restrict__ Y, int64_t nrows, int d, const float* __restrict__ M,
                             int ldm, int m, int fac_f32, uint8_t* __restrict__ out) {
  const int64_t total = nrows * m;
  for (int64_t e = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; e < total; e += int64_t(gridDim.x) * blockDim.x) {
    const int64_t r = e / m;
    const int j = int(e % m);
    float a = 0.f;
    for (int i = 0; i < d; ++i) a += Y[r * d + i] * M[int64_t(i) * ldm + j];
    if (fac_f32) reinterpret_cast<float*>(out)[e] = a;
    else reinterpret_cast<__nv_bfloat16*>(out)[e] = __float2bfloat16_rn(a);
  }
}

__device__ __forceinline__ float ld_fac_any(const uint8_t* p, int64_t i, int f32) {
  return f32 ? reinterpret_cast<const float*>(p)[i] : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(p)[i]);
}

// B[lh][r][i] = sum_j G[lh][r][j] * U_d[i][j] from the stored values (fp32 out), with rows r of
// all (lh, r) pairs flattened. A block covers 32 rows x all D columns; G and U_d pass through
// shared memory 32 values of j at a time; each sum runs over j in order (one fused multiply-add
// per term).
template <int D>
__global__ void __launch_bounds__(256) k_recon_b(const uint8_t* __restrict__ G, const uint8_t* __restrict__ Ud,
                                                 int64_t nrows, int rd, int f32, float* __restrict__ B) {
  constexpr int kGroups = 256 / D, kRows = 32 / kGroups;
  __shared__ float Gs[32][33];
  __shared__ float Us[32][D];
  const int i = threadIdx.x % D, g = threadIdx.x / D;
  const int64_t r0 = int64_t(blockIdx.x) * 32;
  float a[kRows];
#pragma unroll
  for (int k = 0; k < kRows; ++k) a[k] = 0.f;
  for (int j0 = 0; j0 < rd; j0 += 32) {
    const int nj = min(32, rd - j0);
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * 32; e += 256) {
      const int rr = e / 32, jj = e % 32;
      const int64_t r = r0 + rr;
      Gs[rr][jj] = (r < nrows && jj < nj) ? ld_fac_any(G, r * rd + j0 + jj, f32) : 0.f;
    }
    for (int e = threadIdx.x; e < 32 * D; e += 256) {
      const int jj = e / D, ii = e % D;
      Us[jj][ii] = jj < nj ? ld_fac_any(Ud, int64_t(ii) * rd + j0 + jj, f32) : 0.f;
    }
    __syncthreads();
    for (int jj = 0; jj < nj; ++jj) {
      const float u = Us[jj][i];
#pragma unroll
      for (int k = 0; k < kRows; ++k) a[k] += Gs[g + kGroups * k][jj] * u;
    }
  }
#pragma unroll
  for (int k = 0; k < kRows; ++k) {
    const int64_t r = r0 + g + kGroups * k;
    if (r < nrows) B[r * D + i] = a[k];
  }
}

// Residual rows: x = X[row] - Xt[row] (Xt may be null), rotated, quantised and packed.
template <int E, typename TX>
__global__ void __launch_bounds__(256) k_residual(const TX* __restrict__ X, const float* __restrict__ Xt, int64_t rows,
                                                  int b, uint64_t seed, uint8_t* __restrict__ codes,
                                                  __half2* __restrict__ sz, int32_t* err) {
  constexpr int D = 32 * E;
  __shared__ uint8_t stage[8][D];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int64_t warps = int64_t(gridDim.x) * 8;
  const int nbytes = D * b / 8;
  const float isd = rsqrtf(float(D));
  for (int64_t r = int64_t(blockIdx.x) * 8 + w; r < rows; r += warps) {
    float x[E];
#pragma unroll
    for (int i = 0; i < E; ++i) {
      const int64_t idx = r * D + lane * E + i;
      x[i] = ld_as_float(X, idx) - (Xt ? Xt[idx] : 0.f);
    }
    warp_rotate<E>(x, seed, isd);
    uint8_t c[E];
    __half hs, hz;
    bool ok = true;
#pragma unroll
    for (int i = 0; i < E; ++i) ok &= isfinite(x[i]);
    ok = __all_sync(0xffffffffu, ok);
    if (!warp_quantize<E>(x, b, c, &hs, &hz)) ok = false;
    if (!ok && lane == 0) report_error(err, JOLT_ERR_NUMERIC);
    warp_pack_store<E>(c, b, stage[w], codes + r * nbytes);
    if (lane == 0) sz[r] = __halves2half2(hs, hz);
  }
}

// fp64 Gram of the token unfolding: G[a][b] += sum_t Xu[t][a] Xu[t][b], Xu(t, c) = X[c/d][t][c%d].
// grid (n/64, n/64, C*ks); each CTA covers a 64x64 tile over its slice of t.
template <typename TX>
__global__ void __launch_bounds__(256) k_gram64(const TX* __restrict__ X, int64_t cell_elems, int T, int d, int n,
                                                int ks, double* __restrict__ G) {
  __shared__ double As[16][64], Bs[16][64];
  const int a0 = blockIdx.x * 64, b0 = blockIdx.y * 64;
  const int c = blockIdx.z / ks, kz = blockIdx.z % ks;
  const TX* x = X + int64_t(c) * cell_elems;
  const int chunk = (T + ks - 1) / ks;
  const int t_beg = kz * chunk, t_end = min(T, t_beg + chunk);
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[4][4] = {};
  const int la = a0 / d, ja = a0 % d, lb = b0 / d, jb = b0 % d;
  for (int t0 = t_beg; t0 < t_end; t0 += 16) {
    __syncthreads();
    for (int e = threadIdx.x; e < 16 * 64; e += blockDim.x) {
      const int tt = e / 64, cc = e % 64, t = t0 + tt;
      const bool ok = t < t_end;
      As[tt][cc] = ok ? double(ld_as_float(x, (int64_t(la) * T + t) * d + ja + cc)) : 0.0;
      Bs[tt][cc] = ok ? double(ld_as_float(x, (int64_t(lb) * T + t) * d + jb + cc)) : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int tt = 0; tt < 16; ++tt) {
      double av[4], bv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) av[u] = As[tt][ty * 4 + u];
#pragma unroll
      for (int v = 0; v < 4; ++v) bv[v] = Bs[tt][tx * 4 + v];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] += av[u] * bv[v];
    }
  }
  double* g = G + int64_t(c) * n * n;
#pragma unroll
  for (int u = 0; u < 4; ++u)
#pragma unroll
    for (int v = 0; v < 4; ++v) atomicAdd(&g[int64_t(a0 + ty * 4 + u) * n + b0 + tx * 4 + v], acc[u][v]);
}

// U[t][r] = sum_c Xu[t][c] V[c][r] / sqrt(lambda_r)  (fp64 math, fp32 out), r < q; grid (q/64, ceil(T/64), C)
template <typename TX>
__global__ void __launch_bounds__(256) k_xv64(const TX* __restrict__ X, int64_t cell_elems, int T, int d, int n,
                                              const double* __restrict__ Vv, const double* __restrict__ lam, int q,
                                              float* __restrict__ U, int64_t u_cell_stride) {
  __shared__ double As[64][17], Bs[16][64];
  const int r0 = blockIdx.x * 64, t0 = blockIdx.y * 64, c = blockIdx.z;
  const TX* x = X + int64_t(c) * cell_elems;
  const double* vv = Vv + int64_t(c) * n * n;
  const int ty = threadIdx.x / 16, tx = threadIdx.x % 16;
  double acc[4][4] = {};
  for (int c0 = 0; c0 < n; c0 += 16) {
    __syncthreads();
    const int lh = c0 / d, j0 = c0 % d;
    for (int e = threadIdx.x; e < 64 * 16; e += blockDim.x) {
      const int tt = e / 16, cc = e % 16, t = t0 + tt;
      As[tt][cc] = (t < T) ? double(ld_as_float(x, (int64_t(lh) * T + t) * d + j0 + cc)) : 0.0;
      const int rr = e % 64, kk = e / 64;
      Bs[kk][rr] = (r0 + rr < q) ? vv[int64_t(c0 + kk) * n + r0 + rr] : 0.0;
    }
    __syncthreads();
#pragma unroll 4
    for (int kk = 0; kk < 16; ++kk) {
      double av[4], bv[4];
#pragma unroll
      for (int u = 0; u < 4; ++u) av[u] = As[ty * 4 + u][kk];
#pragma unroll
      for (int v = 0; v < 4; ++v) bv[v] = Bs[kk][tx * 4 + v];
#pragma unroll
      for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) acc[u][v] += av[u] * bv[v];
    }
  }
  float* out = U + int64_t(c) * u_cell_stride;
#pragma unroll
  for (int v = 0; v < 4; ++v) {
    const int r = r0 + tx * 4 + v;
    if (r >= q) continue;
    const double lm = lam[int64_t(c) * n + r];
    const double inv = lm > 1e-300 ? 1.0 / sqrt(lm) : 0.0;
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int t = t0 + ty * 4 + u;
      if (t < T) out[int64_t(t) * q + r] = float(acc[u][v] * inv);
    }
  }
}

// S_d = sum over the d x d diagonal blocks of the token-unfolding Gram.
__global__ void k_diag_blocks(const double* __restrict__ G, int n, int d, int nblk, double* __restrict__ Sd) {
  const int c = blockIdx.y;
  for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < d * d; e += gridDim.x * blockDim.x) {
    const int i = e / d, j = e % d;
    double a = 0.0;
    for (int b = 0; b < nblk; ++b) a += G[int64_t(c) * n * n + int64_t(b * d + i) * n + b * d + j];
    Sd[int64_t(c) * d * d + e] = a;
  }
}

int grid1(int64_t n) { return int(std::max<int64_t>(1, std::min<int64_t>((n + 255) / 256, 148 * 16))); }

struct Ctx {
  const jolt_shape* s;
  Plan p;
  uint8_t* ws;
  int32_t* err;
  cudaStream_t st;
  uint8_t* pass() const { return ws + p.off_pass; }
  template <typename Tp> Tp* at(size_t rel) const { return reinterpret_cast<Tp*>(pass() + rel); }
  template <typename Tp> Tp* atc(size_t rel) const { return reinterpret_cast<Tp*>(ws + p.off_cmp + rel); }
};

// Every contraction of the compressor runs in the kernel form the shape names.
jolt_status run_gemm(const Ctx& c, GemmCall& g) {
  g.plan = c.s->gemm_plan;
  return gemm_tc(g, c.st);
}

void report_error_host(const Ctx& c, int32_t code) {
  int32_t cur = 0;
  cudaMemcpyAsync(&cur, c.err, 4, cudaMemcpyDeviceToHost, c.st);
  cudaStreamSynchronize(c.st);
  if (!cur) cudaMemcpyAsync(c.err, &code, 4, cudaMemcpyHostToDevice, c.st);
  cudaStreamSynchronize(c.st);
}

Operand plain(const void* ptr, int major, int64_t inner, int64_t outer, int64_t ld, int64_t batch = 1,
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

// X_(T) of a cell batch: rows t, columns (lh, j); folded inner index (lh, j) with fold d.
Operand xunfold(const void* X, int major, const Plan& p, int C) {
  Operand o;
  o.ptr = X;
  o.major = major;
  o.inner = p.d;
  o.fold = p.d;
  o.nfold = p.LgH;
  o.fold_stride = int64_t(p.T) * p.d;
  o.outer = p.T;
  o.outer_stride = p.d;
  o.batch = C;
  o.batch_stride = p.cell_elems;
  return o;
}

// Orthonormalise the columns of Y [C][rows][l] by CholeskyQR passes with bf16 hi/lo Grams and
// products. Two forms of Y:
//  - fp32 (Yf != nullptr, updated in place): each pass splits Yf into hi/lo buffer 0 first;
//  - bf16 parts already in hi/lo buffer *cur (Yf == nullptr): each pass writes its product's hi/lo
//    split straight from the GEMM epilogue into the other buffer, and *cur follows the result.
// Shifted passes (s = 1e-4 * ||G||_F) run until the Cholesky's smallest pivot ratio R_jj^2 / G_jj
// reaches 0.1; then unshifted passes run until one factors a Gram whose ratio is >= 0.9 (an
// almost orthonormal input, so the output is orthonormal to the hi/lo precision). A breakdown of
// an unshifted factorisation falls back to a shifted pass. At most kMaxOrthPasses passes.
constexpr int kMaxOrthPasses = 8;

// polish = false (inside the power iterations): the basis only feeds the next product, which reads
// its bf16 part. Rounding is harmless once the basis is well conditioned — every direction is then
// kept to 2^-9 of itself — but not before: the product's columns are dominated by the top singular
// directions, and those ~1e-4 of the top one in singular value fall below bf16's resolution of the
// column. So the passes read the product's hi/lo parts (Gram and Y R^-1 in hi/lo terms, as for
// the final basis), and stop after the first unshifted pass, i.e. once a shifted pass has made the
// input well conditioned (ratio >= 0.1) and one more pass has orthonormalised it. The final basis
// (polish = true) gets unshifted passes until the input was nearly orthonormal (ratio >= 0.9).
jolt_status orth(const Ctx& c, float* Yf, int* cur, int rows, int C, bool polish = true) {
  const Plan& p = c.p;
  const int l = p.l;
  __nv_bfloat16* Yh_b[2] = {c.at<__nv_bfloat16>(p.Yh), c.at<__nv_bfloat16>(p.Yh2)};
  __nv_bfloat16* Yl_b[2] = {c.at<__nv_bfloat16>(p.Yl), c.at<__nv_bfloat16>(p.Yl2)};
  float* Gm = c.at<float>(p.Gm);
  __nv_bfloat16* Rh = c.at<__nv_bfloat16>(p.Rh);
  __nv_bfloat16* Rl = c.at<__nv_bfloat16>(p.Rl);
  int b = Yf ? 0 : *cur;
  bool conditioned = false;
  for (int pass = 0; pass < kMaxOrthPasses; ++pass) {
    __nv_bfloat16* Yh = Yh_b[b];
    __nv_bfloat16* Yl = Yl_b[b];
    jolt_status r;
    if (Yf && (r = split_bf16(Yf, l, rows, l, C, int64_t(rows) * l, Yh, Yl, l, int64_t(rows) * l, c.st)))
      return r;
    JOLT_CUDA_TRY(cudaMemsetAsync(Gm, 0, size_t(C) * l * l * 4, c.st));
    GemmCall g;
    g.M = l; g.N = l; g.K = rows; g.n_terms = 3;
    const Operand yh = plain(Yh, kMajorMN, l, rows, l, C, int64_t(rows) * l);
    const Operand yl = plain(Yl, kMajorMN, l, rows, l, C, int64_t(rows) * l);
    g.A[0] = yh; g.B[0] = yh;
    g.A[1] = yh; g.B[1] = yl;
    g.A[2] = yl; g.B[2] = yh;
    g.C = Gm; g.ldc = l; g.c_batch_stride = int64_t(l) * l; g.batch = C;
    g.k_split = 0;
    g.accumulate = true; g.err = c.err;
    g.c_upper = true;  // symmetric: the Cholesky reads the upper triangle
    if ((r = run_gemm(c, g))) return r;
    if (kDebug) {
      std::vector<float> h(size_t(C) * l * l);
      cudaMemcpyAsync(h.data(), Gm, h.size() * 4, cudaMemcpyDeviceToHost, c.st);
      cudaStreamSynchronize(c.st);
      for (int bb = 0; bb < C; ++bb) {
        const float* gb = h.data() + size_t(bb) * l * l;
        int bad = 0;
        float dmn = 1e30f, dmx = 0.f;
        for (int i = 0; i < l; ++i) {
          dmn = std::min(dmn, gb[size_t(i) * l + i]);
          dmx = std::max(dmx, gb[size_t(i) * l + i]);
          for (int j = i; j < l; ++j) bad += !std::isfinite(gb[size_t(i) * l + j]);
        }
        std::fprintf(stderr, "jolt gram: rows %d pass %d cell %d nonfinite %d diag [%g, %g]\n", rows, pass, bb, bad,
                     dmn, dmx);
      }
    }
    const bool last = pass == kMaxOrthPasses - 1;
    float ratio = 0.f;
    double shift = (conditioned || last) ? 0.0 : 1e-4;
    if ((r = chol_inverse(Gm, l, C, l, shift, Rh, Rl, c.pass() + p.chol, c.err, c.st, &ratio))) return r;
    if (!(ratio > 0.f)) {
      if (shift == 0.0 && pass < kMaxOrthPasses - 1) {
        shift = 1e-4;
        if ((r = chol_inverse(Gm, l, C, l, shift, Rh, Rl, c.pass() + p.chol, c.err, c.st, &ratio))) return r;
      }
      if (!(ratio > 0.f)) {
        report_error_host(c, JOLT_ERR_NUMERIC);
        return JOLT_ERR_NUMERIC;
      }
    }
    if (kDebug)
      std::fprintf(stderr, "jolt orth: rows %d pass %d shift %g min pivot ratio %g\n", rows, pass, shift, ratio);
    GemmCall t;
    t.M = rows; t.N = l; t.K = l; t.n_terms = 3;
    const Operand ykh = plain(Yh, kMajorK, l, rows, l, C, int64_t(rows) * l);
    const Operand ykl = plain(Yl, kMajorK, l, rows, l, C, int64_t(rows) * l);
    const Operand rh = plain(Rh, kMajorMN, l, l, l, C, int64_t(l) * l);
    const Operand rl = plain(Rl, kMajorMN, l, l, l, C, int64_t(l) * l);
    t.A[0] = ykh; t.B[0] = rh;
    t.A[1] = ykh; t.B[1] = rl;
    t.A[2] = ykl; t.B[2] = rh;
    if (Yf) {
      t.C = Yf;
    } else {
      // the product cannot overwrite the parts it reads: write the other buffer
      b ^= 1;
      t.Ch = Yh_b[b];
      t.Cl = Yl_b[b];
    }
    t.ldc = l; t.c_batch_stride = int64_t(rows) * l; t.batch = C; t.err = c.err;
    t.b_upper = true;  // R^-1 is upper triangular
    if ((r = run_gemm(c, t))) return r;
    if (cur) *cur = b;
    if (shift == 0.0 && ratio >= 0.9f) return JOLT_OK;
    if (!polish && shift == 0.0) return JOLT_OK;
    if (ratio >= 0.1f) conditioned = true;
  }
  return JOLT_OK;
}

// One pass: cells [bg0, bg0 + C) of kind kv. Writes U_T to the persistent region and the spectra
// (eigenvalues of W and S_d, ||X||^2) to host arrays.
jolt_status analyze_pass(const Ctx& c, const void* Xkind, int kv, int bg0, int C, std::vector<double>& evT,
                         std::vector<double>& evD, std::vector<double>& nrm) {
  const Plan& p = c.p;
  const jolt_shape& s = *c.s;
  const int T = p.T, n = p.n, l = p.l, d = p.d, q = p.qcap;
  const bool io32 = s.io_dtype == JOLT_F32;
  const uint8_t* X = static_cast<const uint8_t*>(Xkind) + int64_t(bg0) * p.cell_elems * (io32 ? 4 : 2);
  jolt_status r;
  // ||X||^2
  double* nr = c.at<double>(p.nrm);
  JOLT_CUDA_TRY(cudaMemsetAsync(nr, 0, C * 8, c.st));
  if (io32) k_norm2<float><<<dim3(148, C), 256, 0, c.st>>>(reinterpret_cast<const float*>(X), p.cell_elems, nr);
  else k_norm2<__nv_bfloat16><<<dim3(148, C), 256, 0, c.st>>>(reinterpret_cast<const __nv_bfloat16*>(X), p.cell_elems, nr);
  // f32 inputs enter the tensor cores as hi + lo bf16 parts (bf16 inputs are exact as they are)
  const void* Xb = X;
  const void* Xlo = nullptr;
  if (io32) {
    __nv_bfloat16* xh = c.at<__nv_bfloat16>(p.xb);
    __nv_bfloat16* xl = xh + int64_t(C) * p.cell_elems;
    if ((r = split_bf16(reinterpret_cast<const float*>(X), 1, int64_t(C) * p.cell_elems, 1, 1, 0, xh, xl, 1, 0, c.st)))
      return r;
    Xb = xh;
    Xlo = xl;
  }
  // S_d = sum_lh X_lh^T X_lh
  float* Sd = c.at<float>(p.Sd);
  JOLT_CUDA_TRY(cudaMemsetAsync(Sd, 0, size_t(C) * d * d * 4, c.st));
  {
    GemmCall g;
    g.M = d; g.N = d; g.K = T;
    const Operand xh = plain(Xb, kMajorMN, d, T, d, int64_t(C) * p.LgH, int64_t(T) * d);
    g.A[0] = xh; g.B[0] = xh;
    if (Xlo) {
      const Operand xl = plain(Xlo, kMajorMN, d, T, d, int64_t(C) * p.LgH, int64_t(T) * d);
      g.n_terms = 3;
      g.A[1] = xh; g.B[1] = xl;
      g.A[2] = xl; g.B[2] = xh;
    }
    g.C = Sd; g.ldc = d; g.c_batch_stride = int64_t(d) * d; g.c_batch_div = p.LgH;
    g.batch = C * p.LgH; g.k_split = 0; g.accumulate = true; g.err = c.err;
    if ((r = run_gemm(c, g))) return r;
  }
  const bool exact = (p.l == p.n);
  if (exact && q > 0) {
    // sketch width == n: the range finder would span all of X_(T); take the exact token-mode
    // spectrum instead, in fp64: G = X_(T)^T X_(T), eig(G), U_T = X_(T) V / sigma.
    double* G64 = c.at<double>(p.g64);
    double* ev64 = c.at<double>(p.ev64);
    double* evec64 = c.at<double>(p.evec64);
    JOLT_CUDA_TRY(cudaMemsetAsync(G64, 0, size_t(C) * n * n * 8, c.st));
    const int nt = (n + 63) / 64;
    const int ks = std::max(1, std::min(64, int((2 * 148 + int64_t(nt) * nt * C - 1) / (int64_t(nt) * nt * C))));
    const dim3 gg(nt, nt, C * ks);
    if (io32) k_gram64<float><<<gg, 256, 0, c.st>>>(reinterpret_cast<const float*>(X), p.cell_elems, T, d, n, ks, G64);
    else k_gram64<__nv_bfloat16><<<gg, 256, 0, c.st>>>(reinterpret_cast<const __nv_bfloat16*>(X), p.cell_elems, T, d, n, ks, G64);
    JOLT_CUDA_TRY(cudaGetLastError());
    if ((r = jacobi_eig64(G64, n, C, n, ev64, evec64, c.pass() + p.jac, 30, 1e-13, c.err, c.st))) return r;
    float* Ut = reinterpret_cast<float*>(c.ws + p.off_ut) + (int64_t(bg0) * 2 + kv) * int64_t(T) * q;
    const dim3 gx((q + 63) / 64, (T + 63) / 64, C);
    if (io32) k_xv64<float><<<gx, 256, 0, c.st>>>(reinterpret_cast<const float*>(X), p.cell_elems, T, d, n, evec64, ev64, q, Ut, 2 * int64_t(T) * q);
    else k_xv64<__nv_bfloat16><<<gx, 256, 0, c.st>>>(reinterpret_cast<const __nv_bfloat16*>(X), p.cell_elems, T, d, n, evec64, ev64, q, Ut, 2 * int64_t(T) * q);
    JOLT_CUDA_TRY(cudaGetLastError());
    std::vector<double> e64(size_t(C) * n);
    JOLT_CUDA_TRY(cudaMemcpyAsync(e64.data(), ev64, size_t(C) * n * 8, cudaMemcpyDeviceToHost, c.st));
    // exact feature Gram from the diagonal blocks
    double* sd64 = c.at<double>(p.sd64);
    double* evd64 = c.at<double>(p.evd64);
    double* evecd64 = c.at<double>(p.evecd64);
    k_diag_blocks<<<dim3(std::max(1, d * d / 256), C), 256, 0, c.st>>>(G64, n, d, p.LgH, sd64);
    if ((r = jacobi_eig64(sd64, d, C, d, evd64, evecd64, c.pass() + p.jac, 30, 1e-13, c.err, c.st))) return r;
    std::vector<double> d64(size_t(C) * d);
    JOLT_CUDA_TRY(cudaMemcpyAsync(d64.data(), evd64, size_t(C) * d * 8, cudaMemcpyDeviceToHost, c.st));
    nrm.resize(C);
    JOLT_CUDA_TRY(cudaMemcpyAsync(nrm.data(), nr, size_t(C) * 8, cudaMemcpyDeviceToHost, c.st));
    JOLT_CUDA_TRY(cudaStreamSynchronize(c.st));
    evT.assign(e64.begin(), e64.end());
    evD.assign(d64.begin(), d64.end());
    return JOLT_OK;
  }
  if (q > 0) {
    float* Z = c.at<float>(p.Z);
    __nv_bfloat16* Yh_b[2] = {c.at<__nv_bfloat16>(p.Yh), c.at<__nv_bfloat16>(p.Yh2)};
    __nv_bfloat16* Yl_b[2] = {c.at<__nv_bfloat16>(p.Yl), c.at<__nv_bfloat16>(p.Yl2)};
    __nv_bfloat16* Zh = c.at<__nv_bfloat16>(p.Zh);
    __nv_bfloat16* Zl = c.at<__nv_bfloat16>(p.Zl);
    const __nv_bfloat16* om = c.at<__nv_bfloat16>(p.om);
    // The sketch Y lives only as bf16 hi and lo parts written by the GEMM epilogues (its fp32 value
    // is never needed beyond its split); every orthonormalisation reads both.
    int cur = 0;
    // Y = X Omega
    {
      GemmCall g;
      g.M = T; g.N = l; g.K = n;
      g.A[0] = xunfold(Xb, kMajorK, p, C);
      g.B[0] = plain(om, kMajorK, n, l, n);
      g.Ch = Yh_b[0];
      g.Cl = Yl_b[0];
      g.ldc = l; g.c_batch_stride = int64_t(T) * l; g.batch = C; g.err = c.err;
      if ((r = run_gemm(c, g))) return r;
    }
    for (int it = 0; it < s.power_iters; ++it) {
      if ((r = orth(c, nullptr, &cur, T, C, false))) return r;
      JOLT_CUDA_TRY(cudaMemsetAsync(Z, 0, size_t(C) * n * l * 4, c.st));
      GemmCall g;
      g.M = n; g.N = l; g.K = T;
      g.A[0] = xunfold(Xb, kMajorMN, p, C);
      g.B[0] = plain(Yh_b[cur], kMajorMN, l, T, l, C, int64_t(T) * l);
      g.C = Z; g.ldc = l; g.c_batch_stride = int64_t(n) * l; g.batch = C;
      g.k_split = 0; g.accumulate = true; g.err = c.err;
      if ((r = run_gemm(c, g))) return r;
      if ((r = orth(c, Z, nullptr, n, C, false))) return r;
      if ((r = split_bf16(Z, l, n, l, C, int64_t(n) * l, Zh, nullptr, l, int64_t(n) * l, c.st))) return r;
      GemmCall h;
      h.M = T; h.N = l; h.K = n;
      h.A[0] = xunfold(Xb, kMajorK, p, C);
      h.B[0] = plain(Zh, kMajorMN, l, n, l, C, int64_t(n) * l);
      cur = 0;
      h.Ch = Yh_b[0];
      h.Cl = Yl_b[0];
      h.ldc = l; h.c_batch_stride = int64_t(T) * l; h.batch = C; h.err = c.err;
      if ((r = run_gemm(c, h))) return r;
    }
    if ((r = orth(c, nullptr, &cur, T, C, true))) return r;  // Q, as hi / lo parts in buffer cur
    __nv_bfloat16* Yh = Yh_b[cur];
    __nv_bfloat16* Yl = Yl_b[cur];
    // B^T = X^T Q  (n x l), hi/lo terms of Q
    JOLT_CUDA_TRY(cudaMemsetAsync(Z, 0, size_t(C) * n * l * 4, c.st));
    {
      GemmCall g;
      g.M = n; g.N = l; g.K = T; g.n_terms = 2;
      g.A[0] = xunfold(Xb, kMajorMN, p, C);
      g.A[1] = g.A[0];
      g.B[0] = plain(Yh, kMajorMN, l, T, l, C, int64_t(T) * l);
      g.B[1] = plain(Yl, kMajorMN, l, T, l, C, int64_t(T) * l);
      if (Xlo) {
        g.n_terms = 3;
        g.A[2] = xunfold(Xlo, kMajorMN, p, C);
        g.B[2] = g.B[0];
      }
      g.C = Z; g.ldc = l; g.c_batch_stride = int64_t(n) * l; g.batch = C;
      g.k_split = 0; g.accumulate = true; g.err = c.err;
      if ((r = run_gemm(c, g))) return r;
    }
    // W = B B^T = (B^T)^T (B^T), hi/lo terms
    if ((r = split_bf16(Z, l, n, l, C, int64_t(n) * l, Zh, Zl, l, int64_t(n) * l, c.st))) return r;
    float* W = c.at<float>(p.Gm);
    JOLT_CUDA_TRY(cudaMemsetAsync(W, 0, size_t(C) * l * l * 4, c.st));
    {
      GemmCall g;
      g.M = l; g.N = l; g.K = n; g.n_terms = 3;
      const Operand zh = plain(Zh, kMajorMN, l, n, l, C, int64_t(n) * l);
      const Operand zl = plain(Zl, kMajorMN, l, n, l, C, int64_t(n) * l);
      g.A[0] = zh; g.B[0] = zh;
      g.A[1] = zh; g.B[1] = zl;
      g.A[2] = zl; g.B[2] = zh;
      g.C = W; g.ldc = l; g.c_batch_stride = int64_t(l) * l; g.batch = C;
      g.k_split = 0; g.accumulate = true; g.err = c.err;
      g.c_upper = true;  // symmetric: the eigensolver reads the upper triangle
      if ((r = run_gemm(c, g))) return r;
    }
    float* ev = c.at<float>(p.ev);
    float* evec = c.at<float>(p.evec);
    if ((r = jacobi_eig(W, l, C, l, ev, evec, c.pass() + p.jac, 30, 1e-6, c.err, c.st))) return r;
    __nv_bfloat16* Vh = c.at<__nv_bfloat16>(p.Vh);
    __nv_bfloat16* Vl = c.at<__nv_bfloat16>(p.Vl);
    if ((r = split_bf16(evec, l, l, l, C, int64_t(l) * l, Vh, Vl, l, int64_t(l) * l, c.st))) return r;
    // U_T = Q V[:, :q]
    {
      float* Ut = reinterpret_cast<float*>(c.ws + p.off_ut) + (int64_t(bg0) * 2 + kv) * int64_t(T) * q;
      GemmCall g;
      g.M = T; g.N = q; g.K = l; g.n_terms = 3;
      const Operand qh = plain(Yh, kMajorK, l, T, l, C, int64_t(T) * l);
      const Operand ql = plain(Yl, kMajorK, l, T, l, C, int64_t(T) * l);
      const Operand vh = plain(Vh, kMajorMN, q, l, l, C, int64_t(l) * l);
      const Operand vl = plain(Vl, kMajorMN, q, l, l, C, int64_t(l) * l);
      g.A[0] = qh; g.B[0] = vh;
      g.A[1] = qh; g.B[1] = vl;
      g.A[2] = ql; g.B[2] = vh;
      g.C = Ut; g.ldc = q; g.c_batch_stride = 2 * int64_t(T) * q; g.batch = C; g.err = c.err;
      if ((r = run_gemm(c, g))) return r;
    }
    std::vector<float> e32(size_t(C) * l);
    JOLT_CUDA_TRY(cudaMemcpyAsync(e32.data(), ev, size_t(C) * l * 4, cudaMemcpyDeviceToHost, c.st));
    JOLT_CUDA_TRY(cudaStreamSynchronize(c.st));
    evT.assign(e32.begin(), e32.end());
  }
  float* evd = c.at<float>(p.evd);
  float* evecd = c.at<float>(p.evecd);
  if ((r = jacobi_eig(Sd, d, C, d, evd, evecd, c.pass() + p.jac, 30, 1e-8, c.err, c.st))) return r;
  std::vector<float> d32(size_t(C) * d);
  nrm.resize(C);
  JOLT_CUDA_TRY(cudaMemcpyAsync(d32.data(), evd, size_t(C) * d * 4, cudaMemcpyDeviceToHost, c.st));
  JOLT_CUDA_TRY(cudaMemcpyAsync(nrm.data(), nr, size_t(C) * 8, cudaMemcpyDeviceToHost, c.st));
  JOLT_CUDA_TRY(cudaStreamSynchronize(c.st));
  evD.assign(d32.begin(), d32.end());
  return JOLT_OK;
}

jolt_status read_err(const Ctx& c) {
  int32_t e = 0;
  JOLT_CUDA_TRY(cudaMemcpyAsync(&e, c.err, 4, cudaMemcpyDeviceToHost, c.st));
  JOLT_CUDA_TRY(cudaStreamSynchronize(c.st));
  return static_cast<jolt_status>(e);
}

}  // namespace

size_t compress_workspace_bytes(const jolt_shape& s) { return make_plan(s).total; }

}  // namespace jolt

using namespace jolt;

namespace jolt {
namespace {
// ready[kv] (optional): an event the stream waits on before the first pass over kind kv's cells
// (the host-to-device copy of that kind, when the inputs are streamed in).
jolt_status analyze_impl(const jolt_shape* shape, const void* k, const void* v, double* norm2_out,
                         double* tail_T_out, double* tail_d_out, void* ws, size_t ws_bytes, void* stream,
                         const cudaEvent_t* ready);
}  // namespace
}  // namespace jolt

extern "C" jolt_status jolt_analyze(const jolt_shape* shape, const void* k, const void* v, double* norm2_out,
                                    double* tail_T_out, double* tail_d_out, void* ws, size_t ws_bytes,
                                    void* stream) {
  return analyze_impl(shape, k, v, norm2_out, tail_T_out, tail_d_out, ws, ws_bytes, stream, nullptr);
}

extern "C" jolt_status jolt_analyze_from_host(const jolt_shape* shape, const void* k_host, const void* v_host,
                                              void* k_dev, void* v_dev, double* norm2_out, double* tail_T_out,
                                              double* tail_d_out, void* ws, size_t ws_bytes, void* stream) {
  if (!shape_ok(shape) || !k_host || !v_host || !k_dev || !v_dev) return JOLT_ERR_INVALID_ARG;
  const jolt_shape& s = *shape;
  const size_t bytes = size_t(s.batch) * s.n_layers * s.n_kv * size_t(s.T) * s.d_h * (s.io_dtype == JOLT_F32 ? 4 : 2);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStream_t cs = nullptr;
  cudaEvent_t ev[3] = {nullptr, nullptr, nullptr};
  auto cleanup = [&]() {
    for (cudaEvent_t& e : ev)
      if (e) cudaEventDestroy(e);
    if (cs) cudaStreamDestroy(cs);
  };
  jolt_status r = JOLT_OK;
  do {
    if (cudaStreamCreateWithFlags(&cs, cudaStreamNonBlocking) != cudaSuccess) { r = JOLT_ERR_CUDA; break; }
    bool ok = true;
    for (cudaEvent_t& e : ev) ok = ok && cudaEventCreateWithFlags(&e, cudaEventDisableTiming) == cudaSuccess;
    if (!ok) { r = JOLT_ERR_CUDA; break; }
    // the copies wait for earlier work on `stream` (which may still read k_dev / v_dev), then K and
    // V cross the bus one after the other while the key cells are being analysed
    if (cudaEventRecord(ev[0], st) != cudaSuccess || cudaStreamWaitEvent(cs, ev[0], 0) != cudaSuccess ||
        cudaMemcpyAsync(k_dev, k_host, bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaEventRecord(ev[1], cs) != cudaSuccess ||
        cudaMemcpyAsync(v_dev, v_host, bytes, cudaMemcpyHostToDevice, cs) != cudaSuccess ||
        cudaEventRecord(ev[2], cs) != cudaSuccess) {
      r = JOLT_ERR_CUDA;
      break;
    }
    r = analyze_impl(shape, k_dev, v_dev, norm2_out, tail_T_out, tail_d_out, ws, ws_bytes, stream, ev + 1);
    if (cudaStreamSynchronize(cs) != cudaSuccess && r == JOLT_OK) r = JOLT_ERR_CUDA;
  } while (false);
  cleanup();
  return r;
}

namespace jolt {
namespace {
jolt_status analyze_impl(const jolt_shape* shape, const void* k, const void* v, double* norm2_out,
                         double* tail_T_out, double* tail_d_out, void* ws, size_t ws_bytes, void* stream,
                         const cudaEvent_t* ready) {
  if (!shape_ok(shape) || !k || !v || !norm2_out || !tail_T_out || !tail_d_out || !ws) return JOLT_ERR_INVALID_ARG;
  const jolt_shape& s = *shape;
  Ctx c;
  c.s = shape;
  c.p = make_plan(s);
  if (ws_bytes < c.p.total) return JOLT_ERR_WORKSPACE;
  c.ws = static_cast<uint8_t*>(ws);
  c.err = reinterpret_cast<int32_t*>(ws);
  c.st = static_cast<cudaStream_t>(stream);
  const Plan& p = c.p;
  WsHeader hdr;
  memset(&hdr, 0, sizeof(hdr));
  JOLT_CUDA_TRY(cudaMemcpyAsync(ws, &hdr, sizeof(hdr), cudaMemcpyHostToDevice, c.st));
  if (p.qcap > 0) {
    k_omega<<<grid1(int64_t(p.l) * p.n), 256, 0, c.st>>>(c.at<__nv_bfloat16>(p.om), p.l, p.n, s.sketch_seed);
    JOLT_CUDA_TRY(cudaGetLastError());
  }
  const int per_kind = s.batch * n_groups(s);
  const int nrt = n_rt(s), nrd = n_rd(s);
  const bool exact_path = (p.l == p.n);
  for (int kv = 0; kv < 2; ++kv) {
    if (ready) JOLT_CUDA_TRY(cudaStreamWaitEvent(c.st, ready[kv], 0));
    for (int bg0 = 0; bg0 < per_kind; bg0 += p.C) {
      const int C = std::min(p.C, per_kind - bg0);
      std::vector<double> evT, evD;
      std::vector<double> nrm;
      jolt_status r = analyze_pass(c, kv ? v : k, kv, bg0, C, evT, evD, nrm);
      if (r) {
        if (kDebug) std::fprintf(stderr, "jolt analyze: pass kv %d bg0 %d status %d\n", kv, bg0, int(r));
        return r;
      }
      if ((r = read_err(c))) {
        if (kDebug) std::fprintf(stderr, "jolt analyze: device error %d after pass kv %d bg0 %d\n", int(r), kv, bg0);
        return r;
      }
      for (int i = 0; i < C; ++i) {
        const int cell = (bg0 + i) * 2 + kv;
        const double n2 = nrm[i];
        if (!std::isfinite(n2)) {
          if (kDebug) std::fprintf(stderr, "jolt analyze: cell %d norm2 %g\n", cell, n2);
          return JOLT_ERR_NUMERIC;
        }
        norm2_out[cell] = n2;
        double cum = 0.0;
        for (int kk = 0; kk < nrt; ++kk) {
          if (kk > 0)
            for (int j = (kk - 1) * kRankStep; j < kk * kRankStep; ++j) cum += std::max(0.0, evT[size_t(i) * (exact_path ? p.n : p.l) + j]);
          tail_T_out[size_t(cell) * nrt + kk] = std::max(0.0, n2 - cum);
        }
        // The eigenvalues of S_d sum to trace(S_d) = ||X||^2. The tensor-core Gram accumulates in
        // fp32 and comes out short by a near-uniform factor (~2e-5 at T = 128K), so the spectrum is
        // rescaled to the fp64 norm before the tail is taken.
        double tr = 0.0;
        for (int j = 0; j < p.d; ++j) tr += std::max(0.0, evD[size_t(i) * p.d + j]);
        const double dsc = (tr > 0.0 && n2 > 0.0) ? n2 / tr : 1.0;
        cum = 0.0;
        for (int jj = 0; jj < nrd; ++jj) {
          if (jj > 0)
            for (int j = (jj - 1) * kRankStep; j < jj * kRankStep; ++j) cum += dsc * std::max(0.0, evD[size_t(i) * p.d + j]);
          tail_d_out[size_t(cell) * nrd + jj] = std::max(0.0, n2 - cum);
        }
      }
    }
  }
  hdr.analyze_tag = shape_tag(s);
  JOLT_CUDA_TRY(cudaMemcpyAsync(&reinterpret_cast<WsHeader*>(ws)->analyze_tag, &hdr.analyze_tag, 8,
                                cudaMemcpyHostToDevice, c.st));
  JOLT_CUDA_TRY(cudaStreamSynchronize(c.st));
  return JOLT_OK;
}
}  // namespace
}  // namespace jolt

// ---- layer alignment (grouping) ----------------------------------------------------------------

namespace jolt {
namespace {

// The single-layer shape whose cells are the layers of `s`: its analyze pass finds each layer's
// top-k token directions (sketch width k + 16 capped at min(T, n_kv*d_h), two power iterations).
bool layer_shape(const jolt_shape& s, int k, jolt_shape* o) {
  if (!shape_ok(&s)) return false;
  *o = s;
  o->layers_per_group = 1;
  const int64_t lim = std::min<int64_t>(int64_t(s.n_kv) * s.d_h, s.T);
  if (k < 16 || k % kRankStep || k > lim) return false;
  int64_t l = std::min<int64_t>(lim, int64_t(k) + 16);
  l -= l % kRankStep;
  o->q_cap = k;
  o->sketch_cols = int(l);
  o->power_iters = 2;
  o->cells_per_pass = std::max(1, std::min(s.batch * s.n_layers, 32));
  return shape_ok(o);
}

// M[pair] += sum_t U1[t][i] U2[t][j] over this block's rows, pair = (b * (L-1) + l) * 2 + kv with
// U1, U2 the token bases (fp32 [T][k]) of layers l and l + 1 of sequence b, kind kv.
constexpr int kAlignMaxK = 128;
__global__ void __launch_bounds__(256) k_align(const float* __restrict__ Ut, int64_t cell_elems, int T, int k,
                                               int L, int rows_per_block, double* __restrict__ M) {
  constexpr int kMaxE = kAlignMaxK * kAlignMaxK / 256;
  __shared__ float s1[32][kAlignMaxK + 1], s2[32][kAlignMaxK + 1];
  const int pair = blockIdx.y;
  const int kv = pair & 1, bl = pair >> 1;
  const int b = bl / (L - 1), l = bl % (L - 1);
  const float* U1 = Ut + int64_t((b * L + l) * 2 + kv) * cell_elems;
  const float* U2 = Ut + int64_t((b * L + l + 1) * 2 + kv) * cell_elems;
  const int t0 = blockIdx.x * rows_per_block, t1 = min(T, t0 + rows_per_block);
  float acc[kMaxE];
#pragma unroll
  for (int j = 0; j < kMaxE; ++j) acc[j] = 0.f;
  for (int r0 = t0; r0 < t1; r0 += 32) {
    __syncthreads();
    for (int e = threadIdx.x; e < 32 * k; e += 256) {
      const int rr = e / k, c = e % k, t = r0 + rr;
      s1[rr][c] = t < t1 ? U1[int64_t(t) * k + c] : 0.f;
      s2[rr][c] = t < t1 ? U2[int64_t(t) * k + c] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int j = 0; j < kMaxE; ++j) {
      const int e = threadIdx.x + 256 * j;
      if (e < k * k) {
        const int i = e / k, c = e % k;
        float a = acc[j];
#pragma unroll 8
        for (int rr = 0; rr < 32; ++rr) a = fmaf(s1[rr][i], s2[rr][c], a);
        acc[j] = a;
      }
    }
  }
#pragma unroll
  for (int j = 0; j < kMaxE; ++j) {
    const int e = threadIdx.x + 256 * j;
    if (e < k * k) atomicAdd(&M[int64_t(pair) * k * k + e], double(acc[j]));
  }
}

}  // namespace
}  // namespace jolt

extern "C" size_t jolt_layer_align_workspace(const jolt_shape* shape, int32_t k) {
  jolt_shape s1;
  if (!shape || !layer_shape(*shape, k, &s1) || k > kAlignMaxK) return 0;
  const size_t npairs = size_t(shape->batch) * std::max(0, shape->n_layers - 1) * 2;
  return align_up(make_plan(s1).total, 256) + npairs * size_t(k) * k * 8;
}

extern "C" jolt_status jolt_layer_align(const jolt_shape* shape, int32_t k, const void* K, const void* V,
                                        double* align, void* ws, size_t ws_bytes, void* stream) {
  jolt_shape s1;
  if (!shape || !layer_shape(*shape, k, &s1) || k > kAlignMaxK || !K || !V || !align || !ws)
    return JOLT_ERR_INVALID_ARG;
  const jolt_shape& s = *shape;
  if (s.n_layers < 2) return JOLT_OK;
  if (ws_bytes < jolt_layer_align_workspace(shape, k)) return JOLT_ERR_WORKSPACE;
  const Plan p = make_plan(s1);
  const int ncell = n_cells(s1);
  std::vector<double> n2(ncell), tT(size_t(ncell) * n_rt(s1)), td(size_t(ncell) * n_rd(s1));
  jolt_status r = jolt_analyze(&s1, K, V, n2.data(), tT.data(), td.data(), ws, p.total, stream);
  if (r) return r;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int npairs = s.batch * (s.n_layers - 1) * 2;
  double* M = reinterpret_cast<double*>(static_cast<uint8_t*>(ws) + align_up(p.total, 256));
  JOLT_CUDA_TRY(cudaMemsetAsync(M, 0, size_t(npairs) * k * k * 8, st));
  const float* Ut = reinterpret_cast<const float*>(static_cast<uint8_t*>(ws) + p.off_ut);
  const int rows_per_block = 2048;
  const dim3 grid(unsigned((s.T + rows_per_block - 1) / rows_per_block), unsigned(npairs));
  k_align<<<grid, 256, 0, st>>>(Ut, int64_t(s.T) * k, s.T, k, s.n_layers, rows_per_block, M);
  JOLT_CUDA_TRY(cudaGetLastError());
  std::vector<double> h(size_t(npairs) * k * k);
  JOLT_CUDA_TRY(cudaMemcpyAsync(h.data(), M, h.size() * 8, cudaMemcpyDeviceToHost, st));
  JOLT_CUDA_TRY(cudaStreamSynchronize(st));
  for (int bl = 0; bl < s.batch * (s.n_layers - 1); ++bl) {
    double f[2] = {0.0, 0.0};
    for (int kv = 0; kv < 2; ++kv) {
      const double* m = h.data() + size_t(bl * 2 + kv) * k * k;
      for (int e = 0; e < k * k; ++e) f[kv] += m[e] * m[e];
    }
    align[bl] = (f[0] + f[1]) / (2.0 * k);
  }
  return JOLT_OK;
}

extern "C" jolt_status jolt_compress(const jolt_shape* shape, const void* k, const void* v,
                                     const jolt_cell_choice* choices, void* cache, uint64_t cache_bytes, void* ws,
                                     size_t ws_bytes, void* stream) {
  if (!shape_ok(shape) || !k || !v || !choices || !cache || !ws) return JOLT_ERR_INVALID_ARG;
  const jolt_shape& s = *shape;
  Ctx c;
  c.s = shape;
  c.p = make_plan(s);
  const Plan& p = c.p;
  if (ws_bytes < p.total) return JOLT_ERR_WORKSPACE;
  c.ws = static_cast<uint8_t*>(ws);
  c.err = reinterpret_cast<int32_t*>(ws);
  c.st = static_cast<cudaStream_t>(stream);
  uint64_t total = 0;
  const int nc = n_cells(s);
  std::vector<uint64_t> offs(size_t(nc) * 5);
  jolt_status r = jolt_cache_layout(shape, choices, offs.data(), &total);
  if (r) return r;
  if (cache_bytes < total) return JOLT_ERR_INVALID_ARG;
  uint64_t tag = 0;
  JOLT_CUDA_TRY(cudaMemcpyAsync(&tag, &reinterpret_cast<WsHeader*>(ws)->analyze_tag, 8, cudaMemcpyDeviceToHost, c.st));
  JOLT_CUDA_TRY(cudaStreamSynchronize(c.st));
  if (tag != shape_tag(s)) return JOLT_ERR_STATE;
  const bool io32 = s.io_dtype == JOLT_F32, f32 = s.factor_dtype == JOLT_F32;
  const int T = p.T, d = p.d, q = p.qcap, LgH = p.LgH;
  uint8_t* cb = static_cast<uint8_t*>(cache);
  // U's GEMM parts for one cell: hi (the stored value for bf16 factors), lo (and mid for fp32 factors)
  auto store_u = [&](int cell, int rT, __nv_bfloat16*& uh, __nv_bfloat16*& ul, __nv_bfloat16*& um) {
    const float* U = reinterpret_cast<const float*>(c.ws + p.off_ut) + int64_t(cell) * T * q;
    uint8_t* cut = cb + offs[5 * cell + 0];
    uh = f32 ? c.atc<__nv_bfloat16>(p.uh) : reinterpret_cast<__nv_bfloat16*>(cut);
    ul = c.atc<__nv_bfloat16>(p.ul);
    um = f32 ? c.atc<__nv_bfloat16>(p.um) : nullptr;
    k_store_ut<<<grid1(int64_t(T) * rT), 256, 0, c.st>>>(U, T, q, rT, f32, cut, f32 ? uh : nullptr, um, ul);
  };
  for (int c0 = 0; c0 < nc; c0 += p.cc) {
    const int c1 = std::min(nc, c0 + p.cc);
    // ---- per cell: Y_lh = U_T^T X_lh [LgH][rT][d] and S_Y (slot = rank among the chunk's
    // cells with r_T > 0) ----
    int nact = 0;
    int slot_of[kCmpChunk];
    for (int cell = c0; cell < c1; ++cell) {
      const jolt_cell_choice ch = choices[cell];
      slot_of[cell - c0] = -1;
      if (ch.r_T <= 0) continue;
      const int slot = nact++;
      slot_of[cell - c0] = slot;
      const int bg = cell / 2, kv = cell % 2, rT = ch.r_T;
      const uint8_t* Xk = static_cast<const uint8_t*>(kv ? v : k) + int64_t(bg) * p.cell_elems * (io32 ? 4 : 2);
      __nv_bfloat16 *uh, *ul, *um;
      store_u(cell, rT, uh, ul, um);
      // the cell's X as bf16 for the tensor cores (f32 inputs: hi + lo copies first)
      const void* Xb = Xk;
      const void* Xlo = nullptr;
      if (io32) {
        __nv_bfloat16* xh = c.at<__nv_bfloat16>(p.xb);
        __nv_bfloat16* xl = xh + p.cell_elems;
        if ((r = split_bf16(reinterpret_cast<const float*>(Xk), 1, p.cell_elems, 1, 1, 0, xh, xl, 1, 0, c.st))) return r;
        Xb = xh;
        Xlo = xl;
      }
      float* ylh = c.atc<float>(p.ylh) + int64_t(slot) * LgH * q * d;
      JOLT_CUDA_TRY(cudaMemsetAsync(ylh, 0, size_t(LgH) * rT * d * 4, c.st));
      {
        // projection with the unrounded basis: (U_hi, X_hi) + (U_hi, X_lo) + (U_2nd, X_hi)
        GemmCall g;
        g.M = rT; g.N = d; g.K = T;
        const Operand xh = plain(Xb, kMajorMN, d, T, d, LgH, int64_t(T) * d);
        const Operand uhh = plain(uh, kMajorMN, rT, T, rT, LgH, 0);
        int nt = 0;
        g.A[nt] = uhh; g.B[nt] = xh; ++nt;
        if (Xlo) { g.A[nt] = uhh; g.B[nt] = plain(Xlo, kMajorMN, d, T, d, LgH, int64_t(T) * d); ++nt; }
        g.A[nt] = plain(f32 ? um : ul, kMajorMN, rT, T, rT, LgH, 0); g.B[nt] = xh; ++nt;
        g.n_terms = nt;
        g.C = ylh; g.ldc = d; g.c_batch_stride = int64_t(rT) * d; g.batch = LgH;
        g.k_split = 0; g.accumulate = true; g.err = c.err;
        if ((r = run_gemm(c, g))) return r;
      }
      float* sy = c.atc<float>(p.sy) + int64_t(slot) * d * d;
      JOLT_CUDA_TRY(cudaMemsetAsync(sy, 0, size_t(d) * d * 4, c.st));
      {
        const int nrows = LgH * rT;
        const int gx = std::max(1, std::min(64, nrows / 256));
        k_gram_small<<<dim3(gx, (d + 31) / 32, (d + 31) / 32), 256, 32 * 64 * 4, c.st>>>(ylh, nrows, d, sy);
      }
    }
    // ---- the chunk's S_Y eigenproblems in one launch ----
    float* evy = c.atc<float>(p.evy);
    float* evecy = c.atc<float>(p.evecy);
    if (nact > 0 &&
        (r = jacobi_eig(c.atc<float>(p.sy), d, nact, d, evy, evecy, c.ws + p.off_cmp + p.jac2, 30, 1e-8, c.err, c.st)))
      return r;
    // ---- per cell: U_d, G, X~, residual ----
    for (int cell = c0; cell < c1; ++cell) {
      const int bg = cell / 2, kv = cell % 2;
      const jolt_cell_choice ch = choices[cell];
      const uint8_t* Xk = static_cast<const uint8_t*>(kv ? v : k) + int64_t(bg) * p.cell_elems * (io32 ? 4 : 2);
      float* Xt = nullptr;
      bool coded = false;  // residual already coded by the fused X~ GEMM
      if (ch.r_T > 0) {
        const int rT = ch.r_T, rd = ch.r_d, slot = slot_of[cell - c0];
        uint8_t* cud = cb + offs[5 * cell + 1];
        uint8_t* cg = cb + offs[5 * cell + 2];
        const float* ylh = c.atc<float>(p.ylh) + int64_t(slot) * LgH * q * d;
        const float* evs = evecy + int64_t(slot) * d * d;
        // U_d = first rd eigenvector columns (stored dtype), then G = Y U_d (stored dtype)
        k_store_ut<<<grid1(int64_t(d) * rd), 256, 0, c.st>>>(evs, d, d, rd, f32, cud, nullptr, nullptr, nullptr);
        k_proj_small<<<grid1(int64_t(LgH) * rT * rd), 256, 0, c.st>>>(ylh, int64_t(LgH) * rT, d, evs, d, rd, f32, cg);
      }
      if (ch.r_T > 0 && ch.b > 0) {
        // X~ = U^s B with B = G^s U_d^s^T, to fp32 accuracy: 3-way bf16 splits, terms of order <= 2
        // (only the residual needs it: a cell without one stores the factors alone)
        const int rT = ch.r_T, rd = ch.r_d;
        uint8_t* cud = cb + offs[5 * cell + 1];
        uint8_t* cg = cb + offs[5 * cell + 2];
        __nv_bfloat16 *uh, *ul, *um;
        if (f32) store_u(cell, rT, uh, ul, um);  // the scratch parts were overwritten by later cells
        else {
          uh = reinterpret_cast<__nv_bfloat16*>(cb + offs[5 * cell + 0]);
          ul = um = nullptr;
        }
        float* xt = c.atc<float>(p.xt);
        __nv_bfloat16* bh = c.atc<__nv_bfloat16>(p.bh);
        __nv_bfloat16* bm = c.atc<__nv_bfloat16>(p.bm);
        __nv_bfloat16* bl = c.atc<__nv_bfloat16>(p.bl);
        float* blh = c.atc<float>(p.blh);
        {
          const int64_t nrows = int64_t(LgH) * rT;
          const unsigned gb = unsigned((nrows + 31) / 32);
          if (d == 128) k_recon_b<128><<<gb, 256, 0, c.st>>>(cg, cud, nrows, rd, f32, blh);
          else k_recon_b<64><<<gb, 256, 0, c.st>>>(cg, cud, nrows, rd, f32, blh);
        }
        if ((r = split3_bf16(blh, int64_t(LgH) * rT * d, bh, bm, bl, c.st))) return r;
        {
          GemmCall g;
          g.M = T; g.N = d; g.K = rT;
          const Operand Bp[3] = {plain(bh, kMajorMN, d, rT, d, LgH, int64_t(rT) * d),
                                 plain(bm, kMajorMN, d, rT, d, LgH, int64_t(rT) * d),
                                 plain(bl, kMajorMN, d, rT, d, LgH, int64_t(rT) * d)};
          const Operand Up[3] = {plain(uh, kMajorK, rT, T, rT, LgH, 0), plain(um, kMajorK, rT, T, rT, LgH, 0),
                                 plain(ul, kMajorK, rT, T, rT, LgH, 0)};
          const int nu = f32 ? 3 : 1;
          int nt = 0;
          for (int i = 0; i < nu; ++i)
            for (int jj = 0; jj < 3; ++jj)
              if (i + jj <= 2) {
                g.A[nt] = Up[i];
                g.B[nt] = Bp[jj];
                ++nt;
              }
          g.n_terms = nt;
          g.batch = LgH; g.err = c.err;
          // d = 128: the GEMM's epilogue codes the residual rows X - X~ directly (X~ never
          // reaches memory); otherwise X~ is stored and coded by k_residual
          uint8_t* codes = cb + offs[5 * cell + 3];
          void* szp = cb + offs[5 * cell + 4];
          ResidualEpi e;
          e.X = Xk; e.x_f32 = io32 ? 1 : 0; e.T = T; e.seed = s.rot_seed; e.b = ch.b;
          e.codes = codes; e.sz = szp;
          const bool fuse = d == 128 && reinterpret_cast<uintptr_t>(codes) % 16 == 0 &&
                            reinterpret_cast<uintptr_t>(Xk) % 16 == 0 && reinterpret_cast<uintptr_t>(szp) % 4 == 0;
          if (fuse) {
            g.res = &e;
            const int64_t rows = int64_t(LgH) * T;
            StatScope sc(JOLT_K_RESIDUAL, c.st, 0.0, double(rows) * d * (io32 ? 4 : 2) + double(rows) * (d * ch.b / 8 + 4));
            if ((r = run_gemm(c, g))) return r;
            coded = true;
          } else {
            g.C = xt; g.ldc = d; g.c_batch_stride = int64_t(T) * d;
            if ((r = run_gemm(c, g))) return r;
            Xt = xt;
          }
        }
      }
      if (ch.b > 0 && !coded) {
        uint8_t* codes = cb + offs[5 * cell + 3];
        __half2* sz = reinterpret_cast<__half2*>(cb + offs[5 * cell + 4]);
        const int64_t rows = int64_t(LgH) * T;
        const int grid = int(std::min<int64_t>((rows + 7) / 8, 148 * 16));
        // algorithmic bytes: read X (io dtype) and X~ (fp32, when present), write codes and sz
        StatScope sc(JOLT_K_RESIDUAL, c.st, 0.0,
                     double(rows) * d * ((io32 ? 4 : 2) + (Xt ? 4 : 0)) + double(rows) * (d * ch.b / 8 + 4));
        if (d == 128) {
          if (io32) k_residual<4, float><<<grid, 256, 0, c.st>>>(reinterpret_cast<const float*>(Xk), Xt, rows, ch.b, s.rot_seed, codes, sz, c.err);
          else k_residual<4, __nv_bfloat16><<<grid, 256, 0, c.st>>>(reinterpret_cast<const __nv_bfloat16*>(Xk), Xt, rows, ch.b, s.rot_seed, codes, sz, c.err);
        } else {
          if (io32) k_residual<2, float><<<grid, 256, 0, c.st>>>(reinterpret_cast<const float*>(Xk), Xt, rows, ch.b, s.rot_seed, codes, sz, c.err);
          else k_residual<2, __nv_bfloat16><<<grid, 256, 0, c.st>>>(reinterpret_cast<const __nv_bfloat16*>(Xk), Xt, rows, ch.b, s.rot_seed, codes, sz, c.err);
        }
        JOLT_CUDA_TRY(cudaGetLastError());
      }
    }
  }
  return read_err(c);
}
