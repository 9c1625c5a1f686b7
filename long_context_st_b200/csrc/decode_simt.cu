// Decode attention over the stored JoLT factors — CUDA-core (fp32 FMA) kernels.
//
// This path serves fp32 caches (where bf16 tensor-core operands would break the fp32 accuracy
// target) and any shape the tensor-core kernels do not cover. Three launches per call:
//   prologue : per query head, q_rot = R q, qsum = sum(q_rot); non-RoPE keys: P = G^K (U_d^K^T q);
//              pre-RoPE keys (per KV head): B_h = G^K_h U_d^K^T  (r_T x d_h)
//   main     : split-T flash decoding; per token tile the scores (U_T P + scale*(q_rot.code) +
//              zero*qsum, or q . RoPE(U_T B_h + R^T deq(codes))), an online softmax, and the value
//              accumulators w += p U_T^V, acc += p deq(codes^V) (rotated domain)
//   merge    : log-sum-exp merge of the splits, out = (U_d^V (G^V^T w) + R^T acc) / l.
#include "common.cuh"
#include "decode.cuh"
#include "pack.cuh"
#include "stats.h"

namespace jolt {

__device__ __forceinline__ SegOffsets cell_segs(const DecodeParams& p, const CellRef& c) {
  return seg_offsets(p.T, p.d_h, p.Lg, p.n_kv, p.fac_f32 ? 4 : 2, c.r_T, c.r_d, c.b);
}

__device__ __forceinline__ float ld_fac(const DecodeParams& p, const uint8_t* base, int64_t i) {
  return p.fac_f32 ? reinterpret_cast<const float*>(base)[i]
                   : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
}
__device__ __forceinline__ float ld_io(const DecodeParams& p, const void* base, int64_t i) {
  return p.io_f32 ? reinterpret_cast<const float*>(base)[i]
                  : __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(base)[i]);
}

// ---- prologue over query heads --------------------------------------------------------------
template <int E>
__global__ void k_prologue_q(DecodeParams p) {
  constexpr int D = 32 * E;
  const int hq = blockIdx.x, li = blockIdx.y, b = blockIdx.z;
  const int layer = p.layer_begin + li, g = layer / p.Lg, ll = layer % p.Lg, h = hq / p.gq;
  const CellRef ck = p.cells[(b * p.Gc + (g - p.g_first)) * 2 + 0];
  const SegOffsets so = cell_segs(p, ck);
  const int64_t qrow = ((int64_t(b) * p.Lc + li) * p.n_q + hq);
  __shared__ float qs[D];
  __shared__ float qhat[128];
  for (int i = threadIdx.x; i < D; i += blockDim.x) qs[i] = ld_io(p, p.q, qrow * D + i);
  __syncthreads();
  if (threadIdx.x < 32) {
    float v[E];
#pragma unroll
    for (int i = 0; i < E; ++i) v[i] = qs[threadIdx.x * E + i];
    warp_rotate<E>(v, p.rot_seed, rsqrtf(float(D)));
    float sum = 0.f;
#pragma unroll
    for (int i = 0; i < E; ++i) {
      p.ws_qrot[qrow * D + threadIdx.x * E + i] = v[i];
      sum += v[i];
    }
    sum = warp_sum(sum);
    if (threadIdx.x == 0) p.ws_qsum[qrow] = sum;
  }
  if (p.pre_rope || p.skip_p || ck.r_T == 0) return;
  const uint8_t* Ud = p.cache + ck.offset + so.ud;
  const uint8_t* G = p.cache + ck.offset + so.g + (int64_t(ll) * p.n_kv + h) * ck.r_T * ck.r_d *
                     (p.fac_f32 ? 4 : 2);
  for (int j = threadIdx.x; j < ck.r_d; j += blockDim.x) {
    float a = 0.f;
    for (int i = 0; i < D; ++i) a += ld_fac(p, Ud, int64_t(i) * ck.r_d + j) * qs[i];
    qhat[j] = a;
  }
  __syncthreads();
  float* P = p.ws_P + qrow * p.q_cap;
  for (int r = threadIdx.x; r < ck.r_T; r += blockDim.x) {
    float a = 0.f;
    for (int j = 0; j < ck.r_d; ++j) a += ld_fac(p, G, int64_t(r) * ck.r_d + j) * qhat[j];
    P[r] = a;
  }
}

// ---- prologue over KV heads (pre-RoPE keys): B_h = G_h U_d^T --------------------------------
__global__ void k_prologue_bh(DecodeParams p) {
  const int h = blockIdx.x, li = blockIdx.y, b = blockIdx.z;
  const int layer = p.layer_begin + li, g = layer / p.Lg, ll = layer % p.Lg;
  const CellRef ck = p.cells[(b * p.Gc + (g - p.g_first)) * 2 + 0];
  if (ck.r_T == 0) return;
  const SegOffsets so = cell_segs(p, ck);
  const uint8_t* Ud = p.cache + ck.offset + so.ud;
  const uint8_t* G = p.cache + ck.offset + so.g + (int64_t(ll) * p.n_kv + h) * ck.r_T * ck.r_d *
                     (p.fac_f32 ? 4 : 2);
  float* Bh = p.ws_Bh + ((int64_t(b) * p.Lc + li) * p.n_kv + h) * int64_t(p.q_cap) * p.d_h;
  const int64_t n = int64_t(ck.r_T) * p.d_h;
  for (int64_t e = threadIdx.x; e < n; e += blockDim.x) {
    const int r = int(e / p.d_h), i = int(e % p.d_h);
    float a = 0.f;
    for (int j = 0; j < ck.r_d; ++j)
      a += ld_fac(p, G, int64_t(r) * ck.r_d + j) * ld_fac(p, Ud, int64_t(i) * ck.r_d + j);
    Bh[e] = a;
  }
}

// ---- main split-T kernel ------------------------------------------------------------------------
// grid (S, n_kv, B*Lc), 256 threads; tiles of 32 tokens; g_q <= 16 query heads per KV head.
constexpr int kTile = 32;
constexpr int kMaxGq = 16;

template <int E>
__global__ void __launch_bounds__(256) k_decode_main(DecodeParams p) {
  constexpr int D = 32 * E;
  const int split = blockIdx.x, h = blockIdx.y;
  const int b = blockIdx.z / p.Lc, li = blockIdx.z % p.Lc;
  const int layer = p.layer_begin + li, g = layer / p.Lg, ll = layer % p.Lg;
  const CellRef ck = p.cells[(b * p.Gc + (g - p.g_first)) * 2 + 0];
  const CellRef cv = p.cells[(b * p.Gc + (g - p.g_first)) * 2 + 1];
  const SegOffsets sk = cell_segs(p, ck), sv = cell_segs(p, cv);
  const int gq = p.gq, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int chunk = ((p.T + p.S - 1) / p.S + kTile - 1) / kTile * kTile;
  const int t_begin = split * chunk, t_end = min(p.T, t_begin + chunk);

  extern __shared__ float smem[];
  float* s_P = smem;                                 // [gq][q_cap]   (non-RoPE)
  float* s_q = s_P + (p.pre_rope ? 0 : gq * p.q_cap);  // [gq][D] q_rot (non-RoPE) or q (pre-RoPE)
  float* s_k = s_q + gq * D;                         // [kTile][D] reconstructed keys (pre-RoPE)
  float* s_s = s_k + (p.pre_rope ? kTile * D : 0);   // [kTile][gq] scores -> probabilities
  float* s_w = s_s + kTile * kMaxGq;                 // [gq][q_cap] value factor accumulators
  float* s_acc = s_w + gq * p.q_cap;                 // [gq][D] rotated residual accumulators
  float* s_m = s_acc + gq * D;                       // [gq]
  float* s_l = s_m + kMaxGq;                         // [gq]
  float* s_alpha = s_l + kMaxGq;                     // [gq]
  float* s_qsum = s_alpha + kMaxGq;                  // [gq]

  const int64_t qrow0 = (int64_t(b) * p.Lc + li) * p.n_q + int64_t(h) * gq;
  for (int e = tid; e < gq * D; e += blockDim.x) {
    const int hq = e / D, i = e % D;
    s_q[e] = p.pre_rope ? ld_io(p, p.q, (qrow0 + hq) * D + i) : p.ws_qrot[(qrow0 + hq) * D + i];
  }
  if (!p.pre_rope)
    for (int e = tid; e < gq * ck.r_T; e += blockDim.x) {
      const int hq = e / ck.r_T, r = e % ck.r_T;
      s_P[hq * p.q_cap + r] = p.ws_P[(qrow0 + hq) * p.q_cap + r];
    }
  for (int e = tid; e < gq * p.q_cap; e += blockDim.x) s_w[e] = 0.f;
  for (int e = tid; e < gq * D; e += blockDim.x) s_acc[e] = 0.f;
  if (tid < kMaxGq) {
    s_m[tid] = -INFINITY;
    s_l[tid] = 0.f;
    s_qsum[tid] = (tid < gq) ? p.ws_qsum[qrow0 + tid] : 0.f;
  }
  __syncthreads();

  const uint8_t* UtK = p.cache + ck.offset + sk.ut;
  const uint8_t* UtV = p.cache + cv.offset + sv.ut;
  const int64_t row_k = (int64_t(ll) * p.n_kv + h) * p.T;  // row index base of this (layer, head)
  const uint8_t* codesK = p.cache + ck.offset + sk.codes;
  const __half2* szK = reinterpret_cast<const __half2*>(p.cache + ck.offset + sk.sz);
  const uint8_t* codesV = p.cache + cv.offset + sv.codes;
  const __half2* szV = reinterpret_cast<const __half2*>(p.cache + cv.offset + sv.sz);
  const int nbK = D * ck.b / 8, nbV = D * cv.b / 8;
  const float* Bh = p.ws_Bh + ((int64_t(b) * p.Lc + li) * p.n_kv + h) * int64_t(p.q_cap) * D;

  for (int t0 = t_begin; t0 < t_end; t0 += kTile) {
    const int nt = min(kTile, t_end - t0);
    // ---- scores ----
    if (!p.pre_rope) {
      // warp w handles tokens w, w+8, w+16, w+24
      for (int tt = warp; tt < nt; tt += 8) {
        const int t = t0 + tt;
        float acc[kMaxGq];
#pragma unroll
        for (int k = 0; k < kMaxGq; ++k) acc[k] = 0.f;
        for (int r = lane; r < ck.r_T; r += 32) {
          const float u = ld_fac(p, UtK, int64_t(t) * ck.r_T + r);
#pragma unroll
          for (int k = 0; k < kMaxGq; ++k)
            if (k < gq) acc[k] += u * s_P[k * p.q_cap + r];
        }
        // residual part: scale * (q_rot . code) + zero * qsum
        float rd[kMaxGq];
#pragma unroll
        for (int k = 0; k < kMaxGq; ++k) rd[k] = 0.f;
        if (ck.b) {
          const uint8_t* row = codesK + (row_k + t) * nbK;
#pragma unroll
          for (int i = 0; i < E; ++i) {
            const float c = float(unpack_code(row, lane * E + i, ck.b));
#pragma unroll
            for (int k = 0; k < kMaxGq; ++k)
              if (k < gq) rd[k] += c * s_q[k * D + lane * E + i];
          }
        }
#pragma unroll
        for (int k = 0; k < kMaxGq; ++k) {
          if (k < gq) {
            const float a = warp_sum(acc[k]);
            const float c = warp_sum(rd[k]);
            if (lane == 0) {
              float sres = 0.f;
              if (ck.b) {
                const __half2 sz = szK[row_k + t];
                sres = __low2float(sz) * c + __high2float(sz) * s_qsum[k];
              }
              s_s[tt * kMaxGq + k] = (a + sres) * p.attn_scale;
            }
          }
        }
      }
    } else {
      // reconstruct keys: k_t = U_T[t] B_h (+ R^T deq(codes)), then RoPE at position pos0 + t
      for (int e = tid; e < nt * D; e += blockDim.x) {
        const int tt = e / D, i = e % D;
        const int t = t0 + tt;
        float a = 0.f;
        for (int r = 0; r < ck.r_T; ++r)
          a += ld_fac(p, UtK, int64_t(t) * ck.r_T + r) * Bh[int64_t(r) * D + i];
        s_k[tt * D + i] = a;
      }
      __syncthreads();
      if (ck.b) {
        for (int tt = warp; tt < nt; tt += 8) {
          const int t = t0 + tt;
          const uint8_t* row = codesK + (row_k + t) * nbK;
          const __half2 sz = szK[row_k + t];
          float v[E];
#pragma unroll
          for (int i = 0; i < E; ++i)
            v[i] = dequant(unpack_code(row, lane * E + i, ck.b), __low2float(sz), __high2float(sz));
          warp_unrotate<E>(v, p.rot_seed, rsqrtf(float(D)));
#pragma unroll
          for (int i = 0; i < E; ++i) s_k[tt * D + lane * E + i] += v[i];
        }
        __syncthreads();
      }
      for (int e = tid; e < nt * (D / 2); e += blockDim.x) {
        const int tt = e / (D / 2), i = e % (D / 2);
        const double ang = double(p.pos_offset + t0 + tt) * double(p.inv_freq[i]);
        const double red = ang - 6.283185307179586 * rint(ang * 0.15915494309189535);
        float sn, cs;
        sincosf(float(red), &sn, &cs);
        cs *= p.rope_scaling;
        sn *= p.rope_scaling;
        const float x1 = s_k[tt * D + i], x2 = s_k[tt * D + i + D / 2];
        s_k[tt * D + i] = x1 * cs - x2 * sn;
        s_k[tt * D + i + D / 2] = x2 * cs + x1 * sn;
      }
      __syncthreads();
      for (int tt = warp; tt < nt; tt += 8) {
#pragma unroll
        for (int k = 0; k < kMaxGq; ++k) {
          if (k < gq) {
            float a = 0.f;
#pragma unroll
            for (int i = 0; i < E; ++i) a += s_k[tt * D + lane * E + i] * s_q[k * D + lane * E + i];
            a = warp_sum(a);
            if (lane == 0) s_s[tt * kMaxGq + k] = a * p.attn_scale;
          }
        }
      }
    }
    __syncthreads();
    // ---- online softmax per query head ----
    if (tid < gq) {
      float mx = s_m[tid];
      for (int tt = 0; tt < nt; ++tt) mx = fmaxf(mx, s_s[tt * kMaxGq + tid]);
      const float alpha = __expf(s_m[tid] - mx);
      float lsum = 0.f;
      for (int tt = 0; tt < nt; ++tt) {
        const float pr = __expf(s_s[tt * kMaxGq + tid] - mx);
        s_s[tt * kMaxGq + tid] = pr;
        lsum += pr;
      }
      s_l[tid] = s_l[tid] * alpha + lsum;
      s_m[tid] = mx;
      s_alpha[tid] = alpha;
    }
    __syncthreads();
    // ---- value accumulators ----
    for (int e = tid; e < gq * cv.r_T; e += blockDim.x) {
      const int hq = e / cv.r_T, r = e % cv.r_T;
      float a = s_w[hq * p.q_cap + r] * s_alpha[hq];
      for (int tt = 0; tt < nt; ++tt)
        a += s_s[tt * kMaxGq + hq] * ld_fac(p, UtV, int64_t(t0 + tt) * cv.r_T + r);
      s_w[hq * p.q_cap + r] = a;
    }
    for (int e = tid; e < gq * D; e += blockDim.x) {
      const int hq = e / D, j = e % D;
      float a = s_acc[e] * s_alpha[hq];
      if (cv.b) {
        for (int tt = 0; tt < nt; ++tt) {
          const int64_t rr = row_k + t0 + tt;
          const __half2 sz = szV[rr];
          const float dv = dequant(unpack_code(codesV + rr * nbV, j, cv.b), __low2float(sz), __high2float(sz));
          a += s_s[tt * kMaxGq + hq] * dv;
        }
      }
      s_acc[e] = a;
    }
    __syncthreads();
  }
  // ---- write partials ----
  const int row = 2 + p.q_cap + D;
  for (int hq = 0; hq < gq; ++hq) {
    float* part = p.ws_part + ((qrow0 + hq) * p.S + split) * int64_t(row);
    if (tid == 0) {
      part[0] = s_m[hq];
      part[1] = s_l[hq];
    }
    for (int r = tid; r < cv.r_T; r += blockDim.x) part[2 + r] = s_w[hq * p.q_cap + r];
    for (int j = tid; j < D; j += blockDim.x) part[2 + p.q_cap + j] = s_acc[hq * D + j];
  }
}

// ---- merge --------------------------------------------------------------------------------------
template <int E>
__global__ void k_decode_merge(DecodeParams p) {
  constexpr int D = 32 * E;
  const int hq = blockIdx.x, li = blockIdx.y, b = blockIdx.z;
  const int layer = p.layer_begin + li, g = layer / p.Lg, ll = layer % p.Lg, h = hq / p.gq;
  const CellRef cv = p.cells[(b * p.Gc + (g - p.g_first)) * 2 + 1];
  const SegOffsets sv = cell_segs(p, cv);
  const int64_t qrow = (int64_t(b) * p.Lc + li) * p.n_q + hq;
  const int row = 2 + p.q_cap + D;
  const float* part = p.ws_part + qrow * p.S * int64_t(row);
  extern __shared__ float sm[];
  float* w = sm;                 // [q_cap]
  float* v = w + p.q_cap;        // [128] G^T w
  float* acc = v + 128;          // [D]
  float* coef = acc + D;         // [S]
  __shared__ float s_M, s_L;
  if (threadIdx.x == 0) {
    float M = -INFINITY;
    for (int s = 0; s < p.S; ++s) M = fmaxf(M, part[s * row]);
    float L = 0.f;
    for (int s = 0; s < p.S; ++s) {
      const float m = part[s * row];
      const float c = (m == -INFINITY) ? 0.f : __expf(m - M);
      coef[s] = c;
      L += c * part[s * row + 1];
    }
    s_M = M;
    s_L = L;
  }
  __syncthreads();
  for (int r = threadIdx.x; r < cv.r_T; r += blockDim.x) {
    float a = 0.f;
    for (int s = 0; s < p.S; ++s) a += coef[s] * part[s * row + 2 + r];
    w[r] = a;
  }
  for (int j = threadIdx.x; j < D; j += blockDim.x) {
    float a = 0.f;
    for (int s = 0; s < p.S; ++s) a += coef[s] * part[s * row + 2 + p.q_cap + j];
    acc[j] = a;
  }
  __syncthreads();
  const uint8_t* Ud = p.cache + cv.offset + sv.ud;
  const uint8_t* G = p.cache + cv.offset + sv.g + (int64_t(ll) * p.n_kv + h) * cv.r_T * cv.r_d *
                     (p.fac_f32 ? 4 : 2);
  for (int j = threadIdx.x; j < cv.r_d; j += blockDim.x) {
    float a = 0.f;
    for (int r = 0; r < cv.r_T; ++r) a += ld_fac(p, G, int64_t(r) * cv.r_d + j) * w[r];
    v[j] = a;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    float x[E];
#pragma unroll
    for (int i = 0; i < E; ++i) x[i] = acc[threadIdx.x * E + i];
    if (cv.b) warp_unrotate<E>(x, p.rot_seed, rsqrtf(float(D)));
#pragma unroll
    for (int i = 0; i < E; ++i) acc[threadIdx.x * E + i] = cv.b ? x[i] : 0.f;
  }
  __syncthreads();
  const float invL = 1.f / s_L;
  for (int i = threadIdx.x; i < D; i += blockDim.x) {
    float a = acc[i];
    for (int j = 0; j < cv.r_d; ++j) a += ld_fac(p, Ud, int64_t(i) * cv.r_d + j) * v[j];
    a *= invL;
    if (p.io_f32) reinterpret_cast<float*>(p.out)[qrow * D + i] = a;
    else reinterpret_cast<__nv_bfloat16*>(p.out)[qrow * D + i] = __float2bfloat16_rn(a);
  }
  if (threadIdx.x == 0 && p.lse) p.lse[qrow] = s_M + logf(s_L);
}

size_t decode_simt_main_smem(const DecodeParams& p) {
  const int D = p.d_h;
  size_t f = 0;
  f += p.pre_rope ? 0 : size_t(p.gq) * p.q_cap;
  f += size_t(p.gq) * D;
  f += p.pre_rope ? size_t(kTile) * D : 0;
  f += size_t(kTile) * kMaxGq;
  f += size_t(p.gq) * p.q_cap;
  f += size_t(p.gq) * D;
  f += 4 * kMaxGq;
  return f * sizeof(float);
}

jolt_status launch_decode_prologue_q(const DecodeParams& p, cudaStream_t st) {
  const dim3 gq_grid(p.n_q, p.Lc, p.B);
  if (p.d_h == 64) k_prologue_q<2><<<gq_grid, 128, 0, st>>>(p);
  else k_prologue_q<4><<<gq_grid, 128, 0, st>>>(p);
  JOLT_CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

jolt_status launch_decode_simt(const DecodeParams& p, cudaStream_t st) {
  if (p.gq > kMaxGq) return JOLT_ERR_INVALID_ARG;
  {
    StatScope sc(JOLT_K_DECODE_AUX, st, 0.0, 0.0);
    jolt_status r = launch_decode_prologue_q(p, st);
    if (r) return r;
    if (p.pre_rope) {
      k_prologue_bh<<<dim3(p.n_kv, p.Lc, p.B), 256, 0, st>>>(p);
      JOLT_CUDA_TRY(cudaGetLastError());
    }
  }
  const size_t smem = decode_simt_main_smem(p);
  if (smem > 227 * 1024) return JOLT_ERR_INVALID_ARG;
  const dim3 grid(p.S, p.n_kv, p.B * p.Lc);
  StatScope sc(JOLT_K_DECODE_MAIN, st, 0.0, p.alg_bytes);
  if (p.d_h == 64) {
    JOLT_CUDA_TRY(cudaFuncSetAttribute(k_decode_main<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    k_decode_main<2><<<grid, 256, smem, st>>>(p);
  } else {
    JOLT_CUDA_TRY(cudaFuncSetAttribute(k_decode_main<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem)));
    k_decode_main<4><<<grid, 256, smem, st>>>(p);
  }
  JOLT_CUDA_TRY(cudaGetLastError());
  StatScope sc2(JOLT_K_DECODE_AUX, st, 0.0, 0.0);
  return launch_decode_merge(p, st);
}

jolt_status launch_decode_merge(const DecodeParams& p, cudaStream_t st) {
  const dim3 gq_grid(p.n_q, p.Lc, p.B);
  const size_t msm = (size_t(p.q_cap) + 128 + p.d_h + p.S) * sizeof(float);
  if (p.d_h == 64) {
    JOLT_CUDA_TRY(cudaFuncSetAttribute(k_decode_merge<2>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(msm)));
    k_decode_merge<2><<<gq_grid, 128, msm, st>>>(p);
  } else {
    JOLT_CUDA_TRY(cudaFuncSetAttribute(k_decode_merge<4>, cudaFuncAttributeMaxDynamicSharedMemorySize, int(msm)));
    k_decode_merge<4><<<gq_grid, 128, msm, st>>>(p);
  }
  JOLT_CUDA_TRY(cudaGetLastError());
  return JOLT_OK;
}

}  // namespace jolt
