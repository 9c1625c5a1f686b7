/*
 * jolt.h — C ABI of the JoLT KV-cache codec for NVIDIA B200 (sm_100a).
 *
 * JoLT compresses a transformer's prefill KV cache by a partial Tucker decomposition of each
 * (layer group, K|V) cell along its token and feature modes, plus a randomly rotated, uniformly
 * quantised residual; one Lagrange multiplier allocates ranks and residual bits across cells
 * under a global byte budget; decode attention runs directly over the stored factors.
 * Sources: "A JoLT for the KV cache: Near-Lossless KV Cache Compression via Joint Rank-bit
 * Allocation" (arXiv:2607.12550v4 summary on paperlayer.ai), §3 Method, §3.1 FlashJoLT,
 * §4.5 Fused decode kernel; "Technische Samenvatting: Een JOLT voor de KV Cache"
 * (gist.science/nl), Methodologie 1-4; "JoLT: совместное распределение ранга и бит в KV-кэше"
 * (sarnas.ru), sections on the KV-cache size and on building cos/sin inside the kernel.
 *
 * Conventions for every call:
 *   - Pointers marked "device" are CUDA device pointers of the current device; "host" are host
 *     pointers. The caller owns every buffer; the library never allocates device memory and
 *     keeps no state between calls except read-only device constants.
 *   - `stream` is a cudaStream_t passed as void* (NULL = legacy default stream).
 *   - Device-side errors (numeric range, bounded waits that gave up) are written to an error
 *     word at the start of the workspace `ws`; calls that synchronise report them, the
 *     asynchronous decode call leaves them for jolt_check().
 *   - Invalid arguments return JOLT_ERR_INVALID_ARG before any launch.
 *
 * Tensor layouts (row-major, last index fastest):
 *   K, V   [batch][n_layers][n_kv][T][d_h]           io dtype
 *   q, out [batch][n_layers_call][n_q][d_h]           io dtype
 *   cells are indexed c = (b * n_groups + g) * 2 + kv, kv = 0 for K and 1 for V; a cell holds
 *   layers [g*L_g, (g+1)*L_g) of sequence b: the tensor X[L_g][n_kv][T][d_h].
 *   Query head h' reads KV head floor(h' / (n_q / n_kv)).
 *
 * Stored cache, per cell, five segments each starting on a 256-byte boundary:
 *   U_T   [T][r_T]                 factor dtype   token basis
 *   U_d   [d_h][r_d]               factor dtype   feature basis
 *   G     [L_g][n_kv][r_T][r_d]    factor dtype   core
 *   codes [L_g][n_kv][T][d_h*b/8]  uint8          packed residual codes (absent when b == 0)
 *   sz    [L_g][n_kv][T][2]        fp16           per-row (scale, zero)  (absent when b == 0)
 * Code j of a row occupies bits [(j*b) mod 8, +b) of byte floor(j*b/8).
 */
#ifndef JOLT_H_
#define JOLT_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  JOLT_OK = 0,
  JOLT_ERR_INVALID_ARG = -1,   /* bad shape, pointer, size or option */
  JOLT_ERR_CUDA = -2,          /* a CUDA runtime/driver call failed */
  JOLT_ERR_TIMEOUT = -3,       /* a bounded device-side wait gave up */
  JOLT_ERR_BUDGET = -4,        /* byte budget below the cheapest allocation */
  JOLT_ERR_NUMERIC = -5,       /* non-finite input or fp16 scale/zero out of range */
  JOLT_ERR_WORKSPACE = -6,     /* workspace smaller than jolt_workspace_bytes() */
  JOLT_ERR_STATE = -7          /* jolt_compress without a matching jolt_analyze */
} jolt_status;

typedef enum { JOLT_F32 = 0, JOLT_BF16 = 1 } jolt_dtype;

typedef enum { JOLT_OP_COMPRESS = 0, JOLT_OP_DECODE = 1 } jolt_op;

/* Problem description shared by all calls. */
/* Kernel form of the tcgen05 GEMMs the compressor and decoder run (all give the same results up to
 * the fp32 summation order):
 *   JOLT_GEMM_DEFAULT     one output tile per CTA, one or two 128-row accumulators, split-K and
 *                         tile shape from a whole-wave time estimate; MN-major operands copied as one
 *                         multi-chunk TMA copy per pipeline stage;
 *   JOLT_GEMM_PER_CHUNK   the same kernel copying MN-major operands one 64-wide chunk at a time;
 *   JOLT_GEMM_PERSISTENT  persistent single CTAs, two TMEM accumulators (epilogue of one tile under
 *                         the main loop of the next), for N > 128 and more than one row tile;
 *   JOLT_GEMM_PAIRS       the persistent form on CTA pairs (cta_group::2, M = 256 per MMA, each SM
 *                         staging half of B). Faster in isolation at a fixed clock; in a whole
 *                         compression pass under the 1 kW power cap it lowers the clock the rest of
 *                         the pass runs at, so it is not the default. */
typedef enum { JOLT_GEMM_DEFAULT = 0, JOLT_GEMM_PER_CHUNK = 1, JOLT_GEMM_PERSISTENT = 2, JOLT_GEMM_PAIRS = 3 } jolt_gemm_plan;

typedef struct {
  int32_t batch;              /* sequences B >= 1 */
  int32_t n_layers;           /* L >= 1 */
  int32_t layers_per_group;   /* L_g, divides L: a cell groups L_g consecutive layers */
  int32_t n_kv;               /* KV heads >= 1 */
  int32_t n_q;                /* query heads, a multiple of n_kv */
  int32_t T;                  /* cached tokens per sequence >= 1 */
  int32_t d_h;                /* head dimension: 64 or 128 */
  int32_t io_dtype;           /* jolt_dtype of K, V, q, out */
  int32_t factor_dtype;       /* jolt_dtype of the stored U_T, U_d, G */
  int32_t keys_pre_rope;      /* 1: keys were captured before RoPE; decode re-applies RoPE */
  int32_t q_cap;              /* token-rank cap, multiple of 16, <= min(T, L_g*n_kv*d_h) */
  int32_t sketch_cols;        /* l: sketch width of the randomized token SVD, q_cap <= l <=
                                 min(T, L_g*n_kv*d_h), multiple of 16 */
  int32_t power_iters;        /* q >= 0 power iterations of the range finder */
  int32_t cells_per_pass;     /* cells processed together by jolt_analyze (>= 1) */
  uint64_t rot_seed;          /* seed of the residual rotation's sign diagonal */
  uint64_t sketch_seed;       /* seed of the Rademacher sketch matrix */
  float attn_scale;           /* softmax scale, usually 1/sqrt(d_h) */
  float rope_attention_scaling; /* multiplies cos and sin (1.0 for plain RoPE) */
  int32_t gemm_plan;          /* jolt_gemm_plan of the compressor's and decoder's GEMMs */
} jolt_shape;

/* Per-cell rank/bit choice: r_T, r_d multiples of 16 (both 0 or both > 0), b in {0,2,4,8}. */
typedef struct {
  int32_t r_T;
  int32_t r_d;
  int32_t b;
} jolt_cell_choice;

/* Human-readable status. Never NULL. */
const char* jolt_status_string(jolt_status s);

/* Library version (major*10000 + minor*100 + patch). */
int32_t jolt_version(void);

/* Checks a shape; JOLT_OK or JOLT_ERR_INVALID_ARG. */
jolt_status jolt_shape_check(const jolt_shape* shape);

/* Dense KV-cache bytes 2 * L * n_kv * d_h * T * dtype_bytes ("JoLT: совместное распределение ранга
 * и бит в KV-кэше", section on the KV-cache size formula). */
uint64_t jolt_kv_bytes(int32_t n_layers, int32_t n_kv, int32_t d_h, int64_t T, int32_t dtype_bytes);

/* Bytes one cell stores for a choice, without alignment padding (the allocator's byte model):
 * s_f*(T*r_T + d_h*r_d + L_g*n_kv*r_T*r_d) + [b>0]*L_g*n_kv*T*(d_h*b/8 + 4).
 * Returns 0 for an invalid choice. */
uint64_t jolt_cell_bytes(const jolt_shape* shape, jolt_cell_choice choice);

/* Layout of the stored cache for per-cell choices (host array, n_cells = 2*B*L/L_g entries).
 * offsets (host, may be NULL): n_cells*5 byte offsets of U_T, U_d, G, codes, sz per cell.
 * total_bytes (host): bytes of the whole cache buffer. */
jolt_status jolt_cache_layout(const jolt_shape* shape, const jolt_cell_choice* choices,
                              uint64_t* offsets, uint64_t* total_bytes);

/* ---- Stored cache as a host blob (persisting a compressed cache, moving it between processes).
 * The pages store the factors, codes and scales per group ("A JoLT for the KV cache", §3, the
 * stored cache); the blob adds a header so a reader can check what it holds:
 *   bytes 0..7   magic "JOLTCACH"; 8..11 format version (2); 12..15 header bytes (h)
 *   16..         jolt_shape (as in this header), int32 n_cells, n_cells jolt_cell_choice,
 *                uint64 cache bytes (c), zero padding up to h (a multiple of 256)
 *   h .. h+c     the cache exactly as jolt_cache_layout places it (device bytes copied verbatim)
 * All fields little-endian. */

/* Blob bytes for a shape and its choices (0 if either is invalid). */
uint64_t jolt_cache_blob_bytes(const jolt_shape* shape, const jolt_cell_choice* choices);

/* Copies the device cache (laid out for `choices`) into the host blob and writes the header.
 *   cache  device, >= the jolt_cache_layout total;  blob  host, >= jolt_cache_blob_bytes
 * Synchronises `stream`. JOLT_ERR_INVALID_ARG on a bad shape, choice or short blob. */
jolt_status jolt_cache_serialize(const jolt_shape* shape, const jolt_cell_choice* choices, const void* cache,
                                 void* blob, uint64_t blob_bytes, void* stream);

/* Reads and checks a blob's header (host only, no device work): magic, version, shape, choices,
 * and that the blob holds the cache bytes the layout needs.
 *   shape_out (host, may be NULL), n_cells_out (host, may be NULL), cache_bytes_out (host, may
 *   be NULL). JOLT_ERR_INVALID_ARG on a malformed or truncated blob. */
jolt_status jolt_cache_blob_info(const void* blob, uint64_t blob_bytes, jolt_shape* shape_out, int32_t* n_cells_out,
                                 uint64_t* cache_bytes_out);

/* Checks the blob as jolt_cache_blob_info does, then writes its choices (host, n_cells entries
 * from jolt_cache_blob_info) and copies the cache into device memory `cache` (>= cache bytes).
 * Synchronises `stream`. */
jolt_status jolt_cache_deserialize(const void* blob, uint64_t blob_bytes, jolt_cell_choice* choices_out,
                                   int32_t n_cells, void* cache, uint64_t cache_bytes, void* stream);

/* Error fraction phi(b) of the rotated b-bit quantiser for b = 0, 2, 4, 8 (phi(0) = 1), measured
 * on n_rows Gaussian rows of dimension d_h drawn from `seed` (host computation). The allocator's
 * surrogate multiplies the discarded mass by it ("A JoLT for the KV cache", §3). */
jolt_status jolt_phi(int32_t d_h, int32_t n_rows, uint64_t seed, double phi_out[4]);

/* Joint allocation with one Lagrange multiplier ("A JoLT for the KV cache", §3): for n_cells
 * cells with spectra tails
 *   norm2[c]                = ||X_c||^2,
 *   tail_T[c*n_rt + k]      = discarded token-mode mass at r_T = 16k  (k < n_rt),
 *   tail_d[c*n_rd + j]      = discarded feature-mode mass at r_d = 16j (j < n_rd),
 * (all host, float64) choose per cell (r_T, r_d, b) minimising sum E subject to
 * sum bytes <= budget, E = phi(b) * (r_T ? min(norm2, tail_T + tail_d) : norm2), bytes from
 * jolt_cell_bytes. Hull segments are bought in order of falling price dE/dbytes while the budget
 * holds; lambda_out (host, may be NULL) is the price of the first segment that did not fit.
 * Host-only and deterministic. JOLT_ERR_BUDGET if the cheapest choices exceed the budget. */
jolt_status jolt_allocate(const jolt_shape* shape, int32_t n_cells, const double* norm2,
                          const double* tail_T, int32_t n_rt, const double* tail_d, int32_t n_rd,
                          const double phi[4], uint64_t budget, jolt_cell_choice* choices_out,
                          double* lambda_out, uint64_t* total_bytes_out);

/* Allocation variants of the pages' ablations ("A JoLT for the KV cache", §4.4 Ablations and
 * App. D Tables 12-13), same inputs and error model as jolt_allocate, cells ordered (sequence,
 * group, K|V) so even cells are keys and odd cells values:
 *   JOLT_ALLOC_JOINT     jolt_allocate itself;
 *   JOLT_ALLOC_KV_SPLIT  K/V-decoupled: keys and values each allocated jointly on their own, with
 *                        budget/2 (rounded down) for keys and the rest for values;
 *   JOLT_ALLOC_UNIFORM   uniform ranks: one (r_T, r_d, b) for every key cell and one for every
 *                        value cell, the pair of least summed error whose bytes fit (ties: fewer
 *                        bytes, then the earlier key choice, then the earlier value choice, choices
 *                        ordered by r_T, r_d, b);
 *   JOLT_ALLOC_COORD     the pages' coordinate-wise rank search ("A JoLT for the KV cache", §3: a
 *                        heuristic over the two truncated modes) under the same single multiplier:
 *                        for a multiplier lam each cell starts at full ranks and alternates the best
 *                        r_T with r_d held (r_T = 0 takes the residual-only choices) and the best r_d
 *                        with r_T held, b chosen with each move, by E + lam * bytes (ties: fewer
 *                        bytes, smaller r_T, r_d, b) until a round changes nothing (at most 32);
 *                        lam is the fitting end of a geometric bisection of [1e-30, 1e30] (200
 *                        halvings, midpoint sqrt(lo * hi)). Never better than jolt_allocate at equal
 *                        bytes; reported beside it to show what the exact search gains.
 * Host-only. JOLT_ERR_BUDGET if nothing fits; JOLT_ERR_INVALID_ARG for an odd n_cells or bad mode. */
typedef enum { JOLT_ALLOC_JOINT = 0, JOLT_ALLOC_KV_SPLIT = 1, JOLT_ALLOC_UNIFORM = 2, JOLT_ALLOC_COORD = 3 } jolt_alloc_mode;
jolt_status jolt_allocate_variant(const jolt_shape* shape, int32_t n_cells, const double* norm2,
                                  const double* tail_T, int32_t n_rt, const double* tail_d, int32_t n_rd,
                                  const double phi[4], uint64_t budget, int32_t mode,
                                  jolt_cell_choice* choices_out, uint64_t* total_bytes_out);

/* Workspace bytes for an operation (device memory the caller allocates and passes as `ws`).
 * JOLT_OP_COMPRESS covers jolt_analyze followed by jolt_compress on the same ws;
 * JOLT_OP_DECODE covers jolt_decode_attn with any n_layers_call <= n_layers. 0 on bad shape. */
size_t jolt_workspace_bytes(const jolt_shape* shape, int32_t op);

/* Spectra of every cell ("A JoLT for the KV cache", §3.1 FlashJoLT): a randomized token-mode SVD
 * (Rademacher sketch, power iterations with CholeskyQR orthonormalisation, Rayleigh-Ritz) gives
 * the top q_cap token directions; the energy it did not find, ||X||^2 minus the captured part,
 * closes the token tail; the feature tail comes from the eigenvalues of the cell's feature Gram.
 *   k, v        device, [B][L][n_kv][T][d_h] io dtype
 *   norm2_out   host [n_cells];  tail_T_out host [n_cells][q_cap/16+1];
 *   tail_d_out  host [n_cells][d_h/16+1]
 *   ws          device, >= jolt_workspace_bytes(shape, JOLT_OP_COMPRESS); on return holds the
 *               cells' token bases for jolt_compress.
 * Synchronises `stream`. */
jolt_status jolt_analyze(const jolt_shape* shape, const void* k, const void* v, double* norm2_out,
                         double* tail_T_out, double* tail_d_out, void* ws, size_t ws_bytes,
                         void* stream);

/* jolt_analyze with the inputs streamed from host memory: K crosses the bus into k_dev, then V
 * into v_dev on a copy stream of the library's own while the key cells are analysed (each kind's
 * passes wait only for that kind's copy). The copies start after the work already queued on
 * `stream` (which may still be reading k_dev / v_dev). k_host, v_host: page-locked host
 * memory [B][L][n_kv][T][d_h] io dtype (pageable memory works but does not overlap); k_dev, v_dev:
 * device buffers of the same size, left holding the inputs for jolt_compress. Otherwise as
 * jolt_analyze. Synchronises `stream`. */
jolt_status jolt_analyze_from_host(const jolt_shape* shape, const void* k_host, const void* v_host,
                                   void* k_dev, void* v_dev, double* norm2_out, double* tail_T_out,
                                   double* tail_d_out, void* ws, size_t ws_bytes, void* stream);

/* Layer alignment for grouping ("A JoLT for the KV cache", §3: JoLT groups consecutive layers
 * whose token-mode singular vectors align, from the cache being compressed). The pages give no
 * measure; the one computed here: for every sequence b and layer l, U^X_{b,l} = the top-k token
 * directions of layer l's own cache X in {K, V} (token unfolding [T][n_kv*d_h]), found by the
 * compressor's randomized token SVD (sketch width k + 16 capped at min(T, n_kv*d_h), two power
 * iterations, Rayleigh-Ritz); then
 *   align[b*(L-1) + l] = ( ||U^K_l^T U^K_{l+1}||_F^2 + ||U^V_l^T U^V_{l+1}||_F^2 ) / (2k),
 * the mean squared cosine of the principal angles, in [0, 1], for l < L-1.
 *   shape   the codec's shape (layers_per_group, q_cap, sketch_cols, power_iters are ignored)
 *   k       multiple of 16, 16 <= k <= min(T, n_kv*d_h)
 *   K, V    device, [B][L][n_kv][T][d_h] io dtype
 *   align   host [B][L-1]
 *   ws      device, >= jolt_layer_align_workspace(shape, k)
 * Synchronises `stream`. JOLT_ERR_INVALID_ARG for a bad shape or k. */
size_t jolt_layer_align_workspace(const jolt_shape* shape, int32_t k);
jolt_status jolt_layer_align(const jolt_shape* shape, int32_t k, const void* K, const void* V, double* align,
                             void* ws, size_t ws_bytes, void* stream);

/* Consecutive layer groups from alignments (host): layer l+1 joins the current group when
 * align[l] >= tau and, if max_group > 0, the group has fewer than max_group layers.
 *   align        host [n_layers - 1];  group_sizes host [n_layers] (first *n_groups entries set)
 * JOLT_ERR_INVALID_ARG for n_layers < 1 or NULL outputs. */
jolt_status jolt_group_layers(const double* align, int32_t n_layers, double tau, int32_t max_group,
                              int32_t* group_sizes, int32_t* n_groups);

/* Largest group size L_g dividing n_layers whose uniform groups keep every consecutive alignment
 * inside a group >= tau (1 always qualifies): the grouping a fixed-L_g shape can use (host). */
jolt_status jolt_uniform_group(const double* align, int32_t n_layers, double tau, int32_t* L_g);

/* Compress every cell with its choice ("A JoLT for the KV cache", §3): U_T = the first r_T token
 * directions found by jolt_analyze, U_d = top-r_d eigenvectors of the feature Gram of U_T^T X,
 * G = U_T^T X U_d, residual R = X - U_T G U_d^T against the stored (rounded) factors, rotated by
 * (1/sqrt(d_h)) H D (Hadamard times seeded signs), quantised per row and packed.
 *   k, v      device, as for jolt_analyze — the same tensors the preceding analyze saw
 *   choices   host [n_cells]
 *   cache     device, cache_bytes >= jolt_cache_layout total
 *   ws        device, the workspace jolt_analyze filled (JOLT_ERR_STATE otherwise)
 * Synchronises `stream`. */
jolt_status jolt_compress(const jolt_shape* shape, const void* k, const void* v,
                          const jolt_cell_choice* choices, void* cache, uint64_t cache_bytes,
                          void* ws, size_t ws_bytes, void* stream);

/* Decode attention of one query token per (sequence, layer, query head) over all T stored
 * tokens, evaluated on the stored factors without materialising dense K/V ("A JoLT for the KV
 * cache", §4.5): scores U_T (G (U_d^T q)) + (R q) . deq(codes) and values
 * U_d G^T (U_T^T p) + R^T (deq(codes)^T p); with keys_pre_rope, each key is rebuilt per token
 * tile and rotated by RoPE at position pos_offset + t before the dot product, cos/sin computed in
 * the kernel from inv_freq ("JoLT: совместное распределение ранга и бит в KV-кэше", section on
 * building cos/sin in the kernel).
 * bf16 I/O and factors with d_h = 128 and g_q <= 16 run on the tensor-core path (tcgen05 key
 * rebuild and value GEMMs, fp32 accumulation); other shapes on the CUDA-core split-T path.
 *   cache        device, filled by jolt_compress (or laid out by jolt_cache_layout); on the
 *                tensor-core path it must be 16-byte aligned (JOLT_ERR_INVALID_ARG otherwise)
 *   layer_begin, n_layers_call: layers [layer_begin, layer_begin + n_layers_call)
 *   q            device [B][n_layers_call][n_q][d_h] io dtype
 *   out          device [B][n_layers_call][n_q][d_h] io dtype
 *   lse          device [B][n_layers_call][n_q] fp32 log-sum-exp of the scaled scores, or NULL
 *   inv_freq     device [d_h/2] fp32 (required when keys_pre_rope), may carry RoPE scaling
 *   pos_offset   position of cached token 0
 *   ws           device, >= jolt_workspace_bytes(shape, JOLT_OP_DECODE); calls sharing a ws
 *                must not overlap in time
 * Asynchronous on `stream`. */
jolt_status jolt_decode_attn(const jolt_shape* shape, const jolt_cell_choice* choices,
                             const void* cache, int32_t layer_begin, int32_t n_layers_call,
                             const void* q, void* out, float* lse, const float* inv_freq,
                             int32_t pos_offset, void* ws, size_t ws_bytes, void* stream);

/* Synchronises `stream` and returns the device error word of `ws` (then clears it). */
jolt_status jolt_check(void* ws, void* stream);

/* Building blocks, exposed for bit-exact testing and for callers that quantise their own data. */

/* Rotate rows by (1/sqrt(d)) H D (inverse = 0) or its transpose D H / sqrt(d) (inverse = 1),
 * D the seeded sign diagonal. in/out device fp32 [n_rows][d], d in {64, 128}; may alias. */
jolt_status jolt_rotate_rows(const float* in, float* out, int64_t n_rows, int32_t d,
                             uint64_t seed, int32_t inverse, void* stream);

/* Quantise fp32 rows per row (fp16 scale = (max-min)/(2^b-1), fp16 zero = min, codes rounded to
 * nearest even and clipped) and pack them. rows device fp32 [n_rows][d]; codes device uint8
 * [n_rows][d*b/8]; sz device fp16 [n_rows][2]; err device int32 (set to JOLT_ERR_NUMERIC when a
 * scale or zero is out of fp16 range; never cleared by the kernel). b in {2,4,8}. */
jolt_status jolt_quantize_pack(const float* rows, int64_t n_rows, int32_t d, int32_t b,
                               uint8_t* codes, void* sz, int32_t* err, void* stream);

/* Unpack and dequantise: out = fp32(code * scale + zero) (one rounding). */
jolt_status jolt_unpack_dequant(const uint8_t* codes, const void* sz, int64_t n_rows, int32_t d,
                                int32_t b, float* out, void* stream);

/* Plain batched GEMM on the tcgen05 tensor cores (the kernel the compressor's contractions use):
 *   C[z][m][n] (+)= sum_k A[z](m,k) * B[z](k,n),  bf16 operands, fp32 accumulation and output.
 * A (device, bf16): element (m,k) at A[z*stride_a + m*lda + k] (a_mn_major = 0) or
 *   A[z*stride_a + k*lda + m] (a_mn_major = 1).  B (device, bf16): element (k,n) at
 *   B[z*stride_b + n*ldb + k] (b_mn_major = 0) or B[z*stride_b + k*ldb + n] (b_mn_major = 1).
 * C (device, fp32): element (m,n) at C[z*stride_c + m*ldc + n]. Strides in elements; lda and ldb
 * must be multiples of 8 and the base pointers 16-byte aligned. k_split > 1 splits K over CTAs
 * and requires accumulate = 1 (atomic adds into C, which the caller zeroes first). plan: a
 * jolt_gemm_plan (JOLT_ERR_INVALID_ARG outside it). */
jolt_status jolt_gemm_bf16(const void* A, int32_t a_mn_major, const void* B, int32_t b_mn_major,
                           float* C, int32_t M, int32_t N, int32_t K, int64_t lda, int64_t ldb,
                           int64_t ldc, int32_t batch, int64_t stride_a, int64_t stride_b,
                           int64_t stride_c, int32_t k_split, int32_t accumulate, int32_t plan, void* stream);

/* The same product with the fp32 result split into bf16 parts by the GEMM's epilogue instead of
 * being stored: Ch = bf16_rn(c), and when Cl is not NULL, Cl = bf16_rn(c - Ch), for every result c
 * (the hi / lo split the compressor's CholeskyQR passes feed back into the tensor cores). Ch, Cl
 * (device, bf16) use C's layout (ldc, stride_c). No split-K and no accumulation. */
jolt_status jolt_gemm_bf16_hilo(const void* A, int32_t a_mn_major, const void* B, int32_t b_mn_major,
                                void* Ch, void* Cl, int32_t M, int32_t N, int32_t K, int64_t lda,
                                int64_t ldb, int64_t ldc, int32_t batch, int64_t stride_a,
                                int64_t stride_b, int64_t stride_c, void* stream);

/* The same product with N = 128 coded as residual rows instead of stored (the compressor's fused
 * reconstruction + residual step): for each output row c = C[z][m][:], x = X[z*M + m][:] - c is
 * rotated as jolt_rotate_rows does, quantised to b bits and packed as jolt_quantize_pack does,
 * into codes [batch*M][16*b] and sz (fp16 pairs) [batch*M][2]. A K-major (lda), B N-major (ldb);
 * X (device) bf16, or fp32 when x_f32, [batch*M][128]. codes, X 16-byte aligned. err (device
 * int32, may be NULL) gets JOLT_ERR_NUMERIC for a non-finite row, scale or zero. b in {2,4,8}. */
jolt_status jolt_gemm_bf16_residual(const void* A, const void* B, int32_t M, int32_t K, int64_t lda,
                                    int64_t ldb, int32_t batch, int64_t stride_a, int64_t stride_b,
                                    const void* X, int32_t x_f32, uint64_t seed, int32_t b,
                                    uint8_t* codes, void* sz, int32_t* err, void* stream);

/* Failure-detection self-test: launches a kernel whose wait nothing will end — which = 0: an
 * mbarrier no thread arrives on (the bounded wait of every TMA / tensor-core pipeline); which = 1:
 * a two-CTA cooperative grid whose second CTA never reaches the grid barrier (the barrier of the
 * Cholesky and Jacobi kernels). The wait gives up after limit_ns (1 ns .. 2 s) and the kernel
 * returns with JOLT_ERR_TIMEOUT in ws's error word, which jolt_check then reports; the context
 * stays usable. ws device, >= 512 bytes (zeroed here). Does not synchronise. */
jolt_status jolt_selftest_timeout(int32_t which, uint64_t limit_ns, void* ws, size_t ws_bytes, void* stream);

/* Symmetric eigendecomposition of `batch` fp32 matrices A [batch][n][n] (device) by block Jacobi
 * (the solver the compressor uses for the Rayleigh-Ritz and feature-mode steps): eigenvalues
 * descending into evals [batch][n], eigenvectors as the columns of evecs [batch][n][n] (device).
 * ws (device) >= jolt_sym_eig_workspace(n, batch). Synchronises `stream`. */
size_t jolt_sym_eig_workspace(int32_t n, int32_t batch);
jolt_status jolt_sym_eig(const float* A, int32_t n, int32_t batch, float* evals, float* evecs,
                         void* ws, size_t ws_bytes, void* stream);

/* Decode attention without a caller-provided workspace: same arguments, results and kernels as
 * jolt_decode_attn, except that its scratch lives in a fixed 32 MiB device array inside this
 * library instead of `ws`. The pages have no counterpart to this call; it exists for callers that
 * cannot allocate device memory when they decode, e.g. a plugin of an inference runtime that is
 * handed a stream but no allocator, or a serving loop whose device memory is planned up front and
 * where an allocation would synchronise the device or fail under memory pressure.
 *   - Every GPU that loads the library reserves the 32 MiB until the process exits.
 *   - The first call on a device looks up the array's device address (once per device and
 *     context, with that device current); make that first call before any stream capture. A
 *     context the device gets later (after cudaDeviceReset, say) is noticed and the address looked
 *     up again on the next call, which then must also come before any capture.
 *   - Arguments are checked as jolt_decode_attn checks them (JOLT_ERR_INVALID_ARG) before the
 *     scratch size.
 *   - A call whose scratch would exceed 32 MiB (jolt_workspace_bytes-style sizing for its
 *     n_layers_call) returns JOLT_ERR_WORKSPACE before launching anything: use smaller
 *     n_layers_call or jolt_decode_attn with your own workspace.
 *   - Calls share the array: calls that overlap on the GPU (different streams, or other devices'
 *     contexts excluded) race and corrupt each other's results. The error word is cleared at the
 *     start of every call; device errors are not reported back by this call.
 *   - Allocates nothing: no cudaMalloc, cudaFree or allocating library routine. */
jolt_status jolt_decode_attn_noalloc(const jolt_shape* shape, const jolt_cell_choice* choices,
                                     const void* cache, int32_t layer_begin, int32_t n_layers_call,
                                     const void* q, void* out, float* lse, const float* inv_freq,
                                     int32_t pos_offset, void* stream);

/* Per-kernel-family device timing (off by default). When enabled, the library records a CUDA event
 * pair on the launching stream around every launch of the families below and accumulates the
 * elapsed device time together with the launch's algorithmic work (FLOPs of a contraction, or
 * bytes a streaming kernel must move). Host-global; not for concurrent use from several threads. */
typedef enum {
  JOLT_K_GEMM = 0,          /* tcgen05 contractions (compressor, and the decode's value GEMMs) */
  JOLT_K_DECODE_MAIN = 1,   /* decode scores: tcgen05 key rebuild (pre-RoPE) or residual scores,
                               or the CUDA-core split-T kernel */
  JOLT_K_RESIDUAL = 2,      /* residual rotate + quantise + pack */
  JOLT_K_DECODE_AUX = 3,    /* decode prologue, softmax, value residual, finalize, split merge */
  JOLT_K_CHOL = 4,          /* fp64 Cholesky + triangular inverse (CholeskyQR) */
  JOLT_K_EIG = 5,           /* fp64 block-Jacobi symmetric eigensolver */
  JOLT_K_COUNT = 6
} jolt_kernel_family;

typedef struct {
  int32_t kernel;       /* jolt_kernel_family */
  uint64_t launches;
  double ms;            /* summed device time of the launches */
  double flops;         /* summed algorithmic FLOPs: each product of the method counted once */
  double bytes;         /* summed algorithmic bytes */
  double flops_issued;  /* summed tensor-core FLOPs issued: a product carried as several bf16
                           terms (hi/lo splits of fp32 operands) counts once per term */
} jolt_kernel_stat;

void jolt_stats_enable(int32_t on);
/* Fills out[JOLT_K_COUNT] (host); synchronises on the pending events; reset != 0 clears. */
jolt_status jolt_stats_read(jolt_kernel_stat* out, int32_t reset);

#ifdef __cplusplus
}
#endif

#endif  /* JOLT_H_ */
