"""Thin Python API over the C ABI: torch tensors in, pointers and sizes to libjolt.so out.

Nothing here computes part of the codec; PyTorch provides device memory and streams only.
"""
import ctypes as C
import math

import numpy as np
import torch

from ._lib import (lib, check, Shape, CellChoice, JOLT_F32, JOLT_BF16, JOLT_OP_COMPRESS,
                   JOLT_OP_DECODE, JoltError)

_DT = {"f32": JOLT_F32, "bf16": JOLT_BF16}


def _stream(stream=None):
    if stream is not None:
        return C.c_void_p(stream)
    if torch.cuda.is_available():
        return C.c_void_p(torch.cuda.current_stream().cuda_stream)
    return C.c_void_p(0)


def _ptr(t):
    return C.c_void_p(0 if t is None else t.data_ptr())


def make_shape(w, **over) -> Shape:
    """Shape for a workload (synth.Workload or any object with the same fields)."""
    s = Shape()
    s.batch = over.get("batch", w.batch)
    s.n_layers = over.get("n_layers", w.n_layers)
    s.layers_per_group = w.layers_per_group
    s.n_kv, s.n_q, s.T, s.d_h = w.n_kv, w.n_q, over.get("T", w.T), w.d_h
    s.io_dtype = _DT[over.get("io_dtype", w.io_dtype)]
    s.factor_dtype = _DT[over.get("factor_dtype", w.factor_dtype)]
    s.keys_pre_rope = int(over.get("keys_pre_rope", w.keys_pre_rope))
    n = w.layers_per_group * w.n_kv * w.d_h
    qcap = min(over.get("q_cap", w.q_cap), n, s.T) // 16 * 16
    s.q_cap = qcap
    s.sketch_cols = over.get("sketch_cols", min(qcap + over.get("oversample", w.oversample), n, s.T) // 16 * 16)
    s.power_iters = over.get("power_iters", w.power_iters)
    s.cells_per_pass = over.get("cells_per_pass", 8)
    s.rot_seed = over.get("rot_seed", 0x5EED0000 + w.seed)
    s.sketch_seed = over.get("sketch_seed", 0xC0FFEE00 + w.seed)
    s.attn_scale = over.get("attn_scale", 1.0 / math.sqrt(w.d_h))
    s.rope_attention_scaling = over.get("rope_attention_scaling", 1.0)
    s.gemm_plan = over.get("gemm_plan", GEMM_PLANS["default"])
    check(lib().jolt_shape_check(C.byref(s)), "jolt_shape_check")
    return s


def n_cells(s: Shape) -> int:
    return 2 * s.batch * (s.n_layers // s.layers_per_group)


def choices_array(choices):
    arr = (CellChoice * len(choices))()
    for i, (rT, rd, b) in enumerate(choices):
        arr[i] = CellChoice(int(rT), int(rd), int(b))
    return arr


def cell_bytes(s: Shape, choice) -> int:
    return int(lib().jolt_cell_bytes(C.byref(s), CellChoice(*map(int, choice))))


def kv_bytes(n_layers, n_kv, d_h, T, dtype_bytes) -> int:
    return int(lib().jolt_kv_bytes(n_layers, n_kv, d_h, T, dtype_bytes))


def cache_layout(s: Shape, choices):
    nc = n_cells(s)
    offs = (C.c_uint64 * (5 * nc))()
    tot = C.c_uint64(0)
    check(lib().jolt_cache_layout(C.byref(s), choices_array(choices), offs, C.byref(tot)),
          "jolt_cache_layout")
    return np.array(offs, dtype=np.uint64).reshape(nc, 5), int(tot.value)


def cache_blob_bytes(s: Shape, choices) -> int:
    return int(lib().jolt_cache_blob_bytes(C.byref(s), choices_array(choices)))


def serialize_cache(s: Shape, choices, cache, stream=None) -> np.ndarray:
    """The stored cache (device uint8 tensor) as a host blob with a checked header."""
    n = cache_blob_bytes(s, choices)
    if n == 0:
        raise JoltError(-1, "jolt_cache_blob_bytes")
    blob = np.empty(n, dtype=np.uint8)
    check(lib().jolt_cache_serialize(C.byref(s), choices_array(choices), _ptr(cache), blob.ctypes.data, n,
                                     _stream(stream)), "jolt_cache_serialize")
    return blob


def cache_blob_info(blob):
    """(shape, n_cells, cache_bytes) of a blob; raises on a malformed or truncated blob."""
    b = np.ascontiguousarray(blob, dtype=np.uint8)
    s = Shape()
    nc = C.c_int32(0)
    cb = C.c_uint64(0)
    check(lib().jolt_cache_blob_info(b.ctypes.data, b.size, C.byref(s), C.byref(nc), C.byref(cb)),
          "jolt_cache_blob_info")
    return s, int(nc.value), int(cb.value)


def deserialize_cache(blob, device="cuda", stream=None):
    """(shape, choices, cache device tensor) from a blob written by serialize_cache."""
    b = np.ascontiguousarray(blob, dtype=np.uint8)
    s, nc, cb = cache_blob_info(b)
    out = (CellChoice * nc)()
    cache = torch.empty(max(cb, 1), dtype=torch.uint8, device=device)
    check(lib().jolt_cache_deserialize(b.ctypes.data, b.size, out, nc, _ptr(cache), cache.numel(),
                                       _stream(stream)), "jolt_cache_deserialize")
    return s, [(c.r_T, c.r_d, c.b) for c in out], cache


def phi(d_h: int, n_rows: int = 1 << 16, seed: int = 1):
    out = (C.c_double * 4)()
    check(lib().jolt_phi(d_h, n_rows, seed, out), "jolt_phi")
    return list(out)


JOLT_ALLOC_JOINT, JOLT_ALLOC_KV_SPLIT, JOLT_ALLOC_UNIFORM, JOLT_ALLOC_COORD = 0, 1, 2, 3


def allocate_variant(s: Shape, norm2, tail_T, tail_d, phi4, budget: int, mode: int):
    """The allocator's ablation variants (joint, K/V-decoupled, uniform ranks). Returns
    (choices [(r_T, r_d, b)], bytes)."""
    norm2 = np.ascontiguousarray(norm2, dtype=np.float64)
    tT = np.ascontiguousarray(tail_T, dtype=np.float64)
    td = np.ascontiguousarray(tail_d, dtype=np.float64)
    nc = norm2.shape[0]
    out = (CellChoice * nc)()
    tot = C.c_uint64(0)
    dp = C.POINTER(C.c_double)
    ph = (C.c_double * 4)(*phi4)
    check(lib().jolt_allocate_variant(C.byref(s), nc, norm2.ctypes.data_as(dp), tT.ctypes.data_as(dp),
                                      tT.shape[1], td.ctypes.data_as(dp), td.shape[1], ph, int(budget),
                                      int(mode), out, C.byref(tot)), "jolt_allocate_variant")
    return [(c.r_T, c.r_d, c.b) for c in out], int(tot.value)


def allocate(s: Shape, norm2, tail_T, tail_d, phi4, budget: int):
    """One allocation over the given cells. Returns (choices [(r_T, r_d, b)], lambda, bytes)."""
    norm2 = np.ascontiguousarray(norm2, dtype=np.float64)
    tT = np.ascontiguousarray(tail_T, dtype=np.float64)
    td = np.ascontiguousarray(tail_d, dtype=np.float64)
    nc = norm2.shape[0]
    out = (CellChoice * nc)()
    lam = C.c_double(0)
    tot = C.c_uint64(0)
    dp = C.POINTER(C.c_double)
    ph = (C.c_double * 4)(*phi4)
    check(lib().jolt_allocate(C.byref(s), nc, norm2.ctypes.data_as(dp), tT.ctypes.data_as(dp),
                              tT.shape[1], td.ctypes.data_as(dp), td.shape[1], ph, int(budget), out,
                              C.byref(lam), C.byref(tot)), "jolt_allocate")
    return [(c.r_T, c.r_d, c.b) for c in out], lam.value, int(tot.value)


def workspace_bytes(s: Shape, op: int) -> int:
    return int(lib().jolt_workspace_bytes(C.byref(s), op))


def new_workspace(s: Shape, op: int, device="cuda"):
    return torch.zeros(workspace_bytes(s, op), dtype=torch.uint8, device=device)


def analyze(s: Shape, k, v, ws, stream=None):
    nc = n_cells(s)
    nrt, nrd = s.q_cap // 16 + 1, s.d_h // 16 + 1
    norm2 = np.zeros(nc)
    tT = np.zeros((nc, nrt))
    td = np.zeros((nc, nrd))
    dp = C.POINTER(C.c_double)
    check(lib().jolt_analyze(C.byref(s), _ptr(k), _ptr(v), norm2.ctypes.data_as(dp),
                             tT.ctypes.data_as(dp), td.ctypes.data_as(dp), _ptr(ws), ws.numel(),
                             _stream(stream)), "jolt_analyze")
    return norm2, tT, td


def layer_align_workspace(s: Shape, rank=32):
    return lib().jolt_layer_align_workspace(C.byref(s), rank)


def layer_align(s: Shape, k, v, rank=32, ws=None, stream=None):
    """Alignment of consecutive layers' top-`rank` token subspaces (mean squared cosine of the
    principal angles, K and V averaged), per sequence: float64 [B, L-1]."""
    nb = lib().jolt_layer_align_workspace(C.byref(s), rank)
    if nb == 0:
        raise JoltError(-1, "jolt_layer_align_workspace")
    if ws is None or ws.numel() < nb:
        ws = torch.zeros(nb, dtype=torch.uint8, device=k.device)
    out = np.zeros((s.batch, max(0, s.n_layers - 1)))
    check(lib().jolt_layer_align(C.byref(s), rank, _ptr(k), _ptr(v), out.ctypes.data_as(C.POINTER(C.c_double)),
                                 _ptr(ws), ws.numel(), _stream(stream)), "jolt_layer_align")
    return out


def group_layers(align, tau, max_group=0):
    """Consecutive layer groups (sizes) from one sequence's alignments [L-1]."""
    a = np.ascontiguousarray(np.asarray(align, dtype=np.float64))
    L = a.size + 1
    sizes = np.zeros(L, dtype=np.int32)
    ng = C.c_int32(0)
    check(lib().jolt_group_layers(a.ctypes.data_as(C.c_void_p), L, float(tau), int(max_group),
                                  sizes.ctypes.data_as(C.c_void_p), C.byref(ng)), "jolt_group_layers")
    return [int(x) for x in sizes[:ng.value]]


def uniform_group(align, tau):
    """Largest uniform group size dividing L that keeps every in-group alignment >= tau."""
    a = np.ascontiguousarray(np.asarray(align, dtype=np.float64))
    out = C.c_int32(0)
    check(lib().jolt_uniform_group(a.ctypes.data_as(C.c_void_p), a.size + 1, float(tau), C.byref(out)),
          "jolt_uniform_group")
    return out.value


def analyze_from_host(s: Shape, k_host, v_host, k_dev, v_dev, ws, stream=None):
    """analyze() with K and V copied from (pinned) host tensors into k_dev / v_dev inside the
    call, the value copy overlapping the key cells' analysis."""
    nc = n_cells(s)
    nrt, nrd = s.q_cap // 16 + 1, s.d_h // 16 + 1
    norm2 = np.zeros(nc)
    tT = np.zeros((nc, nrt))
    td = np.zeros((nc, nrd))
    dp = C.POINTER(C.c_double)
    check(lib().jolt_analyze_from_host(C.byref(s), C.c_void_p(k_host.data_ptr()), C.c_void_p(v_host.data_ptr()),
                                       _ptr(k_dev), _ptr(v_dev), norm2.ctypes.data_as(dp), tT.ctypes.data_as(dp),
                                       td.ctypes.data_as(dp), _ptr(ws), ws.numel(), _stream(stream)),
          "jolt_analyze_from_host")
    return norm2, tT, td


def compress(s: Shape, k, v, choices, cache, ws, stream=None):
    check(lib().jolt_compress(C.byref(s), _ptr(k), _ptr(v), choices_array(choices), _ptr(cache),
                              cache.numel(), _ptr(ws), ws.numel(), _stream(stream)), "jolt_compress")


def decode_attn(s: Shape, choices, cache, q, out, ws, lse=None, inv_freq=None, layer_begin=0,
                n_layers_call=None, pos_offset=0, stream=None, choices_c=None):
    if n_layers_call is None:
        n_layers_call = s.n_layers - layer_begin
    ch = choices_c if choices_c is not None else choices_array(choices)
    check(lib().jolt_decode_attn(C.byref(s), ch, _ptr(cache), layer_begin, n_layers_call, _ptr(q),
                                 _ptr(out), _ptr(lse), _ptr(inv_freq), pos_offset, _ptr(ws),
                                 ws.numel(), _stream(stream)), "jolt_decode_attn")


def decode_attn_noalloc(s: Shape, choices, cache, q, out, lse=None, inv_freq=None, layer_begin=0,
                        n_layers_call=None, pos_offset=0, stream=None):
    """jolt_decode_attn with the library's built-in 32 MiB scratch instead of a workspace."""
    if n_layers_call is None:
        n_layers_call = s.n_layers - layer_begin
    check(lib().jolt_decode_attn_noalloc(C.byref(s), choices_array(choices), _ptr(cache), layer_begin,
                                         n_layers_call, _ptr(q), _ptr(out), _ptr(lse), _ptr(inv_freq),
                                         pos_offset, _stream(stream)), "jolt_decode_attn_noalloc")


def check_ws(ws, stream=None):
    check(lib().jolt_check(_ptr(ws), _stream(stream)), "device error")


def rotate_rows(x, seed, inverse=False, out=None, stream=None):
    out = torch.empty_like(x) if out is None else out
    check(lib().jolt_rotate_rows(_ptr(x), _ptr(out), x.shape[0], x.shape[1], seed, int(inverse),
                                 _stream(stream)), "jolt_rotate_rows")
    return out


def quantize_pack(rows, b, stream=None):
    n, d = rows.shape
    codes = torch.empty(n, d * b // 8, dtype=torch.uint8, device=rows.device)
    sz = torch.empty(n, 2, dtype=torch.float16, device=rows.device)
    err = torch.zeros(1, dtype=torch.int32, device=rows.device)
    check(lib().jolt_quantize_pack(_ptr(rows), n, d, b, _ptr(codes), _ptr(sz), _ptr(err),
                                   _stream(stream)), "jolt_quantize_pack")
    return codes, sz, err


def unpack_dequant(codes, sz, d, b, stream=None):
    n = codes.shape[0]
    out = torch.empty(n, d, dtype=torch.float32, device=codes.device)
    check(lib().jolt_unpack_dequant(_ptr(codes), _ptr(sz), n, d, b, _ptr(out), _stream(stream)),
          "jolt_unpack_dequant")
    return out


# jolt_gemm_plan values by name
GEMM_PLANS = {"default": 0, "perchunk": 1, "persistent": 2, "pairs": 3}


def gemm_bf16(A, B, a_mn_major=False, b_mn_major=False, C=None, k_split=1, accumulate=False,
              plan="default", stream=None):
    """C = A_logical @ B_logical for bf16 tensors, via the library's tcgen05 GEMM.

    A: [batch?, M, K] (a_mn_major False) or [batch?, K, M] (True); B: [batch?, N, K] (b_mn_major
    False) or [batch?, K, N] (True). Returns fp32 [batch?, M, N]."""
    batched = A.dim() == 3
    A3 = A if batched else A[None]
    B3 = B if batched else B[None]
    bt = A3.shape[0]
    M = A3.shape[2] if a_mn_major else A3.shape[1]
    K = A3.shape[1] if a_mn_major else A3.shape[2]
    N = B3.shape[2] if b_mn_major else B3.shape[1]
    if C is None:
        C = torch.zeros(bt, M, N, dtype=torch.float32, device=A.device)
    C3 = C if C.dim() == 3 else C[None]
    check(lib().jolt_gemm_bf16(_ptr(A3), int(a_mn_major), _ptr(B3), int(b_mn_major), _ptr(C3), M, N,
                               K, A3.stride(1), B3.stride(1), C3.stride(1), bt, A3.stride(0),
                               B3.stride(0), C3.stride(0), k_split, int(accumulate), GEMM_PLANS[plan],
                               _stream(stream)), "jolt_gemm_bf16")
    return C3 if batched else C3[0]


def gemm_bf16_hilo(A, B, a_mn_major=False, b_mn_major=False, lo=True, stream=None):
    """The product of gemm_bf16 returned as its bf16 hi / lo split (hi = bf16(c), lo =
    bf16(c - hi)) written by the GEMM epilogue. Returns (hi, lo or None), bf16 [batch?, M, N]."""
    batched = A.dim() == 3
    A3 = A if batched else A[None]
    B3 = B if batched else B[None]
    bt = A3.shape[0]
    M = A3.shape[2] if a_mn_major else A3.shape[1]
    K = A3.shape[1] if a_mn_major else A3.shape[2]
    N = B3.shape[2] if b_mn_major else B3.shape[1]
    hi = torch.empty(bt, M, N, dtype=torch.bfloat16, device=A.device)
    lo_t = torch.empty_like(hi) if lo else None
    check(lib().jolt_gemm_bf16_hilo(_ptr(A3), int(a_mn_major), _ptr(B3), int(b_mn_major), _ptr(hi),
                                    _ptr(lo_t) if lo else None, M, N, K, A3.stride(1), B3.stride(1),
                                    hi.stride(1), bt, A3.stride(0), B3.stride(0), hi.stride(0),
                                    _stream(stream)), "jolt_gemm_bf16_hilo")
    if batched:
        return hi, lo_t
    return hi[0], (lo_t[0] if lo else None)


def gemm_bf16_residual(A, B, X, seed, b, stream=None):
    """Fused reconstruction + residual coding: rows of X - A @ B (A [batch?, M, K] bf16 K-major,
    B [batch?, K, 128] bf16, X [batch?, M, 128] bf16 or fp32) rotated, quantised to b bits and
    packed. Returns (codes uint8 [batch?*M, 16*b], sz fp16 [batch?*M, 2], err int32 [1])."""
    batched = A.dim() == 3
    A3 = A if batched else A[None]
    B3 = B if batched else B[None]
    bt, M, K = A3.shape
    X2 = X.reshape(bt * M, 128)
    codes = torch.empty(bt * M, 16 * b, dtype=torch.uint8, device=A.device)
    sz = torch.empty(bt * M, 2, dtype=torch.float16, device=A.device)
    err = torch.zeros(1, dtype=torch.int32, device=A.device)
    check(lib().jolt_gemm_bf16_residual(_ptr(A3), _ptr(B3), M, K, A3.stride(1), B3.stride(1), bt,
                                        A3.stride(0), B3.stride(0), _ptr(X2),
                                        int(X2.dtype == torch.float32), seed, b, _ptr(codes), _ptr(sz),
                                        _ptr(err), _stream(stream)), "jolt_gemm_bf16_residual")
    return codes, sz, err


def sym_eig(A, stream=None):
    """Eigen-decomposition of symmetric fp32 matrices [batch?, n, n] on the GPU (block Jacobi).
    Returns (evals descending [batch?, n], evecs [batch?, n, n] with eigenvectors as columns)."""
    batched = A.dim() == 3
    A3 = (A if batched else A[None]).contiguous().float()
    bt, n = A3.shape[0], A3.shape[1]
    ev = torch.empty(bt, n, dtype=torch.float32, device=A.device)
    V = torch.empty(bt, n, n, dtype=torch.float32, device=A.device)
    ws = torch.empty(int(lib().jolt_sym_eig_workspace(n, bt)), dtype=torch.uint8, device=A.device)
    check(lib().jolt_sym_eig(_ptr(A3), n, bt, _ptr(ev), _ptr(V), _ptr(ws), ws.numel(), _stream(stream)),
          "jolt_sym_eig")
    return (ev, V) if batched else (ev[0], V[0])


def stats_enable(on=True):
    lib().jolt_stats_enable(int(on))


def stats_read(reset=True):
    """Per kernel family: launches, device ms (CUDA events), algorithmic flops and bytes."""
    from ._lib import KernelStat, KERNEL_FAMILIES
    arr = (KernelStat * len(KERNEL_FAMILIES))()
    check(lib().jolt_stats_read(arr, int(reset)), "jolt_stats_read")
    return {KERNEL_FAMILIES[i]: dict(launches=arr[i].launches, ms=arr[i].ms, flops=arr[i].flops,
                                     bytes=arr[i].bytes, flops_issued=arr[i].flops_issued)
            for i in range(len(KERNEL_FAMILIES))}


__all__ = ["analyze_from_host", "layer_align_workspace", "layer_align", "group_layers", "uniform_group", "gemm_bf16_hilo", "gemm_bf16_residual", "allocate_variant", "JOLT_ALLOC_JOINT", "JOLT_ALLOC_KV_SPLIT", "JOLT_ALLOC_UNIFORM", "JOLT_ALLOC_COORD", "GEMM_PLANS", "serialize_cache", "deserialize_cache", "cache_blob_info", "cache_blob_bytes", "decode_attn_noalloc", "stats_enable", "stats_read", "sym_eig", "gemm_bf16", "make_shape", "n_cells", "choices_array", "cell_bytes", "kv_bytes", "cache_layout", "phi",
           "allocate", "workspace_bytes", "new_workspace", "analyze", "compress", "decode_attn",
           "check_ws", "rotate_rows", "quantize_pack", "unpack_dequant", "JoltError",
           "JOLT_OP_COMPRESS", "JOLT_OP_DECODE"]
