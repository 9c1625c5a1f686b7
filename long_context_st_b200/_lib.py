"""ctypes binding of libjolt.so (include/jolt.h). Argument marshalling only: every step of the
codec runs inside the library's CUDA kernels or its host C++ (allocator, layout).

Raises RuntimeError when the library is missing: there is no fallback implementation.
"""
import ctypes as C
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libjolt.so")

JOLT_OK = 0
STATUS = {0: "ok", -1: "invalid argument", -2: "CUDA error", -3: "device wait timed out",
          -4: "byte budget infeasible", -5: "numeric range error", -6: "workspace too small",
          -7: "workspace not prepared by jolt_analyze"}
JOLT_F32, JOLT_BF16 = 0, 1
JOLT_OP_COMPRESS, JOLT_OP_DECODE = 0, 1


class JoltError(RuntimeError):
    def __init__(self, status, what=""):
        self.status = status
        super().__init__(f"{what}: jolt status {status} ({STATUS.get(status, '?')})")


class Shape(C.Structure):
    _fields_ = [("batch", C.c_int32), ("n_layers", C.c_int32), ("layers_per_group", C.c_int32),
                ("n_kv", C.c_int32), ("n_q", C.c_int32), ("T", C.c_int32), ("d_h", C.c_int32),
                ("io_dtype", C.c_int32), ("factor_dtype", C.c_int32), ("keys_pre_rope", C.c_int32),
                ("q_cap", C.c_int32), ("sketch_cols", C.c_int32), ("power_iters", C.c_int32),
                ("cells_per_pass", C.c_int32), ("rot_seed", C.c_uint64), ("sketch_seed", C.c_uint64),
                ("attn_scale", C.c_float), ("rope_attention_scaling", C.c_float), ("gemm_plan", C.c_int32)]


class KernelStat(C.Structure):
    _fields_ = [("kernel", C.c_int32), ("launches", C.c_uint64), ("ms", C.c_double),
                ("flops", C.c_double), ("bytes", C.c_double), ("flops_issued", C.c_double)]


KERNEL_FAMILIES = ["gemm", "decode_main", "residual", "decode_aux", "chol", "eig"]


class CellChoice(C.Structure):
    _fields_ = [("r_T", C.c_int32), ("r_d", C.c_int32), ("b", C.c_int32)]


# (name, restype, argtypes) of every entry point declared in include/jolt.h
_P = C.c_void_p
SIGNATURES = [
    ("jolt_status_string", C.c_char_p, [C.c_int]),
    ("jolt_version", C.c_int32, []),
    ("jolt_shape_check", C.c_int, [C.POINTER(Shape)]),
    ("jolt_kv_bytes", C.c_uint64, [C.c_int32, C.c_int32, C.c_int32, C.c_int64, C.c_int32]),
    ("jolt_cell_bytes", C.c_uint64, [C.POINTER(Shape), CellChoice]),
    ("jolt_cache_blob_bytes", C.c_uint64, [C.POINTER(Shape), C.POINTER(CellChoice)]),
    ("jolt_cache_serialize", C.c_int, [C.POINTER(Shape), C.POINTER(CellChoice), C.c_void_p, C.c_void_p,
                                       C.c_uint64, C.c_void_p]),
    ("jolt_cache_blob_info", C.c_int, [C.c_void_p, C.c_uint64, C.POINTER(Shape), C.POINTER(C.c_int32),
                                       C.POINTER(C.c_uint64)]),
    ("jolt_cache_deserialize", C.c_int, [C.c_void_p, C.c_uint64, C.POINTER(CellChoice), C.c_int32, C.c_void_p,
                                         C.c_uint64, C.c_void_p]),
    ("jolt_cache_layout", C.c_int, [C.POINTER(Shape), C.POINTER(CellChoice), C.POINTER(C.c_uint64),
                                    C.POINTER(C.c_uint64)]),
    ("jolt_phi", C.c_int, [C.c_int32, C.c_int32, C.c_uint64, C.POINTER(C.c_double)]),
    ("jolt_allocate", C.c_int, [C.POINTER(Shape), C.c_int32, C.POINTER(C.c_double),
                                C.POINTER(C.c_double), C.c_int32, C.POINTER(C.c_double), C.c_int32,
                                C.POINTER(C.c_double), C.c_uint64, C.POINTER(CellChoice),
                                C.POINTER(C.c_double), C.POINTER(C.c_uint64)]),
    ("jolt_allocate_variant", C.c_int, [C.POINTER(Shape), C.c_int32, C.POINTER(C.c_double),
                                        C.POINTER(C.c_double), C.c_int32, C.POINTER(C.c_double), C.c_int32,
                                        C.POINTER(C.c_double), C.c_uint64, C.c_int32, C.POINTER(CellChoice),
                                        C.POINTER(C.c_uint64)]),
    ("jolt_workspace_bytes", C.c_size_t, [C.POINTER(Shape), C.c_int32]),
    ("jolt_analyze", C.c_int, [C.POINTER(Shape), _P, _P, C.POINTER(C.c_double),
                               C.POINTER(C.c_double), C.POINTER(C.c_double), _P, C.c_size_t, _P]),
    ("jolt_compress", C.c_int, [C.POINTER(Shape), _P, _P, C.POINTER(CellChoice), _P, C.c_uint64,
                                _P, C.c_size_t, _P]),
    ("jolt_decode_attn", C.c_int, [C.POINTER(Shape), C.POINTER(CellChoice), _P, C.c_int32,
                                   C.c_int32, _P, _P, _P, _P, C.c_int32, _P, C.c_size_t, _P]),
    ("jolt_check", C.c_int, [_P, _P]),
    ("jolt_decode_attn_noalloc", C.c_int, [C.POINTER(Shape), C.POINTER(CellChoice), _P, C.c_int32,
                                           C.c_int32, _P, _P, _P, _P, C.c_int32, _P]),
    ("jolt_rotate_rows", C.c_int, [_P, _P, C.c_int64, C.c_int32, C.c_uint64, C.c_int32, _P]),
    ("jolt_quantize_pack", C.c_int, [_P, C.c_int64, C.c_int32, C.c_int32, _P, _P, _P, _P]),
    ("jolt_unpack_dequant", C.c_int, [_P, _P, C.c_int64, C.c_int32, C.c_int32, _P, _P]),
    ("jolt_gemm_bf16", C.c_int, [_P, C.c_int32, _P, C.c_int32, _P, C.c_int32, C.c_int32, C.c_int32,
                                 C.c_int64, C.c_int64, C.c_int64, C.c_int32, C.c_int64, C.c_int64,
                                 C.c_int64, C.c_int32, C.c_int32, C.c_int32, _P]),
    ("jolt_gemm_bf16_hilo", C.c_int, [_P, C.c_int32, _P, C.c_int32, _P, _P, C.c_int32, C.c_int32,
                                      C.c_int32, C.c_int64, C.c_int64, C.c_int64, C.c_int32, C.c_int64,
                                      C.c_int64, C.c_int64, _P]),
    ("jolt_gemm_bf16_residual", C.c_int, [_P, _P, C.c_int32, C.c_int32, C.c_int64, C.c_int64, C.c_int32,
                                          C.c_int64, C.c_int64, _P, C.c_int32, C.c_uint64, C.c_int32, _P,
                                          _P, _P, _P]),
    ("jolt_analyze_from_host", C.c_int, [C.POINTER(Shape), _P, _P, _P, _P, _P, _P, _P, _P, C.c_size_t, _P]),
    ("jolt_layer_align_workspace", C.c_size_t, [C.POINTER(Shape), C.c_int32]),
    ("jolt_layer_align", C.c_int, [C.POINTER(Shape), C.c_int32, _P, _P, _P, _P, C.c_size_t, _P]),
    ("jolt_group_layers", C.c_int, [_P, C.c_int32, C.c_double, C.c_int32, _P, _P]),
    ("jolt_uniform_group", C.c_int, [_P, C.c_int32, C.c_double, _P]),
    ("jolt_selftest_timeout", C.c_int, [C.c_int32, C.c_uint64, _P, C.c_size_t, _P]),
    ("jolt_sym_eig_workspace", C.c_size_t, [C.c_int32, C.c_int32]),
    ("jolt_stats_enable", None, [C.c_int32]),
    ("jolt_stats_read", C.c_int, [C.POINTER(KernelStat), C.c_int32]),
    ("jolt_sym_eig", C.c_int, [_P, C.c_int32, C.c_int32, _P, _P, _P, C.c_size_t, _P]),
]

_lib = None


def lib():
    """The loaded library (loads on first use; fails loudly when it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} not built: run `python -m long_context_st_b200.build`")
        L = C.CDLL(LIB_PATH)
        for name, res, args in SIGNATURES:
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def check(status, what=""):
    if status != JOLT_OK:
        raise JoltError(status, what)
    return status
