"""Uniform b-bit quantiser of the rotated residual, bit packing, and the quantiser's error fraction.

[nl Methodologie 2]: the rotated residual is quantised uniformly at b in {0, 2, 4, 8} bits;
[v4 §3]: b = 0 stores no residual. The pages fix neither the granularity nor the parameter
format. Reading: asymmetric min/max quantisation per row (one (layer, head, token) vector of d_h
rotated values) with an fp16 scale and an fp16 zero (4 bytes per row, as the int8 ratio
2T/(T+4) of [v4 App. E] implies), computed in float32 arithmetic, each operation rounded once:

    mn, mx = min(x), max(x)                       (x: float32 row)
    scale  = f16( f32( f32(mx - mn) / f32(2^b - 1) ) )
    zero   = f16( mn )
    code_j = clip( rint( f32( f32(x_j - zero) / scale ) ), 0, 2^b - 1 )   (0 when scale == 0)
    deq_j  = f32( code_j * scale + zero )         (exact product and sum, one rounding)

rint is round-half-to-even. fp16 scale or zero outside +-65504 is a numeric error.
Packing: code j occupies bits [(j*b) mod 8, (j*b) mod 8 + b) of byte floor(j*b/8), little-endian.

The error fraction phi(b) [v4 §3: the surrogate "multiplies the discarded-mass estimate by the
fraction unrecovered by the rotated quantizer"] is measured by Monte Carlo on N(0, I) rows, since a
rotated residual row is close to Gaussian; phi(0) = 1.

Pinned by: the per-element error bound of uniform rounding; decreasing aggregate error in b;
phi(8)/phi(4) ~ ((2^4-1)/(2^8-1))^2 (step-squared law); pack/unpack round trip and hand-packed bytes.
"""
import numpy as np

F16_MAX = 65504.0


class NumericError(ValueError):
    pass


def quantize_rows(x: np.ndarray, b: int):
    """x float32 [..., d] -> (codes uint8 [..., d], scale f16 [...], zero f16 [...])."""
    x = np.asarray(x, dtype=np.float32)
    assert b in (2, 4, 8)
    levels = np.float32((1 << b) - 1)
    mn = x.min(axis=-1)
    mx = x.max(axis=-1)
    step = np.float32(mx - mn) / levels
    step = step.astype(np.float32)
    with np.errstate(over="ignore"):
        scale = step.astype(np.float16)
        zero = mn.astype(np.float16)
    if not (np.all(np.isfinite(scale)) and np.all(np.isfinite(zero))):
        raise NumericError("fp16 scale/zero out of range")
    s32 = scale.astype(np.float32)[..., None]
    z32 = zero.astype(np.float32)[..., None]
    diff = (x - z32).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        qv = (diff / s32).astype(np.float32)
    code = np.rint(qv)
    code = np.where(s32 == 0, 0.0, code)
    code = np.clip(code, 0, (1 << b) - 1).astype(np.uint8)
    return code, scale, zero


def dequantize_rows(code: np.ndarray, scale: np.ndarray, zero: np.ndarray) -> np.ndarray:
    """float32 [..., d] = f32(code * scale + zero), exact in float64 then rounded once."""
    v = code.astype(np.float64) * scale.astype(np.float64)[..., None] \
        + zero.astype(np.float64)[..., None]
    return v.astype(np.float32)


def pack_codes(code: np.ndarray, b: int) -> np.ndarray:
    code = np.asarray(code, dtype=np.uint8)
    d = code.shape[-1]
    per = 8 // b
    assert d % per == 0
    c = code.reshape(*code.shape[:-1], d // per, per).astype(np.uint16)
    out = np.zeros(c.shape[:-1], dtype=np.uint16)
    for k in range(per):
        out |= c[..., k] << (k * b)
    return out.astype(np.uint8)


def unpack_codes(packed: np.ndarray, b: int, d: int) -> np.ndarray:
    packed = np.asarray(packed, dtype=np.uint8)
    per = 8 // b
    mask = (1 << b) - 1
    parts = [(packed >> (k * b)) & mask for k in range(per)]
    out = np.stack(parts, axis=-1).reshape(*packed.shape[:-1], packed.shape[-1] * per)
    assert out.shape[-1] == d
    return out.astype(np.uint8)


_PHI_CACHE = {}


def phi_table(d: int, n_rows: int = 1 << 16, seed: int = 1):
    """[phi(0), phi(2), phi(4), phi(8)] for rows of dimension d (Monte Carlo, N(0, I) rows)."""
    key = (d, n_rows, seed)
    if key in _PHI_CACHE:
        return list(_PHI_CACHE[key])
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n_rows, d)).astype(np.float32)
    tot = float(np.sum(x.astype(np.float64) ** 2))
    phi = [1.0]
    for b in (2, 4, 8):
        c, s, z = quantize_rows(x, b)
        e = x.astype(np.float64) - dequantize_rows(c, s, z).astype(np.float64)
        phi.append(float(np.sum(e * e)) / tot)
    _PHI_CACHE[key] = tuple(phi)
    return phi
