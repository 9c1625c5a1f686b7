"""Whole-cell compression, decompression, RoPE and decode attention (float64 reference).

compress_cell: partial Tucker (oracle.hosvd) -> factors rounded to the storage dtype ->
residual R = X - X~ taken against the STORED factors -> rotated by the seeded rotation ->
rounded to float32 -> quantised and packed (oracle.quant) [v4 §3; nl Methodologie 1-2].

decompress_cell: X^ = U_T G U_d^T + rotation^T deq(codes), all from the stored cache; decoding
inverts the rotation [nl Methodologie 2].

rope: rotate-half RoPE of a pre-RoPE key at its position. [v4 §3]: keys are decomposed before
RoPE; [v4 §4.5]: RoPE does not commute with the factorisation, so keys are reconstructed per
tile and rotated. Angles t * inv_freq_i are taken in float64 from the fp32 inv_freq the model
supplies ([ru "Почему cos/sin строят в ядре"]: the model's own inv_freq and integer positions,
angles up to ~1e5 rad at 128K). Pairs are (i, i + d/2).

decode_attention: textbook softmax attention of one query per query head over all T cached
tokens (no causal mask: every cached token precedes the query), GQA head h' reading KV head
floor(h' / g_q) [ru "Сколько памяти занимает KV-кэш": each KV head serves g_q query heads].

Pinned by: with full ranks and b = 0 decode equals attention on the uncompressed cache
(checked against torch's scaled_dot_product_attention); RoPE preserves norms and relative
positions (q(t1).k(t2) depends on t2 - t1 only).
"""
import numpy as np
import torch

from .hosvd import st_hosvd, reconstruct
from .quant import quantize_rows, dequantize_rows, pack_codes, unpack_codes
from .rotation import rotation_matrix


def to_storage(a: np.ndarray, dtype: str) -> np.ndarray:
    """Round float64 values to the storage dtype; returned as float64 holding the stored values."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float64))
    tdt = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}[dtype]
    return t.to(tdt).to(torch.float64).numpy()


def compress_cell(X, r_T: int, r_d: int, b: int, rot_seed: int, factor_dtype: str):
    X = np.asarray(X, dtype=np.float64)
    L, H, T, d = X.shape
    out = {"r_T": r_T, "r_d": r_d, "b": b, "shape": X.shape}
    if r_T > 0:
        U_T, U_d, G, sig2, lam = st_hosvd(X, r_T, r_d)
        out["U_T"] = to_storage(U_T, factor_dtype)
        out["U_d"] = to_storage(U_d, factor_dtype)
        out["G"] = to_storage(G, factor_dtype)
        Xt = reconstruct(out["U_T"], out["G"], out["U_d"])
    else:
        out["U_T"] = np.zeros((T, 0))
        out["U_d"] = np.zeros((d, 0))
        out["G"] = np.zeros((L, H, 0, 0))
        Xt = np.zeros_like(X)
    if b > 0:
        M = rotation_matrix(d, rot_seed)
        Rrot = ((X - Xt) @ M.T).astype(np.float32)
        code, scale, zero = quantize_rows(Rrot, b)
        out["codes"] = pack_codes(code, b)
        out["scale"] = scale
        out["zero"] = zero
        out["rot_resid"] = Rrot
    return out


def residual_hat(cell, rot_seed: int) -> np.ndarray:
    L, H, T, d = cell["shape"]
    b = cell["b"]
    if b == 0:
        return np.zeros((L, H, T, d))
    code = unpack_codes(cell["codes"], b, d)
    deq = dequantize_rows(code, cell["scale"], cell["zero"]).astype(np.float64)
    M = rotation_matrix(d, rot_seed)
    return deq @ M


def decompress_cell(cell, rot_seed: int) -> np.ndarray:
    L, H, T, d = cell["shape"]
    if cell["r_T"] > 0:
        Xt = reconstruct(cell["U_T"], cell["G"], cell["U_d"])
    else:
        Xt = np.zeros((L, H, T, d))
    return Xt + residual_hat(cell, rot_seed)


def decompress_slice(cell, l: int, h: int, rot_seed: int) -> np.ndarray:
    """X^[l, h] of one cell (layer l of the group, KV head h) without rebuilding the rest:
    U_T (G[l, h] U_d^T) + rotation^T deq(codes[l, h]) — the same stored values as decompress_cell."""
    L, H, T, d = cell["shape"]
    if cell["r_T"] > 0:
        Xt = cell["U_T"] @ (cell["G"][l, h] @ cell["U_d"].T)
    else:
        Xt = np.zeros((T, d))
    if cell["b"] == 0:
        return Xt
    code = unpack_codes(cell["codes"][l, h], cell["b"], d)
    deq = dequantize_rows(code, cell["scale"][l, h], cell["zero"][l, h]).astype(np.float64)
    return Xt + deq @ rotation_matrix(d, rot_seed)


def rope(x: np.ndarray, positions: np.ndarray, inv_freq: np.ndarray) -> np.ndarray:
    """x [..., T, d] float64, positions [T] ints, inv_freq [d/2] float32 -> rotated float64."""
    d = x.shape[-1]
    ang = positions.astype(np.float64)[:, None] * inv_freq.astype(np.float64)[None, :]
    c, s = np.cos(ang), np.sin(ang)
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def decode_attention(K: np.ndarray, V: np.ndarray, q: np.ndarray, scale: float):
    """K, V [n_kv, T, d], q [n_q, d] (float64) -> (out [n_q, d], lse [n_q])."""
    n_kv = K.shape[0]
    n_q = q.shape[0]
    gq = n_q // n_kv
    out = np.empty((n_q, K.shape[2]))
    lse = np.empty(n_q)
    for hq in range(n_q):
        h = hq // gq
        s = (K[h] @ q[hq]) * scale
        m = s.max()
        p = np.exp(s - m)
        ell = p.sum()
        out[hq] = (p @ V[h]) / ell
        lse[hq] = m + np.log(ell)
    return out, lse
