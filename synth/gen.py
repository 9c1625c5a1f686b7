"""Seeded generators for K/V caches, decode queries and other inputs.

Every draw is keyed by (workload seed, purpose, indices) so a cell can be regenerated on its own.
Generation uses torch's generator on the target device: the same seed gives the same tensor on
any CUDA device; CPU draws differ from CUDA draws, so a test generates once and hands the same
tensor to both sides.
"""
import math

import numpy as np
import torch

_DT = {"f32": torch.float32, "bf16": torch.bfloat16, "f16": torch.float16}


def _subseed(*keys) -> int:
    h = 1469598103934665603
    for k in keys:
        if isinstance(k, str):
            k = sum((i + 1) * ord(c) for i, c in enumerate(k))
        h = ((h ^ (int(k) & 0xFFFFFFFFFFFF)) * 1099511628211) % (1 << 62)
    return h


def _gen(device, *keys) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_subseed(*keys))
    return g


def _decay(w, kv: str, b: int, layer: int) -> float:
    lo, hi = w.k_decay if kv == "K" else w.v_decay
    if lo == hi:
        return float(lo)
    u = torch.rand(1, generator=_gen("cpu", w.seed, "decay", kv, b, layer)).item()
    return float(lo + (hi - lo) * u)


def make_layer(w, kv: str, b: int, layer: int, device="cpu", dtype=None) -> torch.Tensor:
    """One layer's [n_kv, T, d_h] K or V slice of sequence b."""
    dtype = dtype or _DT[w.io_dtype]
    R, T, d = w.rank, w.T, w.d_h
    g = _gen(device, w.seed, kv, b, layer)
    f32 = torch.float32
    P = torch.randn(T, R, generator=g, device=device, dtype=f32)
    Q = torch.randn(d, R, generator=g, device=device, dtype=f32)
    C = torch.randn(w.n_kv, R, R, generator=g, device=device, dtype=f32)
    s = torch.tensor([_decay(w, kv, b, layer) ** i for i in range(R)], dtype=f32, device=device)
    PS = P * s[None, :]
    X = torch.empty(w.n_kv, T, d, device=device, dtype=f32)
    QT = Q.t().contiguous()
    for h in range(w.n_kv):
        X[h] = (PS @ C[h]) @ QT
    X += w.noise * torch.randn(w.n_kv, T, d, generator=g, device=device, dtype=f32)
    if kv == "K":
        for c in (d // 8, 3 * d // 8, 5 * d // 8, 7 * d // 8):
            X[:, :, c] *= w.outlier_scale
    return X.to(dtype)


def make_kv(w, device="cpu", dtype=None, batches=None, layers=None):
    """Full K and V tensors [B, L, n_kv, T, d_h] (optionally a subset of batches / layers)."""
    dtype = dtype or _DT[w.io_dtype]
    batches = list(range(w.batch)) if batches is None else list(batches)
    layers = list(range(w.n_layers)) if layers is None else list(layers)
    shape = (len(batches), len(layers), w.n_kv, w.T, w.d_h)
    K = torch.empty(shape, dtype=dtype, device=device)
    V = torch.empty(shape, dtype=dtype, device=device)
    for bi, b in enumerate(batches):
        for li, l in enumerate(layers):
            K[bi, li] = make_layer(w, "K", b, l, device, dtype)
            V[bi, li] = make_layer(w, "V", b, l, device, dtype)
    return K, V


def make_kv_cell(w, kv: str, b: int, group: int, device="cpu", dtype=None) -> torch.Tensor:
    """One cell's tensor [L_g, n_kv, T, d_h]."""
    L0 = group * w.layers_per_group
    return torch.stack([make_layer(w, kv, b, L0 + i, device, dtype)
                        for i in range(w.layers_per_group)])


def make_queries(w, device="cpu", dtype=None, n_layers=None) -> torch.Tensor:
    """Decode queries [B, L, n_q, d_h] ~ N(0, 1), one independent query per (sequence, layer)."""
    dtype = dtype or _DT[w.io_dtype]
    L = w.n_layers if n_layers is None else n_layers
    g = _gen(device, w.seed, "q")
    return torch.randn(w.batch, L, w.n_q, w.d_h, generator=g, device=device,
                       dtype=torch.float32).to(dtype)


def make_inv_freq(d_h: int, theta: float) -> np.ndarray:
    """RoPE inverse frequencies theta^(-2i/d_h), i < d_h/2, computed in float64, stored fp32."""
    i = np.arange(d_h // 2, dtype=np.float64)
    return (theta ** (-2.0 * i / d_h)).astype(np.float32)


def make_gaussian_rows(n_rows: int, d: int, seed: int, device="cpu") -> torch.Tensor:
    return torch.randn(n_rows, d, generator=_gen(device, seed, "rows"), device=device,
                       dtype=torch.float32)


def make_random_tables(n_cells: int, n_rt: int, n_rd: int, seed: int):
    """Random but well-formed spectra tails for allocator tests.

    Returns (norm2[c], tail_T[c][n_rt], tail_d[c][n_rd]) with tail[0] = norm2 and tails
    non-increasing and non-negative, as the tails of a real spectrum are.
    """
    rng = np.random.default_rng(seed)
    norm2 = rng.uniform(1e3, 1e5, size=n_cells)
    tT = np.empty((n_cells, n_rt))
    td = np.empty((n_cells, n_rd))
    for c in range(n_cells):
        for tab, n in ((tT, n_rt), (td, n_rd)):
            w = rng.exponential(1.0, size=n) * np.exp(-rng.uniform(0.01, 0.3) * np.arange(n))
            w = w / w.sum() * norm2[c] * rng.uniform(0.9, 1.0)
            cum = np.concatenate([[0.0], np.cumsum(w[:-1])])
            tab[c] = np.maximum(norm2[c] - cum, 0.0)
    return norm2, tT, td


def make_random_cache_parts(w, r_T: int, r_d: int, b: int, seed: int, device="cpu"):
    """Random stored-cache contents of one cell in storage dtypes (for decode-only tests).

    Returns dict(U_T [T, r_T], U_d [d_h, r_d], G [L_g, n_kv, r_T, r_d], codes u8
    [L_g, n_kv, T, d_h*b/8], sz f16 [L_g, n_kv, T, 2]) with magnitudes like a real cache's.
    """
    g = _gen(device, seed, "cache", r_T, r_d, b)
    fdt = _DT[w.factor_dtype]
    Lg, H, T, d = w.layers_per_group, w.n_kv, w.T, w.d_h
    out = {}
    out["U_T"] = (torch.randn(T, r_T, generator=g, device=device) / math.sqrt(T)).to(fdt)
    out["U_d"] = (torch.randn(d, r_d, generator=g, device=device) / math.sqrt(d)).to(fdt)
    sig = torch.logspace(3, 1, max(r_T, 1), device=device)[:r_T]
    out["G"] = (torch.randn(Lg, H, r_T, r_d, generator=g, device=device)
                * sig[None, None, :, None] / math.sqrt(max(r_d, 1))).to(fdt)
    nbytes = d * b // 8
    out["codes"] = torch.randint(0, 256, (Lg, H, T, nbytes), generator=g, device=device,
                                 dtype=torch.int32).to(torch.uint8)
    scale = torch.rand(Lg, H, T, generator=g, device=device) * 0.5 + 0.05
    zero = -(torch.rand(Lg, H, T, generator=g, device=device) * 2.0 + 0.5)
    out["sz"] = torch.stack([scale, zero], dim=-1).to(torch.float16)
    return out
