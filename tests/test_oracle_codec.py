"""Pins of the oracle's compress/decompress, RoPE and decode attention."""
import numpy as np
import torch
import pytest

from oracle.codec import compress_cell, decompress_cell, decompress_slice, rope, decode_attention
from oracle.hosvd import st_hosvd, reconstruct
from synth import get_workload, make_kv_cell, make_inv_freq


def sdpa(K, V, q, scale):
    n_kv, n_q = K.shape[0], q.shape[0]
    g = n_q // n_kv
    Kt = torch.from_numpy(K).repeat_interleave(g, 0)
    Vt = torch.from_numpy(V).repeat_interleave(g, 0)
    qt = torch.from_numpy(q)[:, None, :]
    o = torch.nn.functional.scaled_dot_product_attention(qt, Kt, Vt, scale=scale)
    return o[:, 0, :].numpy()


def test_decode_matches_sdpa():
    rng = np.random.default_rng(0)
    K = rng.standard_normal((2, 300, 64))
    V = rng.standard_normal((2, 300, 64))
    q = rng.standard_normal((8, 64)) * 3
    out, lse = decode_attention(K, V, q, 0.125)
    assert np.max(np.abs(out - sdpa(K, V, q, 0.125))) < 1e-12
    s = np.einsum("td,d->t", K[0], q[0]) * 0.125
    assert lse[0] == pytest.approx(np.log(np.sum(np.exp(s))), rel=1e-12)


def test_full_rank_no_residual_is_lossless():
    w = get_workload("toy")
    X = make_kv_cell(w, "V", 0, 0, dtype=torch.float64).numpy()
    n = X.shape[0] * X.shape[1] * X.shape[3]
    cell = compress_cell(X, n, X.shape[3], 0, 1, "f32")
    Xh = decompress_cell(cell, 1)
    assert np.linalg.norm(Xh - X) / np.linalg.norm(X) < 1e-6   # fp32 factor storage
    q = np.random.default_rng(1).standard_normal((8, 64))
    o1, _ = decode_attention(Xh[0], Xh[0], q, 0.125)
    o2 = sdpa(X[0], X[0], q, 0.125)
    assert np.max(np.abs(o1 - o2)) / np.max(np.abs(o2)) < 1e-5


def test_residual_error_decreases_with_bits_and_b0_is_tucker_only():
    w = get_workload("toy")
    X = make_kv_cell(w, "K", 0, 0, dtype=torch.float64).numpy()
    errs = []
    for b in (0, 2, 4, 8):
        cell = compress_cell(X, 32, 32, b, 5, "f32")
        errs.append(np.sum((decompress_cell(cell, 5) - X) ** 2))
    U_T, U_d, G, _, _ = st_hosvd(X, 32, 32)
    tucker = np.sum((reconstruct(U_T, G, U_d) - X) ** 2)
    assert errs[0] == pytest.approx(tucker, rel=1e-5)
    assert errs[0] > errs[1] > errs[2] > errs[3]


def test_rope_complex_form_and_relative_position():
    rng = np.random.default_rng(3)
    d = 64
    inv = make_inv_freq(d, 500000.0)
    x = rng.standard_normal((5, d))
    pos = np.array([0, 1, 1000, 65535, 131071])
    y = rope(x, pos, inv)
    z = (x[:, : d // 2] + 1j * x[:, d // 2:]) * np.exp(1j * pos[:, None] * inv.astype(np.float64))
    assert np.max(np.abs(y - np.concatenate([z.real, z.imag], -1))) < 1e-9
    assert np.allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1))
    q, k = rng.standard_normal(d), rng.standard_normal(d)
    a = rope(q[None], np.array([10]), inv) @ rope(k[None], np.array([3]), inv).T
    b = rope(q[None], np.array([1007]), inv) @ rope(k[None], np.array([1000]), inv).T
    assert abs(a - b).max() < 1e-9


@pytest.mark.parametrize("ch", [(32, 32, 4), (0, 0, 2), (48, 16, 0), (16, 64, 8)])
def test_decompress_slice_is_the_cells_slice(ch):
    # every (layer, head) slice of the whole-cell reconstruction, for factor-only, residual-only
    # and mixed cells (an index or transpose slip in the slice path breaks it)
    w = get_workload("toy", n_layers=2, layers_per_group=2)
    X = make_kv_cell(w, "K", 0, 0, dtype=torch.float64).numpy()
    cell = compress_cell(X, *ch, 7, "bf16")
    full = decompress_cell(cell, 7)
    for l in range(X.shape[0]):
        for h in range(X.shape[1]):
            assert np.allclose(decompress_slice(cell, l, h, 7), full[l, h], rtol=0, atol=1e-12)
