"""The full 70B-shaped workload (80 layers, 8 KV heads, 64 query heads, T = 131072, pre-RoPE keys,
3x budget) through analyze -> allocate -> compress -> decode, in the launch configuration the
benchmark times. The oracle cannot redo the whole step, so it checks sampled outputs one by one:
for a few (layer, KV head) pairs it rebuilds K and V from the GPU's own stored factors and codes
(oracle.decompress_slice), applies RoPE and runs dense attention for that head's query heads;
the GPU decode must match to the bf16 bar (1e-2). Properties that hold at any size: bytes within
the budget, tails non-increasing in the rank, stored token bases orthonormal to bf16 storage."""
import numpy as np
import pytest
import torch

import oracle
from synth import get_workload, make_kv, make_queries, make_inv_freq
from cache_io import device_cell, max_rel_err
from long_context_st_b200 import api

pytestmark = pytest.mark.gpu


def test_llama70b_128k_full_size_sampled(cuda_ok):
    w = get_workload("llama70b_128k")
    shape = api.make_shape(w)
    K, V = make_kv(w, device="cuda")
    q = make_queries(w, device="cuda")
    inv = make_inv_freq(w.d_h, w.rope_theta)
    cws = api.new_workspace(shape, api.JOLT_OP_COMPRESS)
    n2, tT, td = api.analyze(shape, K, V, cws)
    assert np.all(np.diff(tT, axis=1) <= 1e-9 * n2[:, None]) and np.all(np.diff(td, axis=1) <= 1e-9 * n2[:, None])
    raw = 2 * w.n_layers * w.n_kv * w.d_h * w.T * w.io_bytes
    budget = raw // 3
    choices, lam, tot = api.allocate(shape, n2, tT, td, api.phi(w.d_h), budget)
    _, total = api.cache_layout(shape, choices)
    assert total <= budget
    cache = torch.empty(total, dtype=torch.uint8, device="cuda")
    api.compress(shape, K, V, choices, cache, cws)
    del cws
    dws = api.new_workspace(shape, api.JOLT_OP_DECODE)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    api.decode_attn(shape, choices, cache, q, out, dws, lse=lse, inv_freq=torch.from_numpy(inv).cuda())
    api.check_ws(dws)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy()
    ls = lse.cpu().numpy()
    qn = q.double().cpu().numpy()
    G, Lg, gq = w.n_layers // w.layers_per_group, w.layers_per_group, w.n_q // w.n_kv
    for l, h in [(0, 0), (41, 5), (79, 7)]:
        g, ll = divmod(l, Lg)
        ck = device_cell(shape, w, cache, choices, 2 * g)
        cv = device_cell(shape, w, cache, choices, 2 * g + 1)
        if ck["r_T"]:
            U = torch.from_numpy(ck["U_T"]).cuda()
            assert torch.max(torch.abs(U.T @ U - torch.eye(U.shape[1], device="cuda", dtype=U.dtype))) < 2e-2
        Kh = oracle.decompress_slice(ck, ll, h, shape.rot_seed)
        Kh = oracle.rope(Kh[None], np.arange(w.T), inv)[0]
        Vh = oracle.decompress_slice(cv, ll, h, shape.rot_seed)
        ref, rl = oracle.decode_attention(Kh[None], Vh[None], qn[0, l, h * gq:(h + 1) * gq], shape.attn_scale)
        assert max_rel_err(o[0, l, h * gq:(h + 1) * gq], ref) <= 1e-2
        assert np.max(np.abs(ls[0, l, h * gq:(h + 1) * gq] - rl)) < 1e-3 * max(1.0, np.abs(rl).max())
