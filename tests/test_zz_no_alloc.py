"""Decode attention through the allocation-free entry point (jolt_decode_attn_noalloc).

For callers that cannot allocate device memory while decoding (a runtime plugin handed only a
stream, a serving loop with pre-planned memory): the call must give the same outputs as
jolt_decode_attn with a caller-provided workspace, on two calls in a row (the built-in scratch is
reused between calls), and refuse calls whose scratch would not fit.
"""
import numpy as np
import pytest
import torch

from synth import get_workload, make_kv, make_queries, make_inv_freq
from cache_io import oracle_cells, cells_to_device, max_rel_err
from long_context_st_b200 import api

pytestmark = pytest.mark.gpu


def setup(w, choices):
    shape = api.make_shape(w)
    K, V = make_kv(w, device="cuda")
    q = make_queries(w, device="cuda")
    cells = oracle_cells(w, K, V, choices, shape.rot_seed)
    cache = cells_to_device(shape, w, cells, choices)
    inv = torch.from_numpy(make_inv_freq(w.d_h, w.rope_theta)).cuda()
    return shape, cache, q, inv


@pytest.mark.parametrize("name,over,choice,tol", [
    ("toy", {}, (32, 32, 4), 1e-3),
    ("llama8b_64k_b4", {"n_layers": 4, "T": 999, "batch": 2}, (48, 64, 4), 1e-2),
])
def test_noalloc_matches_workspace_decode_twice(cuda_ok, name, over, choice, tol):
    w = get_workload(name, **over)
    choices = [choice] * (2 * w.batch * (w.n_layers // w.layers_per_group))
    shape, cache, q, inv = setup(w, choices)
    ws = api.new_workspace(shape, api.JOLT_OP_DECODE)
    ref = torch.empty_like(q)
    ref_lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    api.decode_attn(shape, choices, cache, q, ref, ws, lse=ref_lse, inv_freq=inv)
    api.check_ws(ws)
    for _ in range(2):
        out = torch.full_like(q, float("nan"))
        lse = torch.full(q.shape[:3], float("nan"), dtype=torch.float32, device="cuda")
        # one call per layer, as a decode loop makes them (keeps the scratch well under 32 MiB)
        for l in range(w.n_layers):
            o_l = torch.empty_like(q[:, l:l + 1])
            s_l = torch.empty(q.shape[0], 1, q.shape[2], dtype=torch.float32, device="cuda")
            api.decode_attn_noalloc(shape, choices, cache, q[:, l:l + 1].contiguous(), o_l, lse=s_l,
                                    inv_freq=inv, layer_begin=l, n_layers_call=1)
            out[:, l:l + 1] = o_l
            lse[:, l:l + 1] = s_l
        torch.cuda.synchronize()
        o, r = out.float().cpu().numpy(), ref.float().cpu().numpy()
        assert np.isfinite(o).all()
        for b in range(w.batch):
            for l in range(w.n_layers):
                assert max_rel_err(o[b, l], r[b, l]) <= tol
        assert torch.allclose(lse, ref_lse, rtol=1e-4, atol=1e-4)


def test_noalloc_rejects_scratch_beyond_limit(cuda_ok):
    # all 80 layers of the 70B-shaped workload in one call need ~370 MB of scratch (> 32 MiB);
    # the call must refuse before touching any buffer
    w = get_workload("llama70b_128k")
    shape = api.make_shape(w)
    choices = [(256, 128, 4)] * api.n_cells(shape)
    dummy = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(api.JoltError) as e:
        api.decode_attn_noalloc(shape, choices, dummy, dummy, dummy, inv_freq=dummy)
    assert e.value.status == -6
