"""A compressed cache written to a host blob and read back is byte-identical and decodes to the
same outputs (up to the summation order of the decode's atomic partial sums)."""
import numpy as np
import pytest
import torch

from synth import get_workload, make_kv, make_queries, make_inv_freq
from long_context_st_b200 import api

pytestmark = pytest.mark.gpu


def test_blob_round_trip_decodes_identically(cuda_ok):
    w = get_workload("llama8b_64k_b4", n_layers=4, T=777, batch=2)
    shape = api.make_shape(w)
    K, V = make_kv(w, device="cuda")
    q = make_queries(w, device="cuda")
    inv = torch.from_numpy(make_inv_freq(w.d_h, w.rope_theta)).cuda()
    cws = api.new_workspace(shape, api.JOLT_OP_COMPRESS)
    api.analyze(shape, K, V, cws)
    choices = [(96, 64, 4), (48, 128, 2), (0, 0, 8), (128, 32, 0)]
    _, total = api.cache_layout(shape, choices)
    cache = torch.zeros(total, dtype=torch.uint8, device="cuda")
    api.compress(shape, K, V, choices, cache, cws)
    blob = api.serialize_cache(shape, choices, cache)
    s2, ch2, cache2 = api.deserialize_cache(blob)
    assert ch2 == choices and bytes(s2) == bytes(shape)
    assert torch.equal(cache2[:total], cache)
    dws = api.new_workspace(shape, api.JOLT_OP_DECODE)
    o1 = torch.empty_like(q)
    o2 = torch.empty_like(q)
    api.decode_attn(shape, choices, cache, q, o1, dws, inv_freq=inv)
    api.decode_attn(s2, ch2, cache2, q, o2, dws, inv_freq=inv)
    torch.cuda.synchronize()
    # the bytes are identical (above); decode sums split-K partials with float atomics, whose
    # order (hence last-bit rounding) may differ from one call to the next: the bf16 outputs agree
    # to one unit in the last place
    a, b = o1.float(), o2.float()
    ulp = torch.maximum(a.abs(), b.abs()) * 2.0 ** -7 + 1e-30
    assert bool(((a - b).abs() <= ulp).all())
    assert (a - b).abs().max().item() <= 2.0 ** -7 * a.abs().max().item()
