"""GPU layer alignment (jolt_layer_align: randomized top-k token subspaces of every layer, then
||U_l^T U_{l+1}||_F^2 / k) vs the oracle's exact-SVD alignment, and the grouping it implies."""
import numpy as np
import pytest
import torch

from oracle.grouping import layer_alignment, group_layers
from synth import get_workload
from long_context_st_b200 import api

pytestmark = pytest.mark.gpu


def planted(rng, sizes, B, H, T, d, r, noise):
    """[B, L, H, T, d]: layers of one planted group share a rank-r token subspace."""
    out = np.zeros((B, sum(sizes), H, T, d))
    for b in range(B):
        l = 0
        for size in sizes:
            A, _ = np.linalg.qr(rng.standard_normal((T, r)))
            for _ in range(size):
                W = rng.standard_normal((r, H * d)) * np.linspace(4.0, 1.0, r)[:, None]
                Xu = A @ W + noise * rng.standard_normal((T, H * d))
                out[b, l] = Xu.reshape(T, H, d).transpose(1, 0, 2)
                l += 1
    return out


@pytest.mark.parametrize("io,T,sizes,k", [("bf16", 1000, [3, 2, 1], 16), ("f32", 777, [2, 2, 2, 2], 32),
                                          ("bf16", 4096, [1, 4, 3], 16)])
def test_layer_alignment_and_groups(cuda_ok, io, T, sizes, k):
    rng = np.random.default_rng(T + k)
    B, H, d = 2, 2, 64
    L = sum(sizes)
    K = planted(rng, sizes, B, H, T, d, k, 0.02)
    V = planted(rng, sizes, B, H, T, d, k, 0.02)
    w = get_workload("toy", n_layers=L, T=T, batch=B, n_kv=H, n_q=4 * H, d_h=d, io_dtype=io,
                     layers_per_group=1)
    s = api.make_shape(w)
    dt = torch.bfloat16 if io == "bf16" else torch.float32
    Kd = torch.from_numpy(K).to(dt).cuda()
    Vd = torch.from_numpy(V).to(dt).cuda()
    a_gpu = api.layer_align(s, Kd, Vd, rank=k)
    assert a_gpu.shape == (B, L - 1)
    for b in range(B):
        a_ref = layer_alignment(Kd[b].double().cpu().numpy(), Vd[b].double().cpu().numpy(), k)
        assert np.max(np.abs(a_gpu[b] - a_ref)) < 0.02, (a_gpu[b], a_ref)
        assert api.group_layers(a_gpu[b], 0.5) == sizes == group_layers(a_ref, 0.5)


def test_layer_align_rejects_bad_rank(cuda_ok):
    w = get_workload("toy", n_layers=2, layers_per_group=1)
    s = api.make_shape(w)
    K = torch.zeros(1, 2, w.n_kv, w.T, w.d_h, dtype=torch.float32, device="cuda")
    with pytest.raises(api.JoltError):
        api.layer_align(s, K, K, rank=24)  # not a multiple of 16
