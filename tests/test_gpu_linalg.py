"""GPU block-Jacobi eigensolver (jolt_sym_eig) vs LAPACK on the same matrices."""
import numpy as np
import pytest
import torch

from long_context_st_b200 import api

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n,batch", [(64, 1), (128, 3), (200, 2), (1152, 2)])
def test_sym_eig(cuda_ok, n, batch):
    rng = np.random.default_rng(n)
    A = []
    for b in range(batch):
        Q = np.linalg.qr(rng.standard_normal((n, n)))[0]
        lam = np.sort(rng.exponential(1.0, n) * np.logspace(0, -6, n))[::-1] * 1e4
        lam[: 4] *= 100.0        # a few dominant directions, like outlier channels
        A.append((Q * lam) @ Q.T)
    A = np.array(A)
    ev, V = api.sym_eig(torch.from_numpy(A).float().cuda())
    ev = ev.cpu().double().numpy()
    V = V.cpu().double().numpy()
    for b in range(batch):
        ref = np.sort(np.linalg.eigvalsh(A[b]))[::-1]
        assert np.max(np.abs(ev[b] - ref)) <= 2e-6 * ref[0]
        assert np.max(np.abs(V[b].T @ V[b] - np.eye(n))) <= 1e-5
        R = A[b] @ V[b] - V[b] * ev[b][None, :]
        assert np.max(np.abs(R)) <= 2e-6 * ref[0]
