"""Oracle pins for layer grouping by token-mode subspace alignment ([v4 §3]; the measure and
threshold are this codec's reading, stated in oracle/grouping.py)."""
import numpy as np
import pytest

from oracle.grouping import (layer_token_basis, subspace_alignment, layer_alignment, group_layers,
                             uniform_group)


def orthonormal(rng, T, k):
    Q, _ = np.linalg.qr(rng.standard_normal((T, k)))
    return Q


def test_same_subspace_in_another_basis_is_one():
    rng = np.random.default_rng(1)
    U = orthonormal(rng, 200, 8)
    R, _ = np.linalg.qr(rng.standard_normal((8, 8)))
    assert subspace_alignment(U, U @ R) == pytest.approx(1.0, abs=1e-12)


def test_orthogonal_subspaces_are_zero():
    rng = np.random.default_rng(2)
    Q = orthonormal(rng, 200, 16)
    assert subspace_alignment(Q[:, :8], Q[:, 8:]) == pytest.approx(0.0, abs=1e-12)


@pytest.mark.parametrize("theta", [0.1, 0.7, 1.3])
def test_one_principal_angle(theta):
    # k = 1: e1 vs cos(theta) e1 + sin(theta) e2 -> cos^2(theta)
    T = 10
    U1 = np.zeros((T, 1)); U1[0, 0] = 1.0
    U2 = np.zeros((T, 1)); U2[0, 0] = np.cos(theta); U2[1, 0] = np.sin(theta)
    assert subspace_alignment(U1, U2) == pytest.approx(np.cos(theta) ** 2, abs=1e-14)


def test_j_of_k_shared_directions():
    rng = np.random.default_rng(3)
    Q = orthonormal(rng, 300, 12)
    U1 = Q[:, :6]
    U2 = np.concatenate([Q[:, :2], Q[:, 6:10]], axis=1)  # 2 of 6 shared, rest orthogonal
    assert subspace_alignment(U1, U2) == pytest.approx(2 / 6, abs=1e-12)


def test_layer_token_basis_is_the_top_singular_subspace():
    rng = np.random.default_rng(4)
    H, T, d, k = 2, 64, 8, 3
    A = orthonormal(rng, T, k)
    W = rng.standard_normal((k, H * d)) * np.array([10.0, 5.0, 2.0])[:, None]
    Xu = A @ W + 1e-6 * rng.standard_normal((T, H * d))
    X = Xu.reshape(T, H, d).transpose(1, 0, 2)  # [n_kv, T, d_h]
    U = layer_token_basis(X, k)
    assert np.allclose(U.T @ U, np.eye(k), atol=1e-10)
    assert subspace_alignment(U, A) == pytest.approx(1.0, abs=1e-9)


def test_group_layers_hand_cases():
    assert group_layers([], 0.5) == [1]
    assert group_layers([0.9, 0.8, 0.1, 0.95, 0.2], 0.5) == [3, 2, 1]
    assert group_layers([0.9, 0.9, 0.9, 0.9], 0.5, max_group=2) == [2, 2, 1]
    assert group_layers([0.5, 0.49], 0.5) == [2, 1]  # the threshold is inclusive


def test_uniform_group_hand_cases():
    # 8 layers; breaks at (1,2) and (5,6) -> L_g = 2 keeps every group aligned, 4 does not
    a = [0.9, 0.1, 0.9, 0.9, 0.9, 0.1, 0.9]
    assert uniform_group(a, 8, 0.5) == 2
    assert uniform_group([0.9] * 7, 8, 0.5) == 8
    assert uniform_group([0.1] * 7, 8, 0.5) == 1
    assert uniform_group([0.9, 0.9, 0.1, 0.9, 0.9], 6, 0.5) == 3


def planted_layers(rng, sizes, H, T, d, r, noise=1e-3):
    """K or V [L, H, T, d] whose layers share a token subspace within each planted group."""
    layers = []
    for size in sizes:
        A = orthonormal(rng, T, r)
        for _ in range(size):
            W = rng.standard_normal((r, H * d)) * np.linspace(3.0, 1.0, r)[:, None]
            Xu = A @ W + noise * rng.standard_normal((T, H * d))
            layers.append(Xu.reshape(T, H, d).transpose(1, 0, 2))
    return np.stack(layers)


def test_planted_groups_recovered():
    rng = np.random.default_rng(5)
    sizes = [3, 2, 1]
    K = planted_layers(rng, sizes, 2, 256, 32, 8)
    V = planted_layers(rng, sizes, 2, 256, 32, 8)
    a = layer_alignment(K, V, 8)
    assert a.shape == (5,)
    inside = [0, 1, 3]
    assert np.all(a[inside] > 0.99)
    assert np.all(np.delete(a, inside) < 0.2)
    assert group_layers(a, 0.5) == sizes


def test_grouping_properties_random():
    """group sizes partition the layers; every in-group link is >= tau and every boundary link
    is < tau (without a size cap); the uniform size divides L and respects tau inside groups."""
    rng = np.random.default_rng(11)
    for _ in range(200):
        L = int(rng.integers(1, 40))
        a = rng.uniform(0, 1, size=L - 1)
        tau = float(rng.uniform(0.1, 0.9))
        sizes = group_layers(a, tau)
        assert sum(sizes) == L and min(sizes) >= 1
        edge = np.cumsum(sizes)[:-1] - 1          # last layer of each group but the final one
        inside = np.setdiff1d(np.arange(L - 1), edge)
        assert np.all(a[inside] >= tau) and np.all(a[edge] < tau)
        Lg = uniform_group(a, L, tau)
        assert L % Lg == 0
        assert all(a[l] >= tau for l in range(L - 1) if (l + 1) % Lg)
        # no larger divisor qualifies
        for g in range(Lg + 1, L + 1):
            if L % g == 0:
                assert not all(a[l] >= tau for l in range(L - 1) if (l + 1) % g)
