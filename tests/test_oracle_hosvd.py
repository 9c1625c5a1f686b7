"""Pins of the oracle's ST-HOSVD against exact recovery, the HOSVD error identity and
Eckart-Young."""
import numpy as np
import pytest

from oracle import hosvd
from oracle.hosvd import st_hosvd, reconstruct, spectra_tails, token_unfolding


def planted(L, H, T, d, rT, rd, seed=0, noise=0.0):
    rng = np.random.default_rng(seed)
    U = np.linalg.qr(rng.standard_normal((T, rT)))[0]
    W = np.linalg.qr(rng.standard_normal((d, rd)))[0]
    C = rng.standard_normal((L, H, rT, rd)) * 3
    X = np.einsum("tr,lhrk,jk->lhtj", U, C, W)
    return X + noise * rng.standard_normal(X.shape)


def test_exact_recovery_full_rank():
    X = planted(2, 3, 200, 32, 12, 10, seed=1)
    U_T, U_d, G, _, _ = st_hosvd(X, 12, 10)
    err = np.linalg.norm(X - reconstruct(U_T, G, U_d)) / np.linalg.norm(X)
    assert err < 1e-10


def test_orthonormal_factors():
    X = planted(2, 2, 300, 64, 40, 30, seed=2, noise=0.1)
    U_T, U_d, G, _, _ = st_hosvd(X, 32, 16)
    assert np.max(np.abs(U_T.T @ U_T - np.eye(32))) < 1e-12
    assert np.max(np.abs(U_d.T @ U_d - np.eye(16))) < 1e-12


@pytest.mark.parametrize("rT,rd", [(8, 8), (16, 32), (40, 20), (64, 64)])
def test_st_hosvd_error_identity(rT, rd):
    # Orthogonal projections: ||X - X~||^2 = token tail + feature tail of the projected tensor.
    X = planted(2, 2, 256, 64, 48, 40, seed=3, noise=0.3)
    U_T, U_d, G, sig2, lamY = st_hosvd(X, rT, rd)
    err2 = np.sum((X - reconstruct(U_T, G, U_d)) ** 2)
    pred = np.sum(sig2[rT:]) + np.sum(lamY[rd:])
    assert abs(err2 - pred) <= 1e-9 * np.sum(X ** 2)


def test_eckart_young_single_slice():
    # L_g = n_kv = 1 and r_T = r_d = r: the truncated SVD, error = sum of trailing s^2.
    rng = np.random.default_rng(4)
    A = rng.standard_normal((120, 48)) @ np.diag(0.9 ** np.arange(48)) @ rng.standard_normal((48, 48))
    X = A[None, None]
    ev = np.sort(np.linalg.eigvalsh(A.T @ A))[::-1]
    for r in (4, 16, 30):
        U_T, U_d, G, _, _ = st_hosvd(X, r, r)
        err2 = np.sum((X - reconstruct(U_T, G, U_d)) ** 2)
        assert abs(err2 - ev[r:].sum()) <= 1e-8 * ev.sum()


def test_gram_path_matches_svd_path(monkeypatch):
    X = planted(1, 4, 900, 32, 20, 16, seed=5, noise=0.2)
    XT = token_unfolding(X)
    U1, s1 = hosvd._token_svd(XT, 24)
    monkeypatch.setattr(hosvd, "SVD_MAX_ELEMS", 0)
    U2, s2 = hosvd._token_svd(XT, 24)
    assert np.allclose(s2[:24], s1[:24], rtol=1e-9)
    assert np.max(np.abs(U1 @ U1.T - U2 @ U2.T)) < 1e-8
    assert np.max(np.abs(U2.T @ U2 - np.eye(24))) < 1e-12


def test_spectra_tails():
    X = planted(2, 2, 256, 64, 20, 24, seed=6, noise=0.05)
    n2, tT, td = spectra_tails(X, 128)
    assert tT[0] == pytest.approx(n2) and td[0] == pytest.approx(n2)
    assert np.all(np.diff(tT) <= 1e-9 * n2) and np.all(np.diff(td) <= 1e-9 * n2)
    assert tT[-1] <= 1e-9 * n2 + np.sum(0.05 ** 2 * X.size) * 2
    assert td[-1] <= 1e-9 * n2
    # tails agree with the ST-HOSVD spectra at the same ranks
    _, _, _, sig2, _ = st_hosvd(X, 16, 16)
    assert tT[1] == pytest.approx(sig2[16:].sum(), rel=1e-9)


def _known_spectrum_tensor(L, H, T, d, sig, seed):
    """X[l,h] = A_lh diag(sig) W^T with every A_lh [T, d] having orthonormal columns and W an
    orthogonal d x d basis: X[l,h]^T X[l,h] = W diag(sig^2) W^T for every (l, h), so the feature
    Gram sum_lh X_lh^T X_lh has the eigenvalues L*H*sig_j^2 exactly (up to rounding)."""
    rng = np.random.default_rng(seed)
    W = np.linalg.qr(rng.standard_normal((d, d)))[0]
    X = np.empty((L, H, T, d))
    for l in range(L):
        for h in range(H):
            A = np.linalg.qr(rng.standard_normal((T, d)))[0]
            X[l, h] = (A * sig[None, :]) @ W.T
    return X


@pytest.mark.parametrize("L,H", [(1, 1), (2, 3)])
def test_spectra_tails_feature_closed_form(L, H):
    # [v4 §3] the feature-mode tail is the discarded energy sum_{j > r_d} lambda_j(S_d), lambda in
    # decreasing order. Singular values given in a shuffled order: a tail summed from the
    # smallest eigenvalue first, or over the wrong end, misses the closed form below.
    d, T = 64, 160
    rng = np.random.default_rng(11)
    sig = rng.permutation(np.linspace(5.0, 0.1, d) ** 1.5)
    X = _known_spectrum_tensor(L, H, T, d, sig, seed=12)
    n2, tT, td = spectra_tails(X, 64)
    lam = np.sort(L * H * sig ** 2)[::-1]
    assert n2 == pytest.approx(lam.sum(), rel=1e-12)
    for j in range(d // 16 + 1):
        assert td[j] == pytest.approx(lam[16 * j:].sum(), rel=1e-9, abs=1e-9 * n2), j
    if L * H == 1:
        # one slice: X = A diag(sig) W^T is its own SVD, so the token tail is the same closed form
        for k in range(len(tT)):
            assert tT[k] == pytest.approx(lam[16 * k:].sum(), rel=1e-9, abs=1e-9 * n2), k


def test_spectra_tails_token_closed_form_grouped():
    # token-mode tail of a grouped cell: columns of X_(T) spanned by the orthonormal token basis P
    # with X[l,h] = P diag(s) C_lh^T where the stacked C_lh [n_heads*d, r] has orthonormal columns:
    # X_(T) = P diag(s) C^T is an SVD, so t_T(16k) = sum_{i > 16k} s_i^2 (s in decreasing order).
    L, H, T, d, r = 2, 2, 300, 32, 48
    rng = np.random.default_rng(13)
    P = np.linalg.qr(rng.standard_normal((T, r)))[0]
    C = np.linalg.qr(rng.standard_normal((L * H * d, r)))[0]
    s = rng.permutation(np.geomspace(30.0, 0.5, r))
    XT = (P * s[None, :]) @ C.T                                  # [T, L*H*d], columns (l, h, j)
    X = XT.reshape(T, L, H, d).transpose(1, 2, 0, 3)
    assert np.allclose(token_unfolding(X), XT)
    n2, tT, td = spectra_tails(X, 64)
    s2 = np.sort(s ** 2)[::-1]
    for k in range(len(tT)):
        assert tT[k] == pytest.approx(s2[16 * k:].sum(), rel=1e-9, abs=1e-9 * n2), k
