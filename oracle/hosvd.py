"""Partial Tucker decomposition of one cell by ST-HOSVD, token mode first (exact, float64).

[v4 §3]: a cell is the fourth-order tensor X [L_g, n_kv, T, d_h] of one layer group's keys or
values; JoLT truncates its token and feature modes, keeps the layer and head modes at full rank,
shares the token and feature bases across the group's heads and layers, and truncates the token
mode before the feature mode. [nl Methodologie 1] names the method: sequentially truncated HOSVD.

Steps (reading of "token truncation precedes feature truncation"):
  1. U_T = top-r_T left singular vectors of the token unfolding X_(T) [T, L_g*n_kv*d_h];
  2. Y_lh = U_T^T X_lh [r_T, d_h];  S_Y = sum_lh Y_lh^T Y_lh;  U_d = top-r_d eigenvectors of S_Y;
  3. G_lh = Y_lh U_d [r_T, r_d];  X~_lh = U_T G_lh U_d^T.

Spectra for the allocator [v4 §3, §3.1]: the token-mode tail t_T(r) = ||X||^2 - sum_{i<=r} s_i^2
(the uncomputed energy of the randomized variant is ||X||^2 minus what it found, appended as a
synthetic tail entry; here the spectrum is exact, so the tail is exact too); the feature-mode tail
t_d(r) = ||X||^2 - sum_{j<=r} lambda_j(S_d), S_d = sum_lh X_lh^T X_lh (the full tensor's feature
Gram, because r_T is not known when the tables are built).

Pinned by: exact recovery of a planted low-rank tensor; the ST-HOSVD error identity
||X - X~||^2 = sum_{i>r_T} s_i^2 + sum_{j>r_d} lambda_j(S_Y); the Eckart-Young error for
L_g = n_kv = 1; orthonormal U_T and U_d.
"""
import numpy as np

# Largest T*n for which the token basis comes from a direct SVD; above it, from eigh of the Gram.
SVD_MAX_ELEMS = 2_000_000


def token_unfolding(X: np.ndarray) -> np.ndarray:
    """X [L_g, n_kv, T, d_h] -> X_(T) [T, L_g*n_kv*d_h], column index (layer, head, feature)."""
    L, H, T, d = X.shape
    return np.ascontiguousarray(X.transpose(2, 0, 1, 3).reshape(T, L * H * d))


def _token_svd(XT: np.ndarray, r: int):
    """Top-r left singular vectors and ALL squared singular values of XT (float64)."""
    T, n = XT.shape
    if T * n <= SVD_MAX_ELEMS:
        U, s, _ = np.linalg.svd(XT, full_matrices=False)
        return U[:, :r], s ** 2
    if n <= T:
        lam, V = np.linalg.eigh(XT.T @ XT)
        lam, V = lam[::-1].clip(min=0.0), V[:, ::-1]
        Ur = XT @ V[:, :r]
        Ur /= np.sqrt(np.maximum(lam[:r], 1e-300))[None, :]
        # one Gram-Schmidt pass (QR) to remove the small loss of orthogonality of X V / sigma
        Qr, Rr = np.linalg.qr(Ur)
        Ur = Qr * np.sign(np.diag(Rr))[None, :]
        return Ur, lam
    lam, U = np.linalg.eigh(XT @ XT.T)
    return U[:, ::-1][:, :r], lam[::-1].clip(min=0.0)


def _top_eigvecs(S: np.ndarray, r: int):
    lam, V = np.linalg.eigh(S)
    return V[:, ::-1][:, :r], lam[::-1]


def st_hosvd(X: np.ndarray, r_T: int, r_d: int):
    """Returns (U_T [T,r_T], U_d [d_h,r_d], G [L_g,n_kv,r_T,r_d], sigma2_T, lambda_SY)."""
    X = np.asarray(X, dtype=np.float64)
    L, H, T, d = X.shape
    XT = token_unfolding(X)
    U_T, sig2 = _token_svd(XT, r_T)
    Y = np.matmul(U_T.T, X)                      # [L_g, n_kv, r_T, d_h]
    Yf = Y.reshape(-1, d)
    S_Y = Yf.T @ Yf
    U_d, lam_Y = _top_eigvecs(S_Y, r_d)
    G = np.matmul(Y, U_d)
    return U_T, U_d, G, sig2, lam_Y


def reconstruct(U_T: np.ndarray, G: np.ndarray, U_d: np.ndarray) -> np.ndarray:
    """X~[l,h] = U_T G[l,h] U_d^T, float64 [L_g, n_kv, T, d_h]."""
    U_T = np.asarray(U_T, dtype=np.float64)
    return np.matmul(np.matmul(U_T, np.asarray(G, dtype=np.float64)),
                     np.asarray(U_d, dtype=np.float64).T)


def spectra_tails(X: np.ndarray, qcap: int, step: int = 16):
    """Allocator inputs of one cell: (||X||^2, t_T[k] for r_T = step*k <= qcap, t_d[j] for
    r_d = step*j <= d_h), all float64."""
    X = np.asarray(X, dtype=np.float64)
    L, H, T, d = X.shape
    norm2 = float(np.sum(X * X))
    XT = token_unfolding(X)
    _, sig2 = _token_svd(XT, 0)
    Xf = X.reshape(-1, d)
    S_d = Xf.T @ Xf
    lam_d = np.linalg.eigvalsh(S_d)[::-1]
    csT = np.concatenate([[0.0], np.cumsum(sig2)])
    csd = np.concatenate([[0.0], np.cumsum(lam_d)])
    tT = np.array([norm2 - csT[min(k * step, len(sig2))] for k in range(qcap // step + 1)])
    td = np.array([norm2 - csd[min(j * step, d)] for j in range(d // step + 1)])
    return norm2, np.maximum(tT, 0.0), np.maximum(td, 0.0)
