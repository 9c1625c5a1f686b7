"""Layer grouping by token-mode subspace alignment (exact, float64) — TEST INFRASTRUCTURE ONLY.

[v4 §3]: JoLT groups consecutive layers whose token-mode singular vectors align, computing the
grouping from the cache being compressed (no calibration data); [v4 §3] reports 11 groups for
Mistral-7B-v0.3 at T = 1024. The pages give neither the alignment measure nor the threshold.
Reading taken here (and by the CUDA path):

  * a layer's token basis U_l = top-k left singular vectors of the token unfolding of that layer's
    cache alone, X_l,(T) [T, n_kv*d_h] (column index (head, feature)), for K and for V;
  * alignment of layers l and l+1 = mean squared cosine of the principal angles between their
    token subspaces, ||U_l^T U_{l+1}||_F^2 / k in [0, 1], averaged over K and V;
  * groups: consecutive layers, a layer joining the current group when its alignment with the
    previous layer is >= tau (and the group has fewer than max_group layers, when max_group > 0);
  * uniform group size for a fixed-L_g codec: the largest L_g dividing L whose groups keep every
    consecutive alignment inside a group >= tau.

Pinned by (tests/test_oracle_grouping.py): alignment 1 for the same subspace in another basis, 0
for orthogonal subspaces, cos^2 of a known principal angle, j/k when j of k directions are shared;
hand-worked groupings and uniform group sizes; recovery of planted layer groups.
"""
import numpy as np

from .hosvd import _token_svd


def layer_token_basis(X_layer: np.ndarray, k: int) -> np.ndarray:
    """X_layer [n_kv, T, d_h] -> U [T, k], top-k left singular vectors of its token unfolding."""
    H, T, d = X_layer.shape
    XT = np.ascontiguousarray(X_layer.astype(np.float64).transpose(1, 0, 2).reshape(T, H * d))
    U, _ = _token_svd(XT, k)
    return U


def subspace_alignment(U1: np.ndarray, U2: np.ndarray) -> float:
    """||U1^T U2||_F^2 / k for orthonormal U1, U2 [T, k]: mean squared cosine of principal angles."""
    k = U1.shape[1]
    M = U1.T @ U2
    return float(np.sum(M * M) / k)


def layer_alignment(K: np.ndarray, V: np.ndarray, k: int) -> np.ndarray:
    """K, V [L, n_kv, T, d_h] of one sequence -> alignment of layers (l, l+1), l < L-1."""
    L = K.shape[0]
    UK = [layer_token_basis(K[l], k) for l in range(L)]
    UV = [layer_token_basis(V[l], k) for l in range(L)]
    return np.array([0.5 * (subspace_alignment(UK[l], UK[l + 1]) + subspace_alignment(UV[l], UV[l + 1]))
                     for l in range(L - 1)], dtype=np.float64)


def group_layers(align, tau: float, max_group: int = 0):
    """Consecutive grouping: layer l+1 joins the current group when align[l] >= tau."""
    sizes = [1]
    for a in align:
        if a >= tau and (max_group <= 0 or sizes[-1] < max_group):
            sizes[-1] += 1
        else:
            sizes.append(1)
    return sizes


def uniform_group(align, n_layers: int, tau: float) -> int:
    """Largest L_g dividing n_layers with every within-group consecutive alignment >= tau."""
    best = 1
    for Lg in range(1, n_layers + 1):
        if n_layers % Lg:
            continue
        ok = all(align[l] >= tau for l in range(n_layers - 1) if (l + 1) % Lg != 0)
        if ok:
            best = Lg
    return best
