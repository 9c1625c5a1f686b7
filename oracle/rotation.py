"""The JL residual rotation as an explicit dense matrix.

[v4 §3]: the truncation residual is stored after a seeded feature-axis rotation that is shared
across cells and regenerated at decode; [nl Methodologie 2]: a random JL rotation is applied to
R = X - X~ before uniform quantisation, and decoding inverts the rotation.
Reading: rotation = (1/sqrt(d)) H_d D with H_d the Sylvester Hadamard matrix
(H_1 = [1], H_2m = [[H, H], [H, -H]]) and D the seeded sign diagonal of oracle.rng.

Pinned by: H_ij = (-1)^popcount(i & j) and H H^T = d I; rotation^T rotation = I.
"""
import numpy as np

from .rng import rotation_signs


def hadamard(d: int) -> np.ndarray:
    assert d >= 1 and (d & (d - 1)) == 0, "d must be a power of two"
    H = np.ones((1, 1))
    while H.shape[0] < d:
        H = np.block([[H, H], [H, -H]])
    return H


def rotation_matrix(d: int, seed: int) -> np.ndarray:
    """Dense float64 rotation matrix (1/sqrt(d)) H diag(s); apply to a column vector r as M @ r."""
    return hadamard(d) * rotation_signs(d, seed)[None, :] / np.sqrt(d)
