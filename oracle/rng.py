"""Counter-based randomness the codec draws: the seeded sign diagonal of the residual rotation.

The pages say only that the residual rotation is random, seeded, shared across cells and
regenerated at decode [v4 §3, "stores the residual after a feature-axis rotation"]. Reading: the
rotation is a randomized Hadamard H·D/sqrt(d_h) whose sign diagonal D is drawn from SplitMix64
(Steele, Lea & Flood, "Fast splittable pseudorandom number generators", OOPSLA 2014) used as a
hash of a counter: s_j = +1 if bit 63 of splitmix64(seed * 2^32 + j) is 0, else -1.

Pinned by: the published SplitMix64 output sequence for state 0 (tests/test_oracle_core.py).
"""
import numpy as np

_M64 = (1 << 64) - 1
_GAMMA = 0x9E3779B97F4A7C15


def splitmix64(state):
    """SplitMix64 output for the given 64-bit state (the state is advanced by gamma first).

    Works on Python ints or numpy uint64 arrays (wrapping arithmetic).
    """
    if isinstance(state, (int, np.integer)):
        z = (int(state) + _GAMMA) & _M64
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _M64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _M64
        return z ^ (z >> 31)
    s = np.asarray(state, dtype=np.uint64)
    with np.errstate(over="ignore"):
        z = s + np.uint64(_GAMMA)
        z = (z ^ (z >> np.uint64(30))) * np.uint64(0xBF58476D1CE4E5B9)
        z = (z ^ (z >> np.uint64(27))) * np.uint64(0x94D049BB133111EB)
        return z ^ (z >> np.uint64(31))


def rotation_signs(d: int, seed: int) -> np.ndarray:
    """The +-1 diagonal D of the residual rotation, as float64 [d]."""
    ctr = np.array([((seed << 32) + j) & _M64 for j in range(d)], dtype=np.uint64)
    top = splitmix64(ctr) >> np.uint64(63)
    return np.where(top == 0, 1.0, -1.0)
