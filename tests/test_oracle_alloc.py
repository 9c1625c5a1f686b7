"""Pins of the oracle allocator against brute force (Everett's theorem) and its invariants."""
import numpy as np
import pytest

from oracle.alloc import (build_options, allocate, brute_force_allocate, evaluate, lower_hull,
                          BudgetError)
from synth import make_random_tables

PHI = [1.0, 0.12, 0.0075, 2.9e-5]


def small_instance(n_cells, seed, n_rt=3, n_rd=3, T=64, d=32, Lg=2, H=2, sf=2):
    n2, tT, td = make_random_tables(n_cells, n_rt, n_rd, seed)
    return [build_options(n2[c], tT[c], td[c], PHI, T, d, Lg, H, sf) for c in range(n_cells)]


@pytest.mark.parametrize("seed", range(6))
def test_everett_against_brute_force(seed):
    opts = small_instance(3, seed)
    lo = sum(min(o[0] for o in c) for c in opts)
    hi = sum(max(o[0] for o in c) for c in opts)
    for frac in np.linspace(0.0, 1.0, 9):
        budget = int(lo + frac * (hi - lo))
        ch, lam, total = allocate(opts, budget)
        B, E = evaluate(opts, ch)
        assert B == total <= budget
        best = brute_force_allocate(opts, B)
        assert E <= best[0] * (1 + 1e-12) + 1e-12


def test_lambda_monotone_in_budget():
    opts = small_instance(4, 11, n_rt=5, n_rd=4)
    lo = sum(min(o[0] for o in c) for c in opts)
    hi = sum(max(o[0] for o in c) for c in opts)
    lams, Es = [], []
    for frac in np.linspace(0.0, 1.0, 25):
        ch, lam, total = allocate(opts, int(lo + frac * (hi - lo)))
        lams.append(lam)
        Es.append(evaluate(opts, ch)[1])
    assert all(a >= b for a, b in zip(lams, lams[1:]))
    assert all(a >= b for a, b in zip(Es, Es[1:]))


def test_infeasible_budget():
    opts = small_instance(2, 3)
    lo = sum(min(o[0] for o in c) for c in opts)
    with pytest.raises(BudgetError):
        allocate(opts, lo - 1)
    ch, lam, total = allocate(opts, lo)
    assert total == lo


def test_unbounded_budget_takes_min_error():
    opts = small_instance(3, 5)
    ch, lam, total = allocate(opts, 10 ** 15)
    for c, o in zip(ch, opts):
        best = min(x[1] for x in o)
        assert next(x for x in o if tuple(x[2:5]) == tuple(c))[1] == best
    assert lam == 0.0


def test_hull_is_convex_and_decreasing():
    opts = small_instance(1, 7, n_rt=8, n_rd=5)[0]
    h = lower_hull(opts)
    B = np.array([v[0] for v in h], float)
    E = np.array([v[1] for v in h])
    assert np.all(np.diff(B) > 0) and np.all(np.diff(E) < 0)
    sl = -np.diff(E) / np.diff(B)
    assert np.all(np.diff(sl) <= 1e-12 * sl[:-1])
    # every option lies on or above the hull's piecewise-linear envelope
    for o in opts:
        if B[0] <= o[0] <= B[-1]:
            assert o[1] >= np.interp(o[0], B, E) * (1 - 1e-12)


def test_zero_rank_pairs_with_zero_rank():
    opts = small_instance(1, 2)[0]
    for B, E, rT, rd, b in opts:
        assert (rT == 0) == (rd == 0)


@pytest.mark.parametrize("seed", range(4))
def test_uniform_equals_brute_force_with_one_cell_per_kind(seed):
    # with one key and one value cell every joint choice is uniform: the uniform allocator must
    # reach the exhaustive minimum over all joint choices (a different search)
    from oracle.alloc import allocate_uniform
    opts = small_instance(2, seed)
    lo = sum(min(o[0] for o in c) for c in opts)
    hi = sum(max(o[0] for o in c) for c in opts)
    for frac in np.linspace(0.0, 1.0, 7):
        budget = int(lo + frac * (hi - lo))
        ch, total = allocate_uniform(opts, budget)
        B, E = evaluate(opts, ch)
        assert B == total <= budget
        assert E == pytest.approx(brute_force_allocate(opts, budget)[0], rel=1e-12, abs=1e-12)


@pytest.mark.parametrize("seed", range(4))
def test_ablation_allocations_are_feasible_and_never_beat_the_joint_optimum(seed):
    # both ablations are feasible allocations, so neither goes below the exhaustive joint minimum;
    # uniform shares one choice per kind; the decoupled split keeps keys within half the budget
    from oracle.alloc import allocate_uniform, allocate_kv_split
    opts = small_instance(4, seed)
    lo = sum(min(o[0] for o in c) for c in opts)
    hi = sum(max(o[0] for o in c) for c in opts)
    for frac in (0.3, 0.6, 0.9):
        budget = int(lo + frac * (hi - lo)) + 2 * max(max(o[0] for o in c) for c in opts)
        best = brute_force_allocate(opts, budget)[0]
        cu, tu = allocate_uniform(opts, budget)
        assert len(set(cu[0::2])) == 1 and len(set(cu[1::2])) == 1
        Bu, Eu = evaluate(opts, cu)
        assert Bu == tu <= budget and Eu >= best * (1 - 1e-12)
        ck, tk = allocate_kv_split(opts, budget)
        Bk, Ek = evaluate(opts, ck)
        assert Bk == tk <= budget and Ek >= best * (1 - 1e-12)
        assert evaluate(opts[0::2], ck[0::2])[0] <= budget // 2


# ---- the pages' coordinate-wise rank search (a heuristic under the same multiplier) ----------

@pytest.mark.parametrize("seed", range(5))
def test_coord_never_beats_the_exhaustive_optimum(seed):
    # Everett's bound: no allocation using at most B bytes has less summed error than the best
    # one found by brute force within B; the coordinate search must respect it and the budget.
    from oracle.alloc import allocate_coord
    opts = small_instance(3, 40 + seed, n_rt=4, n_rd=3)
    lo = sum(min(o[0] for o in c) for c in opts)
    hi = sum(max(o[0] for o in c) for c in opts)
    for frac in np.linspace(0.0, 1.0, 7):
        budget = int(lo + frac * (hi - lo))
        ch, lam, total = allocate_coord(opts, budget, iters=80)
        B, E = evaluate(opts, ch)
        assert B == total <= budget
        best = brute_force_allocate(opts, B)
        assert E >= best[0] * (1 - 1e-12) - 1e-12


@pytest.mark.parametrize("seed", range(4))
def test_coord_cell_with_one_feature_rank_is_the_exhaustive_argmin(seed):
    # with a single nonzero r_d the token-mode move already ranges over every option, so the
    # search returns the exact minimiser of E + lam * bytes (ties: bytes, r_T, r_d, b)
    from oracle.alloc import _coord_cell
    opts = small_instance(1, 60 + seed, n_rt=6, n_rd=2)[0]
    for lam in (0.0, 1e-9, 1e-6, 1e-4, 1e-2, 1.0, 1e3):
        got = _coord_cell(opts, lam)
        want = min(opts, key=lambda o: (o[1] + lam * o[0], o[0], o[2], o[3], o[4]))
        assert got == want


def test_coord_descent_can_stop_short_of_the_optimum():
    # a hand-built cell (bytes, error) over r_T in {0, 16, 32}, r_d in {0, 16, 32}, b = 0 only
    # (other b priced out): from full ranks (32, 32) the token move keeps r_T = 32 and the
    # feature move keeps r_d = 32, although (16, 16) has the smaller E + lam * bytes.
    lam = 1.0
    grid = {(0, 0): (0, 100.0), (16, 16): (10, 20.0), (16, 32): (40, 19.0), (32, 16): (40, 19.0),
            (32, 32): (45, 0.0)}
    opts = [(B, E, rT, rd, 0) for (rT, rd), (B, E) in grid.items()]
    from oracle.alloc import _coord_cell
    got = _coord_cell(opts, lam)
    assert got[2:4] == (32, 32)                     # stuck: 45 + 0 < 40 + 19 and < 100
    best = min(opts, key=lambda o: o[1] + lam * o[0])
    assert best[2:4] == (16, 16) and best[1] + lam * best[0] < got[1] + lam * got[0]


def test_coord_infeasible_and_unbounded_budgets():
    from oracle.alloc import allocate_coord
    opts = small_instance(2, 3)
    # the sparsest coordinate choice of every cell is residual-only with b = 0 (zero bytes)
    ch, lam, total = allocate_coord(opts, 0, iters=40)
    assert total == 0 and all(c == (0, 0, 0) for c in ch)
    ch, lam, total = allocate_coord(opts, 10 ** 15, iters=40)
    assert lam == 1e-30
