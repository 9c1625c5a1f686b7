"""Joint rank/bit allocation under a global byte budget with a single Lagrange multiplier.

[v4 §3]: the allocator minimises summed reconstruction error subject to a global byte budget,
jointly choosing Tucker ranks and residual bits per (layer group, K/V) cell; one Lagrangian dual
allocates across all cells [v4 abstract; nl Methodologie 3]. The error surrogate multiplies the
discarded-mass estimate by the fraction the rotated quantiser leaves unrecovered [v4 §3]; the
surrogate prices Frobenius mass uniformly [v4 §3, §5], so the objective is the sum of absolute
squared errors.

Readings (the pages give no formulas):
  * options per cell: r_T in {0, 16, ..., qcap}, r_d in {0, 16, ..., d_h} (r_T = 0 iff r_d = 0),
    b in {0, 2, 4, 8};
  * discarded mass D(0, 0) = ||X||^2 and D(r_T, r_d) = min(||X||^2, t_T(r_T) + t_d(r_d));
    error E = D * phi(b); bytes from oracle.bytes_model.cell_bytes;
  * the dual: for a multiplier lam every cell picks argmin E + lam * bytes; the allocation is the
    one of the smallest lam whose total bytes fit the budget. Written out exactly: each cell's
    choices as lam falls are the vertices of the lower convex hull of its (bytes, E) points, so
    the cells start at their cheapest vertex and hull segments are taken in order of falling
    price dE/dbytes while the budget holds; the first segment that does not fit gives lam.
    Ties: equal bytes keep the smaller E, then smaller r_T, r_d, b; equal prices go to the lower
    cell index. A budget below the cheapest vertices is infeasible.

Pinned by: brute force over all joint choices on small instances (Everett: the Lagrangian
allocation is optimal among allocations using at most its bytes); budget respected; lam monotone
in the budget.
"""
import itertools

import numpy as np

from .bytes_model import cell_bytes

BITS = (0, 2, 4, 8)


class BudgetError(ValueError):
    pass


def build_options(norm2, tT, td, phi, T, d_h, L_g, n_kv, s_f, step=16):
    """All (bytes, E, r_T, r_d, b) options of one cell (python ints / floats)."""
    opts = []
    pairs = [(0, 0)] + [(k, j) for k in range(1, len(tT)) for j in range(1, len(td))]
    for k, j in pairs:
        r_T, r_d = k * step, j * step
        if k == 0:
            D = float(norm2)
        else:
            D = min(float(norm2), float(tT[k]) + float(td[j]))
        for bi, b in enumerate(BITS):
            E = D * float(phi[bi])
            B = cell_bytes(T, d_h, L_g, n_kv, s_f, r_T, r_d, b)
            opts.append((B, E, r_T, r_d, b))
    return opts


def _cross(a, b, c):
    return (float(b[0]) - float(a[0])) * (c[1] - a[1]) - (b[1] - a[1]) * (float(c[0]) - float(a[0]))


def lower_hull(opts):
    """Vertices (bytes, E, r_T, r_d, b) of the decreasing lower convex hull, cheapest first."""
    srt = sorted(opts, key=lambda o: (o[0], o[1], o[2], o[3], o[4]))
    front = []
    for o in srt:
        if front and front[-1][0] == o[0]:
            continue                      # same bytes: first one has the smallest E
        if front and not (o[1] < front[-1][1]):
            continue                      # dominated: more bytes, no less error
        front.append(o)
    hull = []
    for o in front:
        while len(hull) >= 2 and _cross(hull[-2], hull[-1], o) <= 0.0:
            hull.pop()
        hull.append(o)
    return hull


def allocate(cell_options, budget: int):
    """cell_options: list (per cell) of option lists. Returns (choices, lam, total_bytes)
    with choices[c] = (r_T, r_d, b)."""
    hulls = [lower_hull(o) for o in cell_options]
    pos = [0] * len(hulls)
    total = sum(h[0][0] for h in hulls)
    if total > budget:
        raise BudgetError(f"budget {budget} below minimum {total}")
    segs = []
    for c, h in enumerate(hulls):
        prev = float("inf")
        for i in range(1, len(h)):
            dB = h[i][0] - h[i - 1][0]
            dE = h[i - 1][1] - h[i][1]
            price = dE / float(dB)
            price = min(price, prev)
            prev = price
            segs.append((price, c, i, dB))
    segs.sort(key=lambda s: (-s[0], s[1], s[2]))
    lam = 0.0
    for price, c, i, dB in segs:
        if total + dB <= budget:
            assert pos[c] == i - 1
            pos[c] = i
            total += dB
        else:
            lam = price
            break
    choices = [tuple(hulls[c][pos[c]][2:5]) for c in range(len(hulls))]
    return choices, lam, total


def brute_force_allocate(cell_options, budget: int):
    """Exhaustive minimum of summed E over all joint choices with total bytes <= budget."""
    best = None
    for combo in itertools.product(*cell_options):
        B = sum(o[0] for o in combo)
        if B > budget:
            continue
        E = sum(o[1] for o in combo)
        if best is None or E < best[0]:
            best = (E, B, [tuple(o[2:5]) for o in combo])
    return best


def allocate_kv_split(cell_options, budget: int):
    """K/V-decoupled allocation ([v4] §4.4 Ablations, App. D Table 12): keys (even cells) and
    values (odd cells) each allocated jointly on their own; reading: budget // 2 for keys, the
    rest for values. Returns (choices, total bytes)."""
    ck, tk = allocate(cell_options[0::2], budget // 2)[0::2]
    cv, tv = allocate(cell_options[1::2], budget - budget // 2)[0::2]
    choices = [None] * len(cell_options)
    choices[0::2] = ck
    choices[1::2] = cv
    return choices, tk + tv


def allocate_uniform(cell_options, budget: int):
    """Uniform ranks ([v4] §4.4 Ablations, App. D Table 13); reading: one (r_T, r_d, b) for all
    key cells and one for all value cells, the pair with the least summed error whose bytes fit.
    Ties: fewer bytes, then the earlier key option, then the earlier value option (options in
    build_options order). Returns (choices, total bytes); BudgetError if nothing fits."""
    n = len(cell_options)
    half = n // 2
    ng = len(cell_options[0])
    Bo = np.array([o[0] for o in cell_options[0]], dtype=np.int64)
    E = [np.zeros(ng), np.zeros(ng)]
    for c in range(n):
        E[c % 2] = E[c % 2] + np.array([o[1] for o in cell_options[c]])
    Et = E[0][:, None] + E[1][None, :]
    Bt = half * Bo[:, None] + half * Bo[None, :]
    ok = Bt <= budget
    if not ok.any():
        raise BudgetError(f"budget {budget} below the cheapest uniform pair")
    ki, vi = np.nonzero(ok)
    order = np.lexsort((vi, ki, Bt[ki, vi], Et[ki, vi]))
    k, v = int(ki[order[0]]), int(vi[order[0]])
    choices = [tuple(cell_options[c][k if c % 2 == 0 else v][2:5]) for c in range(n)]
    return choices, int(Bt[k, v])


def _coord_cell(opts, lam, max_rounds=32):
    """One cell's choice for multiplier lam by the coordinate-wise rank search: from full ranks,
    alternately the best r_T with r_d held (r_T = 0 forces r_d = 0) and the best r_d with r_T held,
    b chosen with each move, until a round changes nothing. The current option is always a
    candidate, so E + lam * bytes never rises. Ordering key: (E + lam * bytes, bytes, r_T, r_d, b)."""
    def key(o):
        return (o[1] + lam * o[0], o[0], o[2], o[3], o[4])

    kmax = max(o[2] for o in opts)
    jmax = max(o[3] for o in opts)
    cur = min((o for o in opts if o[2] == kmax and o[3] == jmax), key=key)
    for _ in range(max_rounds):
        start = cur
        # token-mode move: r_d held (a zero token rank takes the residual-only option)
        cand = [o for o in opts if o[3] == cur[3] or o[2] == 0]
        cur = min(cand, key=key)
        # feature-mode move: r_T held
        cand = [o for o in opts if o[2] == cur[2]]
        cur = min(cand, key=key)
        if cur == start:
            break
    return cur


def allocate_coord(cell_options, budget: int, iters: int = 200):
    """The pages' coordinate-wise rank search ([v4] §3: a heuristic over the two truncated modes)
    under the same single multiplier and error model. Reading: each cell's choice for a given lam
    comes from _coord_cell; lam is the bracket end of a geometric bisection over [1e-30, 1e30]
    (iters halvings of the bracket, midpoint sqrt(lo * hi)) with the largest total bytes that still
    fit. Returns (choices, lam, total bytes); BudgetError if even the sparsest allocation does not
    fit."""
    def at(lam):
        ch = [_coord_cell(o, lam) for o in cell_options]
        return ch, sum(o[0] for o in ch)

    lo, hi = 1e-30, 1e30
    ch_hi, b_hi = at(hi)
    if b_hi > budget:
        raise BudgetError(f"budget {budget} below the sparsest coordinate allocation {b_hi}")
    ch_lo, b_lo = at(lo)
    if b_lo <= budget:
        return [tuple(o[2:5]) for o in ch_lo], lo, b_lo
    for _ in range(iters):
        mid = float(np.sqrt(lo * hi))
        ch, b = at(mid)
        if b <= budget:
            hi, ch_hi, b_hi = mid, ch, b
        else:
            lo = mid
    return [tuple(o[2:5]) for o in ch_hi], hi, b_hi


def evaluate(cell_options, choices):
    """(total bytes, total E) of a choice vector."""
    B = E = 0
    for opts, ch in zip(cell_options, choices):
        o = next(o for o in opts if tuple(o[2:5]) == tuple(ch))
        B += o[0]
        E += o[1]
    return B, E


def tables_to_options(norm2, tT, td, phi, w):
    """Options of every cell of one sequence from per-cell spectra tails (arrays [cells, ...])."""
    s_f = w.factor_bytes
    return [build_options(norm2[c], tT[c], td[c], phi, w.T, w.d_h, w.layers_per_group, w.n_kv, s_f)
            for c in range(len(norm2))]


def as_arrays(choices):
    return np.array(choices, dtype=np.int64).reshape(-1, 3)
