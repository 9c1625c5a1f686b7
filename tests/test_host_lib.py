"""Host-side library checks (no GPU): exported symbols, byte model, layout, phi, allocator.

The allocator must choose bit-identically to the oracle's when both get identical tables.
"""
import os
import re

import numpy as np
import pytest

import oracle
from oracle.alloc import tables_to_options, allocate as oracle_allocate, BudgetError
from oracle.bytes_model import cell_bytes as oracle_cell_bytes, raw_sequence_bytes
from synth import get_workload, make_random_tables
from long_context_st_b200 import api, _lib
from long_context_st_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module", autouse=True)
def built():
    build()


def header_symbols():
    txt = open(os.path.join(ROOT, "include", "jolt.h")).read()
    txt = re.sub(r"/\*.*?\*/", "", txt, flags=re.S)
    return sorted(set(re.findall(r"\b(jolt_[a-z_0-9]+)\s*\(", txt)))


def test_exports_every_declared_symbol():
    L = _lib.lib()
    syms = header_symbols()
    assert len(syms) >= 14
    for name in syms:
        assert hasattr(L, name), name
    declared = {n for n, _, _ in _lib.SIGNATURES}
    assert set(syms) <= declared, set(syms) - declared


def test_kv_bytes_formula():
    assert api.kv_bytes(80, 8, 128, 1, 2) == 327680
    assert api.kv_bytes(80, 64, 128, 1, 2) == 2621440
    assert api.kv_bytes(80, 8, 128, 131072, 2) == 40 * 2 ** 30
    assert api.kv_bytes(32, 8, 128, 2048, 2) == 268435456


@pytest.mark.parametrize("name", ["toy", "llama8b_layer", "llama8b_32k", "llama70b_128k"])
def test_cell_bytes_matches_oracle(name):
    w = get_workload(name)
    s = api.make_shape(w)
    for ch in [(0, 0, 0), (0, 0, 2), (16, 16, 0), (32, 32, 4), (s.q_cap, w.d_h, 8), (64, 96, 2)]:
        if ch[0] > s.q_cap or ch[1] > w.d_h:
            continue
        want = oracle_cell_bytes(w.T, w.d_h, w.layers_per_group, w.n_kv, w.factor_bytes, *ch)
        assert api.cell_bytes(s, ch) == want


def test_invalid_choices_and_shapes():
    w = get_workload("toy")
    s = api.make_shape(w)
    assert api.cell_bytes(s, (16, 0, 0)) == 0      # r_T > 0 needs r_d > 0
    assert api.cell_bytes(s, (8, 8, 0)) == 0       # not on the 16 grid
    assert api.cell_bytes(s, (16, 16, 3)) == 0     # b not in {0,2,4,8}
    with pytest.raises(api.JoltError):
        api.make_shape(w, q_cap=48, sketch_cols=32)  # sketch narrower than the cap


def test_cache_layout_alignment_and_sizes():
    w = get_workload("llama8b_32k")
    s = api.make_shape(w)
    rng = np.random.default_rng(0)
    nc = api.n_cells(s)
    choices = []
    for _ in range(nc):
        rT = int(rng.integers(0, s.q_cap // 16 + 1)) * 16
        rd = int(rng.integers(1, 9)) * 16 if rT else 0
        choices.append((rT, rd, int(rng.choice([0, 2, 4, 8]))))
    offs, total = api.cache_layout(s, choices)
    assert np.all(offs % 256 == 0)
    alg = sum(api.cell_bytes(s, c) for c in choices)
    assert alg <= total <= alg + nc * 5 * 256
    for c in range(nc - 1):
        assert offs[c + 1, 0] >= offs[c, 4]


def test_phi_agrees_with_oracle_statistically():
    for d in (64, 128):
        a = api.phi(d, 1 << 14, 3)
        b = oracle.phi_table(d, 1 << 14, 1)
        assert a[0] == 1.0
        for x, y in zip(a[1:], b[1:]):
            assert abs(x / y - 1) < 0.03


@pytest.mark.parametrize("seed", range(8))
def test_allocator_bit_exact_vs_oracle(seed):
    w = get_workload(["llama8b_32k", "llama70b_128k", "toy", "llama8b_layer"][seed % 4])
    s = api.make_shape(w)
    nc = 2 * (w.n_layers // w.layers_per_group)
    nrt, nrd = s.q_cap // 16 + 1, w.d_h // 16 + 1
    n2, tT, td = make_random_tables(nc, nrt, nrd, 100 + seed)
    phi = oracle.phi_table(w.d_h, 1 << 12, 1)
    raw = raw_sequence_bytes(w)
    opts = tables_to_options(n2, tT, td, phi, w)
    for ratio in (2.0, 3.0, 5.0, 8.0):
        budget = int(raw / ratio)
        try:
            want, lam_o, tot_o = oracle_allocate(opts, budget)
        except BudgetError:
            with pytest.raises(api.JoltError):
                api.allocate(s, n2, tT, td, phi, budget)
            continue
        got, lam_g, tot_g = api.allocate(s, n2, tT, td, phi, budget)
        assert [tuple(c) for c in got] == [tuple(c) for c in want]
        assert lam_g == lam_o and tot_g == tot_o


@pytest.mark.parametrize("seed", range(3))
def test_allocator_variants_bit_exact_vs_oracle(seed):
    from oracle.alloc import allocate_kv_split, allocate_uniform
    w = get_workload(["llama8b_32k", "llama70b_128k", "llama8b_64k_b4"][seed])
    s = api.make_shape(w)
    nc = 2 * (w.n_layers // w.layers_per_group)
    nrt, nrd = s.q_cap // 16 + 1, w.d_h // 16 + 1
    n2, tT, td = make_random_tables(nc, nrt, nrd, 200 + seed)
    phi = oracle.phi_table(w.d_h, 1 << 12, 1)
    raw = raw_sequence_bytes(w)
    opts = tables_to_options(n2, tT, td, phi, w)
    for ratio in (2.0, 3.0, 5.0):
        budget = int(raw / ratio)
        for mode, fn in ((api.JOLT_ALLOC_KV_SPLIT, allocate_kv_split), (api.JOLT_ALLOC_UNIFORM, allocate_uniform)):
            want, tot_o = fn(opts, budget)
            got, tot_g = api.allocate_variant(s, n2, tT, td, phi, budget, mode)
            assert [tuple(c) for c in got] == [tuple(c) for c in want] and tot_g == tot_o
        got, tot = api.allocate_variant(s, n2, tT, td, phi, budget, api.JOLT_ALLOC_JOINT)
        assert got == api.allocate(s, n2, tT, td, phi, budget)[0]


def test_allocator_zero_budget_stores_nothing():
    # The empty choice (r_T = r_d = b = 0) costs no bytes, so every budget is feasible; at a
    # zero budget every cell keeps nothing and its error is its whole mass.
    w = get_workload("toy")
    s = api.make_shape(w)
    n2, tT, td = make_random_tables(2, s.q_cap // 16 + 1, w.d_h // 16 + 1, 1)
    ch, lam, tot = api.allocate(s, n2, tT, td, [1.0, 0.1, 0.01, 0.0001], 0)
    assert ch == [(0, 0, 0), (0, 0, 0)] and tot == 0 and lam > 0


def test_cache_blob_header_checks():
    # host-only paths of the blob format: size arithmetic and rejection of malformed blobs
    import ctypes as C
    from long_context_st_b200._lib import Shape
    w = get_workload("llama8b_32k", n_layers=8, T=1000)
    shape = api.make_shape(w)
    choices = [(64, 32, 4), (0, 0, 2)] * (api.n_cells(shape) // 2)
    _, total = api.cache_layout(shape, choices)
    n = api.cache_blob_bytes(shape, choices)
    hdr = n - total
    assert hdr % 256 == 0 and hdr >= 16 + C.sizeof(Shape) + 4 + 12 * len(choices) + 8
    with pytest.raises(api.JoltError):
        api.cache_blob_info(np.zeros(n, dtype=np.uint8))           # no magic
    with pytest.raises(api.JoltError):
        api.cache_blob_info(np.frombuffer(b"JOLTCACH", dtype=np.uint8))  # truncated
    # a header written by hand to the documented layout is accepted; one byte short is not
    blob = np.zeros(n, dtype=np.uint8)
    raw = bytearray(b"JOLTCACH") + (2).to_bytes(4, "little") + hdr.to_bytes(4, "little")
    raw += bytes(shape) + len(choices).to_bytes(4, "little", signed=True)
    for c in choices:
        raw += b"".join(int(v).to_bytes(4, "little", signed=True) for v in c)
    raw += total.to_bytes(8, "little")
    blob[:len(raw)] = np.frombuffer(bytes(raw), dtype=np.uint8)
    s2, nc, cb = api.cache_blob_info(blob)
    assert nc == len(choices) and cb == total and s2.T == shape.T and s2.rot_seed == shape.rot_seed
    with pytest.raises(api.JoltError):
        api.cache_blob_info(blob[:-1])
    bad = blob.copy()
    bad[8] = 1                                                   # an older format version
    with pytest.raises(api.JoltError):
        api.cache_blob_info(bad)


def test_group_layers_matches_oracle():
    """Host grouping (jolt_group_layers / jolt_uniform_group) equals the oracle's on random and
    boundary alignments."""
    import numpy as np
    from oracle.grouping import group_layers as o_group, uniform_group as o_uniform
    from long_context_st_b200 import api
    rng = np.random.default_rng(7)
    cases = [rng.uniform(0, 1, size=n) for n in (0, 1, 5, 11, 79)]
    cases.append(np.array([0.5, 0.49999999, 0.5, 1.0, 0.0]))
    for a in cases:
        for tau in (0.3, 0.5, 0.8):
            for mg in (0, 2, 3):
                assert api.group_layers(a, tau, mg) == o_group(list(a), tau, mg)
            assert api.uniform_group(a, tau) == o_uniform(list(a), a.size + 1, tau)


def test_argument_checks_before_any_device_work():
    """Entry points added for streaming, grouping and failure detection reject bad arguments on
    the host (no device needed)."""
    import ctypes as C
    from long_context_st_b200 import api
    from long_context_st_b200._lib import lib
    w = get_workload("toy", n_layers=2)
    s = api.make_shape(w)
    L = lib()
    # streamed analyze: null host or device buffers
    assert L.jolt_analyze_from_host(C.byref(s), None, None, None, None, None, None, None, None, 0, None) == -1
    # layer alignment: rank not a multiple of 16, or above min(T, n_kv*d_h)
    assert L.jolt_layer_align_workspace(C.byref(s), 24) == 0
    assert L.jolt_layer_align_workspace(C.byref(s), 16 * 1000) == 0
    assert L.jolt_layer_align_workspace(C.byref(s), 16) > 0
    # grouping: no layers, null outputs
    assert L.jolt_group_layers(None, 0, 0.5, 0, None, None) == -1
    # self-test: unbounded or zero limits, unknown test, too small a workspace
    assert L.jolt_selftest_timeout(0, 0, None, 512, None) == -1
    assert L.jolt_selftest_timeout(3, 1000, None, 512, None) == -1


@pytest.mark.parametrize("seed", range(3))
def test_coordinate_allocator_bit_exact_vs_oracle(seed):
    # the pages' coordinate-wise rank search: host library and oracle agree bit for bit (choices,
    # bytes) on random tables; small grids keep the pure-Python oracle fast
    from oracle.alloc import allocate_coord
    w = get_workload("toy")
    s = api.make_shape(w)
    nc = 8
    nrt, nrd = s.q_cap // 16 + 1, w.d_h // 16 + 1
    n2, tT, td = make_random_tables(nc, nrt, nrd, 300 + seed)
    phi = oracle.phi_table(w.d_h, 1 << 12, 1)
    opts = tables_to_options(n2, tT, td, phi, w)
    hi = sum(max(o[0] for o in c) for c in opts)
    for frac in (0.05, 0.2, 0.45, 0.8):
        budget = int(frac * hi)
        want, lam, tot_o = allocate_coord(opts, budget)
        got, tot_g = api.allocate_variant(s, n2, tT, td, phi, budget, api.JOLT_ALLOC_COORD)
        assert [tuple(c) for c in got] == [tuple(c) for c in want] and tot_g == tot_o
        # never better than the exact single-multiplier allocation at its own bytes
        ex, _, tot_e = api.allocate(s, n2, tT, td, phi, budget)
        from oracle.alloc import evaluate
        assert evaluate(opts, got)[1] >= evaluate(opts, ex)[1] * (1 - 1e-12) or tot_g > tot_e


def test_noalloc_decode_checks_arguments_before_scratch_size():
    # host-only paths: a malformed call is JOLT_ERR_INVALID_ARG even when its scratch would also
    # exceed the built-in array; a well-formed oversized call is JOLT_ERR_WORKSPACE. Neither
    # reaches the device (fake, non-null pointers).
    import ctypes as C
    from long_context_st_b200._lib import lib
    w = get_workload("llama70b_128k")
    s = api.make_shape(w)
    good = api.choices_array([(256, 128, 4)] * api.n_cells(s))
    bad = api.choices_array([(250, 128, 4)] * api.n_cells(s))   # r_T not a multiple of 16
    fake = C.c_void_p(0x1000)
    inv = C.c_void_p(0x2000)
    r_bad = lib().jolt_decode_attn_noalloc(C.byref(s), bad, fake, 0, w.n_layers, fake, fake, None, inv, 0, None)
    assert r_bad == -1
    r_big = lib().jolt_decode_attn_noalloc(C.byref(s), good, fake, 0, w.n_layers, fake, fake, None, inv, 0, None)
    assert r_big == -6
    r_pos = lib().jolt_decode_attn_noalloc(C.byref(s), good, fake, 0, w.n_layers, fake, fake, None, inv, -1, None)
    assert r_pos == -1
