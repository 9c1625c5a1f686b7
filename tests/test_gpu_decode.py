"""GPU decode attention over the ORACLE's compressed cache vs the oracle's dense attention on the
reconstructed cache: max relative error <= 1e-3 for fp32 I/O, <= 1e-2 for bf16 I/O."""
import numpy as np
import pytest
import torch

from synth import get_workload, make_kv, make_queries, make_inv_freq
from cache_io import oracle_cells, cells_to_device, oracle_decode, max_rel_err
from long_context_st_b200 import api

pytestmark = pytest.mark.gpu


def run_case(w, choices, tol, layer_calls=None, pos_offset=0, shape_over=None):
    shape = api.make_shape(w, **(shape_over or {}))
    K, V = make_kv(w, device="cuda")
    q = make_queries(w, device="cuda")
    cells = oracle_cells(w, K, V, choices, shape.rot_seed)
    cache = cells_to_device(shape, w, cells, choices)
    inv = make_inv_freq(w.d_h, w.rope_theta)
    inv_t = torch.from_numpy(inv).cuda()
    ws = api.new_workspace(shape, api.JOLT_OP_DECODE)
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:3], dtype=torch.float32, device="cuda")
    calls = layer_calls or [(0, w.n_layers)]
    per_call = torch.empty_like(q)
    for l0, n in calls:
        tmp = torch.empty_like(q[:, l0:l0 + n])
        api.decode_attn(shape, choices, cache, q[:, l0:l0 + n].contiguous(), tmp,
                        ws, lse=None, inv_freq=inv_t, layer_begin=l0, n_layers_call=n,
                        pos_offset=pos_offset)
        per_call[:, l0:l0 + n] = tmp
    # one more whole call for the LSE (out rows are overwritten with identical values)
    api.decode_attn(shape, choices, cache, q, out, ws, lse=lse, inv_freq=inv_t,
                    pos_offset=pos_offset)
    api.check_ws(ws)
    ref = oracle_decode(w, cells, q, shape.rot_seed, inv_freq=inv, pos_offset=pos_offset,
                        attn_scale=shape.attn_scale)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy()
    pc = per_call.float().cpu().numpy()
    ls = lse.cpu().numpy()
    worst = 0.0
    for (b, l), (ro, rl) in ref.items():
        worst = max(worst, max_rel_err(o[b, l], ro), max_rel_err(pc[b, l], ro))
        assert np.max(np.abs(ls[b, l] - rl)) < 1e-3 * max(1.0, np.abs(rl).max())
    assert worst <= tol, worst
    return worst


def uniform(w, ch):
    return [ch] * (2 * w.batch * (w.n_layers // w.layers_per_group))


def test_toy_fixed_ranks(cuda_ok):
    w = get_workload("toy")
    run_case(w, uniform(w, w.fixed_choice), 1e-3)


@pytest.mark.parametrize("ch", [(0, 0, 4), (0, 0, 8), (32, 32, 0), (128, 64, 2), (16, 16, 8),
                                (64, 48, 4)])
def test_toy_choice_grid(cuda_ok, ch):
    w = get_workload("toy")
    run_case(w, uniform(w, ch), 1e-3)


def test_toy_mixed_k_v_choices_and_ragged_T(cuda_ok):
    w = get_workload("toy", T=301)
    run_case(w, [(32, 32, 4), (0, 0, 2)], 1e-3)


def test_toy_pre_rope(cuda_ok):
    w = get_workload("toy", keys_pre_rope=True)
    run_case(w, uniform(w, (32, 32, 4)), 1e-3, pos_offset=1000)


def test_llama8b_layer_full(cuda_ok):
    w = get_workload("llama8b_layer")
    run_case(w, uniform(w, w.fixed_choice), 1e-2)


def test_grouped_layers_per_layer_calls(cuda_ok):
    # 8 layers in 2 groups of 4, T ragged, mixed choices, one call per layer and one whole call
    w = get_workload("llama8b_32k", n_layers=8, T=1000, batch=2)
    rng = np.random.default_rng(5)
    ch = []
    for _ in range(2 * 2 * 2):
        rT = int(rng.integers(1, 9)) * 16
        ch.append((rT, int(rng.integers(1, 9)) * 16, int(rng.choice([0, 2, 4, 8]))))
    run_case(w, ch, 1e-2, layer_calls=[(l, 1) for l in range(8)])


def test_grouped_pre_rope_gqa4(cuda_ok):
    w = get_workload("llama8b_64k_b4", n_layers=4, T=777, batch=2)
    rng = np.random.default_rng(6)
    ch = [(int(rng.integers(1, 6)) * 16, int(rng.integers(2, 9)) * 16, int(rng.choice([2, 4])))
          for _ in range(2 * 1 * 2)]
    run_case(w, ch, 1e-2, layer_calls=[(0, 2), (2, 2)], pos_offset=5)


def test_pre_rope_residual_only_keys_and_calls_across_groups(cuda_ok):
    # key cells with r_T = 0 (residual only), b = 0 and b = 8 cells, ragged T, a call that spans
    # two groups and starts mid-group
    w = get_workload("llama8b_64k_b4", n_layers=8, T=450, batch=2)
    ch = [(0, 0, 4), (32, 32, 0), (64, 128, 8), (48, 16, 2),
          (16, 16, 0), (0, 0, 8), (96, 64, 4), (128, 96, 4)]
    run_case(w, ch, 1e-2, layer_calls=[(1, 5), (6, 2), (0, 1)], pos_offset=3)


def test_pre_rope_full_token_rank(cuda_ok):
    # r_T = q_cap = 1024 > any shared-memory-resident tile, T not a multiple of the 128-token tile
    w = get_workload("llama8b_layer", keys_pre_rope=True, T=1100)
    run_case(w, uniform(w, (1024, 128, 4)), 1e-2, pos_offset=70000)


def test_70b_shape_gqa8_two_row_tiles(cuda_ok):
    # 64 query heads x 4 layers = 256 rows: two 128-row tiles in the score and value GEMMs
    for pre in (False, True):
        w = get_workload("llama70b_128k", n_layers=4, T=640, keys_pre_rope=pre)
        rng = np.random.default_rng(7)
        ch = [(int(rng.integers(1, 9)) * 32, 128, int(rng.choice([2, 4]))) for _ in range(2)]
        run_case(w, ch, 1e-2, layer_calls=[(0, 4)], pos_offset=11)


def test_gqa16_value_residual_two_head_tiles(cuda_ok):
    # 16 query heads per KV head: the value-residual MMA runs two 8-head column tiles; ragged T,
    # value codes of every width, keys with and without RoPE
    for pre in (False, True):
        w = get_workload("llama8b_layer", n_kv=2, T=531, keys_pre_rope=pre)
        ch = [(64, 96, 4), (48, 128, 8)] if pre else [(32, 128, 2), (80, 64, 2)]
        run_case(w, ch, 1e-2, pos_offset=9)


def test_pre_rope_more_rows_than_one_finalize_launch(cuda_ok):
    # 17 sequences x 32 layers = 544 (sequence, layer) rows: the output projection runs as two
    # launches (512 rows, then the rest) after every group's values
    w = get_workload("llama8b_64k_b4", batch=17, T=130)
    run_case(w, uniform(w, (32, 32, 4)), 1e-2, pos_offset=2)
