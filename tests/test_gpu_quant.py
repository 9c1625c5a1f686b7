"""GPU parity of the rotation, quantise+pack and unpack+dequantise building blocks against the
oracle: bit-exact codes, scales, zeros and dequantised values given the same fp32 rows."""
import numpy as np
import pytest
import torch

import oracle
from long_context_st_b200 import api

pytestmark = pytest.mark.gpu


def rows_case(n, d, seed):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((n, d)) * rng.uniform(1e-3, 100, (n, 1)) + rng.uniform(-50, 50, (n, 1))
    x[0] = 0.25          # constant row -> scale 0
    x[1, :] = np.arange(d) * 0.5   # exact half-way rounding cases
    x[2] = rng.standard_normal(d) * 1e-6   # tiny range -> subnormal fp16 scale
    return x.astype(np.float32)


@pytest.mark.parametrize("d", [64, 128])
def test_rotation_columns_match_dense_hadamard(cuda_ok, d):
    seed = 0x5EED0004
    M = oracle.rotation_matrix(d, seed)
    eye = torch.eye(d, dtype=torch.float32, device="cuda")
    fwd = api.rotate_rows(eye, seed).cpu().numpy()   # row j = R e_j = column j of M
    assert np.max(np.abs(fwd - M.T)) < 2e-7
    inv = api.rotate_rows(eye, seed, inverse=True).cpu().numpy()   # row j = R^T e_j
    assert np.max(np.abs(inv - M)) < 2e-7
    x = torch.randn(1000, d, device="cuda")
    back = api.rotate_rows(api.rotate_rows(x, seed), seed, inverse=True)
    assert torch.max(torch.abs(back - x)).item() < 1e-5


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("b", [2, 4, 8])
def test_quantize_pack_bit_exact(cuda_ok, d, b):
    x = rows_case(5003, d, seed=d + b)
    codes, sz, err = api.quantize_pack(torch.from_numpy(x).cuda(), b)
    torch.cuda.synchronize()
    c_ref, s_ref, z_ref = oracle.quantize_rows(x, b)
    p_ref = oracle.pack_codes(c_ref, b)
    assert err.item() == 0
    assert np.array_equal(codes.cpu().numpy(), p_ref)
    szn = sz.cpu().numpy()
    assert np.array_equal(szn[:, 0].view(np.uint16), s_ref.view(np.uint16))
    assert np.array_equal(szn[:, 1].view(np.uint16), z_ref.view(np.uint16))
    deq = api.unpack_dequant(codes, sz, d, b).cpu().numpy()
    d_ref = oracle.dequantize_rows(c_ref, s_ref, z_ref)
    assert np.array_equal(deq.view(np.uint32), d_ref.view(np.uint32))


def test_quantize_out_of_range_sets_error(cuda_ok):
    x = np.zeros((4, 128), np.float32)
    x[2, 5] = -1e6
    codes, sz, err = api.quantize_pack(torch.from_numpy(x).cuda(), 4)
    torch.cuda.synchronize()
    assert err.item() == -5


def test_empty_input(cuda_ok):
    x = torch.zeros(0, 128, device="cuda")
    codes, sz, err = api.quantize_pack(x, 4)
    assert codes.shape == (0, 64)
