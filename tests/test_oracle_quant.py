"""Pins of the oracle quantiser and packer: hand-worked rows, the rounding error bound, the
step-squared law of uniform quantisation and round trips."""
import numpy as np
import pytest

from oracle.quant import (quantize_rows, dequantize_rows, pack_codes, unpack_codes, phi_table,
                          NumericError)


def ulp16(x):
    x = np.abs(np.asarray(x, dtype=np.float64))
    e = np.floor(np.log2(np.maximum(x, 2.0 ** -14)))
    return 2.0 ** (e - 10)


def test_hand_worked_rows():
    c, s, z = quantize_rows(np.array([[0.0, 1.0, 2.0, 3.0]], np.float32), 2)
    assert c.tolist() == [[0, 1, 2, 3]] and float(s[0]) == 1.0 and float(z[0]) == 0.0
    # round half to even: 0.5 -> 0, 1.5 -> 2
    c, s, z = quantize_rows(np.array([[0.0, 0.5, 1.5, 3.0]], np.float32), 2)
    assert c.tolist() == [[0, 0, 2, 3]]
    # constant row: scale 0, all codes 0, dequantised value = fp16(mn)
    c, s, z = quantize_rows(np.full((1, 8), 0.3, np.float32), 4)
    assert float(s[0]) == 0.0 and c.max() == 0
    assert dequantize_rows(c, s, z)[0, 0] == np.float32(np.float16(0.3))


@pytest.mark.parametrize("b", [2, 4, 8])
def test_error_bound(b):
    rng = np.random.default_rng(b)
    x = (rng.standard_normal((4000, 128)) * rng.uniform(0.01, 50, (4000, 1))).astype(np.float32)
    c, s, z = quantize_rows(x, b)
    deq = dequantize_rows(c, s, z).astype(np.float64)
    mn = x.min(-1).astype(np.float64)
    sc = s.astype(np.float64)
    bound = sc / 2 + ulp16(mn) / 2 + ((1 << b) - 1) * ulp16(sc) / 2
    bound = bound + 4 * np.abs(x).max(-1) * 2.0 ** -24
    err = np.abs(x.astype(np.float64) - deq).max(-1)
    assert np.all(err <= bound)
    assert c.max() <= (1 << b) - 1


def test_aggregate_error_decreases_with_bits():
    rng = np.random.default_rng(0)
    x = rng.standard_normal((2000, 64)).astype(np.float32)
    errs = [np.sum(x.astype(np.float64) ** 2)]
    for b in (2, 4, 8):
        c, s, z = quantize_rows(x, b)
        errs.append(np.sum((x - dequantize_rows(c, s, z)).astype(np.float64) ** 2))
    assert errs[0] > errs[1] > errs[2] > errs[3] > 0


@pytest.mark.parametrize("b", [2, 4, 8])
def test_pack_roundtrip(b):
    rng = np.random.default_rng(1)
    c = rng.integers(0, 1 << b, size=(5, 7, 128)).astype(np.uint8)
    p = pack_codes(c, b)
    assert p.shape == (5, 7, 128 * b // 8)
    assert np.array_equal(unpack_codes(p, b, 128), c)


def test_pack_hand_bytes():
    assert pack_codes(np.array([1, 2, 3, 0], np.uint8), 2).tolist() == [0b00111001]
    assert pack_codes(np.array([0xA, 0x5], np.uint8), 4).tolist() == [0x5A]
    assert pack_codes(np.array([7, 200], np.uint8), 8).tolist() == [7, 200]


def test_phi_step_squared_law():
    for d in (64, 128):
        phi = phi_table(d, n_rows=1 << 14)
        assert phi[0] == 1.0 and phi[0] > phi[1] > phi[2] > phi[3] > 0
        # uniform rounding error ~ step^2/12 with the same range: phi(8)/phi(4) ~ (15/255)^2
        assert abs(phi[3] / phi[2] / (15 / 255) ** 2 - 1) < 0.1
        assert 0.03 < phi[1] < 0.3


def test_fp16_overflow_is_numeric_error():
    with pytest.raises(NumericError):
        quantize_rows(np.array([[-1e5, 0.0, 1.0, 2.0]], np.float32), 4)
