"""CPU pins of the oracle's transposed V quantiser (oracle.quantize_v_transposed):
the layout (out[b, h, c, n] holds v[b, h, n, c]'s code), the scale, the zero
tensor, and agreement with the per-tensor quantiser of Q and K without rotation."""
import numpy as np
import pytest
import torch

import oracle


@pytest.mark.parametrize("sign", [1.0, -1.0])
@pytest.mark.parametrize("pos", [(0, 0, 4, 1), (0, 1, 2, 0), (0, 1, 0, 2)])
def test_single_value_lands_at_the_transposed_place(sign, pos):
    # one nonzero value a: amax = |a|, so it scales to +-448 (code 0x7e / 0xfe)
    # and every other code is 0; a transposed index would put it elsewhere
    v = np.zeros((1, 2, 5, 3))
    v[pos] = sign * 3.0
    codes, ds = oracle.quantize_v_transposed(v)
    assert codes.shape == (1, 2, 3, 5)
    assert ds == pytest.approx(3.0 / 448.0, rel=1e-15)
    b, h, n, c = pos
    expect = np.zeros_like(codes)
    expect[b, h, c, n] = 0x7E if sign > 0 else 0xFE
    assert np.array_equal(codes, expect)
    assert float(oracle.e4m3_decode(codes[b, h, c, n])) * ds == pytest.approx(sign * 3.0)


def test_zero_tensor():
    codes, ds = oracle.quantize_v_transposed(np.zeros((1, 1, 7, 4)))
    assert ds == 1.0 and codes.shape == (1, 1, 4, 7) and not codes.any()


def test_round_trip_within_e4m3_precision():
    g = torch.Generator().manual_seed(5)
    v = torch.randn(2, 3, 9, 16, generator=g).double().numpy()
    codes, ds = oracle.quantize_v_transposed(v)
    back = np.swapaxes(oracle.e4m3_decode(codes) * ds, -1, -2)
    # e4m3 keeps 3 mantissa bits: half an ulp is 2^-4 relative (normal range),
    # plus the subnormal step 2^-9 in code units
    assert np.all(np.abs(back - v) <= np.abs(v) * 2.0 ** -4 + ds * 2.0 ** -10 + 1e-15)


def test_agrees_with_the_per_tensor_quantiser_without_rotation():
    g = torch.Generator().manual_seed(6)
    v = torch.randn(2, 2, 33, 64, generator=g).to(torch.bfloat16)
    codes_t, ds_t = oracle.quantize_v_transposed(v)
    codes, ds = oracle.quantize_per_tensor(v.reshape(-1, 64), False)
    assert ds_t == ds
    assert np.array_equal(codes_t, np.swapaxes(codes.reshape(2, 2, 33, 64), -1, -2))
