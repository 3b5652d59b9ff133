"""GPU parity of V's transposed e4m3 quantiser (fa_quant_v_transposed through
the C ABI) against the oracle: codes code by code (either neighbour within the
fp32 product's error of a rounding midpoint), the descale, ragged sizes and
rows whose length is not a multiple of 4; and bit equality with the unrotated
per-tensor quantiser's codes, transposed."""
import numpy as np
import pytest
import torch

import oracle
import io_aware_exact_17_b200 as fa
from io_aware_exact_17_b200 import inputs

pytestmark = pytest.mark.gpu


def _status_ok():
    torch.cuda.synchronize()
    code, site, block = fa.device_status()
    assert code == 0, f"device wait ran out at site {site}, block {block}"


def _check(v):
    codes, ds = fa.quant_v_transposed(v.cuda())
    _status_ok()
    codes = codes.cpu().numpy()
    ds = float(ds.item())
    ref, ref_ds, scaled = oracle.quantize_v_transposed(v, return_scaled=True)
    # the kernel multiplies by 448 / amax in fp32: a relative 1e-6 of the value
    assert abs(ds - ref_ds) <= 1e-6 * ref_ds
    diff = np.where(codes == 0x80, 0, codes) != np.where(ref == 0x80, 0, ref)
    if np.any(diff):
        grid = oracle.e4m3_decode(np.arange(0, 127, dtype=np.uint8))
        mids = (grid[:-1] + grid[1:]) / 2
        a = np.abs(scaled[diff])
        tol = 1e-6 * a + 1e-12
        near = np.min(np.abs(a[:, None] - mids[None, :]), axis=1) <= tol
        assert np.all(near), (int((~near).sum()), a[~near][:5])
    return codes, ds


@pytest.mark.parametrize("B,H,N,d", [(1, 1, 1, 64), (2, 3, 100, 128), (1, 2, 130, 256), (2, 2, 256, 128),
                                     (1, 1, 1000, 64), (1, 2, 67, 256), (4, 16, 2048, 128)])
def test_v_quant_matches_oracle(B, H, N, d):
    v = inputs.qkv_normal(B, H, N, d, 60 + N + d)[2]
    _check(v)


def test_v_quant_equals_unrotated_quantiser_transposed():
    B, H, N, d = 2, 4, 384, 128
    v = inputs.qkv_normal(B, H, N, d, 61)[2].cuda()
    codes_t, ds_t = fa.quant_v_transposed(v)
    codes, ds = fa.hadamard_quant(v, rotate=False)
    _status_ok()
    assert torch.equal(codes_t, codes.transpose(-1, -2).contiguous())
    assert float(ds_t.item()) == float(ds.item())


def test_v_quant_repeatable_and_zero_tensor():
    v = inputs.qkv_normal(2, 2, 700, 64, 62)[2].cuda()
    first, ds0 = fa.quant_v_transposed(v)
    for _ in range(5):
        again, ds = fa.quant_v_transposed(v)
        assert torch.equal(again, first) and float(ds.item()) == float(ds0.item())
    z, dz = fa.quant_v_transposed(torch.zeros(1, 1, 50, 128, dtype=torch.bfloat16, device="cuda"))
    _status_ok()
    assert float(dz.item()) == 1.0 and not bool(z.any())
