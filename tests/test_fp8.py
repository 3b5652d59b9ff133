"""GPU parity of the FP8 path: fa_hadamard_quant against the oracle's rotation,
amax and e4m3 codec; the e4m3-QK attention against (a) the oracle on the same
dequantised inputs (the kernel's own parity) and (b) exact fp64 attention on the
unquantised inputs (the relative-RMSE bound), with and without the Hadamard
rotation, and the outlier claim: on inputs with outlier feature channels the
error with the rotation is strictly lower ("FlashAttention-3 (PT)", section
"Inovações técnicas", subsection 3)."""
import numpy as np
import pytest
import torch

import oracle
import io_aware_exact_17_b200 as fa
from io_aware_exact_17_b200 import inputs
from helpers import (BF16_LSE_ATOL, BF16_O_ATOL, FP8_REL_RMSE, max_abs, record, rel_rmse, rotation_error_bound,
                     to_np)

pytestmark = pytest.mark.gpu


def _quant_check(x, rotate, signs):
    codes, ds = fa.hadamard_quant(x.cuda(), rotate=rotate, signs=None if signs is None else signs.cuda())
    torch.cuda.synchronize()
    codes = codes.cpu().numpy().reshape(-1, x.shape[-1])
    ds = float(ds.item())
    ref, ref_ds, scaled = oracle.quantize_per_tensor(x.reshape(-1, x.shape[-1]), rotate,
                                                     None if signs is None else signs.numpy(), return_scaled=True)
    # The kernel decides each code in fp32 (the rotation as a tensor-core
    # product with fp32 sums, then the scale 448/amax in fp32); the oracle in
    # fp64. Codes must agree exactly except where the oracle's value lies within
    # the kernel's error of a rounding midpoint, where either neighbour is
    # correct: the rotation's error bound (helpers.rotation_error_bound), scaled,
    # plus a relative 1e-5 for the two final multiplies. The descale is amax/448
    # of the kernel's values: within the same bound of the oracle's.
    d = x.shape[-1]
    xf = x.reshape(-1, d).double().numpy()
    bound = rotation_error_bound(xf, rotate)
    assert abs(ds - ref_ds) <= 1e-5 * ref_ds + float(bound.max(initial=0.0)) / 448.0
    # +0 and -0 are one value; which sign a cancelled sum keeps is rounding noise.
    diff = np.where(codes == 0x80, 0, codes) != np.where(ref == 0x80, 0, ref)
    if np.any(diff):
        tol_all = 1e-5 * np.abs(scaled) + bound / ref_ds
        grid = oracle.e4m3_decode(np.arange(0, 127, dtype=np.uint8))
        mids = (grid[:-1] + grid[1:]) / 2
        a = np.abs(scaled[diff])
        tol = tol_all[diff]
        near = np.min(np.abs(a[:, None] - mids[None, :]), axis=1) <= tol
        near |= a >= 448.0 - tol
        assert np.all(near), (int((~near).sum()), a[~near][:5], tol[~near][:5])
        step = np.abs(oracle.e4m3_decode(codes[diff]) - oracle.e4m3_decode(ref[diff]))
        assert np.all(step <= 2 * np.maximum(a, 2.0**-6) * 2.0**-3 + 1e-12)
    return codes, ds


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("rotate", [False, True])
@pytest.mark.parametrize("rows", [1, 7, 1000, 33333, 150001])
def test_quant_matches_oracle(d, rotate, rows):
    g = torch.Generator().manual_seed(rows + d)
    x = torch.randn(rows, d, generator=g).to(torch.bfloat16)
    _quant_check(x, rotate, None)
    if rotate:
        _quant_check(x, True, inputs.hadamard_signs(d, seed=rows))


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("rotate", [False, True])
def test_quant_is_repeatable_at_scale(d, rotate):
    # The quantiser streams every row block through a shared-memory ring twice;
    # a race between a stage's readers and its refill would show up as codes
    # that change from launch to launch. 20 launches on 32 M elements must agree
    # bit for bit (the arithmetic is deterministic), and the first with the oracle.
    rows = (32 << 20) // d
    g = torch.Generator().manual_seed(d + 7)
    x = torch.randn(rows, d, generator=g).to(torch.bfloat16)
    signs = inputs.hadamard_signs(d, seed=d) if rotate else None
    codes0, ds0 = _quant_check(x, rotate, signs)
    xc = x.cuda()
    sc = signs.cuda() if signs is not None else None
    first, _ = fa.hadamard_quant(xc, rotate=rotate, signs=sc)
    for _ in range(20):
        again, ds = fa.hadamard_quant(xc, rotate=rotate, signs=sc)
        assert torch.equal(again, first) and float(ds.item()) == ds0
    assert np.array_equal(first.cpu().numpy().reshape(-1, d), codes0)
    assert fa.device_status()[0] == 0


@pytest.mark.parametrize("n", [1, 2, 3, 8])
@pytest.mark.parametrize("rotate", [False, True])
def test_quant_multi_equals_one_call_per_tensor(n, rotate):
    # tensors of very different ranges, one launch, one scale each
    xs = []
    for i in range(n):
        q, _, _ = inputs.qkv_normal(2, 3, 700, 128, 70 + i)
        xs.append((q.float() * 10.0 ** (2 * i - 2)).to(torch.bfloat16).cuda())
    signs = inputs.hadamard_signs(128, 70).cuda() if rotate else None
    codes, ds = fa.hadamard_quant_multi(xs, rotate=rotate, signs=signs)
    torch.cuda.synchronize()
    for i, x in enumerate(xs):
        c1, d1 = fa.hadamard_quant(x, rotate=rotate, signs=signs)
        torch.cuda.synchronize()
        assert torch.equal(codes[i], c1)
        assert float(ds[i].item()) == float(d1.item())


@pytest.mark.parametrize("n", [2, 3])
def test_quant_multi_larger_than_l2_equals_one_call_per_tensor(n):
    # Tensors of 64 MB each: two of them do not fit in L2 together, so the
    # launch takes the short-lead schedule (the next tensor's first tiles ahead
    # of this one's second pass) instead of the whole next first pass.
    g = torch.Generator(device="cuda").manual_seed(81)
    xs = [(torch.randn(1 << 18, 128, device="cuda", generator=g) * (1.0 + i)).to(torch.bfloat16) for i in range(n)]
    signs = inputs.hadamard_signs(128, 81).cuda()
    codes, ds = fa.hadamard_quant_multi(xs, rotate=True, signs=signs)
    torch.cuda.synchronize()
    for i, x in enumerate(xs):
        c1, d1 = fa.hadamard_quant(x, rotate=True, signs=signs)
        torch.cuda.synchronize()
        assert torch.equal(codes[i], c1)
        assert float(ds[i].item()) == float(d1.item())
    assert fa.device_status()[0] == 0


def test_quant_zero_and_empty():
    codes, ds = fa.hadamard_quant(torch.zeros(5, 128, dtype=torch.bfloat16, device="cuda"))
    assert float(ds.item()) == 1.0 and int(codes.abs().sum()) == 0
    codes, ds = fa.hadamard_quant(torch.zeros(0, 128, dtype=torch.bfloat16, device="cuda"))
    assert float(ds.item()) == 1.0 and codes.numel() == 0


def test_quant_outlier_spread():
    # One outlier channel per head (R1): rotation cuts the tensor amax.
    q, k, _ = inputs.qkv_normal(1, 4, 512, 128, 40)
    q1, _ = inputs.with_outliers_r1(q, k, 40)
    _, ds_plain = fa.hadamard_quant(q1.cuda(), rotate=False)
    _, ds_rot = fa.hadamard_quant(q1.cuda(), rotate=True)
    assert float(ds_rot.item()) < 0.5 * float(ds_plain.item())


def _fp8_attention(q, k, v, causal, rotate, signs=None):
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    sc = None if signs is None else signs.cuda()
    q8, dq = fa.hadamard_quant(qc, rotate=rotate, signs=sc)
    k8, dk = fa.hadamard_quant(kc, rotate=rotate, signs=sc)
    o, lse = fa.fwd(q8, k8, vc, causal=causal, qk_descale=torch.cat([dq, dk]))
    torch.cuda.synchronize()
    code, site, block = fa.device_status()
    assert code == 0, f"device wait ran out at site {site}, block {block}"
    return o, lse, q8, dq, k8, dk


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_fp8_kernel_parity_on_dequantised_inputs(d, causal):
    B, H, N = 1, 3, 700
    q, k, v = inputs.qkv_normal(B, H, N, d, 41)
    o, lse, q8, dq, k8, dk = _fp8_attention(q, k, v, causal, rotate=True)
    qd = oracle.e4m3_decode(q8.cpu().numpy()) * float(dq.item())
    kd = oracle.e4m3_decode(k8.cpu().numpy()) * float(dk.item())
    o_ref, lse_ref = oracle.attention(qd, kd, v, causal, d ** -0.5)
    assert max_abs(to_np(o), o_ref) <= BF16_O_ATOL
    assert max_abs(to_np(lse), lse_ref) <= BF16_LSE_ATOL


def test_fp8_config_rel_rmse_sampled():
    # B=2, H=16, N=8192, d=128, plain N(0,1): relative RMSE against exact
    # attention on the unquantised inputs, with and without the rotation.
    B, H, N, d = 2, 16, 8192, 128
    q, k, v = inputs.qkv_normal(B, H, N, d, 1003)
    rows = inputs.sample_rows(B, H, N, per_head=16, seed=3).numpy()
    o_ref, _ = oracle.attention(q, k, v, False, d ** -0.5, rows=rows)
    for rotate in (False, True):
        o, *_ = _fp8_attention(q, k, v, False, rotate, inputs.hadamard_signs(d, 1003) if rotate else None)
        err = rel_rmse(to_np(o).reshape(-1, d)[rows], o_ref)
        record(f"e4m3 QK B{B} H{H} N{N} d{d} N(0,1) {'rotated' if rotate else 'unrotated'} (sampled rows)",
               rel_rmse=err)
        assert err <= FP8_REL_RMSE, (rotate, err)


def test_fp8_outliers_rotation_strictly_better():
    B, H, N, d = 2, 16, 8192, 128
    q, k, v = inputs.qkv_normal(B, H, N, d, 1003)
    q1, k1 = inputs.with_outliers_r1(q, k, 1003)
    rows = inputs.sample_rows(B, H, N, per_head=16, seed=4).numpy()
    o_ref, _ = oracle.attention(q1, k1, v, False, d ** -0.5, rows=rows)
    err = {}
    for rotate in (False, True):
        o, *_ = _fp8_attention(q1, k1, v, False, rotate, inputs.hadamard_signs(d, 1003) if rotate else None)
        err[rotate] = rel_rmse(to_np(o).reshape(-1, d)[rows], o_ref)
    record(f"e4m3 QK B{B} H{H} N{N} d{d} outliers (sampled rows)", rel_rmse_rotated=err[True],
           rel_rmse_unrotated=err[False])
    assert err[True] < err[False], err


@pytest.mark.parametrize("causal", [False, True])
def test_fp8_small_full_rel_rmse(causal):
    B, H, N, d = 1, 4, 1024, 128
    q, k, v = inputs.qkv_normal(B, H, N, d, 42)
    o_ref, _ = oracle.attention(q, k, v, causal, d ** -0.5)
    o, *_ = _fp8_attention(q, k, v, causal, True)
    assert rel_rmse(to_np(o), o_ref) <= FP8_REL_RMSE
