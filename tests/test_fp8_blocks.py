"""GPU parity of FP8 with one scale per 128-row block of a head
(fa_hadamard_quant_blocks and the FA_E4M3_BLOCK attention): the codes and
descales against the oracle's per-block quantiser, the attention against the
oracle on the same dequantised inputs, and the relative RMSE against exact
attention on the unquantised inputs."""
import numpy as np
import pytest
import torch

import oracle
import io_aware_exact_17_b200 as fa
from io_aware_exact_17_b200 import inputs
from helpers import (BF16_LSE_ATOL, BF16_O_ATOL, FP8_REL_RMSE, max_abs, record, rel_rmse, rotation_error_bound,
                     to_np)

pytestmark = pytest.mark.gpu

BLOCK = 128


def _status_ok():
    torch.cuda.synchronize()
    code, site, block = fa.device_status()
    assert code == 0, f"device wait ran out at site {site}, block {block}"


def _check_block_codes(x, rotate, signs):
    """Codes and descales of fa_hadamard_quant_blocks against the oracle. As for
    one scale per tensor, the kernel decides each code in fp32 and the oracle in
    fp64: codes agree exactly except within the kernel's error (the rotation's
    bound, helpers.rotation_error_bound, plus a relative 1e-5) of a rounding
    midpoint, where either neighbour is correct; each descale within the bound's
    largest value in its block / 448 plus a relative 1e-5."""
    sg = None if signs is None else signs.cuda()
    codes, ds = fa.hadamard_quant_blocks(x.cuda(), rotate=rotate, signs=sg)
    _status_ok()
    codes, ds = codes.cpu().numpy(), ds.cpu().double().numpy()
    ref, ref_ds = oracle.quantize_per_block(x, rotate, None if signs is None else signs.numpy(), BLOCK)
    assert ds.shape == ref_ds.shape
    B, H, N, d = x.shape
    bound = rotation_error_bound(x.double().numpy(), rotate)
    nb = ref_ds.shape[2]
    pad = np.zeros((B, H, nb * BLOCK - N, d))
    block_bound = np.concatenate([bound, pad], axis=2).reshape(B, H, nb, BLOCK * d).max(axis=-1)
    assert np.all(np.abs(ds - ref_ds) <= 1e-5 * ref_ds + block_bound / 448.0)
    xr = oracle.rotate(x, None if signs is None else signs.numpy()) if rotate else x.double().numpy()
    ds_rows = np.repeat(ref_ds, BLOCK, axis=2)[:, :, :N, None]
    scaled = xr / ds_rows
    diff = np.where(codes == 0x80, 0, codes) != np.where(ref == 0x80, 0, ref)
    if np.any(diff):
        tol_all = 1e-5 * np.abs(scaled) + bound / ds_rows
        grid = oracle.e4m3_decode(np.arange(0, 127, dtype=np.uint8))
        mids = (grid[:-1] + grid[1:]) / 2
        a = np.abs(scaled[diff])
        tol = tol_all[diff]
        near = np.min(np.abs(a[:, None] - mids[None, :]), axis=1) <= tol
        near |= a >= 448.0 - tol
        assert np.all(near), (int((~near).sum()), a[~near][:5], tol[~near][:5])
    return codes, ds


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("N", [1, 127, 128, 300, 1000])
@pytest.mark.parametrize("rotate", [False, True])
def test_block_quant_matches_oracle(d, N, rotate):
    q, _, _ = inputs.qkv_normal(2, 3, N, d, 90 + N + d)
    signs = inputs.hadamard_signs(d, 90) if rotate else None
    _check_block_codes(q, rotate, signs)


@pytest.mark.parametrize("d", [64, 128, 256])
def test_block_quant_many_stages_per_cta_and_repeatable(d):
    # 2 x 16 heads of 4096 rows: every CTA streams many stages of several heads
    q, _, _ = inputs.qkv_normal(2, 16, 4096, d, 95 + d)
    signs = inputs.hadamard_signs(d, 95)
    codes, ds = _check_block_codes(q, True, signs)
    qc, sg = q.cuda(), signs.cuda()
    for _ in range(10):
        c2, d2 = fa.hadamard_quant_blocks(qc, rotate=True, signs=sg)
        assert np.array_equal(c2.cpu().numpy(), codes) and np.array_equal(d2.cpu().double().numpy(), ds)
    _status_ok()


def test_block_quant_blocks_of_different_ranges_and_a_zero_block():
    q, _, _ = inputs.qkv_normal(1, 2, 384, 128, 91)
    q = q.float()
    q[0, 0, 128:256] *= 300.0
    q[0, 1, 256:] = 0.0
    _, ds = _check_block_codes(q.to(torch.bfloat16), True, inputs.hadamard_signs(128, 91))
    assert ds[0, 1, 2] == 1.0 and ds[0, 0, 1] > 100 * ds[0, 0, 0]


def _block_attention(q, k, v, causal, signs, Nq=None):
    sg = signs.cuda()
    q8, dq = fa.hadamard_quant_blocks(q.cuda(), rotate=True, signs=sg)
    k8, dk = fa.hadamard_quant_blocks(k.cuda(), rotate=True, signs=sg)
    if q.shape[2] == k.shape[2]:
        o, lse = fa.fwd(q8, k8, v.cuda(), causal=causal, qk_descale=(dq, dk))
    else:
        o, lse = fa.fwd_splitkv(q8, k8, v.cuda(), causal=causal, qk_descale=(dq, dk))
    _status_ok()
    return o, lse, q8, dq, k8, dk


def _dequant(codes, ds, N):
    return oracle.e4m3_decode(codes.cpu().numpy()) * np.repeat(ds.cpu().double().numpy(), BLOCK, axis=2)[:, :, :N,
                                                                                                         None]


@pytest.mark.parametrize("d", [128, 256])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_split", [0, 1])
def test_block_attention_on_dequantised_inputs(d, causal, n_split):
    B, H, N = 1, 3, 700
    q, k, v = inputs.qkv_normal(B, H, N, d, 92)
    sg = inputs.hadamard_signs(d, 92).cuda()
    q8, dq = fa.hadamard_quant_blocks(q.cuda(), rotate=True, signs=sg)
    k8, dk = fa.hadamard_quant_blocks(k.cuda(), rotate=True, signs=sg)
    o, lse = fa.fwd(q8, k8, v.cuda(), causal=causal, qk_descale=(dq, dk), n_split=n_split)
    _status_ok()
    o_ref, lse_ref = oracle.attention(_dequant(q8, dq, N), _dequant(k8, dk, N), v, causal, d ** -0.5)
    assert max_abs(to_np(o), o_ref) <= BF16_O_ATOL
    assert max_abs(to_np(lse), lse_ref) <= BF16_LSE_ATOL


def test_block_attention_decode_and_split_on_dequantised_inputs():
    # decode layout (Nq <= 32) and split keys read the per-block key descales too
    B, H, Nq, Nk, d = 2, 2, 16, 3000, 128
    q, k, v = inputs.qkv_decode(B, H, Nq, Nk, d, 93)
    o, lse, q8, dq, k8, dk = _block_attention(q, k, v, True, inputs.hadamard_signs(d, 93))
    o_ref, lse_ref = oracle.attention(_dequant(q8, dq, Nq), _dequant(k8, dk, Nk), v, True, d ** -0.5)
    assert max_abs(to_np(o), o_ref) <= BF16_O_ATOL
    assert max_abs(to_np(lse), lse_ref) <= BF16_LSE_ATOL


def test_block_fp8_config_rel_rmse_and_outliers():
    # B=2, H=16, N=8192, d=128 (the FP8 workload's shape), sampled rows: plain
    # N(0,1) within the bound, and R1 outliers reported beside one scale per tensor
    B, H, N, d = 2, 16, 8192, 128
    q, k, v = inputs.qkv_normal(B, H, N, d, 1003)
    signs = inputs.hadamard_signs(d, 1003)
    rows = inputs.sample_rows(B, H, N, per_head=16, seed=6).numpy()
    o_ref, _ = oracle.attention(q, k, v, False, d ** -0.5, rows=rows)
    o, *_ = _block_attention(q, k, v, False, signs)
    err = rel_rmse(to_np(o).reshape(-1, d)[rows], o_ref)
    record(f"e4m3 QK per-block B{B} H{H} N{N} d{d} N(0,1) rotated (sampled rows)", rel_rmse=err)
    assert err <= FP8_REL_RMSE
    q1, k1 = inputs.with_outliers_r1(q, k, 1003)
    o_ref1, _ = oracle.attention(q1, k1, v, False, d ** -0.5, rows=rows)
    o_b, *_ = _block_attention(q1, k1, v, False, signs)
    err_b = rel_rmse(to_np(o_b).reshape(-1, d)[rows], o_ref1)
    sg = signs.cuda()
    q8, dq1 = fa.hadamard_quant(q1.cuda(), rotate=True, signs=sg)
    k8, dk1 = fa.hadamard_quant(k1.cuda(), rotate=True, signs=sg)
    o_t, _ = fa.fwd(q8, k8, v.cuda(), qk_descale=torch.cat([dq1, dk1]))
    _status_ok()
    err_t = rel_rmse(to_np(o_t).reshape(-1, d)[rows], o_ref1)
    record(f"e4m3 QK per-block vs per-tensor B{B} H{H} N{N} d{d} outliers rotated (sampled rows)",
           rel_rmse_block=err_b, rel_rmse_tensor=err_t)
    # a block's scale is never coarser than the tensor's
    assert err_b <= err_t * 1.05
