"""Pins for the oracle's FP8 pieces: the e4m3 codec, the Hadamard rotation and
the per-tensor quantiser ("FlashAttention-3 (PT)", section "Inovações técnicas",
subsection 3 "Baixa precisão (FP8)").

The codec is checked against the OCP e4m3 values in tests/golden/e4m3_codes.json
and against torch's float8_e4m3fn conversion (a library routine); the Sylvester
matrix against scipy.linalg.hadamard; the rotation against orthogonality and the
invariance the pages state (step 4: Q Kᵀ is unchanged).
"""
import json
from pathlib import Path

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from io_aware_exact_17_b200 import inputs

GOLDEN = Path(__file__).resolve().parent / "golden"


def test_e4m3_golden_table():
    g = json.loads((GOLDEN / "e4m3_codes.json").read_text())
    for code, val in g["decode"]:
        got = oracle.e4m3_decode(np.array([code], dtype=np.uint8))[0]
        assert got == val and np.signbit(got) == np.signbit(val), (code, got, val)
    assert np.all(np.isnan(oracle.e4m3_decode(np.array(g["decode_nan"], dtype=np.uint8))))
    for x, code in g["encode"]:
        assert int(oracle.e4m3_encode(np.array([x]))[0]) == code, (x, code)


def test_e4m3_decode_matches_torch_for_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    ours = oracle.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    assert np.array_equal(np.signbit(ours[~nan]), np.signbit(ref[~nan]))


def test_e4m3_encode_matches_torch_in_range():
    rng = np.random.default_rng(0)
    # fp32-representable values over the whole finite range, subnormals included,
    # plus every exact midpoint between neighbouring codes (the tie cases).
    mags = np.exp2(rng.uniform(-12, np.log2(448.0), 200000)).astype(np.float32)
    vals = mags * np.where(rng.random(mags.size) < 0.5, -1, 1).astype(np.float32)
    grid = oracle.e4m3_decode(np.arange(0, 127, dtype=np.uint8))
    mids = ((grid[:-1] + grid[1:]) / 2).astype(np.float32)
    vals = np.concatenate([vals, mids, -mids, np.float32([0.0, 448.0, -448.0])])
    ours = oracle.e4m3_encode(vals.astype(np.float64))
    ref = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    bad = np.nonzero(ours != ref)[0]
    assert bad.size == 0, [(float(vals[i]), int(ours[i]), int(ref[i])) for i in bad[:5]]


def test_e4m3_roundtrip_monotone_and_error_bound():
    codes = np.array([c for c in range(256) if (c & 0x7F) != 0x7F], dtype=np.uint8)
    assert np.array_equal(oracle.e4m3_encode(oracle.e4m3_decode(codes)), codes)
    x = np.sort(np.random.default_rng(1).uniform(-500, 500, 100001))
    dec = oracle.e4m3_decode(oracle.e4m3_encode(x))
    assert np.all(np.diff(dec) >= 0)
    a = np.minimum(np.abs(x), 448.0)
    # half the spacing: 2^(floor(log2 a) - 4) for normals, 2^-10 below 2^-6
    half = np.where(a >= 2.0**-6, np.exp2(np.floor(np.log2(np.maximum(a, 1e-300))) - 4), 2.0**-10)
    assert np.all(np.abs(dec - np.sign(x) * a) <= half * (1 + 1e-12))


@pytest.mark.parametrize("d", [1, 2, 4, 8, 16, 32, 64, 128, 256])
def test_sylvester_matches_scipy_and_is_orthogonal(d):
    h = oracle.sylvester_hadamard(d)
    assert np.array_equal(h, scipy.linalg.hadamard(d).astype(np.float64))
    np.testing.assert_array_equal(h @ h.T, d * np.eye(d))
    signs = inputs.hadamard_signs(d, seed=3).numpy()
    for s in (None, signs):
        m = oracle.rotation_matrix(d, s)
        np.testing.assert_allclose(m @ m.T, np.eye(d), atol=1e-14)


@pytest.mark.parametrize("use_signs", [False, True])
def test_rotation_leaves_qkT_unchanged(use_signs):
    d = 128
    rng = np.random.default_rng(2)
    q, k = rng.standard_normal((64, d)), rng.standard_normal((80, d)) * 3
    s = inputs.hadamard_signs(d, seed=9).numpy() if use_signs else None
    np.testing.assert_allclose(oracle.rotate(q, s) @ oracle.rotate(k, s).T, q @ k.T, atol=1e-12)


def rotation_golden_holds(rotation_matrix) -> bool:
    """True iff ``rotation_matrix(d, signs)`` reproduces every hand-derived
    case of tests/golden/rotation_sign_order.json: signs applied first, then
    the Hadamard (M = D H_d / sqrt(d), subsection 3, step 1), and none of the
    values the other order (H_d D) would give."""
    g = json.loads((GOLDEN / "rotation_sign_order.json").read_text())
    ok = True
    for c in g["cases"]:
        x = np.array(c["x"], dtype=np.float64)
        got = x @ rotation_matrix(c["d"], np.array(c["signs"], dtype=np.float64))
        want = np.array(c["expected"]["numer"], dtype=np.float64) / np.sqrt(c["expected"]["denom_sqrt"])
        wrong = np.array(c["wrong_order"]["numer"], dtype=np.float64) / np.sqrt(c["wrong_order"]["denom_sqrt"])
        ok &= bool(np.allclose(got, want, rtol=0, atol=1e-15))
        ok &= not np.allclose(got, wrong, rtol=0, atol=1e-15)
    return bool(ok)


def test_rotation_sign_order_golden():
    assert rotation_golden_holds(oracle.rotation_matrix)
    # rotate() and the quantisers go through the same matrix
    g = json.loads((GOLDEN / "rotation_sign_order.json").read_text())
    for c in g["cases"]:
        x = np.array(c["x"], dtype=np.float64)
        signs = np.array(c["signs"], dtype=np.float64)
        want = np.array(c["expected"]["numer"], dtype=np.float64) / np.sqrt(c["expected"]["denom_sqrt"])
        np.testing.assert_allclose(oracle.rotate(x[None], signs)[0], want, rtol=0, atol=1e-15)
        _, ds, scaled = oracle.quantize_per_tensor(x[None], True, signs, return_scaled=True)
        np.testing.assert_allclose(scaled[0] * ds, want, rtol=0, atol=1e-14)


def test_signs_flip_input_coordinates_before_mixing():
    # Flipping coordinate c of x and the sign s_c together leaves x D unchanged,
    # so x M is unchanged; the other order would not have this property.
    d = 64
    rng = np.random.default_rng(5)
    x = rng.standard_normal(d)
    s = inputs.hadamard_signs(d, seed=4).numpy().astype(np.float64)
    for c in (0, 17, 63):
        x2, s2 = x.copy(), s.copy()
        x2[c], s2[c] = -x2[c], -s2[c]
        np.testing.assert_allclose(oracle.rotate(x2[None], s2), oracle.rotate(x[None], s), rtol=0, atol=1e-13)


def test_rotation_spreads_a_single_coordinate():
    # An outlier on one coordinate becomes +-|x|/sqrt(d) on every coordinate
    # (subsection 3, step 2: the transform spreads large values over all coordinates).
    d = 128
    for c in (0, 5, 127):
        e = np.zeros(d)
        e[c] = 20.0
        r = oracle.rotate(e)
        np.testing.assert_allclose(np.abs(r), 20.0 / np.sqrt(d), atol=1e-13)


def test_quantiser_zero_tensor_and_extremes():
    codes, ds = oracle.quantize_per_tensor(np.zeros((3, 8)), rotate_qk=True)
    assert ds == 1.0 and np.all(codes == 0)
    x = np.random.default_rng(3).standard_normal((16, 64))
    for rot in (False, True):
        codes, ds, scaled = oracle.quantize_per_tensor(x, rot, return_scaled=True)
        xr = oracle.rotate(x) if rot else x
        assert ds == pytest.approx(np.max(np.abs(xr)) / 448.0, rel=1e-15)
        assert np.max(np.abs(oracle.e4m3_decode(codes))) == 448.0
        deq = oracle.e4m3_decode(codes) * ds
        a = np.abs(xr)
        bound = np.where(a / ds >= 2.0**-6, a * 2.0**-4, ds * 2.0**-10)
        assert np.all(np.abs(deq - xr) <= bound * (1 + 1e-9))


def test_rotation_lowers_logit_error_with_shared_outlier_channels():
    # The qualitative claim of subsection 3 (steps 2-3 and its closing sentence):
    # with outlier feature channels, rotating before quantising lowers the error.
    q, k, _ = inputs.qkv_normal(1, 2, 256, 128, seed=11)
    q, k = inputs.with_outliers_r1(q, k, seed=11)
    qd, kd = q.double().numpy()[0], k.double().numpy()[0]
    exact = np.einsum("hid,hjd->hij", qd, kd)
    err = {}
    for rot in (False, True):
        cq, dq = oracle.quantize_per_tensor(qd, rot)
        ck, dk = oracle.quantize_per_tensor(kd, rot)
        approx = np.einsum("hid,hjd->hij", oracle.e4m3_decode(cq) * dq, oracle.e4m3_decode(ck) * dk)
        err[rot] = np.linalg.norm(approx - exact) / np.linalg.norm(exact)
    assert err[True] < err[False] / 3, err


# ------------------------------------------------------ per-block scales --
def _rand_bf16(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g).to(torch.bfloat16).double().numpy()


def test_per_block_one_block_equals_per_tensor():
    x = _rand_bf16((1, 1, 100, 64), 60)
    c1, d1 = oracle.quantize_per_tensor(x, True)
    c2, d2 = oracle.quantize_per_block(x, True)
    assert np.array_equal(c1, c2) and d2.shape == (1, 1, 1) and d2[0, 0, 0] == d1


def test_per_block_max_maps_to_448_and_blocks_are_independent():
    x = _rand_bf16((2, 3, 300, 64), 61).astype(np.float64)  # 3 blocks per head, the last of 44 rows
    codes, desc = oracle.quantize_per_block(x, False)
    assert desc.shape == (2, 3, 3)
    for b in range(2):
        for h in range(3):
            for i, (lo, hi) in enumerate(((0, 128), (128, 256), (256, 300))):
                blk = np.abs(x[b, h, lo:hi])
                assert desc[b, h, i] == pytest.approx(blk.max() / 448.0, rel=0, abs=0)
                # the block's largest magnitude is coded as +-448 (0x7e / 0xfe)
                at = np.unravel_index(np.argmax(blk), blk.shape)
                assert codes[b, h, lo + at[0], at[1]] & 0x7F == 0x7E
    # scaling one block by a power of two changes only that block's descale
    y = x.copy()
    y[1, 2, 128:256] *= 8.0
    codes2, desc2 = oracle.quantize_per_block(y, False)
    assert np.array_equal(codes2, codes)
    assert desc2[1, 2, 1] == 8.0 * desc[1, 2, 1]
    mask = np.ones(desc.shape, dtype=bool)
    mask[1, 2, 1] = False
    assert np.array_equal(desc2[mask], desc[mask])


def test_per_block_zero_block_and_error_bound():
    x = _rand_bf16((1, 2, 256, 128), 62).astype(np.float64)
    x[0, 1, :128] = 0.0
    x[0, 0, 128:] *= 65536.0  # blocks of very different ranges
    codes, desc = oracle.quantize_per_block(x, True)
    assert desc[0, 1, 0] == 1.0 and np.all(codes[0, 1, :128] & 0x7F == 0)
    xr = oracle.rotate(x)
    deq = oracle.e4m3_decode(codes) * np.repeat(desc, 128, axis=2)[..., None]
    # within half an e4m3 spacing (relative 2^-4) of the block's scale, per element
    scale = np.repeat(desc, 128, axis=2)[..., None] * 448.0
    assert np.all(np.abs(deq - xr) <= np.maximum(np.abs(xr) * 2.0 ** -4, scale * 2.0 ** -10) + 1e-12)
    # e4m3 is a floating-point code, so a scale only matters where it pushes
    # values into the subnormal range: with one scale for the whole tensor, the
    # block 65536x smaller than the largest lands there and loses precision
    c_t, d_t = oracle.quantize_per_tensor(x, True)
    small = (0, 0, slice(0, 128))
    err_t = np.linalg.norm(oracle.e4m3_decode(c_t)[small] * d_t - xr[small])
    err_b = np.linalg.norm(deq[small] - xr[small])
    assert err_b < 0.5 * err_t
