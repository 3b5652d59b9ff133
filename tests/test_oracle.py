"""Pins for the CPU attention oracle, none of which re-types its formula.

What fixes the oracle's answer, per the pages: the IO-aware method returns
exactly standard attention ("Flash Attention" glossary page, first paragraph),
whose standard form builds the N x N matrix (same page, second paragraph). So
the oracle is pinned by (a) hand-derived closed forms on a 2-token problem, (b)
a second, independently written routine that materialises the N x N matrix,
(c) closed forms and invariants that any correct attention satisfies.
"""
import json
import math
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_17_b200 import inputs

GOLDEN = Path(__file__).resolve().parent / "golden"


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def test_golden_two_token_closed_form():
    g = json.loads((GOLDEN / "attention_closed_form.json").read_text())
    q = np.array(g["q"], dtype=np.float64)[None, None]
    k = np.array(g["k"], dtype=np.float64)[None, None]
    v = np.array(g["v"], dtype=np.float64)[None, None]
    for mode, causal in (("non_causal", False), ("causal", True)):
        o, lse = oracle.attention(q, k, v, causal, g["scale"])
        np.testing.assert_allclose(o[0, 0, :, 0], g[mode]["O"]["value"], rtol=0, atol=1e-15)
        np.testing.assert_allclose(lse[0, 0], g[mode]["LSE"]["value"], rtol=0, atol=1e-15)
        o2, lse2 = oracle.attention_naive(q, k, v, causal, g["scale"])
        np.testing.assert_allclose(o2[0, 0, :, 0], g[mode]["O"]["value"], rtol=0, atol=1e-15)
        np.testing.assert_allclose(lse2[0, 0], g[mode]["LSE"]["value"], rtol=0, atol=1e-15)


@pytest.mark.parametrize("shape", [(1, 2, 1, 8), (2, 2, 17, 16), (1, 3, 64, 64), (1, 1, 33, 3), (2, 1, 40, 128)])
@pytest.mark.parametrize("causal", [False, True])
def test_rowwise_matches_materialised(shape, causal):
    q, k, v = _rand(shape, 1), _rand(shape, 2), _rand(shape, 3)
    scale = 0.37
    o, lse = oracle.attention(q, k, v, causal, scale)
    o2, lse2 = oracle.attention_naive(q, k, v, causal, scale)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-12)


def test_row_subset_equals_full_and_threads_do_not_matter():
    shape = (2, 3, 50, 16)
    q, k, v = _rand(shape, 4), _rand(shape, 5), _rand(shape, 6)
    o, lse = oracle.attention(q, k, v, True, 0.25, threads=1)
    o4, lse4 = oracle.attention(q, k, v, True, 0.25, threads=4)
    assert np.array_equal(o, o4) and np.array_equal(lse, lse4)
    rows = np.array([0, 49, 50, 77, 299])
    os_, ls_ = oracle.attention(q, k, v, True, 0.25, rows=rows, threads=3)
    assert np.array_equal(os_, o.reshape(-1, 16)[rows])
    assert np.array_equal(ls_, lse.reshape(-1)[rows])


def test_single_key_returns_its_value():
    shape = (2, 2, 1, 32)
    q, k, v = _rand(shape, 7), _rand(shape, 8), _rand(shape, 9)
    for causal in (False, True):
        o, lse = oracle.attention(q, k, v, causal, 0.5)
        np.testing.assert_array_equal(o, v)
        np.testing.assert_allclose(lse, 0.5 * np.sum(q * k, axis=-1), rtol=0, atol=1e-14)


def test_zero_queries_average_the_visible_values():
    B, H, N, d = 1, 2, 37, 8
    q = np.zeros((B, H, N, d))
    k, v = _rand((B, H, N, d), 10), _rand((B, H, N, d), 11)
    o, lse = oracle.attention(q, k, v, False, 1.0)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2, keepdims=True), o.shape), atol=1e-14)
    np.testing.assert_allclose(lse, math.log(N), atol=1e-14)
    o, lse = oracle.attention(q, k, v, True, 1.0)
    prefix_mean = np.cumsum(v, axis=2) / np.arange(1, N + 1)[None, None, :, None]
    np.testing.assert_allclose(o, prefix_mean, atol=1e-14)
    np.testing.assert_allclose(lse, np.log(np.arange(1, N + 1))[None, None, :].repeat(H, 1), atol=1e-14)


def test_causal_first_row_is_first_value_and_ones_stay_ones():
    shape = (1, 2, 20, 16)
    q, k = _rand(shape, 12), _rand(shape, 13)
    v = _rand(shape, 14)
    o, lse = oracle.attention(q, k, v, True, 0.3)
    np.testing.assert_array_equal(o[:, :, 0], v[:, :, 0])
    np.testing.assert_allclose(lse[:, :, 0], 0.3 * np.sum(q[:, :, 0] * k[:, :, 0], -1), atol=1e-14)
    o1, _ = oracle.attention(q, k, np.ones(shape), False, 0.3)
    np.testing.assert_allclose(o1, 1.0, rtol=0, atol=1e-14)


def test_dominant_key_wins():
    # One key aligned with every query and a logit gap of ~1000: the weights of
    # the others are below exp(-900), so O equals that key's value to fp64.
    N, d = 16, 4
    q = np.zeros((1, 1, N, d))
    q[..., 0] = 1.0
    k = _rand((1, 1, N, d), 15) * 0.1
    k[0, 0, 5, 0] = 1000.0
    v = _rand((1, 1, N, d), 16)
    o, lse = oracle.attention(q, k, v, False, 1.0)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(v[0, 0, 5], (N, d)), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], 1000.0, rtol=0, atol=1e-9)


def test_probabilities_rows_sum_to_one_and_respect_the_mask():
    shape = (1, 2, 24, 8)
    q, k, v = _rand(shape, 17), _rand(shape, 18), _rand(shape, 19)
    for causal in (False, True):
        _, _, p = oracle.attention_naive(q, k, v, causal, 0.7, return_probs=True)
        np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-14)
        assert np.all(p >= 0)
        if causal:
            assert np.all(np.triu(p[0, 0], k=1) == 0)


def test_causal_rows_ignore_future_keys_bitwise():
    shape = (1, 2, 30, 16)
    q, k, v = _rand(shape, 20), _rand(shape, 21), _rand(shape, 22)
    o, lse = oracle.attention(q, k, v, True, 0.4)
    i = 11
    k2, v2 = k.copy(), v.copy()
    k2[:, :, i + 1:] += 5.0 * _rand(k2[:, :, i + 1:].shape, 23)
    v2[:, :, i + 1:] -= 3.0
    o2, lse2 = oracle.attention(q, k2, v2, True, 0.4)
    assert np.array_equal(o[:, :, : i + 1], o2[:, :, : i + 1])
    assert np.array_equal(lse[:, :, : i + 1], lse2[:, :, : i + 1])
    assert not np.array_equal(o[:, :, i + 1:], o2[:, :, i + 1:])


def test_key_permutation_invariance():
    shape = (1, 2, 45, 16)
    q, k, v = _rand(shape, 24), _rand(shape, 25), _rand(shape, 26)
    perm = np.random.default_rng(27).permutation(45)
    o, lse = oracle.attention(q, k, v, False, 0.25)
    o2, lse2 = oracle.attention(q, k[:, :, perm], v[:, :, perm], False, 0.25)
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, atol=1e-13)


def test_bf16_inputs_are_widened_exactly():
    q, k, v = inputs.qkv_normal(1, 2, 64, 32, seed=5)
    o, lse = oracle.attention(q, k, v, False, 0.2)
    o2, lse2 = oracle.attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), False, 0.2)
    assert np.array_equal(o, o2) and np.array_equal(lse, lse2)


def test_bad_rows_are_rejected():
    q = np.zeros((1, 1, 4, 2))
    with pytest.raises(RuntimeError):
        oracle.attention(q, q, q, False, 1.0, rows=[4])
    with pytest.raises(RuntimeError):
        oracle.attention(q, q, q, False, 1.0, rows=[-1])
