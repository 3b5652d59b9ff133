"""Pins for the oracle's generalisations: fewer queries than keys (the queries
are the last positions of the sequence), attention restricted to a block of
keys (a partial result, O = 0 and LSE = -inf where a row sees no key), and the
merge of partial results by their LSEs.

What fixes them: softmax over a union of disjoint key sets equals the
LSE-weighted combination of the softmaxes over each set (the accumulation of
partial results of the "Flash Attention" glossary page, second paragraph), so
splitting the keys into blocks and merging must give the full result; closed
forms (Q = 0 averages exactly the visible values, with LSE = ln of their count);
and the materialised routine, which builds the masks independently.
"""
import inspect
import math

import numpy as np
import pytest

import oracle


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


@pytest.mark.parametrize("nq,nk", [(1, 1), (1, 40), (5, 13), (17, 17), (16, 64), (3, 129)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("key_range", [None, (0, 7), (4, 11), (9, 200)])
def test_rectangular_and_ranged_match_materialised(nq, nk, causal, key_range):
    q = _rand((2, 2, nq, 16), 1)
    k, v = _rand((2, 2, nk, 16), 2), _rand((2, 2, nk, 16), 3)
    o, lse = oracle.attention(q, k, v, causal, 0.41, key_range=key_range)
    o2, lse2 = oracle.attention_naive(q, k, v, causal, 0.41, key_range=key_range)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-12)
    assert np.array_equal(np.isneginf(lse), np.isneginf(lse2))
    fin = np.isfinite(lse)
    np.testing.assert_allclose(lse[fin], lse2[fin], rtol=0, atol=1e-12)


@pytest.mark.parametrize("nq,nk", [(1, 9), (4, 9), (9, 9)])
@pytest.mark.parametrize("key_range", [None, (2, 6), (3, 100)])
def test_zero_queries_average_exactly_the_visible_values(nq, nk, key_range):
    # Q = 0: every visible key has weight 1, so O_i is the mean of the visible
    # values and LSE_i = ln(count). Causal row i sees keys <= i + nk - nq.
    d = 4
    q = np.zeros((1, 1, nq, d))
    k = _rand((1, 1, nk, d), 5)
    v = _rand((1, 1, nk, d), 6)
    lo, hi = key_range or (0, nk)
    for causal in (False, True):
        o, lse = oracle.attention(q, k, v, causal, 1.0, key_range=key_range)
        for i in range(nq):
            last = min(hi, nk) - 1
            if causal:
                last = min(last, i + nk - nq)
            idx = list(range(lo, last + 1))
            if not idx:
                assert np.all(o[0, 0, i] == 0) and np.isneginf(lse[0, 0, i])
                continue
            np.testing.assert_allclose(o[0, 0, i], v[0, 0, idx].mean(axis=0), rtol=0, atol=1e-14)
            assert lse[0, 0, i] == pytest.approx(math.log(len(idx)), abs=1e-14)


def test_single_query_causal_sees_every_key():
    q = _rand((1, 3, 1, 8), 7)
    k, v = _rand((1, 3, 30, 8), 8), _rand((1, 3, 30, 8), 9)
    oc, lc = oracle.attention(q, k, v, True, 0.5)
    on, ln = oracle.attention(q, k, v, False, 0.5)
    assert np.array_equal(oc, on) and np.array_equal(lc, ln)


def test_last_query_rows_equal_the_square_problem_rows():
    # The last nq rows of the square causal problem are the rectangular problem.
    n, nq = 23, 6
    q = _rand((1, 2, n, 8), 10)
    k, v = _rand((1, 2, n, 8), 11), _rand((1, 2, n, 8), 12)
    o_sq, l_sq = oracle.attention(q, k, v, True, 0.3)
    o_r, l_r = oracle.attention(q[:, :, n - nq:], k, v, True, 0.3)
    assert np.array_equal(o_r, o_sq[:, :, n - nq:]) and np.array_equal(l_r, l_sq[:, :, n - nq:])


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("bounds", [(0, 40), (0, 13, 40), (0, 1, 2, 39, 40), (0, 10, 20, 30, 40)])
def test_split_keys_then_merge_equals_full(causal, bounds):
    q = _rand((2, 2, 11, 16), 13) * 2.0
    k, v = _rand((2, 2, 40, 16), 14), _rand((2, 2, 40, 16), 15)
    parts = [oracle.attention(q, k, v, causal, 0.6, key_range=(a, b)) for a, b in zip(bounds[:-1], bounds[1:])]
    o, lse = oracle.lse_merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    o_full, lse_full = oracle.attention(q, k, v, causal, 0.6)
    np.testing.assert_allclose(o, o_full, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_full, rtol=0, atol=1e-12)


def test_merge_identities():
    o1 = _rand((3, 5, 8), 16)
    l1 = _rand((3, 5), 17)
    # one part: unchanged
    o, lse = oracle.lse_merge(o1[None], l1[None])
    np.testing.assert_allclose(o, o1, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, l1, rtol=0, atol=1e-15)
    # an empty part (LSE -inf, O 0) changes nothing
    o, lse = oracle.lse_merge(np.stack([o1, np.zeros_like(o1)]), np.stack([l1, np.full_like(l1, -np.inf)]))
    np.testing.assert_allclose(o, o1, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, l1, rtol=0, atol=1e-15)
    # two parts of equal mass: the mean, and LSE + ln 2
    o2 = _rand((3, 5, 8), 18)
    o, lse = oracle.lse_merge(np.stack([o1, o2]), np.stack([l1, l1]))
    np.testing.assert_allclose(o, (o1 + o2) / 2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, l1 + math.log(2.0), rtol=0, atol=1e-14)
    # masses e^0 and e^ln3: weights 1/4 and 3/4
    o, lse = oracle.lse_merge(np.stack([o1, o2]), np.stack([np.zeros_like(l1), np.full_like(l1, math.log(3.0))]))
    np.testing.assert_allclose(o, 0.25 * o1 + 0.75 * o2, rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse, np.full_like(l1, math.log(4.0)), rtol=0, atol=1e-14)
    # all parts empty: O = 0, LSE = -inf
    o, lse = oracle.lse_merge(np.zeros((2, 3, 5, 8)), np.full((2, 3, 5), -np.inf))
    assert np.all(o == 0) and np.all(np.isneginf(lse))
    # order of the parts does not matter; large LSEs do not overflow
    big = np.stack([l1 + 800.0, l1 + 801.0])
    oa, la = oracle.lse_merge(np.stack([o1, o2]), big)
    ob, lb = oracle.lse_merge(np.stack([o2, o1]), big[::-1])
    np.testing.assert_allclose(oa, ob, rtol=0, atol=1e-14)
    np.testing.assert_allclose(la, lb, rtol=0, atol=1e-12)
    assert np.all(np.isfinite(oa))


MERGE_MUTANTS = {
    "weight_sign": ("np.exp(lse_parts - np.where", "np.exp(np.where(empty, 0.0, m)[None] - lse_parts + 0 * np.where"),
    "no_normalisation": ("/ np.where(empty, 1.0, total)[..., None]", "/ 1.0"),
    "lse_without_max": ("m + np.log(np.where(empty, 1.0, total))", "np.log(np.where(empty, 1.0, total))"),
    "max_instead_of_sum": ("total = w.sum(axis=0)", "total = w.max(axis=0)"),
}


def _merge_pins_pass(merge) -> bool:
    ok = True
    o1, o2 = _rand((3, 5, 8), 16), _rand((3, 5, 8), 18)
    o, lse = merge(np.stack([o1, o2]), np.stack([np.zeros((3, 5)), np.full((3, 5), math.log(3.0))]))
    ok &= np.allclose(o, 0.25 * o1 + 0.75 * o2, rtol=0, atol=1e-14)
    ok &= np.allclose(lse, math.log(4.0), rtol=0, atol=1e-14)
    q = _rand((1, 2, 7, 8), 19)
    k, v = _rand((1, 2, 30, 8), 20), _rand((1, 2, 30, 8), 21)
    parts = [oracle.attention(q, k, v, True, 0.5, key_range=r) for r in ((0, 12), (12, 30))]
    o, lse = merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    o_full, lse_full = oracle.attention(q, k, v, True, 0.5)
    ok &= np.allclose(o, o_full, rtol=0, atol=1e-12) and np.allclose(lse, lse_full, rtol=0, atol=1e-12)
    return bool(ok)


def _load_merge(src):
    ns = {"np": np, "_as_f64": oracle._as_f64}
    exec(compile(src, "<lse_merge>", "exec"), ns)
    return ns["lse_merge"]


def test_unmutated_merge_passes_its_pins():
    assert _merge_pins_pass(_load_merge(inspect.getsource(oracle.lse_merge)))


@pytest.mark.parametrize("name", sorted(MERGE_MUTANTS))
def test_each_planted_merge_mistake_is_caught(name):
    src = inspect.getsource(oracle.lse_merge)
    old, new = MERGE_MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    with np.errstate(all="ignore"):
        assert not _merge_pins_pass(_load_merge(src.replace(old, new)))
