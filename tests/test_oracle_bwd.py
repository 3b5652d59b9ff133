"""Pins of the backward oracle (oracle.attention_bwd), none of which re-types its
formulas:

* central finite differences of the forward oracle (itself pinned elsewhere):
  with L = Σ dO ∘ O, dL/dx for every element of Q, K and V;
* closed forms: one key (dV = dO, dQ = dK = 0), identical value rows (O does not
  depend on Q or K, so dQ = dK = 0), the first causal row (a single visible key,
  so dQ_0 = 0);
* invariants: Σ_j dK_j = 0 (adding one vector to every key leaves each softmax
  unchanged), Σ_j dV_j = Σ_i dO_i (each row of P sums to 1),
  Σ_i q_i·dQ_i = Σ_j k_j·dK_j (both are scale · dL/dscale), causal locality (dK_j
  and dV_j do not depend on queries before j), and the error envelope bounds
  each gradient entry;
* planted mistakes in a private copy of the function, each of which some pin
  must reject.
"""
import inspect

import numpy as np
import pytest

import oracle


def _loss_grad_fd(q, k, v, do, causal, scale, h=1e-5):
    """Central differences of L = Σ dO ∘ O(q, k, v) w.r.t. every input element."""
    def loss(q_, k_, v_):
        o, _ = oracle.attention(q_, k_, v_, causal, scale, threads=1)
        return float(np.sum(do * o))

    grads = []
    for which in range(3):
        base = [q.copy(), k.copy(), v.copy()]
        g = np.zeros_like(base[which])
        for idx in np.ndindex(*g.shape):
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[which][idx] += h
            minus[which][idx] -= h
            g[idx] = (loss(*plus) - loss(*minus)) / (2 * h)
        grads.append(g)
    return grads


def _inputs(B, H, N, d, seed):
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal((B, H, N, d)) for _ in range(4))


def _fd_pin(fn, N, d, causal, seed):
    q, k, v, do = _inputs(1, 2, N, d, seed)
    scale = d ** -0.5
    got = fn(q, k, v, do, causal, scale)
    want = _loss_grad_fd(q, k, v, do, causal, scale)
    return max(float(np.max(np.abs(g - w))) for g, w in zip(got, want))


@pytest.mark.parametrize("N,d", [(1, 4), (5, 4), (9, 8)])
@pytest.mark.parametrize("causal", [False, True])
def test_matches_finite_differences_of_the_forward_oracle(N, d, causal):
    assert _fd_pin(oracle.attention_bwd, N, d, causal, 10 + N + d) <= 1e-7


def test_single_key():
    q, k, v, do = _inputs(2, 3, 1, 16, 1)
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, False, 0.25)
    assert np.array_equal(dv, do)
    assert np.all(dq == 0) and np.all(dk == 0)


@pytest.mark.parametrize("causal", [False, True])
def test_equal_value_rows_give_no_query_or_key_gradient(causal):
    q, k, v, do = _inputs(1, 2, 33, 8, 2)
    v[:] = v[:, :, :1]
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal, 0.3)
    assert np.max(np.abs(dq)) <= 1e-13 and np.max(np.abs(dk)) <= 1e-13
    assert np.max(np.abs(dv)) > 0.1


def test_first_causal_row_has_no_query_gradient():
    q, k, v, do = _inputs(1, 2, 20, 8, 3)
    dq, _, _ = oracle.attention_bwd(q, k, v, do, True, 0.3)
    assert np.all(np.abs(dq[:, :, 0]) <= 1e-15)
    assert np.min(np.abs(dq[:, :, 1:]).max(axis=-1)) > 1e-6


@pytest.mark.parametrize("causal", [False, True])
def test_sum_invariants(causal):
    q, k, v, do = _inputs(2, 2, 47, 16, 4)
    scale = 0.2
    dq, dk, dv = oracle.attention_bwd(q, k, v, do, causal, scale)
    assert np.max(np.abs(dk.sum(axis=2))) <= 1e-11
    np.testing.assert_allclose(dv.sum(axis=2), do.sum(axis=2), rtol=0, atol=1e-11)
    np.testing.assert_allclose((q * dq).sum(axis=(2, 3)), (k * dk).sum(axis=(2, 3)), rtol=0, atol=1e-10)


def test_causal_locality():
    q, k, v, do = _inputs(1, 1, 30, 8, 5)
    _, dk, dv = oracle.attention_bwd(q, k, v, do, True, 0.3)
    q2, do2 = q.copy(), do.copy()
    q2[:, :, :12] += 3.0
    do2[:, :, :12] -= 2.0
    _, dk2, dv2 = oracle.attention_bwd(q2, k, v, do2, True, 0.3)
    assert np.array_equal(dk[:, :, 12:], dk2[:, :, 12:]) or np.max(np.abs(dk[:, :, 12:] - dk2[:, :, 12:])) <= 1e-13
    assert np.max(np.abs(dv[:, :, 12:] - dv2[:, :, 12:])) <= 1e-13
    assert np.max(np.abs(dk[:, :, :12] - dk2[:, :, :12])) > 1e-3


@pytest.mark.parametrize("causal", [False, True])
def test_envelope_bounds_each_entry(causal):
    q, k, v, do = _inputs(1, 2, 40, 16, 6)
    grads, bounds = oracle.attention_bwd(q, k, v, do, causal, 0.25, return_bounds=True)
    for g, m in zip(grads, bounds):
        assert np.all(np.abs(g) <= m * (1 + 1e-12) + 1e-15)
    assert np.array_equal(grads[0], oracle.attention_bwd(q, k, v, do, causal, 0.25)[0])


# -------------------------------------------------------------- mutants --
MUTANTS = {
    "no_softmax_jacobian_term": ("ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))", "ds = p * dp"),
    "jacobian_sum_over_queries": ("(p * dp).sum(axis=1, keepdims=True)", "(p * dp).sum(axis=0, keepdims=True)"),
    "dq_without_scale": ("dq[b, h] = scale * (ds @ kh)", "dq[b, h] = ds @ kh"),
    "dq_transposed_ds": ("dq[b, h] = scale * (ds @ kh)", "dq[b, h] = scale * (ds.T @ kh)"),
    "dk_from_keys": ("dk[b, h] = scale * (ds.T @ qh)", "dk[b, h] = scale * (ds.T @ kh)"),
    "dv_untransposed_p": ("dv[b, h] = p.T @ doh", "dv[b, h] = p @ doh"),
    "dp_from_queries": ("dp = doh @ vh.T", "dp = doh @ qh.T"),
    "mask_off_by_one": ("np.triu(np.ones((N, N), dtype=bool), 1)", "np.triu(np.ones((N, N), dtype=bool), 2)"),
}


def _mutant(name):
    src = inspect.getsource(oracle.attention_bwd)
    old, new = MUTANTS[name]
    assert src.count(old) == 1, name
    ns = dict(vars(oracle))
    exec(src.replace(old, new), ns)
    return ns["attention_bwd"]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_every_planted_mistake_is_caught(name):
    fn = _mutant(name)
    errs = [_fd_pin(fn, N, d, causal, 10 + N + d) for N, d in [(5, 4), (9, 8)] for causal in (False, True)]
    assert max(errs) > 1e-4, (name, errs)
