"""The backward parity tolerance is derived from the kernel's arithmetic, not
fitted to its output. This CPU test replays that arithmetic's rounding steps in
fp64 (P and dS rounded to bf16 before their products, D from the bf16 O the
kernel is given, each gradient rounded to bf16 once) and checks the result
against the oracle's exact gradients with the bound the GPU tests apply:
|G - G_ref| <= 3u·M + 2u·|G_ref| + 1e-6 per entry and relative RMSE <= 1e-2,
u = 2^-8. It also checks that the bound is not loose enough to pass a gradient
with one term dropped."""
import numpy as np
import pytest
import torch

import oracle
from io_aware_exact_17_b200 import inputs

U = 2.0 ** -8


def _bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16).double().numpy()


def _emulate(q, k, v, do, causal, scale, drop_d=False):
    """The kernel's rounding steps, per head, in fp64."""
    B, H, N, d = q.shape
    out = [np.zeros_like(q) for _ in range(3)]
    hidden = np.triu(np.ones((N, N), dtype=bool), 1) if causal else np.zeros((N, N), dtype=bool)
    for b in range(B):
        for h in range(H):
            qh, kh, vh, doh = q[b, h], k[b, h], v[b, h], do[b, h]
            s = np.where(hidden, -np.inf, scale * qh @ kh.T)
            m = s.max(axis=1, keepdims=True)
            lse = m + np.log(np.exp(s - m).sum(axis=1, keepdims=True))
            p = np.exp(s - lse)
            o_bf = _bf16(p @ vh)                       # the forward's bf16 O
            dvec = 0.0 if drop_d else (doh * o_bf).sum(axis=1, keepdims=True)
            dp = doh @ vh.T
            ds_bf = _bf16(p * (dp - dvec))
            out[0][b, h] = _bf16(scale * ds_bf @ kh)
            out[1][b, h] = _bf16(scale * ds_bf.T @ qh)
            out[2][b, h] = _bf16(_bf16(p).T @ doh)
    return out


def _within(got, q, k, v, do, causal, scale):
    (gq, gk, gv), (mq, mk, mv) = oracle.attention_bwd(q, k, v, do, causal, scale, return_bounds=True)
    ok, rels = True, []
    for g, ref, m in zip(got, (gq, gk, gv), (mq, mk, mv)):
        ok &= bool(np.all(np.abs(g - ref) <= 3 * U * m + 2 * U * np.abs(ref) + 1e-6))
        rel = float(np.linalg.norm(g - ref) / np.linalg.norm(ref))
        rels.append(rel)
        ok &= rel <= 1e-2
    return ok, rels


@pytest.mark.parametrize("N,d", [(300, 64), (256, 128)])
@pytest.mark.parametrize("causal", [False, True])
def test_rounding_model_meets_the_bound(N, d, causal):
    q, k, v = (t.double().numpy() for t in inputs.qkv_normal(1, 2, N, d, 31 + N))
    do = inputs.grad_out(1, 2, N, d, 32 + N).double().numpy()
    ok, rels = _within(_emulate(q, k, v, do, causal, d ** -0.5), q, k, v, do, causal, d ** -0.5)
    assert ok, rels
    assert max(rels) < 5e-3  # a few 1e-3, as the u/sqrt(3)-per-rounding estimate says


def test_bound_rejects_a_dropped_term():
    N, d = 256, 64
    q, k, v = (t.double().numpy() for t in inputs.qkv_normal(1, 2, N, d, 40))
    do = inputs.grad_out(1, 2, N, d, 41).double().numpy()
    ok, rels = _within(_emulate(q, k, v, do, False, d ** -0.5, drop_d=True), q, k, v, do, False, d ** -0.5)
    assert not ok and max(rels) > 0.1, rels
