"""GPU parity of the backward pass (fa_bwd through the C ABI) against the fp64
oracle's gradients (oracle.attention_bwd), on the same seeded inputs.

Tolerance, from the kernel's arithmetic (u = 2^-8, the unit roundoff of bf16):
the kernel rounds P to bf16 before dV = Pᵀ dO and dS to bf16 before
dK = scale dSᵀ Q and dQ = scale dS K, forms D_i from the bf16 O it is given, and
rounds each gradient to bf16. Each term of a product is then off by at most
about 2u of its size, and a bound on every entry is 3u·M + 2u·|G|, with M the
oracle's absolute-value envelope (the same products over |P|, |dO|, P(|dP| + A),
|Q|, |K|). On top of that worst case, rounding errors of random sign leave a
relative RMSE of about u/√3 per rounding step, a few 1e-3 in all; the tests
gate it at 1e-2. A wrong index, sign or dropped term moves the gradient by its
own size: a relative RMSE near 1.
"""
import numpy as np
import pytest
import torch

import oracle
import io_aware_exact_17_b200 as fa
from io_aware_exact_17_b200 import inputs
from helpers import record, rel_rmse, to_np

pytestmark = pytest.mark.gpu

U = 2.0 ** -8
REL_RMSE_MAX = 1e-2


def _status_ok():
    torch.cuda.synchronize()
    code, site, block = fa.device_status()
    assert code == 0, f"device wait ran out at site {site}, block {block}"


def _problem(B, H, N, d, seed):
    q, k, v = inputs.qkv_normal(B, H, N, d, seed)
    do = inputs.grad_out(B, H, N, d, seed + 500)
    return q, k, v, do


def _check(got, q, k, v, do, causal, scale, label=None):
    (gq, gk, gv), (mq, mk, mv) = oracle.attention_bwd(q, k, v, do, causal, scale, return_bounds=True)
    errs = {}
    for name, g, ref, m in (("dq", got[0], gq, mq), ("dk", got[1], gk, mk), ("dv", got[2], gv, mv)):
        g = to_np(g)
        assert np.all(np.isfinite(g)), name
        bound = 3 * U * m + 2 * U * np.abs(ref) + 1e-6
        over = np.abs(g - ref) > bound
        assert not over.any(), (name, int(over.sum()), float(np.max(np.abs(g - ref) - bound)))
        errs[name] = rel_rmse(g, ref) if np.any(ref != 0) else float(np.max(np.abs(g)))
        assert errs[name] <= REL_RMSE_MAX, (name, errs[name])
    if label:
        record(label, **{f"{n}_rel_rmse": e for n, e in errs.items()})
    return errs


def _oracle_fwd(q, k, v, causal, scale):
    """O (bf16) and LSE (fp32) from the oracle, as the kernel's inputs."""
    o, lse = oracle.attention(q, k, v, causal, scale)
    return torch.from_numpy(o).to(torch.bfloat16), torch.from_numpy(lse).float()


@pytest.mark.parametrize("B,H,N,d", [(1, 2, 128, 64), (1, 2, 300, 128), (2, 2, 700, 64), (1, 3, 512, 128),
                                     (1, 2, 129, 128), (1, 1, 1000, 128)])
@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_oracle(B, H, N, d, causal):
    q, k, v, do = _problem(B, H, N, d, 200 + N + d)
    scale = d ** -0.5
    o, lse = _oracle_fwd(q, k, v, causal, scale)
    got = fa.bwd(q.cuda(), k.cuda(), v.cuda(), o.cuda(), lse.cuda(), do.cuda(), causal=causal, scale=scale)
    _status_ok()
    _check(got, q, k, v, do, causal, scale)


@pytest.mark.parametrize("causal", [False, True])
def test_single_position(causal):
    # One key: P = 1, so dV = dO exactly and, in exact arithmetic, dQ = dK = 0.
    # The kernel's dS = P (dP - D) subtracts two fp32 sums of the same d products
    # (dO_c v_c) taken in different orders, so |dS| <= 2 d 2^-24 Σ_c |dO_c v_c|,
    # and |dQ_c| <= scale |dS| |k_c|, |dK_c| <= scale |dS| |q_c|.
    d, scale = 128, 0.1
    q, k, v, do = _problem(2, 3, 1, d, 7)
    o, lse = _oracle_fwd(q, k, v, causal, scale)
    dq, dk, dv = fa.bwd(q.cuda(), k.cuda(), v.cuda(), o.cuda(), lse.cuda(), do.cuda(), causal=causal, scale=scale)
    _status_ok()
    assert torch.equal(dv.cpu(), do)
    ds_max = 2 * d * 2.0 ** -24 * (do.double() * v.double()).abs().sum(-1, keepdim=True).numpy() * (1 + 2 * U)
    assert np.all(np.abs(to_np(dq)) <= scale * ds_max * np.abs(k.double().numpy()) * (1 + U))
    assert np.all(np.abs(to_np(dk)) <= scale * ds_max * np.abs(q.double().numpy()) * (1 + U))


def test_forward_then_backward_through_the_library():
    # O and LSE from the library's own forward, gradients against the oracle's
    B, H, N, d = 2, 4, 640, 128
    q, k, v, do = _problem(B, H, N, d, 11)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    for causal in (False, True):
        o, lse = fa.fwd(qc, kc, vc, causal=causal)
        got = fa.bwd(qc, kc, vc, o, lse, do.cuda(), causal=causal)
        _status_ok()
        _check(got, q, k, v, do, causal, d ** -0.5)


def test_other_scales():
    q, k, v, do = _problem(1, 2, 384, 64, 12)
    for scale in (0.05, 0.5):
        o, lse = _oracle_fwd(q, k, v, True, scale)
        got = fa.bwd(q.cuda(), k.cuda(), v.cuda(), o.cuda(), lse.cuda(), do.cuda(), causal=True, scale=scale)
        _status_ok()
        _check(got, q, k, v, do, True, scale)


@pytest.mark.parametrize("causal", [False, True])
def test_b4_h16_n2048_d128_sampled_heads(causal):
    # The training-shaped workload at its full size; the oracle recomputes a few
    # whole heads (every gradient entry of those heads).
    B, H, N, d = 4, 16, 2048, 128
    q, k, v, do = _problem(B, H, N, d, 1001)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o, lse = fa.fwd(qc, kc, vc, causal=causal)
    dq, dk, dv = fa.bwd(qc, kc, vc, o, lse, do.cuda(), causal=causal)
    _status_ok()
    g = torch.Generator().manual_seed(5)
    heads = torch.randperm(B * H, generator=g)[:3].tolist() + [B * H - 1]
    for bh in heads:
        b, h = divmod(bh, H)
        sl = (slice(b, b + 1), slice(h, h + 1))
        _check((dq[sl].cpu(), dk[sl].cpu(), dv[sl].cpu()), q[sl], k[sl], v[sl], do[sl], causal, d ** -0.5,
               label=f"bf16 bwd B{B} H{H} N{N} d{d} {'causal' if causal else 'non-causal'} head {bh}")


def test_unsupported_head_dim():
    q = torch.zeros(1, 1, 128, 256, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, 128, device="cuda")
    with pytest.raises(fa.FaError, match="unsupported"):
        fa.bwd(q, q, q, q, lse, q)
