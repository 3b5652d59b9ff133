"""GPU parity of the BF16 forward (fa_fwd through the C ABI) against the fp64
oracle, element by element, on seeded N(0,1) inputs; plus the invariants the
definition fixes (causal rows ignore future keys, key order does not matter,
V = 1 gives O = 1) and ragged / degenerate sizes."""
import numpy as np
import pytest
import torch

import oracle
import io_aware_exact_17_b200 as fa
from io_aware_exact_17_b200 import inputs
from helpers import BF16_LSE_ATOL, BF16_O_ATOL, bf16_out_tol, max_abs, record, to_np

pytestmark = pytest.mark.gpu


def _run(q, k, v, causal, scale=None, n_split=0):
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=causal, scale=scale, n_split=n_split)
    torch.cuda.synchronize()
    code, site, block = fa.device_status()
    assert code == 0, f"device wait ran out at site {site}, block {block}"
    return o, lse


def _check_full(B, H, N, d, causal, seed, n_split=0):
    q, k, v = inputs.qkv_normal(B, H, N, d, seed)
    scale = d ** -0.5
    o, lse = _run(q, k, v, causal, n_split=n_split)
    o_ref, lse_ref = oracle.attention(q, k, v, causal, scale)
    eo, el = max_abs(to_np(o), o_ref), max_abs(to_np(lse), lse_ref)
    record(f"bf16 B{B} H{H} N{N} d{d} {'causal' if causal else 'non-causal'}", o_max_abs=eo, lse_max_abs=el)
    assert eo <= BF16_O_ATOL and el <= BF16_LSE_ATOL, (eo, el)
    return eo, el


@pytest.mark.parametrize("causal", [False, True])
def test_tiny_config(causal):
    # B=1, H=2, N=128, d=64, scale 1/8
    _check_full(1, 2, 128, 64, causal, 1000)


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("N", [1, 17, 129, 200, 384, 700])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_split", [0, 1])
def test_ragged_sizes(d, N, causal, n_split):
    # n_split 0: the automatic schedule (these few heads: keys split and merged);
    # 1: one CTA per query block (fa_fwd)
    _check_full(2, 3, N, d, causal, 7 + N + d, n_split)


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_split", [0, 1])
def test_b4_h16_n2048_d128_full(causal, n_split):
    _check_full(4, 16, 2048, 128, causal, 1001, n_split)


def test_few_heads_long_sequence_split_keys():
    # 2 heads x 8 two-tile query blocks = 16 CTAs on 148 SMs: the automatic
    # schedule splits every block's keys and merges
    B, H, N, d = 1, 2, 2048, 128
    q, k, v = inputs.qkv_normal(B, H, N, d, 1010)
    for causal in (False, True):
        o, lse = _run(q, k, v, causal)
        o_ref, lse_ref = oracle.attention(q, k, v, causal, d ** -0.5)
        eo, el = max_abs(to_np(o), o_ref), max_abs(to_np(lse), lse_ref)
        assert eo <= BF16_O_ATOL and el <= BF16_LSE_ATOL, (causal, eo, el)


@pytest.mark.parametrize("n", [512, 1024, 2048, 4096, 8192, 16384])
@pytest.mark.parametrize("causal", [False, True])
def test_sequence_sweep_sampled_rows(n, causal):
    B, H, d = 16384 // n, 16, 128
    q, k, v = inputs.qkv_normal(B, H, n, d, 1002)
    o, lse = _run(q, k, v, causal)
    rows = inputs.sample_rows(B, H, n, per_head=8, seed=n)
    o_ref, lse_ref = oracle.attention(q, k, v, causal, d ** -0.5, rows=rows.numpy())
    got_o = to_np(o).reshape(-1, d)[rows.numpy()]
    got_l = to_np(lse).reshape(-1)[rows.numpy()]
    eo, el = max_abs(got_o, o_ref), max_abs(got_l, lse_ref)
    record(f"bf16 B{B} H{H} N{n} d{d} {'causal' if causal else 'non-causal'} (sampled rows)", o_max_abs=eo,
           lse_max_abs=el)
    assert eo <= BF16_O_ATOL
    assert el <= BF16_LSE_ATOL


@pytest.mark.parametrize("d", [64, 128, 256])
def test_head_dim_sweep_sampled_rows(d):
    B, H, N = 2, 2048 // d, 4096
    q, k, v = inputs.qkv_normal(B, H, N, d, 1004)
    o, lse = _run(q, k, v, True)
    rows = inputs.sample_rows(B, H, N, per_head=8, seed=d)
    o_ref, lse_ref = oracle.attention(q, k, v, True, d ** -0.5, rows=rows.numpy())
    eo = max_abs(to_np(o).reshape(-1, d)[rows.numpy()], o_ref)
    el = max_abs(to_np(lse).reshape(-1)[rows.numpy()], lse_ref)
    record(f"bf16 B{B} H{H} N{N} d{d} causal (sampled rows)", o_max_abs=eo, lse_max_abs=el)
    assert eo <= BF16_O_ATOL
    assert el <= BF16_LSE_ATOL


@pytest.mark.parametrize("d", [64, 128, 256])
def test_causal_rows_ignore_future_keys_bitwise(d):
    B, H, N = 1, 2, 600
    q, k, v = inputs.qkv_normal(B, H, N, d, 31)
    o1, l1 = _run(q, k, v, True)
    for i0 in (0, 127, 128, 255, 256, 383, 500):
        k2, v2 = k.clone(), v.clone()
        k2[:, :, i0 + 1:] = (k2[:, :, i0 + 1:].float() * -3 + 1).to(torch.bfloat16)
        v2[:, :, i0 + 1:] = (v2[:, :, i0 + 1:].float() * 5 - 2).to(torch.bfloat16)
        o2, l2 = _run(q, k2, v2, True)
        assert torch.equal(o1[:, :, : i0 + 1], o2[:, :, : i0 + 1]), i0
        assert torch.equal(l1[:, :, : i0 + 1], l2[:, :, : i0 + 1]), i0


def test_key_permutation_invariance():
    B, H, N, d = 1, 4, 777, 128
    q, k, v = inputs.qkv_normal(B, H, N, d, 32)
    perm = torch.randperm(N, generator=torch.Generator().manual_seed(3))
    o1, l1 = _run(q, k, v, False)
    o2, l2 = _run(q, k[:, :, perm], v[:, :, perm], False)
    assert max_abs(to_np(o1), to_np(o2)) <= BF16_O_ATOL
    assert max_abs(to_np(l1), to_np(l2)) <= BF16_LSE_ATOL


@pytest.mark.parametrize("causal", [False, True])
def test_ones_values_give_ones(causal):
    q, k, _ = inputs.qkv_normal(1, 2, 300, 128, 33)
    v = torch.ones_like(q)
    o, _ = _run(q, k, v, causal)
    assert max_abs(to_np(o), np.ones(o.shape)) <= BF16_O_ATOL


def test_large_logits_and_scale():
    # Scale 1 with N(0,1) data gives logits of size ~11 and row maxima that grow
    # across tiles: exercises the reference-max moves and the O rescale.
    B, H, N, d = 1, 2, 1024, 128
    q, k, v = inputs.qkv_normal(B, H, N, d, 34)
    for causal in (False, True):
        o, lse = _run(q, k, v, causal, scale=1.0)
        o_ref, lse_ref = oracle.attention(q, k, v, causal, 1.0)
        assert np.all(np.abs(to_np(o) - o_ref) <= bf16_out_tol(o_ref))
        assert max_abs(to_np(lse), lse_ref) <= BF16_LSE_ATOL


def test_increasing_logits_force_rescales():
    # Keys whose scores rise tile after tile: every tile moves the reference max.
    B, H, N, d = 1, 1, 1024, 64
    q = torch.ones(B, H, N, d).to(torch.bfloat16)
    ramp = torch.linspace(0, 6, N).view(1, 1, N, 1)
    k = (torch.ones(B, H, N, d) * ramp).to(torch.bfloat16)
    _, _, v = inputs.qkv_normal(B, H, N, d, 35)
    for causal in (False, True):
        o, lse = _run(q, k, v, causal, scale=1.0)
        o_ref, lse_ref = oracle.attention(q, k, v, causal, 1.0)
        assert np.all(np.abs(to_np(o) - o_ref) <= bf16_out_tol(o_ref))
        # LSE here reaches ~380: fp32 carries ~2^-24 relative, so allow 1e-3 per 100.
        assert max_abs(to_np(lse), lse_ref) <= BF16_LSE_ATOL * max(1.0, float(np.max(np.abs(lse_ref))) / 100)


@pytest.mark.parametrize("causal", [False, True])
def test_growth_in_the_second_half_of_key_tiles(causal):
    # Scores that stay flat over keys 0..63 of every 128-key tile and jump over
    # keys 64..127, higher tile after tile: the row max grows by more than 2^8
    # (log2 units) inside the second half, after P V of the first half is already
    # issued against the old reference. Exercises the wait for that product and
    # the rescale of O that follow.
    B, H, N, d = 1, 2, 640, 64
    q = torch.full((B, H, N, d), 0.125).to(torch.bfloat16)
    t = torch.zeros(N)
    for j in range(128, N):
        if j % 128 >= 64:
            t[j] = 2.0 * (j // 128)  # score 8 t: +16 per tile (23 in log2 units)
    k = (torch.ones(B, H, N, d) * t.view(1, 1, N, 1)).to(torch.bfloat16)
    _, _, v = inputs.qkv_normal(B, H, N, d, 38)
    o, lse = _run(q, k, v, causal, scale=1.0)
    o_ref, lse_ref = oracle.attention(q, k, v, causal, 1.0)
    assert np.all(np.abs(to_np(o) - o_ref) <= bf16_out_tol(o_ref))
    assert max_abs(to_np(lse), lse_ref) <= BF16_LSE_ATOL * max(1.0, float(np.max(np.abs(lse_ref))) / 100)


def test_deterministic():
    q, k, v = inputs.qkv_normal(2, 4, 1000, 128, 36)
    o1, l1 = _run(q, k, v, True)
    o2, l2 = _run(q, k, v, True)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_lse_optional_and_no_nxn_buffer():
    # Linear memory. One CTA per query block (n_split=1): nothing is allocated
    # beyond O (and LSE when asked). The automatic schedule (these 128 query
    # blocks are fewer than the SMs, so keys are split) adds a workspace of fp32
    # partial outputs: O(N d) per head, far below one N x N matrix.
    B, H, N, d = 1, 8, 4096, 128
    q, k, v = (t.cuda() for t in inputs.qkv_normal(B, H, N, d, 37))
    o = torch.empty_like(q)
    torch.cuda.synchronize()
    before = torch.cuda.memory_allocated()
    fa.fwd(q, k, v, causal=False, out=o, return_lse=False, n_split=1)
    torch.cuda.synchronize()
    assert torch.cuda.memory_allocated() == before
    o2, _ = fa.fwd(q, k, v, causal=False, n_split=1)
    assert torch.equal(o, o2)
    o3 = torch.empty_like(q)
    fa.fwd(q, k, v, causal=False, out=o3, return_lse=False)
    torch.cuda.synchronize()
    grown = torch.cuda.memory_allocated() - before
    assert 0 < grown <= 8 * B * H * N * d * 4 < B * H * N * N * 4
    o4, _ = fa.fwd(q, k, v, causal=False)
    assert torch.equal(o3, o4)
    assert max_abs(to_np(o3), to_np(o)) <= 2 * BF16_O_ATOL
