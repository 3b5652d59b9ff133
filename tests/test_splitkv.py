"""GPU parity of attention with few queries over long key sequences
(fa_fwd_splitkv, fa_fwd_partial, fa_lse_merge through the C ABI) against the
fp64 oracle: the per-block partial results (O = 0 and LSE = -inf exactly where a
row sees no key of a block), the merge, and the merged output for split counts
from 1 (no split) up to more blocks than key tiles. Up to 32 queries per head
run the decode layout (each softmax warp on one quarter of every key tile);
the cases include 32 and 33 queries and key counts that leave whole quarters
without a visible key."""
import math

import numpy as np
import pytest
import torch

import oracle
import io_aware_exact_17_b200 as fa
from io_aware_exact_17_b200 import inputs
from helpers import BF16_LSE_ATOL, BF16_O_ATOL, FP8_REL_RMSE, max_abs, record, rel_rmse, to_np

pytestmark = pytest.mark.gpu

KEY_TILE = 128


def _status_ok():
    torch.cuda.synchronize()
    code, site, block = fa.device_status()
    assert code == 0, f"device wait ran out at site {site}, block {block}"


def _qkv(B, H, Nq, Nk, d, seed):
    return inputs.qkv_decode(B, H, Nq, Nk, d, seed)


def _block_bounds(Nk, n_split):
    """Key range [lo, hi) of each block: ceil(tiles / n_split) key tiles each."""
    tiles = math.ceil(Nk / KEY_TILE)
    per = math.ceil(tiles / n_split)
    return [(min(Nk, s * per * KEY_TILE), min(Nk, (s + 1) * per * KEY_TILE)) for s in range(n_split)]


@pytest.mark.parametrize("B,H,Nq,Nk,d", [(1, 2, 1, 1, 128), (2, 3, 1, 777, 128), (1, 2, 5, 300, 64),
                                         (1, 2, 32, 40, 128), (2, 2, 16, 70, 256), (1, 2, 33, 500, 64),
                                         (1, 2, 128, 1000, 128), (1, 1, 200, 4100, 128), (2, 2, 3, 2000, 256),
                                         (1, 2, 700, 700, 64)])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("n_split", [1, 2, 3, 0])
def test_splitkv_matches_oracle(B, H, Nq, Nk, d, causal, n_split):
    q, k, v = _qkv(B, H, Nq, Nk, d, 50 + Nq + Nk + d)
    o, lse = fa.fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=causal, n_split=n_split)
    _status_ok()
    o_ref, lse_ref = oracle.attention(q, k, v, causal, d ** -0.5)
    eo, el = max_abs(to_np(o), o_ref), max_abs(to_np(lse), lse_ref)
    assert eo <= BF16_O_ATOL and el <= BF16_LSE_ATOL, (eo, el)


@pytest.mark.parametrize("causal", [False, True])
def test_partial_blocks_match_oracle_key_ranges(causal):
    # 4 blocks of 2 key tiles over Nk = 1000 (the last block is ragged); causal
    # queries are the last Nq = 300 positions, so the first query rows see no key
    # of the last blocks.
    B, H, Nq, Nk, d, n_split = 1, 2, 300, 1000, 128, 4
    q, k, v = _qkv(B, H, Nq, Nk, d, 77)
    o_part, lse_part = fa.fwd_partial(q.cuda(), k.cuda(), v.cuda(), causal=causal, n_split=n_split)
    _status_ok()
    o_part, lse_part = o_part.cpu().double().numpy(), lse_part.cpu().double().numpy()
    for s, (lo, hi) in enumerate(_block_bounds(Nk, n_split)):
        o_ref, lse_ref = oracle.attention(q, k, v, causal, d ** -0.5, key_range=(lo, hi))
        empty = np.isneginf(lse_ref)
        assert np.array_equal(np.isneginf(lse_part[s]), empty), s
        assert np.all(o_part[s][empty] == 0.0)
        assert max_abs(o_part[s][~empty], o_ref[~empty]) <= 5e-3
        assert max_abs(lse_part[s][~empty], lse_ref[~empty]) <= BF16_LSE_ATOL
    if causal:
        # the case the check above must cover: rows with no key in a block
        assert np.isneginf(lse_part[-1]).any()


def test_more_blocks_than_key_tiles():
    B, H, Nq, Nk, d = 1, 2, 4, 300, 128  # 3 key tiles, 5 blocks: the last two are empty
    q, k, v = _qkv(B, H, Nq, Nk, d, 78)
    o_part, lse_part = fa.fwd_partial(q.cuda(), k.cuda(), v.cuda(), n_split=5)
    o, lse = fa.fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), n_split=5)
    _status_ok()
    assert torch.isneginf(lse_part[3:]).all() and (o_part[3:] == 0).all()
    o_ref, lse_ref = oracle.attention(q, k, v, False, d ** -0.5)
    assert max_abs(to_np(o), o_ref) <= BF16_O_ATOL and max_abs(to_np(lse), lse_ref) <= BF16_LSE_ATOL


@pytest.mark.parametrize("d", [64, 128, 256])
@pytest.mark.parametrize("n_part", [1, 2, 7, 40])
def test_merge_kernel_matches_oracle_merge(d, n_part):
    g = torch.Generator().manual_seed(d + n_part)
    rows = 333
    o_part = torch.randn(n_part, rows, d, generator=g) * 2.0
    lse_part = torch.randn(n_part, rows, generator=g) * 4.0 + 100.0
    lse_part[0, :50] = -math.inf  # blocks a row did not see
    if n_part > 1:
        lse_part[:, 50:60] = -math.inf  # rows that saw no key at all
        o_part[:, 50:60] = 0.0
    o, lse = fa.lse_merge(o_part.cuda(), lse_part.cuda())
    _status_ok()
    o_ref, lse_ref = oracle.lse_merge(o_part.double().numpy(), lse_part.double().numpy())
    got_o, got_l = to_np(o), to_np(lse)
    # one bf16 rounding of the merged value, plus fp32 arithmetic
    assert np.all(np.abs(got_o - o_ref) <= 2.0 ** -8 * np.abs(o_ref) + 1e-5)
    fin = np.isfinite(lse_ref)
    assert np.array_equal(np.isneginf(got_l), ~fin)
    assert max_abs(got_l[fin], lse_ref[fin]) <= 1e-4
    assert np.all(got_o[~fin] == 0.0)


def test_no_split_is_the_square_kernel_bitwise():
    # Nq = Nk and one block: the same kernel and arithmetic as fa_fwd.
    q, k, v = inputs.qkv_normal(2, 3, 700, 128, 79)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    for causal in (False, True):
        o1, l1 = fa.fwd(q, k, v, causal=causal, n_split=1)
        o2, l2 = fa.fwd_splitkv(q, k, v, causal=causal, n_split=1)
        _status_ok()
        assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_causal_single_query_sees_every_key():
    q, k, v = _qkv(2, 2, 1, 3000, 128, 80)
    q, k, v = q.cuda(), k.cuda(), v.cuda()
    oc, lc = fa.fwd_splitkv(q, k, v, causal=True, n_split=4)
    on, ln = fa.fwd_splitkv(q, k, v, causal=False, n_split=4)
    _status_ok()
    assert torch.equal(oc, on) and torch.equal(lc, ln)


def test_split_count_choice():
    # one CTA per SM: few heads and a long key sequence get several blocks, a
    # grid that already fills the GPU gets one
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert fa.splitkv_splits(1, 1, 1, 1 << 16, 128) > 1
    assert fa.splitkv_splits(4, sms, 1, 1 << 16, 128) == 1
    assert fa.splitkv_splits(1, 1, 1, 128, 128) == 1


@pytest.mark.parametrize("Nq,causal", [(1, False), (128, True)])
def test_decode_b4_h16_nk32768_d128_sampled_rows(Nq, causal):
    # The decode-shaped workload at its full size: B=4, H=16, Nk=32768, d=128.
    B, H, Nk, d = 4, 16, 32768, 128
    q, k, v = _qkv(B, H, Nq, Nk, d, 1005)
    o, lse = fa.fwd_splitkv(q.cuda(), k.cuda(), v.cuda(), causal=causal, n_split=0)
    _status_ok()
    rows = np.arange(B * H * Nq) if Nq == 1 else inputs.sample_rows(B, H, Nq, per_head=4, seed=Nq).numpy()
    o_ref, lse_ref = oracle.attention(q, k, v, causal, d ** -0.5, rows=rows)
    eo = max_abs(to_np(o).reshape(-1, d)[rows], o_ref)
    el = max_abs(to_np(lse).reshape(-1)[rows], lse_ref)
    record(f"bf16 decode B{B} H{H} Nq{Nq} Nk{Nk} d{d} {'causal' if causal else 'non-causal'}", o_max_abs=eo,
           lse_max_abs=el)
    assert eo <= BF16_O_ATOL and el <= BF16_LSE_ATOL, (eo, el)


def test_e4m3_decode_matches_oracle():
    B, H, Nq, Nk, d = 2, 4, 16, 3000, 128
    q, k, v = _qkv(B, H, Nq, Nk, d, 81)
    signs = inputs.hadamard_signs(d, 81).cuda()
    q8, dq = fa.hadamard_quant(q.cuda(), rotate=True, signs=signs)
    k8, dk = fa.hadamard_quant(k.cuda(), rotate=True, signs=signs)
    o, lse = fa.fwd_splitkv(q8, k8, v.cuda(), causal=True, qk_descale=torch.cat([dq, dk]), n_split=3)
    _status_ok()
    # against exact attention on the dequantised codes (what the kernel computes) ...
    qd = oracle.e4m3_decode(q8.cpu().numpy()) * float(dq.item())
    kd = oracle.e4m3_decode(k8.cpu().numpy()) * float(dk.item())
    o_ref, lse_ref = oracle.attention(qd, kd, v, True, d ** -0.5)
    assert max_abs(to_np(o), o_ref) <= BF16_O_ATOL and max_abs(to_np(lse), lse_ref) <= BF16_LSE_ATOL
    # ... and against exact attention on the unquantised inputs
    o_exact, _ = oracle.attention(q, k, v, True, d ** -0.5)
    assert rel_rmse(to_np(o), o_exact) <= FP8_REL_RMSE
