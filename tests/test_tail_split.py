"""GPU parity of the automatic schedule's tail split (fa_fwd_splitkv with
n_split = 0, the default of ``fwd``): without causal masking, when a
persistent launch's last round of query blocks is at most half full, each of
those blocks is computed as 2-4 pieces over disjoint key ranges, and the warp
that completes a block's group merges the pieces by their LSEs inside the
kernel. Checked against the fp64 oracle (whole heads and sampled rows), for 2,
3 and 4 pieces, d = 64, 128 and 256, ragged sizes, bf16 and e4m3 Q/K; and that
repeated launches give identical bits (the merge order does not depend on which
piece finishes last)."""
import numpy as np
import pytest
import torch

import oracle
import io_aware_exact_17_b200 as fa
from io_aware_exact_17_b200 import inputs
from helpers import BF16_LSE_ATOL, BF16_O_ATOL, max_abs, record, to_np

pytestmark = pytest.mark.gpu


def _status_ok():
    torch.cuda.synchronize()
    code, site, block = fa.device_status()
    assert code == 0, f"device wait ran out at site {site}, block {block}"


def _tail_pieces(B, H, N, d):
    """Pieces per tail block of the automatic schedule on this device (the rule
    that tests/test_abi.py restates; 0 when there is no tail split)."""
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    nq = 2 if (d <= 128 and N > 128) else 1
    units = B * H * -(-N // (128 * nq))
    tiles = -(-N // 128)
    tail = units % sms
    if units < sms or tail == 0 or 2 * tail > sms or tiles < 4:
        return 0
    ns = min(4, sms // tail, tiles)
    span = -(-tiles // ns)
    ns = -(-tiles // span)
    return ns if ns >= 2 else 0


# (B, H, N, d): 148 SMs give 4 pieces (152 blocks: 4 in the last round), 4 pieces
# of 2 tiles over a ragged last key tile (d = 64, 160 blocks), 3 pieces (d = 256,
# 156 one-tile blocks, 6 key tiles), 2 pieces (B=4, H=16, N=2048: 512 blocks)
CASES = [(1, 19, 2048, 128), (2, 20, 1000, 64), (2, 13, 700, 256)]


@pytest.mark.parametrize("B,H,N,d", CASES)
def test_tail_split_matches_oracle(B, H, N, d):
    ns = _tail_pieces(B, H, N, d)
    q, k, v = inputs.qkv_normal(B, H, N, d, 300 + N + d)
    o, lse = fa.fwd(q.cuda(), k.cuda(), v.cuda(), causal=False)
    _status_ok()
    # the last round's heads in full, the others on sampled rows
    BH = B * H
    nq = 2 if (d <= 128 and N > 128) else 1
    rows_per_head = -(-N // (128 * nq))
    first_tail_head = (BH * rows_per_head - (BH * rows_per_head) % torch.cuda.get_device_properties(
        0).multi_processor_count) // rows_per_head
    heads = sorted(set(range(max(0, first_tail_head), BH)) | {0})
    rows = np.concatenate([np.arange(h * N, (h + 1) * N) for h in heads])
    o_ref, lse_ref = oracle.attention(q, k, v, False, d ** -0.5, rows=rows)
    eo = max_abs(to_np(o).reshape(-1, d)[rows], o_ref)
    el = max_abs(to_np(lse).reshape(-1)[rows], lse_ref)
    record(f"bf16 tail split B{B} H{H} N{N} d{d} ({ns} pieces)", o_max_abs=eo, lse_max_abs=el)
    assert eo <= BF16_O_ATOL and el <= BF16_LSE_ATOL, (eo, el)


def test_tail_split_cases_take_the_split():
    # the cases above (and the B=4, H=16, N=2048 config) do exercise the split
    # on a 148-SM B200
    if torch.cuda.get_device_properties(0).multi_processor_count != 148:
        pytest.skip("piece counts stated for 148 SMs")
    assert [_tail_pieces(*c) for c in CASES] == [4, 4, 3]
    assert _tail_pieces(4, 16, 2048, 128) == 2


@pytest.mark.parametrize("B,H,N,d", CASES + [(4, 16, 2048, 128)])
def test_tail_split_is_deterministic_and_close_to_one_cta_per_block(B, H, N, d):
    q, k, v = (t.cuda() for t in inputs.qkv_normal(B, H, N, d, 310 + d))
    o1, l1 = fa.fwd(q, k, v)
    o2, l2 = fa.fwd(q, k, v)
    o3, l3 = fa.fwd(q, k, v)
    _status_ok()
    assert torch.equal(o1, o2) and torch.equal(o1, o3)
    assert torch.equal(l1, l2) and torch.equal(l1, l3)
    # against one CTA per query block over all keys (fa_fwd): the same sums in
    # another grouping, so within the rounding of the bf16 output and the fp32 LSE
    o0, l0 = fa.fwd(q, k, v, n_split=1)
    _status_ok()
    do = (o1.float() - o0.float()).abs()
    assert float(do.max()) <= 2 * 2.0 ** -8 * max(1.0, float(o0.float().abs().max()))
    assert float((l1 - l0).abs().max()) <= 2e-5 * max(1.0, float(l0.abs().max()))


@pytest.mark.parametrize("per_block", [False, True])
def test_tail_split_e4m3(per_block):
    # e4m3 Q and K (one scale per tensor, or per 128-row block: the pieces read
    # the key-block descales of their own key range) on the dequantised inputs
    B, H, N, d = 1, 19, 2048, 128
    q, k, v = inputs.qkv_normal(B, H, N, d, 320)
    sg = inputs.hadamard_signs(d, 320).cuda()
    if per_block:
        q8, dq = fa.hadamard_quant_blocks(q.cuda(), rotate=True, signs=sg)
        k8, dk = fa.hadamard_quant_blocks(k.cuda(), rotate=True, signs=sg)
        desc = (dq, dk)
        deq = lambda c, s: oracle.e4m3_decode(c.cpu().numpy()) * np.repeat(s.cpu().double().numpy(), 128,
                                                                           axis=2)[:, :, :N, None]
    else:
        q8, dq = fa.hadamard_quant(q.cuda(), rotate=True, signs=sg)
        k8, dk = fa.hadamard_quant(k.cuda(), rotate=True, signs=sg)
        desc = torch.cat([dq, dk])
        deq = lambda c, s: oracle.e4m3_decode(c.cpu().numpy()) * float(s.cpu().double())
    o, lse = fa.fwd(q8, k8, v.cuda(), causal=False, qk_descale=desc)
    _status_ok()
    heads = [0, 15, 16, 17, 18]  # the last round holds the last head's blocks
    rows = np.concatenate([np.arange(h * N, (h + 1) * N) for h in heads])
    o_ref, lse_ref = oracle.attention(deq(q8, dq), deq(k8, dk), v, False, d ** -0.5, rows=rows)
    assert max_abs(to_np(o).reshape(-1, d)[rows], o_ref) <= BF16_O_ATOL
    assert max_abs(to_np(lse).reshape(-1)[rows], lse_ref) <= BF16_LSE_ATOL


def test_tail_split_in_a_replayed_cuda_graph():
    # a captured launch replays with the parameters it was captured with (the
    # same ticket tag every time): each replay must still merge every group
    B, H, N, d = 1, 19, 2048, 128
    q, k, v = (t.cuda() for t in inputs.qkv_normal(B, H, N, d, 330))
    o_ref, l_ref = fa.fwd(q, k, v)
    _status_ok()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    o = torch.empty_like(o_ref)
    lse = torch.empty_like(l_ref)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        fa.fwd(q, k, v, out=o, lse=lse)  # the stream's workspace exists before the capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            fa.fwd(q, k, v, out=o, lse=lse)
    torch.cuda.current_stream().wait_stream(s)
    for _ in range(4):
        o.zero_()
        lse.zero_()
        g.replay()
        _status_ok()
        assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    del g
