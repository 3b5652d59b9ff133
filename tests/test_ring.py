"""Ring attention (io_aware_exact_17_b200.ring).

On CPU: the block schedule, and the whole ring over 2 and 3 gloo ranks (real
point-to-point exchange) with the fp64 oracle as the per-chunk compute and merge,
against the oracle's attention over the full sequence. On the GPU (one device):
the same per-rank computation for 4 emulated ranks through the CUDA kernels
(fa_fwd_partial per chunk, fa_lse_merge), against the oracle.
"""
import os
import socket
import sys
from pathlib import Path

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parents[1]
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))

import oracle  # noqa: E402
from io_aware_exact_17_b200 import inputs  # noqa: E402
from io_aware_exact_17_b200.ring import DIAGONAL, FULL, SKIP, ring_blocks  # noqa: E402


def test_ring_blocks_cover_every_chunk_once():
    for world in (1, 2, 3, 5):
        for rank in range(world):
            for causal in (False, True):
                b = ring_blocks(rank, world, causal)
                assert sorted(c for c, _ in b) == list(range(world))
                assert b[0] == (rank, DIAGONAL if causal else FULL)
                for c, kind in b:
                    want = FULL if (not causal or c < rank) else (DIAGONAL if c == rank else SKIP)
                    assert kind == want


def _oracle_partial(scale):
    def run(q, k, v, causal):
        o, lse = oracle.attention(q.double().numpy(), k.double().numpy(), v.double().numpy(), causal, scale)
        return torch.from_numpy(o), torch.from_numpy(lse)

    return run


def _oracle_merge(o_parts, lse_parts):
    o, lse = oracle.lse_merge(o_parts.double().numpy(), lse_parts.double().numpy())
    return torch.from_numpy(o), torch.from_numpy(lse)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


SHAPE = (1, 2, 24, 16)  # B, H, L (positions per rank), d


def _rank_main(rank, world, port, causal, q_out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    sys.path.insert(0, str(ROOT))
    import datetime

    import torch.distributed as dist

    from io_aware_exact_17_b200.ring import ring_attention

    dist.init_process_group("gloo", timeout=datetime.timedelta(seconds=60))
    B, H, L, d = SHAPE
    q, k, v = inputs.qkv_normal(B, H, world * L, d, 77)
    sl = slice(rank * L, (rank + 1) * L)
    scale = d ** -0.5
    o, lse = ring_attention(q[:, :, sl].float(), k[:, :, sl].float(), v[:, :, sl].float(), causal=causal,
                            partial_fn=_oracle_partial(scale), merge_fn=_oracle_merge)
    dist.barrier()
    dist.destroy_process_group()
    q_out.put((rank, o.numpy(), lse.numpy()))


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("causal", [False, True])
def test_ring_over_gloo_ranks_matches_full_attention(world, causal):
    ctx = mp.get_context("spawn")
    q_out = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, causal, q_out)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    for _ in range(world):
        r, o, lse = q_out.get(timeout=180)
        results[r] = (o, lse)
    for p in procs:
        p.join(timeout=60)
        if p.is_alive():
            p.kill()
            pytest.fail("a rank did not finish")
        assert p.exitcode == 0
    B, H, L, d = SHAPE
    q, k, v = inputs.qkv_normal(B, H, world * L, d, 77)
    o_ref, lse_ref = oracle.attention(q, k, v, causal, d ** -0.5)
    for r in range(world):
        o, lse = results[r]
        sl = slice(r * L, (r + 1) * L)
        # partial outputs are kept in fp32 between the steps
        np.testing.assert_allclose(o, o_ref[:, :, sl], rtol=0, atol=1e-5)
        np.testing.assert_allclose(lse, lse_ref[:, :, sl], rtol=0, atol=1e-5)


@pytest.mark.gpu
@pytest.mark.parametrize("causal", [False, True])
def test_ring_emulated_ranks_on_one_gpu(causal):
    import io_aware_exact_17_b200 as fa
    from io_aware_exact_17_b200.ring import ring_attention_local
    from helpers import BF16_LSE_ATOL, BF16_O_ATOL, max_abs, to_np

    world, B, H, L, d = 4, 1, 4, 384, 128
    q, k, v = inputs.qkv_normal(B, H, world * L, d, 78)
    chunks = [tuple(t[:, :, r * L:(r + 1) * L].contiguous().cuda() for t in (q, k, v)) for r in range(world)]
    res = ring_attention_local([c[0] for c in chunks], [c[1] for c in chunks], [c[2] for c in chunks], causal=causal)
    torch.cuda.synchronize()
    code, site, block = fa.device_status()
    assert code == 0, (site, block)
    o_ref, lse_ref = oracle.attention(q, k, v, causal, d ** -0.5)
    for r, (o, lse) in enumerate(res):
        sl = slice(r * L, (r + 1) * L)
        assert max_abs(to_np(o), o_ref[:, :, sl]) <= BF16_O_ATOL
        assert max_abs(to_np(lse), lse_ref[:, :, sl]) <= BF16_LSE_ATOL
