"""Ring attention: exact attention over a sequence split across ranks.

"Flash Attention" glossary page, fourth paragraph: ring attention spreads the
tiling of Flash Attention over several devices so that sequences longer than one
device's memory fit. (The page says "all-to-all"; a ring passes each key/value
chunk from rank to rank, point to point, which is what this module does.)

Each of the ``world`` ranks holds one contiguous chunk of the sequence: its
queries ``q`` and its keys and values ``k``, ``v``, all ``[B, H, L, d]``. Over
``world`` steps every rank sees every key/value chunk. At step s it holds the
chunk of rank ``(rank - s) mod world``, computes the attention of its queries
over that chunk alone, and passes the chunk on to rank ``rank + 1`` while
receiving the next from ``rank - 1``. The per-chunk results are partial results
in the sense of the same page's second paragraph: a normalised output and an LSE
per query row, combined at the end by their LSEs.

Causal masking over the whole sequence (key position <= query position) makes
the chunk of an earlier rank fully visible, the rank's own chunk causal within
itself, and a later rank's chunk invisible, so that block is skipped.

The per-chunk compute and the merge are the library's CUDA kernels
(``fwd_partial`` and ``lse_merge``) unless other callables are given; the
exchange uses ``torch.distributed`` point-to-point operations (NCCL on GPUs),
issued before the chunk's compute so that they overlap it.
"""
from __future__ import annotations

from typing import Callable, List, Optional, Tuple

import torch

FULL, DIAGONAL, SKIP = "full", "diagonal", "skip"


def ring_blocks(rank: int, world: int, causal: bool) -> List[Tuple[int, str]]:
    """(source chunk, kind) for each ring step of ``rank``: at step s the rank
    holds the key/value chunk of rank (rank - s) mod world; kind is FULL (every
    key visible), DIAGONAL (the rank's own chunk under a causal mask) or SKIP (a
    later chunk under a causal mask: no key visible)."""
    out = []
    for s in range(world):
        c = (rank - s) % world
        if not causal:
            out.append((c, FULL))
        elif c == rank:
            out.append((c, DIAGONAL))
        elif c < rank:
            out.append((c, FULL))
        else:
            out.append((c, SKIP))
    return out


def _default_partial(scale):
    from . import binding

    def run(q, k, v, causal):
        o, lse = binding.fwd_partial(q, k, v, causal=causal, scale=scale, n_split=1)
        return o[0], lse[0]

    return run


def _default_merge(o_parts, lse_parts):
    from . import binding

    return binding.lse_merge(o_parts, lse_parts)


def _run_blocks(q, blocks, chunk_at, partial_fn, merge_fn, step_done=None):
    """Shared by the distributed and the single-device rings: partial results of
    ``q`` over each block's chunk, then the merge. ``chunk_at(s)`` gives step s's
    key/value chunk (the distributed ring also posts the exchange of the next
    one there); ``step_done(s)``, if given, runs after step s's compute (the
    distributed ring waits for that exchange)."""
    B, H, L, d = q.shape
    n = len(blocks)
    o_parts = torch.zeros((n, B, H, L, d), dtype=torch.float32, device=q.device)
    lse_parts = torch.full((n, B, H, L), float("-inf"), dtype=torch.float32, device=q.device)
    for s, (c, kind) in enumerate(blocks):
        k_c, v_c = chunk_at(s)
        if kind != SKIP:
            o, lse = partial_fn(q, k_c, v_c, kind == DIAGONAL)
            o_parts[s].copy_(o)
            lse_parts[s].copy_(lse)
        if step_done is not None:
            step_done(s)
    return merge_fn(o_parts, lse_parts)


def ring_attention(q, k, v, causal: bool = False, scale: Optional[float] = None, group=None,
                   partial_fn: Optional[Callable] = None, merge_fn: Optional[Callable] = None):
    """Exact attention of this rank's queries over the keys of all ranks.

    q, k, v: this rank's chunk ``[B, H, L, d]`` of a sequence of ``world * L``
    positions, rank r holding positions ``r*L .. r*L + L - 1``. Returns
    ``(O, LSE)`` for this rank's queries (by default bf16 O and fp32 LSE from
    ``lse_merge``). Every rank must call it with the same shapes and ``causal``.
    ``partial_fn(q, k, v, causal) -> (O_fp32, LSE)`` and ``merge_fn(O_parts,
    LSE_parts)`` replace the CUDA kernels (the tests run the ring on CPU ranks
    with the CPU oracle in their place).
    """
    import torch.distributed as dist

    if partial_fn is None:
        partial_fn = _default_partial(scale)
    if merge_fn is None:
        merge_fn = _default_merge
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    blocks = ring_blocks(rank, world, causal)
    nxt, prv = (rank + 1) % world, (rank - 1) % world
    if group is not None:
        nxt, prv = dist.get_global_rank(group, nxt), dist.get_global_rank(group, prv)
    cur = torch.stack([k, v]).contiguous()  # one message per step: K and V of a chunk
    state = {"cur": cur}

    def chunk_at(s):
        cur = state["cur"]
        reqs = []
        if s + 1 < world:
            # pass the chunk on and take the next one, overlapping this step's compute
            nb = torch.empty_like(cur)
            ops = [dist.P2POp(dist.isend, cur, nxt, group), dist.P2POp(dist.irecv, nb, prv, group)]
            reqs = dist.batch_isend_irecv(ops)
            state["next"] = nb
        state["reqs"] = reqs
        return cur[0], cur[1]

    def step_done(s):
        for r in state["reqs"]:
            r.wait()
        if s + 1 < world:
            state["cur"] = state["next"]

    return _run_blocks(q, blocks, chunk_at, partial_fn, merge_fn, step_done)


def ring_attention_local(q_chunks, k_chunks, v_chunks, causal: bool = False, scale: Optional[float] = None,
                         partial_fn: Optional[Callable] = None, merge_fn: Optional[Callable] = None):
    """The ring's per-rank computation for every rank on one device, without the
    exchange: rank r's result from ``q_chunks[r]`` and the chunks in ring order.
    Returns a list of ``(O, LSE)``, one per rank."""
    if partial_fn is None:
        partial_fn = _default_partial(scale)
    if merge_fn is None:
        merge_fn = _default_merge
    world = len(q_chunks)
    out = []
    for r in range(world):
        blocks = ring_blocks(r, world, causal)
        out.append(_run_blocks(q_chunks[r], blocks, lambda s, b=blocks: (k_chunks[b[s][0]], v_chunks[b[s][0]]),
                               partial_fn, merge_fn))
    return out
