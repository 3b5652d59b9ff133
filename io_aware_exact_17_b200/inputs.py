"""Seeded synthetic inputs shared by the tests, the smoke check and the benchmark.

This module draws random numbers and nothing else: it holds none of the
attention or quantisation arithmetic, so both the CUDA path and the CPU oracle
can be fed from it without sharing any of the method.

Recipe (all on the CPU, ``torch.Generator`` seeded, then moved as needed):

* Q, K, V: fp32 standard normal, drawn in that order from one generator, cast to
  bf16 (round to nearest even). Layout ``[B, H, N, d]``.
* Decode-shaped problems (few queries, long keys): Q ``[B, H, Nq, d]`` then K and
  V ``[B, H, Nk, d]``, fp32 standard normal drawn in that order from one
  generator, cast to bf16.
* Outliers, reading R1 (default): per head one feature channel, chosen from the
  seed, multiplied by 20 in both Q and K for every token (0.1% of 128 channels
  rounds up to one channel per head).
* Outliers, reading R2: each element of Q and K independently multiplied by 20
  with probability 0.001.
* Output gradients dO for the backward pass: fp32 standard normal from a
  generator seeded with the given seed, cast to bf16, layout ``[B, H, N, d]``.
* Hadamard signs: d independent fair +-1 draws (the random diagonal of the
  rotation); ``None`` means no sign flips.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import torch

OUTLIER_FACTOR = 20.0
OUTLIER_FRACTION = 0.001


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def qkv_normal(B: int, H: int, N: int, d: int, seed: int, dtype=torch.bfloat16):
    """Q, K, V ~ N(0, 1) i.i.d., drawn in that order, returned as CPU tensors."""
    g = _gen(seed)
    shape = (B, H, N, d)
    q = torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)
    k = torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)
    v = torch.randn(shape, generator=g, dtype=torch.float32).to(dtype)
    return q, k, v


def qkv_decode(B: int, H: int, Nq: int, Nk: int, d: int, seed: int, dtype=torch.bfloat16):
    """Q ``[B, H, Nq, d]``, then K and V ``[B, H, Nk, d]``, all N(0, 1) i.i.d.,
    drawn in that order; CPU tensors."""
    g = _gen(seed)
    q = torch.randn((B, H, Nq, d), generator=g, dtype=torch.float32).to(dtype)
    k = torch.randn((B, H, Nk, d), generator=g, dtype=torch.float32).to(dtype)
    v = torch.randn((B, H, Nk, d), generator=g, dtype=torch.float32).to(dtype)
    return q, k, v


def grad_out(B: int, H: int, N: int, d: int, seed: int, dtype=torch.bfloat16) -> torch.Tensor:
    """dLoss/dO for the backward pass: standard normal, cast to ``dtype``."""
    g = _gen(seed)
    return torch.randn((B, H, N, d), generator=g, dtype=torch.float32).to(dtype)


def outlier_channels(H: int, d: int, seed: int) -> torch.Tensor:
    """Reading R1: ``[H, c]`` channel indices, c = max(1, round(0.001*d))."""
    c = max(1, round(OUTLIER_FRACTION * d))
    g = _gen(seed + 7919)
    return torch.stack([torch.randperm(d, generator=g)[:c] for _ in range(H)])


def with_outliers_r1(q: torch.Tensor, k: torch.Tensor, seed: int):
    """Copies of q, k with each head's R1 channels scaled by 20 (same channels in q and k)."""
    B, H, N, d = q.shape
    ch = outlier_channels(H, d, seed)
    mult = torch.ones(H, d, dtype=torch.float32)
    for h in range(H):
        mult[h, ch[h]] = OUTLIER_FACTOR
    mult = mult.view(1, H, 1, d)
    return (q.float() * mult).to(q.dtype), (k.float() * mult).to(k.dtype)


def with_outliers_r2(q: torch.Tensor, k: torch.Tensor, seed: int):
    """Copies of q, k with i.i.d. Bernoulli(0.001) elements scaled by 20, independently in q and k."""
    g = _gen(seed + 104729)
    mq = torch.rand(q.shape, generator=g) < OUTLIER_FRACTION
    mk = torch.rand(k.shape, generator=g) < OUTLIER_FRACTION
    fq = torch.where(mq, OUTLIER_FACTOR, 1.0)
    fk = torch.where(mk, OUTLIER_FACTOR, 1.0)
    return (q.float() * fq).to(q.dtype), (k.float() * fk).to(k.dtype)


def hadamard_signs(d: int, seed: int) -> torch.Tensor:
    """d fair +-1 draws as fp32."""
    g = _gen(seed + 31337)
    return torch.randint(0, 2, (d,), generator=g).float() * 2.0 - 1.0


def sample_rows(B: int, H: int, N: int, per_head: int, seed: int, tile: int = 128) -> torch.Tensor:
    """Flat row ids ``(b*H + h)*N + i`` to check at sizes where the oracle cannot do
    every row: ``per_head`` seeded rows per (b, h) plus rows 0, N-1 and both sides
    of every ``tile`` boundary."""
    g = _gen(seed + 4242)
    fixed = {0, N - 1}
    for t in range(tile, N, tile):
        fixed.update((t - 1, t))
    fixed = sorted(i for i in fixed if 0 <= i < N)
    out = []
    for bh in range(B * H):
        pick = torch.randint(0, N, (per_head,), generator=g).tolist()
        rows = sorted(set(pick) | set(fixed))
        out.extend(bh * N + i for i in rows)
    return torch.tensor(out, dtype=torch.int64)


@dataclass(frozen=True)
class Workload:
    """One attention problem: sizes, mask mode and the seed of its inputs."""

    name: str
    B: int
    H: int
    N: int
    d: int
    causal: bool
    seed: int
    fp8: bool = False

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def flops(self) -> float:
        """4*B*H*N^2*d, halved when causal (the usual attention FLOP count)."""
        f = 4.0 * self.B * self.H * self.N * self.N * self.d
        return f / 2 if self.causal else f


def workloads():
    """The five workload families, seeds 1000 + family index. (The decode-shaped
    problems, family 5, are not square and use :func:`qkv_decode`.)"""
    w = []
    for causal in (False, True):
        w.append(Workload(f"tiny_b1h2n128d64_{'c' if causal else 'nc'}", 1, 2, 128, 64, causal, 1000))
        w.append(Workload(f"b4h16n2048d128_{'c' if causal else 'nc'}", 4, 16, 2048, 128, causal, 1001))
        for n in (512, 1024, 2048, 4096, 8192, 16384):
            w.append(Workload(f"sweep_b{16384 // n}h16n{n}d128_{'c' if causal else 'nc'}", 16384 // n, 16, n,
                              128, causal, 1002))
    w.append(Workload("fp8_b2h16n8192d128_nc", 2, 16, 8192, 128, False, 1003, fp8=True))
    for d in (64, 128, 256):
        w.append(Workload(f"dsweep_b2h{2048 // d}n4096d{d}_c", 2, 2048 // d, 4096, d, True, 1004))
    return w
