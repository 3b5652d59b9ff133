"""Benchmark of the fused attention forward on B200.

One step = one pass of the whole hot path over one batch of synthetic input of
the B=4, H=16, N=2048, d=128 workload (Q, K, V ~ N(0,1) bf16, scale 1/sqrt(128)):
  1. BF16 forward, non-causal;   2. BF16 forward, causal;
  3. Hadamard rotate + e4m3 quantise of Q and K (one launch, a scale each);   4. e4m3-QK forward, non-causal.
Metric: attention TFLOPS = sum of 4*B*H*N^2*d (halved when causal) over the
three forward passes / step time. L2 (126 MB) is flushed between steps by
writing a 512 MB buffer outside the timed events, since the inputs (100 MB)
would otherwise stay resident.

``--impl reference`` times the CPU oracle instead (rank 0 only), on a bounded
row sample of the same workload per step.

``--workload decode`` measures the decode-shaped problem instead: B=4, H=16
single-query heads (Nq=1) over Nk=32768 keys, d=128, bf16: one step is the
split-key attention kernel (fp32 partial results per block of keys) and the LSE
merge. It is HBM-bound (the 1.07 GB of K and V are read once per step), so its
metric is GB/s of algorithmic traffic.

``--workload bwd`` measures the backward pass on the B=4, H=16, N=2048, d=128
workload: one step is fa_bwd non-causal then fa_bwd causal (each a prologue, the
tcgen05 kernel and the dQ conversion), given O and LSE from the library's
forward (computed once, outside the timed region). Metric: backward TFLOPS =
10*B*H*N^2*d (the five N x N x d products; halved when causal) / step time.

Launch: ``python bench.py --gpus N --steps K --warmup W`` (N > 1 under
torch.distributed.run, one rank per GPU, each rank its own batch: weak scaling,
no collective on the data path).
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

ROOT = Path(__file__).resolve().parent
if str(ROOT) not in sys.path:
    sys.path.insert(0, str(ROOT))

import torch  # noqa: E402

from io_aware_exact_17_b200 import inputs as fa_inputs  # noqa: E402

METRIC = "attention fwd TFLOPS (4·B·H·N²·d, ½ if causal) and % of B200 BF16/FP8 peak"
DECODE = {"B": 4, "H": 16, "Nq": 1, "Nk": 32768, "d": 128, "seed": 1005}
DECODE_METRIC = "decode attention GB/s (algorithmic HBM bytes: K, V, Q read; O, LSE written)"
BWD_METRIC = "attention bwd TFLOPS (10·B·H·N²·d, ½ if causal) and % of B200 BF16 peak"
B, H, N, D = 4, 16, 2048, 128
SEED = 1001
WORKLOAD = f"b{B}h{H}n{N}d{D}: bf16 fwd non-causal + bf16 fwd causal + rotate/quantise Q,K + e4m3-QK fwd non-causal"
PEAKS_FALLBACK = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of the
# bf16 non-causal attention kernel on this workload, from one ncu capture, and
# the SHA-256 of the kernel's sources at that capture. When the sources differ
# the figure no longer describes the kernel and `traffic` is reported as null.
KERNEL_SOURCES = ("io_aware_exact_17_b200/csrc/attn_fwd.cuh", "io_aware_exact_17_b200/csrc/sm100.cuh")
NCU_TRAFFIC_BYTES = 109134336  # 100.744192 MB read + 8.390144 MB written
NCU_TRAFFIC_SHA256 = "1cd88edb5ead5007262af6e353d6d14f4f7c22db05befff7ab8ab3ffc1717029"


def kernel_sources_sha256() -> str:
    import hashlib

    h = hashlib.sha256()
    for rel in KERNEL_SOURCES:
        h.update((ROOT / rel).read_bytes())
    return h.hexdigest()


def measured_traffic():
    if NCU_TRAFFIC_BYTES is None or NCU_TRAFFIC_SHA256 != kernel_sources_sha256():
        return None
    return NCU_TRAFFIC_BYTES


def flops_fwd(causal: bool) -> float:
    f = 4.0 * B * H * N * N * D
    return f / 2 if causal else f


STEP_FLOPS = flops_fwd(False) + flops_fwd(True) + flops_fwd(False)


def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        try:
            d = json.loads(p.read_text())
            return {k: float(d[k]) for k in PEAKS_FALLBACK}, "measured"
        except Exception:
            pass
    return dict(PEAKS_FALLBACK), "fallback"


# ------------------------------------------------------------- distributed --
def dist_setup():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist

        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return world, rank, local


def dist_max(x: float, world: int) -> float:
    """Max of a per-rank value over all ranks (identity for one rank)."""
    if world <= 1:
        return x
    import torch.distributed as dist

    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dist_barrier(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.barrier()


def dist_done(world: int):
    if world > 1:
        import torch.distributed as dist

        dist.destroy_process_group()


# ------------------------------------------------------------------ clocks --
class ClockSampler:
    """SM clocks and throttle reasons sampled while the timed region runs: NVML
    every 5 ms from a thread (a timed region can be a few tens of ms), else
    nvidia-smi every 200 ms. Reads only; changes no setting."""

    REASON_BITS = {"sw_power_cap": 0x4, "hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20,
                   "hw_thermal_slowdown": 0x40}
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        # nvidia-smi and NVML number GPUs physically; address ours by UUID instead.
        try:
            uuid = str(torch.cuda.get_device_properties(gpu_index).uuid)
            self.gpu = uuid if uuid.startswith("GPU-") else "GPU-" + uuid
        except Exception:
            self.gpu = str(gpu_index)
        self.proc = None
        self.thread = None
        self.samples = []  # (sm_mhz, max_mhz, reasons bitmask)
        self.lines = []

    def _nvml_loop(self, handle, nv):
        import time as _t

        while not self.stop:
            try:
                sm = nv.nvmlDeviceGetClockInfo(handle, nv.NVML_CLOCK_SM)
                mx = nv.nvmlDeviceGetMaxClockInfo(handle, nv.NVML_CLOCK_SM)
                rs = nv.nvmlDeviceGetCurrentClocksEventReasons(handle)
                self.samples.append((float(sm), float(mx), int(rs)))
            except Exception:
                pass
            _t.sleep(0.005)

    def __enter__(self):
        self.stop = False
        try:
            import threading

            import pynvml as nv

            nv.nvmlInit()
            try:
                handle = nv.nvmlDeviceGetHandleByUUID(self.gpu)
            except Exception:
                handle = nv.nvmlDeviceGetHandleByUUID(self.gpu.encode())
            self.thread = threading.Thread(target=self._nvml_loop, args=(handle, nv), daemon=True)
            self.thread.start()
            return self
        except Exception:
            self.thread = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        self.stop = True
        if self.thread is not None:
            self.thread.join(timeout=2)
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except Exception:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [ln for ln in out.splitlines() if ln.strip()]
        return False

    def summary(self):
        sm, smax, reasons = [], None, set()
        for mhz, mx, bits in self.samples:
            sm.append(mhz)
            smax = mx
            reasons.update(nm for nm, b in self.REASON_BITS.items() if bits & b)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                smax = float(parts[2])
            except ValueError:
                continue
            for nm, val in zip(names, parts[5:9]):
                if val.lower() == "active":
                    reasons.add(nm)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(sm),
                "source": "nvml 5 ms" if self.samples else ("nvidia-smi 200 ms" if self.lines else None)}


# --------------------------------------------------------------- GPU step --
class Step:
    """All buffers of one step, allocated once; run() enqueues the step's kernels
    on the current stream, bracketing each kernel group with CUDA events."""

    def __init__(self, seed: int):
        import io_aware_exact_17_b200 as fa

        self.fa = fa
        q, k, v = fa_inputs.qkv_normal(B, H, N, D, seed)
        self.signs = fa_inputs.hadamard_signs(D, seed).cuda()
        self.q_h, self.k_h, self.v_h = (t.pin_memory() for t in (q, k, v))
        shp = (B, H, N, D)
        # two sets of device inputs and outputs, so that pipelined end-to-end steps
        # can copy one set while computing on the other (the timed device-only
        # steps use set 0)
        self.bufs = []
        for _ in range(2):
            self.bufs.append({
                "q": q.cuda(), "k": k.cuda(), "v": v.cuda(),
                "o": [torch.empty(shp, dtype=torch.bfloat16, device="cuda") for _ in range(3)],
                "lse": [torch.empty((B, H, N), dtype=torch.float32, device="cuda") for _ in range(3)],
            })
        self.q, self.k, self.v = self.bufs[0]["q"], self.bufs[0]["k"], self.bufs[0]["v"]
        self.o, self.lse = self.bufs[0]["o"], self.bufs[0]["lse"]
        self.q8 = torch.empty(shp, dtype=torch.uint8, device="cuda")
        self.k8 = torch.empty(shp, dtype=torch.uint8, device="cuda")
        self.desc = torch.empty(2, dtype=torch.float32, device="cuda")
        self.o_h = [torch.empty(shp, dtype=torch.bfloat16).pin_memory() for _ in range(3)]
        self.lse_h = [torch.empty((B, H, N), dtype=torch.float32).pin_memory() for _ in range(3)]
        self.flush_buf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        self.launches_per_step = 4  # 3 attention kernels + 1 quantisation of Q and K
        self.groups = 4  # breakdown: bf16 nc, bf16 causal, quantise Q+K, e4m3 nc

    def flush_l2(self):
        self.flush_buf.zero_()

    def run(self, ev=None, b=0):
        fa = self.fa
        q, k, v, o, lse = (self.bufs[b][n] for n in ("q", "k", "v", "o", "lse"))
        if ev is not None:
            ev[0].record()
        fa.fwd(q, k, v, causal=False, out=o[0], lse=lse[0])
        if ev is not None:
            ev[1].record()
        fa.fwd(q, k, v, causal=True, out=o[1], lse=lse[1])
        if ev is not None:
            ev[2].record()
        fa.hadamard_quant_multi([q, k], rotate=True, signs=self.signs, outs=[self.q8, self.k8], descales=self.desc)
        if ev is not None:
            ev[3].record()
        fa.fwd(self.q8, self.k8, v, causal=False, qk_descale=self.desc, out=o[2], lse=lse[2])
        if ev is not None:
            ev[4].record()

    # End to end, through the same public calls with host buffers: pinned
    # host -> device copies of Q, K, V, the step, device -> host copies of every
    # O and LSE, each part on the current stream, for buffer set b.
    def h2d(self, b):
        for n, h in (("q", self.q_h), ("k", self.k_h), ("v", self.v_h)):
            self.bufs[b][n].copy_(h, non_blocking=True)

    def compute(self, b):
        self.run(b=b)

    def d2h(self, b):
        for i in range(3):
            self.o_h[i].copy_(self.bufs[b]["o"][i], non_blocking=True)
            self.lse_h[i].copy_(self.bufs[b]["lse"][i], non_blocking=True)

    @property
    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in (self.q_h, self.k_h, self.v_h))

    @property
    def d2h_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.o_h + self.lse_h)


class DecodeStep:
    """The decode-shaped problem: fp32 partial results per block of keys
    (fwd_partial) then the LSE merge (lse_merge), the two kernels fwd_splitkv
    runs, called separately so each is timed. The K/V cache stays on the device
    between steps, as a decode step's cache does."""

    def __init__(self, seed: int):
        import io_aware_exact_17_b200 as fa

        self.fa = fa
        c = DECODE
        self.B, self.H, self.Nq, self.Nk, self.d = c["B"], c["H"], c["Nq"], c["Nk"], c["d"]
        q, k, v = fa_inputs.qkv_decode(self.B, self.H, self.Nq, self.Nk, self.d, seed)
        self.q_h = q.pin_memory()
        self.q, self.k, self.v = (t.cuda() for t in (q, k, v))
        self.qs = [self.q, q.cuda()]  # two query buffers for pipelined end-to-end steps
        self.n_split = fa.splitkv_splits(self.B, self.H, self.Nq, self.Nk, self.d)
        rows = (self.B, self.H, self.Nq)
        self.o_part = torch.empty((self.n_split, *rows, self.d), dtype=torch.float32, device="cuda")
        self.lse_part = torch.empty((self.n_split, *rows), dtype=torch.float32, device="cuda")
        self.o = torch.empty((*rows, self.d), dtype=torch.bfloat16, device="cuda")
        self.lse = torch.empty(rows, dtype=torch.float32, device="cuda")
        self.o_h = torch.empty((*rows, self.d), dtype=torch.bfloat16).pin_memory()
        self.lse_h = torch.empty(rows, dtype=torch.float32).pin_memory()
        self.flush_buf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        self.launches_per_step = 2
        self.groups = 2  # breakdown: split-key attention, merge
        n = self.B * self.H
        # algorithmic bytes: K, V (bf16) and Q read; O (bf16) and LSE written
        self.kv_bytes = 2.0 * n * self.Nk * self.d * 2
        self.bytes = self.kv_bytes + n * self.Nq * self.d * 2 * 2 + n * self.Nq * 4
        self.part_bytes = self.o_part.numel() * 4 + self.lse_part.numel() * 4

    def flush_l2(self):
        self.flush_buf.zero_()

    def run(self, ev=None):
        fa = self.fa
        if ev is not None:
            ev[0].record()
        fa.fwd_partial(self.q, self.k, self.v, n_split=self.n_split, o_part=self.o_part, lse_part=self.lse_part)
        if ev is not None:
            ev[1].record()
        fa.lse_merge(self.o_part, self.lse_part, out=self.o, lse=self.lse)
        if ev is not None:
            ev[2].record()

    # End to end: Q copied in from pinned host memory, the step, O and LSE
    # copied out (the K/V cache stays on the device).
    def h2d(self, b):
        self.qs[b].copy_(self.q_h, non_blocking=True)

    def compute(self, b):
        fa = self.fa
        fa.fwd_partial(self.qs[b], self.k, self.v, n_split=self.n_split, o_part=self.o_part, lse_part=self.lse_part)
        fa.lse_merge(self.o_part, self.lse_part, out=self.o, lse=self.lse)

    def d2h(self, b):
        self.o_h.copy_(self.o, non_blocking=True)
        self.lse_h.copy_(self.lse, non_blocking=True)

    @property
    def h2d_bytes(self):
        return self.q_h.numel() * self.q_h.element_size()

    @property
    def d2h_bytes(self):
        return self.o_h.numel() * 2 + self.lse_h.numel() * 4


class BwdStep:
    """The backward pass: fa_bwd non-causal, then fa_bwd causal, over the same
    Q, K, V and dO, each with the O and LSE the library's forward returned for
    that mask (computed once at set-up)."""

    def __init__(self, seed: int):
        import io_aware_exact_17_b200 as fa

        self.fa = fa
        q, k, v = fa_inputs.qkv_normal(B, H, N, D, seed)
        do = fa_inputs.grad_out(B, H, N, D, seed + 500)
        dev = [t.cuda() for t in (q, k, v, do)]
        fwd = [fa.fwd(dev[0], dev[1], dev[2], causal=c) for c in (False, True)]
        torch.cuda.synchronize()
        # host copies of every input, pinned, for the end-to-end steps
        self.host_in = [t.pin_memory() for t in (q, k, v, do)]
        for o, lse in fwd:
            self.host_in += [o.cpu().pin_memory(), lse.cpu().pin_memory()]
        # two device sets of the inputs (q, k, v, do, o_nc, lse_nc, o_c, lse_c) and workspaces
        self.sets = [[t.to("cuda", non_blocking=False).clone() for t in self.host_in] for _ in range(2)]
        nbytes = fa.bwd_workspace_bytes(B, H, N, D)
        self.ws = [torch.empty(nbytes, dtype=torch.uint8, device="cuda") for _ in range(2)]
        self.out = [None, None]
        self.host_out = [torch.empty((B, H, N, D), dtype=torch.bfloat16).pin_memory() for _ in range(6)]
        self.flush_buf = torch.empty(512 * 1024 * 1024, dtype=torch.uint8, device="cuda")
        self.launches_per_step = 6
        self.groups = 2  # breakdown: bwd non-causal, bwd causal

    def flush_l2(self):
        self.flush_buf.zero_()

    def _bwd(self, b, causal):
        q, k, v, do, o_nc, lse_nc, o_c, lse_c = self.sets[b]
        o, lse = (o_c, lse_c) if causal else (o_nc, lse_nc)
        return self.fa.bwd(q, k, v, o, lse, do, causal=causal, workspace=self.ws[b])

    def run(self, ev=None):
        if ev is not None:
            ev[0].record()
        self.out[0] = self._bwd(0, False)
        if ev is not None:
            ev[1].record()
        self.out[1] = self._bwd(0, True)
        if ev is not None:
            ev[2].record()

    def h2d(self, b):
        for dst, src in zip(self.sets[b], self.host_in):
            dst.copy_(src, non_blocking=True)

    def compute(self, b):
        self.out[b] = self._bwd(b, False) + self._bwd(b, True)

    def d2h(self, b):
        for dst, src in zip(self.host_out, self.out[b]):
            dst.copy_(src, non_blocking=True)

    @property
    def h2d_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.host_in)

    @property
    def d2h_bytes(self):
        return sum(t.numel() * t.element_size() for t in self.host_out)


def flops_bwd(causal: bool) -> float:
    """The five N x N x d products of the backward pass (S, dP, dV, dK, dQ)."""
    return 10.0 * B * H * N * N * D * (0.5 if causal else 1.0)


def capture_step(step):
    """The step's kernels captured once as a CUDA graph, so a timed step carries
    no host launch overhead (the quantiser kernels are ~10 us each)."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        step.run()  # every lazy set-up (attributes, occupancy) done before capture
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            step.run()
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    return g


def time_steps(step, graph, steps: int, warmup: int, world: int):
    """K timed steps (graph replays, L2 flushed between them outside the events),
    then K eager steps with events around each kernel group for the breakdown."""
    for _ in range(warmup):
        step.flush_l2()
        graph.replay()
    torch.cuda.synchronize()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    dist_barrier(world)
    torch.cuda.synchronize()
    for i in range(steps):
        step.flush_l2()
        ev[i][0].record()
        graph.replay()
        ev[i][1].record()
    torch.cuda.synchronize()
    dist_barrier(world)
    step_ms = [a.elapsed_time(b) for a, b in ev]
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(step.groups + 1)] for _ in range(steps)]
    for i in range(steps):
        step.flush_l2()
        step.run(evs[i])
    torch.cuda.synchronize()
    per = [[evs[i][j].elapsed_time(evs[i][j + 1]) for j in range(step.groups)] for i in range(steps)]
    return step_ms, per  # per: ms of each kernel group per eager step


def time_e2e(step, steps: int, warmup: int, world: int):
    """End-to-end steps, pipelined as a serving loop would run them: three CUDA
    streams (host -> device copies, compute, device -> host copies) and two
    sets of device buffers, so that step i+1's inputs travel in and step i-1's
    results travel out while step i computes. Every step still copies all of its
    inputs in and all of its results out. Returns ms per step over the timed
    steps (events on the current stream, which waits for all three)."""
    s_in, s_c, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev_in = [torch.cuda.Event() for _ in range(2)]
    ev_c = [torch.cuda.Event() for _ in range(2)]
    ev_out = [torch.cuda.Event() for _ in range(2)]

    def one(i):
        b = i % 2
        with torch.cuda.stream(s_in):
            if i >= 2:
                s_in.wait_event(ev_c[b])  # step i-2 has finished reading set b's inputs
            step.h2d(b)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_c):
            s_c.wait_event(ev_in[b])
            if i >= 2:
                s_c.wait_event(ev_out[b])  # step i-2's results in set b are copied out
            step.compute(b)
            ev_c[b].record(s_c)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_c[b])
            step.d2h(b)
            ev_out[b].record(s_out)

    for i in range(warmup):
        one(i)
    torch.cuda.synchronize()
    dist_barrier(world)
    step.flush_l2()
    torch.cuda.synchronize()
    cur = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(cur)
    for s in (s_in, s_c, s_out):
        s.wait_stream(cur)
    for i in range(steps):
        one(i)
    for s in (s_in, s_c, s_out):
        cur.wait_stream(s)
    e1.record(cur)
    e1.synchronize()
    dist_barrier(world)
    return e0.elapsed_time(e1) / steps


# ------------------------------------------------------------ CPU oracle --
def oracle_sample(target_s: float, seed: int):
    """Time the oracle (as it stands) on a row sample of the three attention
    passes of the step, sized for about ``target_s`` seconds. Returns
    (flops, seconds, threads, rows_per_pass)."""
    import numpy as np

    import oracle

    q, k, v = fa_inputs.qkv_normal(B, H, N, D, seed)
    qd, kd, vd = (t.double().numpy() for t in (q, k, v))
    threads = oracle.default_threads()
    rng = np.random.default_rng(seed)

    def run(rows_n):
        rows = rng.integers(0, B * H * N, rows_n)
        fl = 0.0
        t0 = time.perf_counter()
        for causal in (False, True, False):
            oracle.attention(qd, kd, vd, causal, D ** -0.5, rows=rows, threads=threads)
            i = rows % N
            fl += float(np.sum(4.0 * D * (i + 1))) if causal else 4.0 * N * D * rows_n
        return fl, time.perf_counter() - t0

    probe_rows = max(threads * 4, 64)
    fl, dt = run(probe_rows)
    rows_n = int(min(B * H * N, max(probe_rows, probe_rows * target_s / max(dt, 1e-3))))
    fl, dt = run(rows_n)
    return fl, dt, threads, rows_n


def oracle_bwd_sample(target_s: float, seed: int):
    """Time the backward oracle (as it stands) on whole heads of the workload,
    non-causal and causal alternately, for about ``target_s`` seconds.
    Returns (flops, seconds, threads, heads)."""
    import oracle

    q, k, v = fa_inputs.qkv_normal(B, H, N, D, seed)
    do = fa_inputs.grad_out(B, H, N, D, seed + 500)
    fl, heads = 0.0, 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < target_s or heads < 2:
        b, h = divmod(heads % (B * H), H)
        causal = heads % 2 == 1
        sl = (slice(b, b + 1), slice(h, h + 1))
        oracle.attention_bwd(q[sl], k[sl], v[sl], do[sl], causal, D ** -0.5)
        fl += flops_bwd(causal) / (B * H)
        heads += 1
    return fl, time.perf_counter() - t0, oracle.default_threads(), heads


def time_call_graph(step, causal: bool, steps: int):
    """ms per fa_bwd call for one mask: the call captured alone as a CUDA graph
    and replayed, L2 flushed between replays outside the events."""
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        step._bwd(0, causal)
        torch.cuda.synchronize()
        with torch.cuda.graph(g, stream=s):
            step._bwd(0, causal)
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    for _ in range(3):
        step.flush_l2()
        g.replay()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    for e0, e1 in ev:
        step.flush_l2()
        e0.record()
        g.replay()
        e1.record()
    torch.cuda.synchronize()
    return statistics.mean(a.elapsed_time(b) for a, b in ev)


def run_bwd(args, world: int, rank: int):
    step = BwdStep(SEED + rank)
    graph = capture_step(step)
    with ClockSampler(torch.cuda.current_device()) as clk:
        step_ms, _ = time_steps(step, graph, args.steps, args.warmup, world)
    comp = [dist_max(time_call_graph(step, c, args.steps), world) for c in (False, True)]
    e2e_ms = dist_max(time_e2e(step, max(8, args.steps // 2), 3, world), world)
    ms = dist_max(statistics.mean(step_ms), world)
    peaks, peak_src = load_peaks()
    clocks = clk.summary()
    if rank == 0:
        step_flops = flops_bwd(False) + flops_bwd(True)
        achieved = flops_bwd(False) / (comp[0] * 1e-3) / 1e12
        line = {
            "metric": BWD_METRIC, "value": world * step_flops / (ms * 1e-3) / 1e12, "unit": "TFLOPS",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16)",
            "config": {"workload": f"bwd b{B}h{H}n{N}d{D}: fa_bwd non-causal + fa_bwd causal", "B": B, "H": H,
                       "N": N, "d": D, "parallelism": f"replicas x{world}",
                       "l2": "flushed between steps (512 MB write outside the timed events)"},
            "timing": "value: CUDA-graph replay of the step; breakdown: each fa_bwd call replayed alone as a CUDA graph",
            "breakdown_ms": {"bwd_noncausal": comp[0], "bwd_causal": comp[1]},
            "breakdown_tflops": {"bwd_noncausal": flops_bwd(False) / comp[0] / 1e9,
                                 "bwd_causal": flops_bwd(True) / comp[1] / 1e9},
            "roofline": {"kernel": "fa_bwd non-causal (prologue + attn_bwd_kernel<128,nc> + dQ conversion)",
                         "bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"], "traffic": None,
                         "peak_source": f"{peak_src} cuBLAS bf16 (burst)"},
            "e2e": {"value": world * step_flops / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS",
                    "h2d_bytes_per_step": step.h2d_bytes, "d2h_bytes_per_step": step.d2h_bytes,
                    "note": "Q, K, V, dO and both masks' O and LSE copied in, the six gradients copied out, per "
                            "step; steps pipelined over three CUDA streams (copy in, compute, copy out)"},
            "gpu_launches": step.launches_per_step * args.steps,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"], "source": clocks["source"]},
        }
        if not args.no_cpu_baseline and world == 1:
            fl, sec, cores, heads = oracle_bwd_sample(args.cpu_seconds, SEED)
            line["cpu_baseline"] = {"value": fl / sec / 1e12, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                                    "sample": f"{heads} whole heads (N={N}, d={D}) of the workload, non-causal and "
                                              f"causal alternately, fp64 numpy, {sec:.1f} s"}
        print(json.dumps(line), flush=True)
    dist_done(world)


# ------------------------------------------------------------------- main --
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--workload", choices=["step", "decode", "bwd"], default="step")
    args = ap.parse_args()
    world, rank, local = dist_setup()

    if args.impl == "reference" and args.workload == "bwd":
        if rank == 0:
            oracle_bwd_sample(1.0, SEED + 100)
            runs = [oracle_bwd_sample(args.cpu_seconds / 2, SEED + i) for i in range(args.steps)]
            fl, sec = sum(r[0] for r in runs), sum(r[1] for r in runs)
            val = fl / sec / 1e12
            line = {
                "impl": "reference", "metric": BWD_METRIC, "value": val, "unit": "TFLOPS", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sec / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded N(0,1))",
                "config": {"workload": f"bwd b{B}h{H}n{N}d{D}: fa_bwd non-causal + fa_bwd causal", "B": B, "H": H,
                           "N": N, "d": D, "l2": "n/a (CPU)"},
                "cpu_baseline": {"value": val, "unit": "TFLOPS", "cores": runs[0][2], "kind": "oracle",
                                 "sample": f"{runs[0][3]} whole heads per step, non-causal and causal alternately, "
                                           "fp64 numpy"},
                "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            }
            print(json.dumps(line), flush=True)
        dist_done(world)
        return

    if args.impl == "reference":
        if rank == 0:
            warm = [oracle_sample(2.0, SEED + 100 + i) for i in range(args.warmup)]
            del warm
            runs = [oracle_sample(args.cpu_seconds / 2, SEED + i) for i in range(args.steps)]
            fl = sum(r[0] for r in runs)
            sec = sum(r[1] for r in runs)
            val = fl / sec / 1e12
            line = {
                "impl": "reference", "metric": METRIC, "value": val, "unit": "TFLOPS", "n_gpus": args.gpus,
                "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * sec / args.steps,
                "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                "data": "synthetic (seeded N(0,1))",
                "config": {"workload": WORKLOAD, "B": B, "H": H, "N": N, "d": D, "l2": "n/a (CPU)"},
                "cpu_baseline": {"value": val, "unit": "TFLOPS", "cores": runs[0][2], "kind": "oracle",
                                 "sample": f"{runs[0][3]} random query rows per attention pass per step, "
                                           "3 passes (non-causal, causal, non-causal), exact fp64"},
                "e2e": {"value": val, "unit": "TFLOPS", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
            }
            print(json.dumps(line), flush=True)
        dist_done(world)
        return

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device for --impl ours")
    torch.cuda.set_device(local)
    if args.workload == "decode":
        run_decode(args, world, rank)
        return
    if args.workload == "bwd":
        run_bwd(args, world, rank)
        return
    step = Step(SEED + rank)
    graph = capture_step(step)
    with ClockSampler(local) as clk:
        step_ms, per = time_steps(step, graph, args.steps, args.warmup, world)
    e2e_ms = time_e2e(step, max(8, args.steps // 2), 3, world)
    ms_local = statistics.mean(step_ms)
    ms = dist_max(ms_local, world)
    e2e_ms = dist_max(e2e_ms, world)
    comp = [statistics.mean(p[j] for p in per) for j in range(4)]
    comp = [dist_max(c, world) for c in comp]
    peaks, peak_src = load_peaks()
    clocks = clk.summary()

    if rank == 0:
        value = world * STEP_FLOPS / (ms * 1e-3) / 1e12
        nc_ms = comp[0]
        achieved = flops_fwd(False) / (nc_ms * 1e-3) / 1e12
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOPS", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic (seeded N(0,1) bf16)",
            "config": {"workload": WORKLOAD, "B": B, "H": H, "N": N, "d": D, "parallelism": f"replicas x{world}",
                       "l2": "flushed between steps (512 MB write outside the timed events)"},
            "timing": "value: CUDA-graph replay of the step; breakdown: eager calls, events per kernel group",
            "breakdown_ms": {"bf16_noncausal": comp[0], "bf16_causal": comp[1], "rotate_quant_qk": comp[2],
                             "e4m3qk_noncausal": comp[3]},
            "breakdown_tflops": {"bf16_noncausal": flops_fwd(False) / comp[0] / 1e9,
                                 "bf16_causal": flops_fwd(True) / comp[1] / 1e9,
                                 "e4m3qk_noncausal": flops_fwd(False) / comp[3] / 1e9},
            "roofline": {"kernel": "attn_fwd_kernel<128,2,nc,bf16>", "bound": "tensor", "achieved": achieved,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": achieved / peaks["bf16_tflops"], "traffic": measured_traffic(),
                         "traffic_unit": "bytes per launch (ncu dram read + write)",
                         "peak_source": f"{peak_src} cuBLAS bf16 (burst)"},
            "e2e": {"value": world * STEP_FLOPS / (e2e_ms * 1e-3) / 1e12, "unit": "TFLOPS",
                    "h2d_bytes_per_step": step.h2d_bytes, "d2h_bytes_per_step": step.d2h_bytes,
                    "note": "steps pipelined over three CUDA streams (copy in, compute, copy out) with two sets of "
                            "device buffers; every step copies its inputs in and its results out"},
            "gpu_launches": step.launches_per_step * args.steps,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"], "source": clocks["source"]},
        }
        if not args.no_cpu_baseline and world == 1:
            fl, sec, cores, rows_n = oracle_sample(args.cpu_seconds, SEED)
            line["cpu_baseline"] = {"value": fl / sec / 1e12, "unit": "TFLOPS", "cores": cores, "kind": "oracle",
                                    "sample": f"{rows_n} random query rows x 3 attention passes of the workload, "
                                              f"exact fp64, {sec:.1f} s"}
        print(json.dumps(line), flush=True)
    dist_done(world)


def run_decode(args, world: int, rank: int):
    step = DecodeStep(DECODE["seed"] + rank)
    graph = capture_step(step)
    with ClockSampler(torch.cuda.current_device()) as clk:
        step_ms, per = time_steps(step, graph, args.steps, args.warmup, world)
    e2e_ms = dist_max(time_e2e(step, max(8, args.steps // 2), 3, world), world)
    ms = dist_max(statistics.mean(step_ms), world)
    comp = [dist_max(statistics.mean(p[j] for p in per), world) for j in range(2)]
    peaks, peak_src = load_peaks()
    clocks = clk.summary()
    if rank == 0:
        # the dominant kernel's algorithmic bytes: K, V, Q read and the partial
        # results written
        attn_bytes = step.kv_bytes + step.q_h.numel() * 2 + step.part_bytes
        achieved = attn_bytes / (comp[0] * 1e-3) / 1e9
        c = DECODE
        line = {
            "metric": DECODE_METRIC, "value": world * step.bytes / (ms * 1e-3) / 1e9, "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic (seeded N(0,1) bf16)",
            "config": {"workload": f"decode b{c['B']}h{c['H']} nq{c['Nq']} nk{c['Nk']} d{c['d']}: split-key attention "
                                   f"({step.n_split} blocks) + LSE merge", **{k: c[k] for k in ("B", "H", "Nq", "Nk", "d")},
                       "n_split": step.n_split, "parallelism": f"replicas x{world}",
                       "l2": "flushed between steps (512 MB write outside the timed events); K+V 1.07 GB > L2"},
            "timing": "value: CUDA-graph replay of the step; breakdown: eager calls, events per kernel",
            "breakdown_ms": {"splitkv_attention": comp[0], "lse_merge": comp[1]},
            "roofline": {"kernel": "attn_fwd_kernel<128,1,nc,bf16> (partial mode)", "bound": "hbm",
                         "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": achieved / peaks["hbm_gbs"], "traffic": None,
                         "peak_source": f"{peak_src} HBM copy bandwidth"},
            "e2e": {"value": world * step.bytes / (e2e_ms * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": step.h2d_bytes, "d2h_bytes_per_step": step.d2h_bytes,
                    "note": "K/V cache resident on the device; Q in, O and LSE out per step; steps pipelined over "
                            "three CUDA streams (copy in, compute, copy out)"},
            "gpu_launches": step.launches_per_step * args.steps,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"], "source": clocks["source"]},
        }
        print(json.dumps(line), flush=True)
    dist_done(world)


if __name__ == "__main__":
    main()
