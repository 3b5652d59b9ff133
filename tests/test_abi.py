"""The C ABI without a GPU: libfa.so builds for sm_100a, loads, exports every
function include/fa.h declares, and rejects bad arguments with the documented
status before touching the device."""
import ctypes
import re
from pathlib import Path

import pytest

from io_aware_exact_17_b200 import binding

ROOT = Path(__file__).resolve().parents[1]


def _declared_functions():
    text = (ROOT / "include" / "fa.h").read_text()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\**\s+\**(fa_\w+)\s*\(", text, flags=re.M)))


@pytest.fixture(scope="module")
def lib():
    return binding.load_library()


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert {"fa_fwd", "fa_hadamard_quant", "fa_status_string", "fa_device_status", "fa_abi_version"} <= set(names)
    for n in names:
        assert hasattr(lib, n), n
    assert {"fa_fwd_splitkv", "fa_fwd_splitkv_workspace_bytes", "fa_fwd_splitkv_splits", "fa_fwd_partial",
            "fa_lse_merge"} <= set(names)
    assert {"fa_bwd", "fa_bwd_workspace_bytes", "fa_fwd_fp8_qrot", "fa_quant_v_transposed"} <= set(names)
    assert lib.fa_abi_version() == 6


def test_status_strings(lib):
    for code in range(6):
        assert lib.fa_status_string(code)
    assert b"alignment" in lib.fa_status_string(binding.FA_ERR_ALIGNMENT) or b"misaligned" in lib.fa_status_string(
        binding.FA_ERR_ALIGNMENT)


# Fake device addresses: the checks below must fail before any CUDA call.
A = 0x10000
MIS = 0x10008


def _fwd(lib, q=A, k=A, v=A, o=A, lse=None, B=1, H=1, N=16, d=128, causal=0, scale=0.1, dtype=0, desc=None):
    return lib.fa_fwd(q, k, v, o, lse, B, H, N, d, causal, scale, dtype, desc, None)


def test_fwd_argument_errors(lib):
    assert _fwd(lib, q=None) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, o=None) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, B=0) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, N=0) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, H=-1) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=0.0) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("inf")) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, scale=float("nan")) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, dtype=7) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, d=96) == binding.FA_ERR_UNSUPPORTED
    assert _fwd(lib, d=64, dtype=1, desc=A) == binding.FA_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=1, desc=None) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, q=MIS) == binding.FA_ERR_ALIGNMENT
    assert _fwd(lib, v=MIS) == binding.FA_ERR_ALIGNMENT
    assert _fwd(lib, o=MIS) == binding.FA_ERR_ALIGNMENT
    assert _fwd(lib, lse=A + 2) == binding.FA_ERR_ALIGNMENT
    assert _fwd(lib, B=1 << 20, H=1 << 12) == binding.FA_ERR_INVALID_ARG


def _quant(lib, x=A, out=A, ds=A, rows=4, d=128, rot=1, signs=None, ws=A, wsb=256):
    return lib.fa_hadamard_quant(x, out, ds, rows, d, rot, signs, ws, wsb, None)


def test_quant_argument_errors(lib):
    assert _quant(lib, x=None) == binding.FA_ERR_INVALID_ARG
    assert _quant(lib, ws=None) == binding.FA_ERR_INVALID_ARG
    assert _quant(lib, wsb=64) == binding.FA_ERR_INVALID_ARG
    assert _quant(lib, rows=-1) == binding.FA_ERR_INVALID_ARG
    assert _quant(lib, rot=2) == binding.FA_ERR_INVALID_ARG
    assert _quant(lib, d=96) == binding.FA_ERR_UNSUPPORTED
    assert _quant(lib, x=MIS) == binding.FA_ERR_ALIGNMENT
    assert _quant(lib, out=MIS) == binding.FA_ERR_ALIGNMENT
    assert _quant(lib, signs=A + 4) == binding.FA_ERR_ALIGNMENT
    assert _quant(lib, ws=A + 4) == binding.FA_ERR_ALIGNMENT


def _skv(lib, q=A, k=A, v=A, o=A, lse=None, B=1, H=1, Nq=1, Nk=300, d=128, causal=0, scale=0.1, dtype=0, desc=None,
         ns=1, ws=None, wsb=0):
    return lib.fa_fwd_splitkv(q, k, v, o, lse, B, H, Nq, Nk, d, causal, scale, dtype, desc, ns, ws, wsb, None)


def test_splitkv_argument_errors(lib):
    assert _skv(lib, q=None) == binding.FA_ERR_INVALID_ARG
    assert _skv(lib, o=None) == binding.FA_ERR_INVALID_ARG
    assert _skv(lib, Nq=0) == binding.FA_ERR_INVALID_ARG
    assert _skv(lib, Nk=0) == binding.FA_ERR_INVALID_ARG
    assert _skv(lib, ns=-1) == binding.FA_ERR_INVALID_ARG
    assert _skv(lib, Nq=301, causal=1) == binding.FA_ERR_INVALID_ARG  # a query would see no key
    assert _skv(lib, scale=-1.0) == binding.FA_ERR_INVALID_ARG
    assert _skv(lib, d=32) == binding.FA_ERR_UNSUPPORTED
    assert _skv(lib, k=MIS) == binding.FA_ERR_ALIGNMENT
    assert _skv(lib, o=MIS) == binding.FA_ERR_ALIGNMENT
    # a split needs a workspace of the stated size, 256-byte aligned
    need = lib.fa_fwd_splitkv_workspace_bytes(1, 1, 1, 300, 128, 3)
    assert need >= 3 * 128 * 4 + 3 * 4
    assert _skv(lib, ns=3) == binding.FA_ERR_INVALID_ARG
    assert _skv(lib, ns=3, ws=A, wsb=need - 1) == binding.FA_ERR_INVALID_ARG
    assert _skv(lib, ns=3, ws=A + 16, wsb=need) == binding.FA_ERR_ALIGNMENT
    assert lib.fa_fwd_splitkv_workspace_bytes(1, 1, 1, 300, 128, 1) == 0
    assert lib.fa_fwd_splitkv_workspace_bytes(0, 1, 1, 300, 128, 2) == 0


def _sms():
    import torch
    return torch.cuda.get_device_properties(0).multi_processor_count if torch.cuda.is_available() else 148


def _tail_plan(B, H, N, d, sms):
    """The automatic schedule's tail split, restated: without causal masking, a
    persistent launch whose last round is at most half full splits that round's
    query blocks into min(4, sms // tail, key tiles) pieces of equal key-tile
    spans (no empty piece). Returns (pieces, tail blocks, query tiles per block)."""
    nq = 2 if (d <= 128 and N > 128) else 1
    units = B * H * -(-N // (128 * nq))
    tiles = -(-N // 128)
    tail = units % sms
    if units < sms or tail == 0 or 2 * tail > sms or tiles < 4 or (nq == 1 and N <= 32):
        return 0, 0, nq
    ns = min(4, sms // tail, tiles)
    span = -(-tiles // ns)
    ns = -(-tiles // span)
    return (ns if ns >= 2 else 0), tail, nq


def test_tail_split_workspace(lib):
    # B=4, H=16, N=2048, d=128: 512 two-tile query blocks on 148 SMs leave 68 for
    # a last round: two pieces of 8 key tiles each
    sms = _sms()
    for (B, H, N, d) in [(4, 16, 2048, 128), (1, 19, 2048, 128), (2, 20, 1000, 64), (2, 13, 700, 256),
                         (1, 16, 16384, 128), (8, 16, 2048, 128)]:
        ns, tail, nq = _tail_plan(B, H, N, d, sms)
        up = lambda x: (x + 255) // 256 * 256
        groups = tail * nq
        want = up(groups * ns * 128 * d * 4) + up(groups * ns * 128 * 4) + up(groups * 4 * 8) if ns else 0
        if ns == 0 and B * H * -(-N // (128 * nq)) < sms:
            continue  # a key split instead
        assert lib.fa_fwd_splitkv_workspace_bytes(B, H, N, N, d, 0) == want, (B, H, N, d)
    if sms == 148:
        assert _tail_plan(4, 16, 2048, 128, sms)[:2] == (2, 68)
        assert _tail_plan(2, 13, 700, 256, sms)[:2] == (3, 8)
        need = lib.fa_fwd_splitkv_workspace_bytes(4, 16, 2048, 2048, 128, 0)
        assert need == 17969408
        # the automatic schedule then needs the workspace, 256-byte aligned
        big = dict(B=4, H=16, Nq=2048, Nk=2048, ns=0)
        assert _skv(lib, **big) == binding.FA_ERR_INVALID_ARG
        assert _skv(lib, ws=A, wsb=need - 1, **big) == binding.FA_ERR_INVALID_ARG
        assert _skv(lib, ws=A + 16, wsb=need, **big) == binding.FA_ERR_ALIGNMENT


def test_v_transposed_quant_argument_errors(lib):
    def q(v=A, o=A, ds=A, BH=2, N=100, d=128, ws=A, wsb=256):
        return lib.fa_quant_v_transposed(v, o, ds, BH, N, d, ws, wsb, None)
    assert q(v=None) == binding.FA_ERR_INVALID_ARG
    assert q(o=None) == binding.FA_ERR_INVALID_ARG
    assert q(ds=None) == binding.FA_ERR_INVALID_ARG
    assert q(ws=None) == binding.FA_ERR_INVALID_ARG
    assert q(BH=0) == binding.FA_ERR_INVALID_ARG
    assert q(BH=65536) == binding.FA_ERR_INVALID_ARG
    assert q(N=0) == binding.FA_ERR_INVALID_ARG
    assert q(wsb=255) == binding.FA_ERR_INVALID_ARG
    assert q(d=96) == binding.FA_ERR_UNSUPPORTED
    assert q(v=MIS) == binding.FA_ERR_ALIGNMENT
    assert q(o=MIS) == binding.FA_ERR_ALIGNMENT
    assert q(ds=A + 2) == binding.FA_ERR_ALIGNMENT


def test_partial_and_merge_argument_errors(lib):
    part = lambda **kw: lib.fa_fwd_partial(kw.get("q", A), A, A, kw.get("op", A), kw.get("lp", A), 1, 1, 4, 64, 128,
                                           kw.get("causal", 0), 0.1, 0, None, kw.get("ns", 1), None)
    assert part(q=None) == binding.FA_ERR_INVALID_ARG
    assert part(op=None) == binding.FA_ERR_INVALID_ARG
    assert part(lp=None) == binding.FA_ERR_INVALID_ARG
    assert part(ns=0) == binding.FA_ERR_INVALID_ARG
    assert part(op=MIS) == binding.FA_ERR_ALIGNMENT
    assert part(lp=A + 2) == binding.FA_ERR_ALIGNMENT
    merge = lambda **kw: lib.fa_lse_merge(kw.get("op", A), kw.get("lp", A), kw.get("n", 2), kw.get("rows", 8),
                                          kw.get("d", 128), kw.get("o", A), None, None)
    assert merge(op=None) == binding.FA_ERR_INVALID_ARG
    assert merge(o=None) == binding.FA_ERR_INVALID_ARG
    assert merge(n=0) == binding.FA_ERR_INVALID_ARG
    assert merge(rows=0) == binding.FA_ERR_INVALID_ARG
    assert merge(d=80) == binding.FA_ERR_UNSUPPORTED
    assert merge(op=MIS) == binding.FA_ERR_ALIGNMENT
    assert merge(o=MIS) == binding.FA_ERR_ALIGNMENT


def test_quant_multi_argument_errors(lib):
    arr = (ctypes.c_void_p * 9)(*([A] * 9))
    mq = lambda **kw: lib.fa_hadamard_quant_multi(kw.get("xs", arr), kw.get("outs", arr), kw.get("ds", A),
                                                  kw.get("n", 2), kw.get("rows", 4), kw.get("d", 128),
                                                  kw.get("rot", 1), None, kw.get("ws", A), kw.get("wsb", 256), None)
    assert mq(xs=None) == binding.FA_ERR_INVALID_ARG
    assert mq(ws=None) == binding.FA_ERR_INVALID_ARG
    assert mq(n=0) == binding.FA_ERR_INVALID_ARG
    assert mq(n=9) == binding.FA_ERR_INVALID_ARG
    assert mq(wsb=8) == binding.FA_ERR_INVALID_ARG
    assert mq(rows=-1) == binding.FA_ERR_INVALID_ARG
    assert mq(d=96) == binding.FA_ERR_UNSUPPORTED
    assert mq(ds=A + 2) == binding.FA_ERR_ALIGNMENT
    mis = (ctypes.c_void_p * 2)(A, MIS)
    assert mq(xs=mis) == binding.FA_ERR_ALIGNMENT


def test_block_quant_argument_errors(lib):
    bq = lambda **kw: lib.fa_hadamard_quant_blocks(kw.get("x", A), kw.get("out", A), kw.get("ds", A), kw.get("BH", 2),
                                                   kw.get("N", 300), kw.get("d", 128), kw.get("rot", 1), None, None)
    assert bq(x=None) == binding.FA_ERR_INVALID_ARG
    assert bq(ds=None) == binding.FA_ERR_INVALID_ARG
    assert bq(BH=0) == binding.FA_ERR_INVALID_ARG
    assert bq(N=0) == binding.FA_ERR_INVALID_ARG
    assert bq(rot=3) == binding.FA_ERR_INVALID_ARG
    assert bq(d=96) == binding.FA_ERR_UNSUPPORTED
    assert bq(x=MIS) == binding.FA_ERR_ALIGNMENT
    assert bq(ds=A + 2) == binding.FA_ERR_ALIGNMENT
    # per-block descales are an e4m3 dtype: not for d = 64, and they are required
    assert _fwd(lib, dtype=2, desc=A, d=64) == binding.FA_ERR_UNSUPPORTED
    assert _fwd(lib, dtype=2, desc=None) == binding.FA_ERR_INVALID_ARG
    assert _fwd(lib, dtype=3, desc=A) == binding.FA_ERR_INVALID_ARG


def test_python_binding_rejects_cpu_tensors():
    import torch

    q = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(binding.FaError):
        binding.fwd(q, q, q)
    with pytest.raises(binding.FaError):
        binding.hadamard_quant(q)
    with pytest.raises(binding.FaError):
        binding.fwd_splitkv(q, q, q)
    with pytest.raises(binding.FaError):
        binding.fwd_partial(q, q, q)
    with pytest.raises(binding.FaError):
        binding.lse_merge(q.float(), q.float()[..., 0])


def test_bwd_argument_errors(lib):
    need = lib.fa_bwd_workspace_bytes(2, 3, 300, 128)
    # dQ accumulator (fp32, 256-byte padded) plus the per-row D and LSE over whole 128-row tiles
    assert need == 2 * 3 * 300 * 128 * 4 + 2 * ((2 * 3 * 384 * 4 + 255) // 256 * 256)
    assert lib.fa_bwd_workspace_bytes(2, 3, 300, 256) == 0
    assert lib.fa_bwd_workspace_bytes(0, 3, 300, 128) == 0

    def bwd(**kw):
        ptrs = [kw.get(n, A) for n in ("q", "k", "v", "o", "do", "lse", "dq", "dk", "dv")]
        return lib.fa_bwd(*ptrs, kw.get("B", 2), 3, kw.get("N", 300), kw.get("d", 128), kw.get("causal", 0),
                          kw.get("scale", 0.1), kw.get("ws", A), kw.get("wsb", need), None)

    for name in ("q", "k", "v", "o", "do", "lse", "dq", "dk", "dv", "ws"):
        assert bwd(**{name: None}) == binding.FA_ERR_INVALID_ARG, name
    assert bwd(B=0) == binding.FA_ERR_INVALID_ARG
    assert bwd(N=0) == binding.FA_ERR_INVALID_ARG
    assert bwd(scale=0.0) == binding.FA_ERR_INVALID_ARG
    assert bwd(scale=float("nan")) == binding.FA_ERR_INVALID_ARG
    assert bwd(d=256) == binding.FA_ERR_UNSUPPORTED
    assert bwd(d=96) == binding.FA_ERR_UNSUPPORTED
    assert bwd(wsb=need - 1) == binding.FA_ERR_INVALID_ARG
    for name in ("q", "k", "v", "o", "do", "dq", "dk", "dv"):
        assert bwd(**{name: MIS}) == binding.FA_ERR_ALIGNMENT, name
    assert bwd(lse=A + 2) == binding.FA_ERR_ALIGNMENT
    assert bwd(ws=A + 16) == binding.FA_ERR_ALIGNMENT


def test_bwd_binding_rejects_host_tensors_and_bad_shapes():
    import torch

    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 1, 8)
    with pytest.raises(binding.FaError):
        binding.bwd(q, q, q, q, lse, q)  # host tensors: no CPU path


def test_tensor_argument_checks_run_before_any_launch():
    """Every caller-supplied tensor (outputs, workspaces, descales, signs) is
    checked before its pointer reaches the library: dtype, exact shape,
    contiguity, size, and that it is a CUDA tensor on the inputs' device."""
    import torch

    dev = torch.device("cuda:0")
    ok = torch.zeros(2, 3, dtype=torch.float32)
    with pytest.raises(binding.FaError, match="CUDA"):           # a host tensor
        binding._tensor_arg(ok, "out", dev, (torch.float32,), (2, 3))
    with pytest.raises(binding.FaError, match="dtype"):
        binding._tensor_arg(ok.double(), "out", dev, (torch.float32,), (2, 3))
    with pytest.raises(binding.FaError, match="shape"):          # a short output
        binding._tensor_arg(torch.zeros(2, 2), "out", dev, (torch.float32,), (2, 3))
    with pytest.raises(binding.FaError, match="contiguous"):     # a strided view
        binding._tensor_arg(torch.zeros(3, 2).t(), "out", dev, (torch.float32,), (2, 3))
    with pytest.raises(binding.FaError, match="bytes"):          # a short workspace
        binding._tensor_arg(torch.zeros(255, dtype=torch.uint8), "workspace", dev, min_bytes=256)
    with pytest.raises(binding.FaError, match="torch tensor"):
        binding._tensor_arg([0.0], "descale", dev)
    with pytest.raises(binding.FaError, match="signs"):
        binding._signs_arg(torch.ones(64), 128, dev)
    with pytest.raises(binding.FaError, match="pair"):
        binding._descale_arg((ok,), 1, 1, 128, 128, dev)
    with pytest.raises(binding.FaError):
        binding._descale_arg(ok.reshape(-1)[:2], 1, 1, 128, 128, dev)   # host descale
    with pytest.raises(binding.FaError):
        binding._descale_arg(None, 1, 1, 128, 128, dev)


def test_fused_q_argument_errors(lib):
    def call(**kw):
        return lib.fa_fwd_fp8_qrot(kw.get("q", A), kw.get("k", A), kw.get("v", A), kw.get("o", A), kw.get("lse", A),
                                   1, 2, kw.get("N", 300), kw.get("d", 128), kw.get("causal", 0), kw.get("scale", 0.1),
                                   kw.get("dk", A), kw.get("rotate", 1), kw.get("signs", None), kw.get("dq", None),
                                   None)
    lib.fa_fwd_fp8_qrot.argtypes = [ctypes.c_void_p] * 5 + [ctypes.c_int] * 5 + [ctypes.c_float, ctypes.c_void_p,
                                                                                   ctypes.c_int] + [ctypes.c_void_p] * 3
    lib.fa_fwd_fp8_qrot.restype = ctypes.c_int
    for name in ("q", "k", "v", "o", "dk"):
        assert call(**{name: None}) == binding.FA_ERR_INVALID_ARG, name
    assert call(d=64) == binding.FA_ERR_UNSUPPORTED
    assert call(d=256) == binding.FA_ERR_UNSUPPORTED
    assert call(rotate=2) == binding.FA_ERR_INVALID_ARG
    assert call(N=0) == binding.FA_ERR_INVALID_ARG
    assert call(scale=0.0) == binding.FA_ERR_INVALID_ARG
    assert call(q=MIS) == binding.FA_ERR_ALIGNMENT
    assert call(signs=A + 4) == binding.FA_ERR_ALIGNMENT
    assert call(dq=A + 2) == binding.FA_ERR_ALIGNMENT
