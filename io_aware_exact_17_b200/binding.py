"""ctypes binding of libfa.so (include/fa.h). Argument marshalling only: every
step of the computation runs in the library's CUDA kernels. PyTorch supplies
device memory and the current stream.

If the library is missing it is built from csrc/ with nvcc; if that fails, or
there is no CUDA device, the calls raise :class:`FaError`. There is no CPU or
PyTorch fallback.
"""
from __future__ import annotations

import ctypes
import math
import threading
from pathlib import Path

import torch

_PKG = Path(__file__).resolve().parent
_lock = threading.Lock()
_lib = None
_workspaces: dict[tuple[int, int], torch.Tensor] = {}

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(6)
FA_BF16, FA_E4M3, FA_E4M3_BLOCK = 0, 1, 2
BLOCK_ROWS = 128  # rows per scale block of fa_hadamard_quant_blocks
QUANT_WORKSPACE_BYTES = 256
E4M3_DTYPES = (torch.uint8, torch.float8_e4m3fn)


class FaError(RuntimeError):
    """A libfa call returned an error status (the message names it)."""


def library_path() -> Path:
    return _PKG / "libfa.so"


def load_library():
    """Load (building first if needed) libfa.so and declare its signatures."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        from . import build as _build

        try:
            path = _build.build()
        except Exception as e:  # no nvcc, or it failed: there is nothing else to run
            raise FaError(f"libfa.so is not built and could not be built: {e}") from e
        lib = ctypes.CDLL(str(path))
        vp, i, f, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int64, ctypes.c_size_t
        lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, vp]
        lib.fa_fwd.restype = i
        lib.fa_hadamard_quant.argtypes = [vp, vp, vp, i64, i, i, vp, vp, sz, vp]
        lib.fa_hadamard_quant.restype = i
        lib.fa_status_string.argtypes = [i]
        lib.fa_status_string.restype = ctypes.c_char_p
        lib.fa_device_status.argtypes = [ctypes.POINTER(i), ctypes.POINTER(ctypes.c_uint),
                                         ctypes.POINTER(ctypes.c_uint)]
        lib.fa_device_status.restype = i
        lib.fa_abi_version.argtypes = []
        lib.fa_abi_version.restype = i
        lib.fa_fwd_splitkv.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, i, vp, sz, vp]
        lib.fa_fwd_splitkv.restype = i
        lib.fa_fwd_splitkv_workspace_bytes.argtypes = [i, i, i, i, i, i]
        lib.fa_fwd_splitkv_workspace_bytes.restype = sz
        lib.fa_fwd_splitkv_splits.argtypes = [i, i, i, i, i]
        lib.fa_fwd_splitkv_splits.restype = i
        lib.fa_fwd_partial.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, f, i, vp, i, vp]
        lib.fa_fwd_partial.restype = i
        lib.fa_lse_merge.argtypes = [vp, vp, i, i64, i, vp, vp, vp]
        lib.fa_lse_merge.restype = i
        lib.fa_hadamard_quant_blocks.argtypes = [vp, vp, vp, i, i, i, i, vp, vp]
        lib.fa_hadamard_quant_blocks.restype = i
        lib.fa_hadamard_quant_multi.argtypes = [vp, vp, vp, i, i64, i, i, vp, vp, sz, vp]
        lib.fa_hadamard_quant_multi.restype = i
        lib.fa_bwd_workspace_bytes.argtypes = [i, i, i, i]
        lib.fa_bwd_workspace_bytes.restype = sz
        lib.fa_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, sz, vp]
        lib.fa_bwd.restype = i
        lib.fa_fwd_fp8_qrot.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, i, vp, vp, vp]
        lib.fa_fwd_fp8_qrot.restype = i
        lib.fa_quant_v_transposed.argtypes = [vp, vp, vp, i, i, i, vp, sz, vp]
        lib.fa_quant_v_transposed.restype = i
        _lib = lib
        return lib


def _check(rc: int, what: str):
    if rc != FA_OK:
        msg = load_library().fa_status_string(rc).decode()
        raise FaError(f"{what} failed: {msg} (status {rc})")


def _ptr(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _tensor_arg(t, name: str, device, dtypes=None, shape=None, min_bytes: int | None = None):
    """Check one tensor argument before its pointer reaches the library: a CUDA
    tensor on ``device``, of one of ``dtypes``, of exactly ``shape``, contiguous
    (a pointer to a strided view would be read or written as if it were dense),
    and holding at least ``min_bytes`` bytes. Raises FaError otherwise."""
    if not isinstance(t, torch.Tensor):
        raise FaError(f"{name} must be a torch tensor")
    if dtypes is not None and t.dtype not in dtypes:
        raise FaError(f"{name} must have dtype {' or '.join(str(x) for x in dtypes)} (got {t.dtype})")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise FaError(f"{name} must have shape {tuple(shape)} (got {tuple(t.shape)})")
    if not t.is_contiguous():
        raise FaError(f"{name} must be contiguous")
    if min_bytes is not None and _nbytes(t) < min_bytes:
        raise FaError(f"{name} holds {_nbytes(t)} bytes, needs at least {min_bytes}")
    if not t.is_cuda:
        raise FaError(f"{name} must be on a CUDA device (got {t.device})")
    if t.device != torch.device(device):
        raise FaError(f"{name} is on {t.device}, the other tensors on {device}")
    return t


def _nbytes(t) -> int:
    return t.numel() * t.element_size()


def _descale_arg(qk_descale, B, H, Nq, Nk, device):
    """(fa_dtype, fp32 CUDA tensor) for e4m3 inputs: a 2-element tensor [dq, dk]
    is one scale per tensor; a pair (dq_blocks [B, H, ceil(Nq/128)], dk_blocks
    [B, H, ceil(Nk/128)]) is one scale per 128-row block."""
    f32 = (torch.float32,)
    if isinstance(qk_descale, (tuple, list)):
        if len(qk_descale) != 2:
            raise FaError("per-block descales must be a pair (dq_blocks, dk_blocks)")
        dq, dk = qk_descale
        nbq, nbk = -(-Nq // BLOCK_ROWS), -(-Nk // BLOCK_ROWS)
        for t, name, nb in ((dq, "dq_blocks", nbq), (dk, "dk_blocks", nbk)):
            if not isinstance(t, torch.Tensor) or t.numel() != B * H * nb:
                raise FaError(f"per-block descales must hold B*H*ceil(N/128) values ({B * H * nbq}, {B * H * nbk})")
            _tensor_arg(t, name, device, f32)
        return FA_E4M3_BLOCK, torch.cat([dq.reshape(-1), dk.reshape(-1)])
    if qk_descale is None:
        raise FaError("e4m3 q/k need qk_descale = CUDA fp32 tensor [dq, dk] or a pair of per-block tensors")
    _tensor_arg(qk_descale, "qk_descale", device, f32)
    if qk_descale.numel() != 2:
        raise FaError("qk_descale must hold exactly two values [dq, dk]")
    return FA_E4M3, qk_descale


def _require_cuda(*ts):
    """The input tensors are CUDA tensors on one device (a CUDA device must exist)."""
    if not torch.cuda.is_available():
        raise FaError("no CUDA device")
    dev = None
    for t in ts:
        if t is None:
            continue
        if not isinstance(t, torch.Tensor) or not t.is_cuda:
            raise FaError("tensors must be on a CUDA device")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise FaError(f"tensors must be on one device (got {dev} and {t.device})")


def _signs_arg(signs, d: int, device):
    """The d Hadamard signs as a contiguous fp32 tensor on ``device``."""
    if signs is None:
        return None
    if not isinstance(signs, torch.Tensor) or signs.numel() != d:
        raise FaError(f"signs must be a tensor of d = {d} values")
    return signs.to(device=device, dtype=torch.float32).reshape(d).contiguous()


def fwd(q, k, v, causal: bool = False, scale: float | None = None, qk_descale=None, out=None, lse=None,
        return_lse: bool = True, n_split: int = 0):
    """Attention forward of ``[B, H, N, d]`` inputs.

    q, k: bf16, or e4m3 codes (uint8 / float8_e4m3fn) with ``qk_descale`` a
    CUDA fp32 tensor ``[dq, dk]`` (one scale per tensor, as ``hadamard_quant``
    gives) or a pair of per-block descales (as ``hadamard_quant_blocks`` gives);
    v: bf16. Returns ``(O, LSE)``: bf16
    ``[B, H, N, d]`` and fp32 ``[B, H, N]`` (natural log); LSE is ``None`` when
    ``return_lse`` is false.

    ``n_split=0`` (default) runs ``fa_fwd_splitkv`` with its automatic
    schedule, which splits the keys of some query blocks (all of them when
    there are fewer blocks than SMs, else those of a mostly empty last wave)
    and merges by LSE, with a workspace cached per device. ``n_split=1`` runs
    ``fa_fwd``: one CTA per query block over all its keys, no workspace.
    """
    _require_cuda(q, k, v)
    lib = load_library()
    if q.dim() != 4 or q.shape != k.shape or q.shape != v.shape:
        raise FaError("q, k, v must share one [B, H, N, d] shape")
    B, H, N, d = q.shape
    fp8 = q.dtype in E4M3_DTYPES
    if fp8 != (k.dtype in E4M3_DTYPES) or (not fp8 and (q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16)):
        raise FaError("q and k must both be bf16 or both e4m3")
    if v.dtype != torch.bfloat16:
        raise FaError("v must be bf16")
    if n_split not in (0, 1):
        raise FaError("n_split must be 0 (automatic) or 1 (no split); use fwd_splitkv for a fixed split")
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    _tensor_arg(out, "out", q.device, (torch.bfloat16,), (B, H, N, d))
    if return_lse:
        if lse is None:
            lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
        _tensor_arg(lse, "lse", q.device, (torch.float32,), (B, H, N))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    dt, desc_t = _descale_arg(qk_descale, B, H, N, N, q.device) if fp8 else (FA_BF16, None)
    desc = _ptr(desc_t)
    with torch.cuda.device(q.device):
        if n_split == 1:
            rc = lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse) if return_lse else None, B, H, N, d,
                            int(bool(causal)), float(scale), dt, desc, _stream(q.device))
            _check(rc, "fa_fwd")
        else:
            need = int(lib.fa_fwd_splitkv_workspace_bytes(B, H, N, N, d, 0))
            ws = _split_workspace(q.device, need)
            rc = lib.fa_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse) if return_lse else None, B, H,
                                    N, N, d, int(bool(causal)), float(scale), dt, desc, 0,
                                    _ptr(ws) if need > 0 else None, need, _stream(q.device))
            _check(rc, "fa_fwd_splitkv")
    return out, (lse if return_lse else None)


def fwd_fp8_qrot(q, k8, v, dk_blocks, causal: bool = False, scale: float | None = None, rotate: bool = True,
                 signs=None, out=None, lse=None, return_lse: bool = True, return_dq: bool = False):
    """e4m3 attention with Q rotated and quantised inside the attention kernel
    (``fa_fwd_fp8_qrot``): ``q`` bf16 ``[B, H, N, 128]``; ``k8`` the e4m3 codes
    of K with one descale per 128-row block, ``dk_blocks`` fp32 ``[B, H,
    ceil(N/128)]`` (as ``hadamard_quant_blocks(k, rotate, signs)`` gives); ``v``
    bf16. Each 128-row query tile is rotated with the same ``signs`` (if
    ``rotate``) and quantised with its own scale in shared memory. Returns ``(O,
    LSE)`` and, with ``return_dq``, also the query-block descales the kernel
    computed, fp32 ``[B, H, ceil(N/128)]``."""
    _require_cuda(q, k8, v, dk_blocks)
    lib = load_library()
    if q.dim() != 4 or q.dtype != torch.bfloat16 or v.dtype != torch.bfloat16 or tuple(v.shape) != tuple(q.shape):
        raise FaError("q and v must be bf16 [B, H, N, d] of one shape")
    B, H, N, d = q.shape
    dev = q.device
    _tensor_arg(k8, "k8", dev, E4M3_DTYPES, (B, H, N, d))
    nb = -(-N // BLOCK_ROWS)
    _tensor_arg(dk_blocks, "dk_blocks", dev, (torch.float32,), (B, H, nb))
    q, v = q.contiguous(), v.contiguous()
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=dev)
    _tensor_arg(out, "out", dev, (torch.bfloat16,), (B, H, N, d))
    if return_lse:
        if lse is None:
            lse = torch.empty((B, H, N), dtype=torch.float32, device=dev)
        _tensor_arg(lse, "lse", dev, (torch.float32,), (B, H, N))
    dq = torch.empty((B, H, nb), dtype=torch.float32, device=dev) if return_dq else None
    signs = _signs_arg(signs, d, dev) if rotate else None
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(dev):
        rc = lib.fa_fwd_fp8_qrot(_ptr(q), _ptr(k8), _ptr(v), _ptr(out), _ptr(lse) if return_lse else None, B, H, N,
                                 d, int(bool(causal)), float(scale), _ptr(dk_blocks), int(bool(rotate)), _ptr(signs),
                                 _ptr(dq), _stream(dev))
    _check(rc, "fa_fwd_fp8_qrot")
    res = (out, lse if return_lse else None)
    return res + (dq,) if return_dq else res


_split_workspaces: dict[tuple[int, int], torch.Tensor] = {}


def _stream_key(device) -> tuple[int, int]:
    dev = torch.device(device)
    return dev.index, torch.cuda.current_stream(dev).cuda_stream


def _split_workspace(device, nbytes: int):
    """A device buffer of at least ``nbytes`` for the split schedules, cached per
    (device, current stream) and grown when a call needs more. Calls on one
    stream run in order, so they can share it; calls on different streams get
    different buffers. A buffer is allocated while its stream is current, so
    the caching allocator reuses its memory only in that stream's order when it
    is replaced."""
    if nbytes <= 0:
        return None
    key = _stream_key(device)
    ws = _split_workspaces.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(nbytes, 1 << 20), dtype=torch.uint8, device=device)
        _split_workspaces[key] = ws
    return ws


def _qkv_kinds(q, k, v, qk_descale):
    """Shapes and dtypes of q [B, H, Nq, d] against k, v [B, H, Nk, d]; returns
    (B, H, Nq, Nk, d, fp8)."""
    if q.dim() != 4 or k.dim() != 4 or k.shape != v.shape or q.shape[:2] != k.shape[:2] or q.shape[3] != k.shape[3]:
        raise FaError("q must be [B, H, Nq, d] and k, v one [B, H, Nk, d] shape")
    fp8 = q.dtype in E4M3_DTYPES
    if fp8 != (k.dtype in E4M3_DTYPES) or (not fp8 and (q.dtype != torch.bfloat16 or k.dtype != torch.bfloat16)):
        raise FaError("q and k must both be bf16 or both e4m3")
    if v.dtype != torch.bfloat16:
        raise FaError("v must be bf16")
    B, H, Nq, d = q.shape
    return B, H, Nq, k.shape[2], d, fp8


def splitkv_splits(B: int, H: int, Nq: int, Nk: int, d: int, device=None) -> int:
    """The split count ``fwd_splitkv`` picks for ``n_split=0`` on ``device``."""
    lib = load_library()
    with torch.cuda.device(device if device is not None else torch.cuda.current_device()):
        return int(lib.fa_fwd_splitkv_splits(B, H, Nq, Nk, d))


def fwd_splitkv(q, k, v, causal: bool = False, scale: float | None = None, qk_descale=None, n_split: int = 0,
                out=None, lse=None, workspace=None, return_lse: bool = True):
    """Attention of ``q`` ``[B, H, Nq, d]`` over ``k``, ``v`` ``[B, H, Nk, d]``
    through ``fa_fwd_splitkv``: the keys are split into ``n_split`` blocks (0 =
    automatic) processed in parallel and merged by their LSEs. With ``causal``,
    query i is position ``Nk - Nq + i`` (Nq <= Nk). Returns ``(O, LSE)`` as
    :func:`fwd`. ``workspace``: optional uint8 CUDA tensor of at least
    ``fa_fwd_splitkv_workspace_bytes`` bytes (allocated here if not given)."""
    _require_cuda(q, k, v)
    lib = load_library()
    B, H, Nq, Nk, d, fp8 = _qkv_kinds(q, k, v, qk_descale)
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    if out is None:
        out = torch.empty((B, H, Nq, d), dtype=torch.bfloat16, device=q.device)
    _tensor_arg(out, "out", q.device, (torch.bfloat16,), (B, H, Nq, d))
    if return_lse:
        if lse is None:
            lse = torch.empty((B, H, Nq), dtype=torch.float32, device=q.device)
        _tensor_arg(lse, "lse", q.device, (torch.float32,), (B, H, Nq))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(q.device):
        if n_split == 0:
            n_split = int(lib.fa_fwd_splitkv_splits(B, H, Nq, Nk, d))
        need = int(lib.fa_fwd_splitkv_workspace_bytes(B, H, Nq, Nk, d, int(n_split)))
        if need > 0:
            if workspace is None:
                workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
            _tensor_arg(workspace, "workspace", q.device, min_bytes=need)
        ws_bytes = _nbytes(workspace) if workspace is not None else 0
        dt, desc_t = _descale_arg(qk_descale, B, H, Nq, Nk, q.device) if fp8 else (FA_BF16, None)
        rc = lib.fa_fwd_splitkv(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse) if return_lse else None, B, H, Nq,
                                Nk, d, int(bool(causal)), float(scale), dt, _ptr(desc_t), int(n_split),
                                _ptr(workspace) if need > 0 else None, ws_bytes, _stream(q.device))
    _check(rc, "fa_fwd_splitkv")
    return out, (lse if return_lse else None)


def fwd_partial(q, k, v, causal: bool = False, scale: float | None = None, qk_descale=None, n_split: int = 1,
                o_part=None, lse_part=None):
    """Per-block attention results through ``fa_fwd_partial``: for each of the
    ``n_split`` blocks of keys, fp32 ``O_s`` ``[n_split, B, H, Nq, d]``
    (normalised over the block) and ``LSE_s`` ``[n_split, B, H, Nq]`` (natural
    log; -inf and O = 0 where a row sees no key of the block)."""
    _require_cuda(q, k, v)
    lib = load_library()
    B, H, Nq, Nk, d, fp8 = _qkv_kinds(q, k, v, qk_descale)
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    if int(n_split) < 1:
        raise FaError("n_split must be at least 1")
    if o_part is None:
        o_part = torch.empty((n_split, B, H, Nq, d), dtype=torch.float32, device=q.device)
    if lse_part is None:
        lse_part = torch.empty((n_split, B, H, Nq), dtype=torch.float32, device=q.device)
    _tensor_arg(o_part, "o_part", q.device, (torch.float32,), (n_split, B, H, Nq, d))
    _tensor_arg(lse_part, "lse_part", q.device, (torch.float32,), (n_split, B, H, Nq))
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(q.device):
        dt, desc_t = _descale_arg(qk_descale, B, H, Nq, Nk, q.device) if fp8 else (FA_BF16, None)
        rc = lib.fa_fwd_partial(_ptr(q), _ptr(k), _ptr(v), _ptr(o_part), _ptr(lse_part), B, H, Nq, Nk, d,
                                int(bool(causal)), float(scale), dt, _ptr(desc_t), int(n_split), _stream(q.device))
    _check(rc, "fa_fwd_partial")
    return o_part, lse_part


def lse_merge(o_part, lse_part, out=None, lse=None, return_lse: bool = True):
    """Merge per-block results ``o_part`` ``[S, ..., d]`` (fp32) and ``lse_part``
    ``[S, ...]`` through ``fa_lse_merge`` into bf16 ``O`` ``[..., d]`` and fp32
    ``LSE`` ``[...]``."""
    _require_cuda(o_part, lse_part)
    lib = load_library()
    if o_part.dtype != torch.float32 or lse_part.dtype != torch.float32:
        raise FaError("o_part and lse_part must be fp32")
    if o_part.dim() < 2 or tuple(o_part.shape[:-1]) != tuple(lse_part.shape):
        raise FaError("o_part must be [S, ..., d] and lse_part [S, ...]")
    n_part, d = o_part.shape[0], o_part.shape[-1]
    rows = lse_part[0].numel()
    o_part, lse_part = o_part.contiguous(), lse_part.contiguous()
    if out is None:
        out = torch.empty(tuple(o_part.shape[1:]), dtype=torch.bfloat16, device=o_part.device)
    _tensor_arg(out, "out", o_part.device, (torch.bfloat16,), tuple(o_part.shape[1:]))
    if return_lse:
        if lse is None:
            lse = torch.empty(tuple(lse_part.shape[1:]), dtype=torch.float32, device=o_part.device)
        _tensor_arg(lse, "lse", o_part.device, (torch.float32,), tuple(lse_part.shape[1:]))
    with torch.cuda.device(o_part.device):
        rc = lib.fa_lse_merge(_ptr(o_part), _ptr(lse_part), n_part, rows, d, _ptr(out),
                              _ptr(lse) if return_lse else None, _stream(o_part.device))
    _check(rc, "fa_lse_merge")
    return out, (lse if return_lse else None)


def bwd(q, k, v, o, lse, dout, causal: bool = False, scale: float | None = None, workspace=None):
    """Gradients ``(dQ, dK, dV)`` (bf16 ``[B, H, N, d]``) of a loss through
    ``fwd(q, k, v, causal, scale)``, given its output ``o``, its ``lse`` and
    ``dout`` = dLoss/dO, through ``fa_bwd``. d is 64 or 128. ``workspace``: an
    optional CUDA uint8 tensor of at least ``fa_bwd_workspace_bytes`` bytes."""
    _require_cuda(q, k, v, o, lse, dout)
    lib = load_library()
    for t, name in ((q, "q"), (k, "k"), (v, "v"), (o, "o"), (dout, "dout")):
        if t.dtype != torch.bfloat16 or t.dim() != 4 or tuple(t.shape) != tuple(q.shape):
            raise FaError(f"{name} must be bf16 [B, H, N, d] like q")
    B, H, N, d = q.shape
    if lse.dtype != torch.float32 or tuple(lse.shape) != (B, H, N):
        raise FaError("lse must be fp32 [B, H, N]")
    scale = d ** -0.5 if scale is None else scale
    q, k, v, o, dout, lse = (t.contiguous() for t in (q, k, v, o, dout, lse))
    need = int(lib.fa_bwd_workspace_bytes(B, H, N, d))
    if workspace is None:
        workspace = torch.empty(max(need, 1), dtype=torch.uint8, device=q.device)
    _tensor_arg(workspace, "workspace", q.device, min_bytes=need)
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    with torch.cuda.device(q.device):
        rc = lib.fa_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(o), _ptr(dout), _ptr(lse), _ptr(dq), _ptr(dk), _ptr(dv),
                        B, H, N, d, int(bool(causal)), float(scale), _ptr(workspace),
                        workspace.numel() * workspace.element_size(), _stream(q.device))
    _check(rc, "fa_bwd")
    return dq, dk, dv


def bwd_workspace_bytes(B: int, H: int, N: int, d: int) -> int:
    """Bytes of device workspace ``fa_bwd`` needs (0 for an unsupported shape)."""
    return int(load_library().fa_bwd_workspace_bytes(B, H, N, d))


def _workspace(device) -> torch.Tensor:
    """The quantisers' 256-byte workspace (amax words and grid-barrier counter),
    cached per (device, current stream): each call zeroes it on its stream, so
    calls on one stream may share it and calls on two streams must not."""
    key = _stream_key(device)
    ws = _workspaces.get(key)
    if ws is None:
        ws = torch.empty(QUANT_WORKSPACE_BYTES, dtype=torch.uint8, device=device)
        _workspaces[key] = ws
    return ws


def hadamard_quant(x, rotate: bool = True, signs=None, out=None, descale=None, workspace=None):
    """Rotate (optionally) and quantise ``x`` (bf16, last dim d) to e4m3 through
    ``fa_hadamard_quant``. Returns ``(codes, descale)``: uint8 codes shaped like
    ``x`` and a CUDA fp32 tensor of one element, ``amax / 448``."""
    _require_cuda(x)
    lib = load_library()
    if x.dtype != torch.bfloat16:
        raise FaError("x must be bf16")
    x = x.contiguous()
    d = x.shape[-1]
    rows = x.numel() // d if d else 0
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if descale is None:
        descale = torch.empty(1, dtype=torch.float32, device=x.device)
    if workspace is None:
        workspace = _workspace(x.device)
    _tensor_arg(out, "out", x.device, E4M3_DTYPES, tuple(x.shape))
    _tensor_arg(descale, "descale", x.device, (torch.float32,), min_bytes=4)
    _tensor_arg(workspace, "workspace", x.device, min_bytes=QUANT_WORKSPACE_BYTES)
    signs = _signs_arg(signs, d, x.device)
    with torch.cuda.device(x.device):
        rc = lib.fa_hadamard_quant(_ptr(x), _ptr(out), _ptr(descale), rows, d, int(bool(rotate)),
                                   _ptr(signs) if (rotate and signs is not None) else None, _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(x.device))
    _check(rc, "fa_hadamard_quant")
    return out, descale


def quant_v_transposed(v, out=None, descale=None, workspace=None):
    """V's e4m3 codes with one scale per tensor and no rotation, transposed per
    head, through ``fa_quant_v_transposed``: ``v`` bf16 ``[B, H, N, d]``.
    Returns ``(codes, descale)``: uint8 codes ``[B, H, d, N]`` (``codes[b, h, c,
    n]`` is v[b, h, n, c]'s code) and a CUDA fp32 tensor of one element, ``amax /
    448``."""
    _require_cuda(v)
    lib = load_library()
    if v.dtype != torch.bfloat16 or v.dim() != 4:
        raise FaError("v must be bf16 [B, H, N, d]")
    v = v.contiguous()
    B, H, N, d = v.shape
    if out is None:
        out = torch.empty((B, H, d, N), dtype=torch.uint8, device=v.device)
    if descale is None:
        descale = torch.empty(1, dtype=torch.float32, device=v.device)
    if workspace is None:
        workspace = _workspace(v.device)
    _tensor_arg(out, "out", v.device, E4M3_DTYPES, (B, H, d, N))
    _tensor_arg(descale, "descale", v.device, (torch.float32,), min_bytes=4)
    _tensor_arg(workspace, "workspace", v.device, min_bytes=QUANT_WORKSPACE_BYTES)
    with torch.cuda.device(v.device):
        rc = lib.fa_quant_v_transposed(_ptr(v), _ptr(out), _ptr(descale), B * H, N, d, _ptr(workspace),
                                       workspace.numel() * workspace.element_size(), _stream(v.device))
    _check(rc, "fa_quant_v_transposed")
    return out, descale


def hadamard_quant_multi(xs, rotate: bool = True, signs=None, outs=None, descales=None, workspace=None):
    """Rotate (optionally) and quantise up to 8 bf16 tensors of one shape (e.g.
    Q and K) in one launch through ``fa_hadamard_quant_multi``, each with its own
    scale. Returns ``(codes, descales)``: a list of uint8 code tensors and a CUDA
    fp32 tensor of one descale per input; the same as ``hadamard_quant`` per
    tensor."""
    xs = [x.contiguous() for x in xs]
    _require_cuda(*xs)
    lib = load_library()
    if not xs or any(x.dtype != torch.bfloat16 or x.shape != xs[0].shape for x in xs):
        raise FaError("xs must be bf16 tensors of one shape")
    d = xs[0].shape[-1]
    rows = xs[0].numel() // d if d else 0
    dev = xs[0].device
    if outs is None:
        outs = [torch.empty(x.shape, dtype=torch.uint8, device=dev) for x in xs]
    if descales is None:
        descales = torch.empty(len(xs), dtype=torch.float32, device=dev)
    if workspace is None:
        workspace = _workspace(dev)
    if len(outs) != len(xs):
        raise FaError("outs must hold one tensor per input")
    for i, o in enumerate(outs):
        _tensor_arg(o, f"outs[{i}]", dev, E4M3_DTYPES, tuple(xs[0].shape))
    _tensor_arg(descales, "descales", dev, (torch.float32,), min_bytes=4 * len(xs))
    _tensor_arg(workspace, "workspace", dev, min_bytes=QUANT_WORKSPACE_BYTES)
    signs = _signs_arg(signs, d, dev)
    n = len(xs)
    x_arr = (ctypes.c_void_p * n)(*[x.data_ptr() for x in xs])
    o_arr = (ctypes.c_void_p * n)(*[o.data_ptr() for o in outs])
    with torch.cuda.device(xs[0].device):
        rc = lib.fa_hadamard_quant_multi(x_arr, o_arr, _ptr(descales), n, rows, d, int(bool(rotate)),
                                         _ptr(signs) if (rotate and signs is not None) else None, _ptr(workspace),
                                         workspace.numel() * workspace.element_size(), _stream(xs[0].device))
    _check(rc, "fa_hadamard_quant_multi")
    return outs, descales


def hadamard_quant_blocks(x, rotate: bool = True, signs=None, out=None, descales=None):
    """Rotate (optionally) and quantise ``x`` (bf16 ``[B, H, N, d]``) to e4m3
    with one scale per block of 128 rows of each head, through
    ``fa_hadamard_quant_blocks``. Returns ``(codes, descales)``: uint8 codes
    shaped like ``x`` and CUDA fp32 ``[B, H, ceil(N/128)]``."""
    _require_cuda(x)
    lib = load_library()
    if x.dtype != torch.bfloat16 or x.dim() != 4:
        raise FaError("x must be bf16 [B, H, N, d]")
    x = x.contiguous()
    B, H, N, d = x.shape
    nb = -(-N // BLOCK_ROWS)
    if out is None:
        out = torch.empty(x.shape, dtype=torch.uint8, device=x.device)
    if descales is None:
        descales = torch.empty((B, H, nb), dtype=torch.float32, device=x.device)
    _tensor_arg(out, "out", x.device, E4M3_DTYPES, tuple(x.shape))
    _tensor_arg(descales, "descales", x.device, (torch.float32,), (B, H, nb))
    signs = _signs_arg(signs, d, x.device)
    with torch.cuda.device(x.device):
        rc = lib.fa_hadamard_quant_blocks(_ptr(x), _ptr(out), _ptr(descales), B * H, N, d, int(bool(rotate)),
                                          _ptr(signs) if (rotate and signs is not None) else None,
                                          _stream(x.device))
    _check(rc, "fa_hadamard_quant_blocks")
    return out, descales


def device_status():
    """(code, site, block) of the first device-side wait that ran out since the
    last call (code 0 = none); synchronises the current device."""
    lib = load_library()
    code, site, block = ctypes.c_int(), ctypes.c_uint(), ctypes.c_uint()
    _check(lib.fa_device_status(ctypes.byref(code), ctypes.byref(site), ctypes.byref(block)), "fa_device_status")
    return code.value, site.value, block.value
