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
_workspaces: dict[int, torch.Tensor] = {}

FA_OK, FA_ERR_INVALID_ARG, FA_ERR_UNSUPPORTED, FA_ERR_ALIGNMENT, FA_ERR_CUDA, FA_ERR_TIMEOUT = range(6)
FA_BF16, FA_E4M3 = 0, 1
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


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise FaError("tensors must be on a CUDA device")
    if not torch.cuda.is_available():
        raise FaError("no CUDA device")


def fwd(q, k, v, causal: bool = False, scale: float | None = None, qk_descale=None, out=None, lse=None,
        return_lse: bool = True):
    """Attention forward through ``fa_fwd``.

    q, k: ``[B, H, N, d]`` bf16, or e4m3 codes (uint8 / float8_e4m3fn) with
    ``qk_descale`` a CUDA fp32 tensor ``[dq, dk]``; v: bf16 ``[B, H, N, d]``.
    Returns ``(O, LSE)``: bf16 ``[B, H, N, d]`` and fp32 ``[B, H, N]`` (natural log);
    LSE is ``None`` when ``return_lse`` is false.
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
    if fp8 and (qk_descale is None or qk_descale.dtype != torch.float32 or qk_descale.numel() < 2):
        raise FaError("e4m3 q/k need qk_descale = CUDA fp32 tensor [dq, dk]")
    q, k, v = q.contiguous(), k.contiguous(), v.contiguous()
    if out is None:
        out = torch.empty((B, H, N, d), dtype=torch.bfloat16, device=q.device)
    if return_lse and lse is None:
        lse = torch.empty((B, H, N), dtype=torch.float32, device=q.device)
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    with torch.cuda.device(q.device):
        rc = lib.fa_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse) if return_lse else None, B, H, N, d,
                        int(bool(causal)), float(scale), FA_E4M3 if fp8 else FA_BF16,
                        _ptr(qk_descale.contiguous()) if fp8 else None, _stream(q.device))
    _check(rc, "fa_fwd")
    return out, (lse if return_lse else None)


def _workspace(device) -> torch.Tensor:
    idx = torch.device(device).index
    ws = _workspaces.get(idx)
    if ws is None:
        ws = torch.empty(QUANT_WORKSPACE_BYTES, dtype=torch.uint8, device=device)
        _workspaces[idx] = ws
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
    if signs is not None:
        signs = signs.to(device=x.device, dtype=torch.float32).contiguous()
    with torch.cuda.device(x.device):
        rc = lib.fa_hadamard_quant(_ptr(x), _ptr(out), _ptr(descale), rows, d, int(bool(rotate)),
                                   _ptr(signs) if (rotate and signs is not None) else None, _ptr(workspace),
                                   workspace.numel() * workspace.element_size(), _stream(x.device))
    _check(rc, "fa_hadamard_quant")
    return out, descale


def device_status():
    """(code, site, block) of the first device-side wait that ran out since the
    last call (code 0 = none); synchronises the current device."""
    lib = load_library()
    code, site, block = ctypes.c_int(), ctypes.c_uint(), ctypes.c_uint()
    _check(lib.fa_device_status(ctypes.byref(code), ctypes.byref(site), ctypes.byref(block)), "fa_device_status")
    return code.value, site.value, block.value
