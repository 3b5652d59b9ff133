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
    assert lib.fa_abi_version() == 1


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


def test_python_binding_rejects_cpu_tensors():
    import torch

    q = torch.zeros(1, 1, 4, 64, dtype=torch.bfloat16)
    with pytest.raises(binding.FaError):
        binding.fwd(q, q, q)
    with pytest.raises(binding.FaError):
        binding.hadamard_quant(q)
