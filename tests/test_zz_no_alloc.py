"""fa_hadamard_quant_noalloc: the quantiser for callers that cannot allocate
device memory (no workspace; its scratch is an array inside the library).

Called through the C ABI and checked against fa_hadamard_quant (the entry point
with a caller-provided workspace), on two calls in a row: the second call uses
inputs of much smaller magnitude, so a scratch word left over from the first
call would show up as a wrong scale. This file is collected last so that a
failure here does not stop the rest of a stop-at-first-failure run.
"""
import ctypes

import pytest
import torch

from io_aware_exact_17_b200 import binding, inputs

pytestmark = pytest.mark.gpu


def _lib():
    lib = binding.load_library()
    f = lib.fa_hadamard_quant_noalloc
    f.argtypes = [ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_void_p), ctypes.c_void_p, ctypes.c_int,
                  ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p]
    f.restype = ctypes.c_int
    return lib


def _noalloc(lib, xs, outs, descales, rotate, signs):
    n = len(xs)
    rows, d = xs[0].numel() // xs[0].shape[-1], xs[0].shape[-1]
    x_arr = (ctypes.c_void_p * n)(*[x.data_ptr() for x in xs])
    o_arr = (ctypes.c_void_p * n)(*[o.data_ptr() for o in outs])
    return lib.fa_hadamard_quant_noalloc(
        x_arr, o_arr, ctypes.c_void_p(descales.data_ptr()), n, rows, d, int(rotate),
        ctypes.c_void_p(signs.data_ptr()) if signs is not None else None,
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("rotate", [True, False])
def test_noalloc_matches_workspace_entry_point_on_two_calls(rotate):
    lib = _lib()
    B, H, N, d = 2, 4, 1000, 128
    signs = inputs.hadamard_signs(d, seed=5).cuda() if rotate else None
    q, k, _ = inputs.qkv_normal(B, H, N, d, seed=61)
    q, k = inputs.with_outliers_r1(q, k, seed=61)            # call 1: large amax
    q2, k2, _ = inputs.qkv_normal(B, H, N, d, seed=62)
    q2, k2 = (q2.float() * 0.01).to(torch.bfloat16), (k2.float() * 0.01).to(torch.bfloat16)  # call 2: small amax
    for xs in ((q, k), (q2, k2)):
        xs = [x.cuda() for x in xs]
        outs = [torch.empty(x.shape, dtype=torch.uint8, device="cuda") for x in xs]
        desc = torch.empty(len(xs), dtype=torch.float32, device="cuda")
        assert _noalloc(lib, xs, outs, desc, rotate, signs) == binding.FA_OK
        torch.cuda.synchronize()
        for i, x in enumerate(xs):
            ref_codes, ref_desc = binding.hadamard_quant(x, rotate=rotate, signs=signs)
            torch.cuda.synchronize()
            assert torch.equal(outs[i], ref_codes)
            assert float(desc[i].item()) == float(ref_desc.item())


def test_noalloc_rejects_more_tensors_than_its_scratch_holds():
    lib = _lib()
    x = torch.zeros(4, 128, dtype=torch.bfloat16, device="cuda")
    o = torch.empty(4, 128, dtype=torch.uint8, device="cuda")
    desc = torch.empty(65, dtype=torch.float32, device="cuda")
    assert _noalloc(lib, [x] * 65, [o] * 65, desc, True, None) == binding.FA_ERR_INVALID_ARG
    assert _noalloc(lib, [x] * 64, [o] * 64, desc, True, None) == binding.FA_OK
    torch.cuda.synchronize()
    assert torch.all(desc[:64] == 1.0)
