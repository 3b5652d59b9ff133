"""A bounded wait that runs out, on purpose, without faulting or hanging the GPU.

Every mbarrier wait in the kernels gives up after a time limit, records
(FA_ERR_TIMEOUT, site, block) in the library's device status word, and makes
every role of the CTA stop and drain its copies and tensor-core operations in
flight before tensor memory is freed. This test runs that path: it loads the
test build of the library (``libfa_testhooks.so``: the same sources with a 5 ms
wait limit and one test hook), arms the hook so that one softmax warp of CTA 0
leaves out its plain software arrival on the P barrier at key tile 1, and
checks that

* the launch returns and block 0 reports a wait that the missing arrival
  starves first: the MMA issuer's wait for that P (site 23), or the TMA
  producer's wait for a ring slot that only the MMAs after that P would free
  (site 10; it can start a little earlier than the issuer's);
* the next launch of the same library, hook cleared, matches the oracle and
  reports no error;
* the product library on the same device still matches the oracle.
"""
import ctypes

import pytest
import torch

import oracle
import io_aware_exact_17_b200 as fa
from io_aware_exact_17_b200 import binding, build, inputs
from helpers import BF16_LSE_ATOL, BF16_O_ATOL, max_abs, to_np

pytestmark = pytest.mark.gpu

SITE_MMA_WAITS_FOR_P = 23  # the MMA issuer's wait on the P barrier of a query tile
SITE_PRODUCER_WAITS_FOR_SLOT = 10  # the TMA producer's wait for a free K/V ring slot


def _test_lib():
    lib = ctypes.CDLL(str(build.build_test_hooks()))
    vp, i, f = ctypes.c_void_p, ctypes.c_int, ctypes.c_float
    lib.fa_fwd.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, vp, vp]
    lib.fa_fwd.restype = i
    lib.fa_device_status.argtypes = [ctypes.POINTER(i), ctypes.POINTER(ctypes.c_uint), ctypes.POINTER(ctypes.c_uint)]
    lib.fa_device_status.restype = i
    lib.fa_test_withhold_p_arrive.argtypes = [i]
    lib.fa_test_withhold_p_arrive.restype = i
    return lib


def _status(lib):
    code, site, block = ctypes.c_int(), ctypes.c_uint(), ctypes.c_uint()
    assert lib.fa_device_status(ctypes.byref(code), ctypes.byref(site), ctypes.byref(block)) == binding.FA_OK
    return code.value, site.value, block.value


def _fwd(lib, q, k, v, o, lse):
    B, H, N, d = q.shape
    return lib.fa_fwd(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()), ctypes.c_void_p(v.data_ptr()),
                      ctypes.c_void_p(o.data_ptr()), ctypes.c_void_p(lse.data_ptr()), B, H, N, d, 0, d ** -0.5,
                      binding.FA_BF16, None, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _check_parity(o, lse, q, k, v):
    d = q.shape[-1]
    o_ref, lse_ref = oracle.attention(q, k, v, False, d ** -0.5)
    assert max_abs(to_np(o), o_ref) <= BF16_O_ATOL
    assert max_abs(to_np(lse), lse_ref) <= BF16_LSE_ATOL


def test_withheld_arrival_times_out_and_the_device_recovers():
    lib = _test_lib()
    B, H, N, d = 1, 2, 1024, 128
    q, k, v = inputs.qkv_normal(B, H, N, d, seed=90)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qc)
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    assert _status(lib)[0] == 0

    # 1. one arrival withheld: the launch returns and reports where it gave up
    assert lib.fa_test_withhold_p_arrive(1) == 0
    assert _fwd(lib, qc, kc, vc, o, lse) == binding.FA_OK
    torch.cuda.synchronize()
    code, site, block = _status(lib)
    assert code == binding.FA_ERR_TIMEOUT and block == 0, (code, site, block)
    assert site in (SITE_MMA_WAITS_FOR_P, SITE_PRODUCER_WAITS_FOR_SLOT), site

    # 2. the hook cleared itself: the same library computes the right result
    o.zero_()
    assert _fwd(lib, qc, kc, vc, o, lse) == binding.FA_OK
    torch.cuda.synchronize()
    assert _status(lib) == (0, 0, 0)
    _check_parity(o, lse, q, k, v)

    # 3. the product library on the same device is unaffected
    o2, lse2 = fa.fwd(qc, kc, vc, n_split=1)
    torch.cuda.synchronize()
    assert fa.device_status()[0] == 0
    _check_parity(o2, lse2, q, k, v)
