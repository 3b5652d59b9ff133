"""GPU parity of the e4m3 attention with Q rotated and quantised inside the
attention kernel (fa_fwd_fp8_qrot): each 128-row query tile is rotated and
quantised with its own scale in shared memory ("FlashAttention-3 (PT)",
section "Inovações técnicas", subsection 3, steps 1-3, one scale per block of
128 rows), so the FP8 step needs no separate pass over Q.

* Bit for bit the same query-block descales as quantising Q first with
  fa_hadamard_quant_blocks and running the FA_E4M3_BLOCK attention (the
  in-kernel rotation is the same tensor-core product with the same operand,
  followed by the same amax and rounding steps, so the codes are the same),
  and, where both run two query tiles per CTA (N > 128), bit for bit the same
  O and LSE. For N <= 128 the FA_E4M3_BLOCK launch takes one query tile per
  CTA, which sums in another order, so O and LSE are compared there within
  the bf16 tolerance.
* The query-block descales against the oracle's per-block quantiser, and the
  output against oracle attention on the oracle's dequantised Q and K.
* The relative RMSE at the FP8 workload's shape against exact attention.
"""
import numpy as np
import pytest
import torch

import oracle
import io_aware_exact_17_b200 as fa
from io_aware_exact_17_b200 import inputs
from helpers import BF16_LSE_ATOL, BF16_O_ATOL, FP8_REL_RMSE, max_abs, record, rel_rmse, to_np

pytestmark = pytest.mark.gpu

BLOCK = 128


def _status_ok():
    torch.cuda.synchronize()
    code, site, block = fa.device_status()
    assert code == 0, f"device wait ran out at site {site}, block {block}"


@pytest.mark.parametrize("N", [1, 100, 128, 129, 300, 700, 2048])
@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("rotate,use_signs", [(True, True), (True, False), (False, False)])
def test_fused_q_equals_quantise_then_attend(N, causal, rotate, use_signs):
    B, H, d = 2, 3, 128
    q, k, v = (t.cuda() for t in inputs.qkv_normal(B, H, N, d, 100 + N))
    signs = inputs.hadamard_signs(d, 100).cuda() if use_signs else None
    k8, dk = fa.hadamard_quant_blocks(k, rotate=rotate, signs=signs)
    q8, dq = fa.hadamard_quant_blocks(q, rotate=rotate, signs=signs)
    o_ref, lse_ref = fa.fwd(q8, k8, v, causal=causal, qk_descale=(dq, dk), n_split=1)
    o, lse, dq_fused = fa.fwd_fp8_qrot(q, k8, v, dk, causal=causal, rotate=rotate, signs=signs, return_dq=True)
    _status_ok()
    assert torch.equal(dq_fused, dq)
    if N > 128:
        assert torch.equal(o, o_ref)
        assert torch.equal(lse, lse_ref)
    else:
        assert max_abs(to_np(o), to_np(o_ref)) <= BF16_O_ATOL
        assert max_abs(to_np(lse), to_np(lse_ref)) <= BF16_LSE_ATOL


@pytest.mark.parametrize("causal", [False, True])
def test_fused_q_against_the_oracle(causal):
    B, H, N, d = 1, 3, 700, 128
    q, k, v = inputs.qkv_normal(B, H, N, d, 110)
    signs = inputs.hadamard_signs(d, 110)
    k8, dk = fa.hadamard_quant_blocks(k.cuda(), rotate=True, signs=signs.cuda())
    o, lse, dq = fa.fwd_fp8_qrot(q.cuda(), k8, v.cuda(), dk, causal=causal, signs=signs.cuda(), return_dq=True)
    _status_ok()
    q_codes, q_ds = oracle.quantize_per_block(q, True, signs.numpy(), BLOCK)
    k_codes, k_ds = oracle.quantize_per_block(k, True, signs.numpy(), BLOCK)
    np.testing.assert_allclose(dq.cpu().double().numpy(), q_ds, rtol=1e-5, atol=0)

    def deq(codes, ds):
        return oracle.e4m3_decode(codes) * np.repeat(ds, BLOCK, axis=2)[:, :, :N, None]

    o_ref, lse_ref = oracle.attention(deq(q_codes, q_ds), deq(k_codes, k_ds), v, causal, d ** -0.5)
    # Codes decided in fp32 (kernel) and fp64 (oracle) may differ by one step
    # where a value sits at a rounding midpoint; the attention tolerance covers it.
    assert max_abs(to_np(o), o_ref) <= BF16_O_ATOL
    assert max_abs(to_np(lse), lse_ref) <= BF16_LSE_ATOL


def test_fused_q_fp8_config_rel_rmse():
    B, H, N, d = 2, 16, 8192, 128  # the FP8 workload's shape, plain N(0,1), sampled rows
    q, k, v = inputs.qkv_normal(B, H, N, d, 1003)
    signs = inputs.hadamard_signs(d, 1003).cuda()
    rows = inputs.sample_rows(B, H, N, per_head=16, seed=7).numpy()
    o_ref, _ = oracle.attention(q, k, v, False, d ** -0.5, rows=rows)
    k8, dk = fa.hadamard_quant_blocks(k.cuda(), rotate=True, signs=signs)
    o, _ = fa.fwd_fp8_qrot(q.cuda(), k8, v.cuda(), dk, signs=signs)
    _status_ok()
    err = rel_rmse(to_np(o).reshape(-1, d)[rows], o_ref)
    record(f"e4m3 QK, Q quantised in the kernel, B{B} H{H} N{N} d{d} N(0,1) rotated (sampled rows)", rel_rmse=err)
    assert err <= FP8_REL_RMSE


def test_fused_q_rejects_bad_arguments():
    q, k, v = (t.cuda() for t in inputs.qkv_normal(1, 1, 256, 64, 111))
    k8 = torch.zeros_like(k, dtype=torch.uint8)
    dk = torch.ones(1, 1, 2, device="cuda")
    with pytest.raises(fa.FaError):  # d = 64: only d = 128 is rotated in the kernel
        fa.fwd_fp8_qrot(q, k8, v, dk)
    q, k, v = (t.cuda() for t in inputs.qkv_normal(1, 1, 256, 128, 111))
    with pytest.raises(fa.FaError, match="shape"):
        fa.fwd_fp8_qrot(q, torch.zeros_like(k, dtype=torch.uint8), v, torch.ones(1, 1, 3, device="cuda"))
