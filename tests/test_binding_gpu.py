"""The Python binding on a GPU: caller-supplied outputs and workspaces that do
not fit are refused before any launch, and calls issued on two CUDA streams at
once (each stream with its own cached split-key and quantiser workspace) both
match the fp64 oracle."""
import numpy as np
import pytest
import torch

import oracle
import io_aware_exact_17_b200 as fa
from io_aware_exact_17_b200 import inputs
from helpers import BF16_LSE_ATOL, BF16_O_ATOL, max_abs, to_np

pytestmark = pytest.mark.gpu


def test_bad_outputs_and_workspaces_are_refused():
    q, k, v = (t.cuda() for t in inputs.qkv_normal(1, 2, 256, 128, seed=71))
    good = torch.empty_like(q)
    with pytest.raises(fa.FaError, match="CUDA"):
        fa.fwd(q, k, v, out=torch.empty(q.shape, dtype=torch.bfloat16))            # host output
    with pytest.raises(fa.FaError, match="shape"):
        fa.fwd(q, k, v, out=good[:, :, :255])                                       # short output
    with pytest.raises(fa.FaError, match="contiguous"):
        fa.fwd(q, k, v, out=good.transpose(2, 3).contiguous().transpose(2, 3))      # strided output
    with pytest.raises(fa.FaError, match="dtype"):
        fa.fwd(q, k, v, lse=torch.empty(1, 2, 256, dtype=torch.float16, device="cuda"))
    with pytest.raises(fa.FaError, match="bytes"):
        fa.fwd_splitkv(q, k, v, n_split=2, workspace=torch.empty(16, dtype=torch.uint8, device="cuda"))
    with pytest.raises(fa.FaError, match="shape"):
        fa.fwd_partial(q, k, v, n_split=2, o_part=torch.empty(1, 1, 2, 256, 128, device="cuda"))
    with pytest.raises(fa.FaError, match="CUDA"):
        fa.hadamard_quant(q, descale=torch.empty(1))                                # host descale
    with pytest.raises(fa.FaError, match="bytes"):
        fa.hadamard_quant(q, workspace=torch.empty(255, dtype=torch.uint8, device="cuda"))
    with pytest.raises(fa.FaError, match="shape"):
        fa.hadamard_quant_multi([q, k], outs=[torch.empty_like(q, dtype=torch.uint8),
                                              torch.empty(3, dtype=torch.uint8, device="cuda")])
    with pytest.raises(fa.FaError, match="signs"):
        fa.hadamard_quant(q, signs=torch.ones(64))
    with pytest.raises(fa.FaError, match="bytes"):
        fa.bwd(q, k, v, good, torch.empty(1, 2, 256, device="cuda"), good,
               workspace=torch.empty(64, dtype=torch.uint8, device="cuda"))
    torch.cuda.synchronize()
    assert fa.device_status()[0] == 0


def test_two_streams_at_once_match_the_oracle():
    # Few query blocks, so fwd() takes the split-key schedule and its workspace;
    # the quantiser uses its amax workspace. Both run on two streams at once.
    B, H, N, d = 1, 4, 2048, 128
    cases = [inputs.qkv_normal(B, H, N, d, seed=80 + i) for i in range(2)]
    dev = [tuple(t.cuda() for t in c) for c in cases]
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    results = [None, None]
    for rep in range(3):
        for i, s in enumerate(streams):
            with torch.cuda.stream(s):
                q, k, v = dev[i]
                o, lse = fa.fwd(q, k, v, causal=bool(i))
                codes, ds = fa.hadamard_quant(q, rotate=True)
                results[i] = (o, lse, codes, ds)
        torch.cuda.synchronize()
        for i, (q, k, v) in enumerate(cases):
            o, lse, codes, ds = results[i]
            rows = np.arange(0, B * H * N, 97)
            o_ref, lse_ref = oracle.attention(q, k, v, bool(i), d ** -0.5, rows=rows)
            got_o = to_np(o).reshape(-1, d)[rows]
            got_lse = to_np(lse).reshape(-1)[rows]
            assert max_abs(got_o, o_ref) <= BF16_O_ATOL and max_abs(got_lse, lse_ref) <= BF16_LSE_ATOL
            _, ref_ds = oracle.quantize_per_tensor(q.reshape(-1, d), True)
            assert float(ds.item()) == pytest.approx(ref_ds, rel=1e-5)
    assert fa.device_status()[0] == 0
