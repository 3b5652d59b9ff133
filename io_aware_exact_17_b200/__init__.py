"""Fused exact-attention forward for B200 (sm_100a): BF16 and FP8-e4m3 kernels,
the BF16 backward pass, the Hadamard rotate-and-quantise step of the FP8 path,
and attention of few
queries over long key sequences with the keys split across CTAs and merged by
their LSEs.

The compute lives in ``libfa.so`` (CUDA, built from ``csrc/``); this package is
its Python binding. Importing the package does not load the library; the first
call does, and fails loudly if the library or a GPU is missing.
"""
from .binding import (  # noqa: F401
    FaError,
    bwd,
    bwd_workspace_bytes,
    device_status,
    fwd,
    fwd_fp8_qrot,
    fwd_partial,
    fwd_splitkv,
    hadamard_quant,
    hadamard_quant_blocks,
    hadamard_quant_multi,
    quant_v_transposed,
    library_path,
    load_library,
    lse_merge,
    splitkv_splits,
)

__all__ = ["fwd", "fwd_fp8_qrot", "bwd", "bwd_workspace_bytes", "fwd_splitkv", "fwd_partial", "lse_merge", "splitkv_splits", "hadamard_quant",
           "hadamard_quant_blocks", "hadamard_quant_multi", "quant_v_transposed", "device_status", "load_library", "library_path", "FaError"]
