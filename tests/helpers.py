"""Small shared pieces of the GPU parity tests (comparison and tolerances)."""
import numpy as np
import torch

# Tolerances of the forward pass against the fp64 oracle (N(0,1) inputs):
# BF16 O max-abs 1e-2 and LSE max-abs 1e-3; FP8 relative RMSE 5e-2.
BF16_O_ATOL = 1e-2
BF16_LSE_ATOL = 1e-3
FP8_REL_RMSE = 5e-2


def bf16_out_tol(o_ref: np.ndarray) -> np.ndarray:
    """Element tolerance for inputs outside the N(0,1), scale 1/sqrt(d) regime:
    the 1e-2 bound plus the bf16 half-ulp of the exact output (2^-8 |O|), since
    O is returned rounded to bf16 and large-logit rows can have |O| near max|V|."""
    return BF16_O_ATOL + 2.0**-8 * np.abs(o_ref)


def to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().double().numpy()


def rel_rmse(a: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(a - ref) / np.linalg.norm(ref))


def max_abs(a: np.ndarray, ref: np.ndarray) -> float:
    return float(np.max(np.abs(a - ref))) if a.size else 0.0


def record(case: str, **values) -> None:
    """Append one JSON line {case, values...} to the file named by the
    FA_PARITY_LOG environment variable, if set: the measured errors of a GPU
    parity run, kept for reporting. Does nothing otherwise."""
    import json
    import os

    path = os.environ.get("FA_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": case, **{k: float(v) for k, v in values.items()}}) + "\n")


def rotation_error_bound(x: np.ndarray, rotate: bool) -> np.ndarray:
    """Bound on |x'_kernel - x'_exact| for each element of x' = x D H_d / sqrt(d)
    (rows of x along the last axis, fp64), as the kernels compute it: each value
    of x D H_d is a tensor-core sum of d exact products +-x_k in fp32, in an
    order and with a rounding (nearest or towards zero) the hardware does not
    document. Each of its d - 1 additions errs by at most one fp32 unit (2^-23)
    of a partial sum bounded by sum_k |x_k|, so the error is below
    d 2^-23 sum_k |x_k| (at d = 256 this also covers the one fp32 addition of
    the last butterfly stage); then / sqrt(d). Without rotation the kernels
    reproduce x exactly (a product with the identity): bound 0."""
    if not rotate:
        return np.zeros_like(x)
    d = x.shape[-1]
    l1 = np.abs(x).sum(axis=-1, keepdims=True)
    return np.broadcast_to(d * 2.0**-23 * l1 / np.sqrt(d), x.shape)
