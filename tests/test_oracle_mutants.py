"""The oracle's pins must be able to fail. Each case here plants one
plausible mistake in a private copy of the oracle's C source (a dropped scale,
a dropped mask, an off-by-one key range, a wrong operand index, a transposed
value operand, a dropped normalisation, an LSE without the max, an unshifted
exponent, a causal mask that ignores the query offset, a key range whose start
or end is ignored, an empty row with a finite LSE), builds it, and checks that
at least one pin rejects it. Nothing here touches the real oracle library.
"""
import ctypes
import json
import subprocess
from pathlib import Path

import numpy as np
import pytest

import oracle

ROOT = Path(__file__).resolve().parents[1]
SRC = (ROOT / "oracle" / "attn_oracle.c").read_text()
GOLDEN = json.loads((ROOT / "tests" / "golden" / "attention_closed_form.json").read_text())

MUTANTS = {
    "dropped_scale": ("z[j] = jb->scale * dot;", "z[j] = dot;"),
    "dropped_mask": ("if (jb->causal && i + (Nk - Nq) < last) last = i + (Nk - Nq);", ""),
    "off_by_one_keys": ("int last = (jb->hi < Nk ? jb->hi : Nk) - 1;", "int last = (jb->hi < Nk ? jb->hi : Nk) - 2 + (Nk == 1);"),
    "causal_offset_ignored": ("i + (Nk - Nq) < last) last = i + (Nk - Nq);", "i < last) last = i;"),
    "range_start_ignored": ("const int first = jb->lo;", "const int first = 0;"),
    "range_end_ignored": ("int last = (jb->hi < Nk ? jb->hi : Nk) - 1;", "int last = Nk - 1;"),
    "empty_row_not_empty": ("jb->lse[out_idx] = -INFINITY;", "jb->lse[out_idx] = 0.0;"),
    "wrong_k_index": ("dot += qi[c] * kj[c];", "dot += qi[c] * kj[0];"),
    "transposed_v": ("oi[c] += z[j] * vj[c];", "oi[c] += z[j] * vj[d - 1 - c];"),
    "no_normalisation": ("oi[c] /= l;", "oi[c] /= 1.0;"),
    "lse_without_max": ("jb->lse[out_idx] = m + log(l);", "jb->lse[out_idx] = log(l);"),
    "unshifted_exp": ("z[j] = exp(z[j] - m);", "z[j] = exp(z[j]);"),
}


def _build(tmp_path, name, src):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(src)
    subprocess.run(["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-pthread", "-o", str(so), str(c), "-lm"],
                   check=True)
    lib = ctypes.CDLL(str(so))
    dp = ctypes.POINTER(ctypes.c_double)
    lib.oracle_attn_rows.argtypes = [dp, dp, dp] + [ctypes.c_int] * 5 + [
        ctypes.c_double, ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, dp, dp, ctypes.c_int]
    lib.oracle_attn_rows.restype = ctypes.c_int
    lib.oracle_attn_range_rows.argtypes = [dp, dp, dp] + [ctypes.c_int] * 6 + [
        ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, dp, dp,
        ctypes.c_int]
    lib.oracle_attn_range_rows.restype = ctypes.c_int
    return lib


def _run(lib, q, k, v, causal, scale):
    B, H, N, d = q.shape
    dp = ctypes.POINTER(ctypes.c_double)
    q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
    o = np.zeros((B * H * N, d))
    lse = np.zeros(B * H * N)
    with np.errstate(all="ignore"):
        rc = lib.oracle_attn_rows(q.ctypes.data_as(dp), k.ctypes.data_as(dp), v.ctypes.data_as(dp), B, H, N, d,
                                  int(causal), scale, None, B * H * N, o.ctypes.data_as(dp),
                                  lse.ctypes.data_as(dp), 1)
    assert rc == 0
    return o.reshape(B, H, N, d), lse.reshape(B, H, N)


def _run_range(lib, q, k, v, causal, scale, lo, hi):
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    dp = ctypes.POINTER(ctypes.c_double)
    q, k, v = (np.ascontiguousarray(x, dtype=np.float64) for x in (q, k, v))
    o = np.zeros((B * H * Nq, d))
    lse = np.zeros(B * H * Nq)
    with np.errstate(all="ignore"):
        rc = lib.oracle_attn_range_rows(q.ctypes.data_as(dp), k.ctypes.data_as(dp), v.ctypes.data_as(dp), B, H, Nq,
                                        Nk, d, int(causal), scale, lo, hi, None, B * H * Nq, o.ctypes.data_as(dp),
                                        lse.ctypes.data_as(dp), 1)
    assert rc == 0
    return o.reshape(B, H, Nq, d), lse.reshape(B, H, Nq)


def _same(o, lse, o2, lse2) -> bool:
    with np.errstate(all="ignore"):
        return bool(np.allclose(o, o2, rtol=0, atol=1e-12) and np.array_equal(np.isneginf(lse), np.isneginf(lse2))
                    and np.allclose(np.where(np.isinf(lse), 0, lse), np.where(np.isinf(lse2), 0, lse2), rtol=0,
                                    atol=1e-12))


def _pins_pass(lib) -> bool:
    """The oracle pins, run against `lib`; True only if every one holds."""
    ok = True
    q = np.array(GOLDEN["q"])[None, None]
    k = np.array(GOLDEN["k"])[None, None]
    v = np.array(GOLDEN["v"])[None, None]
    for mode, causal in (("non_causal", False), ("causal", True)):
        o, lse = _run(lib, q, k, v, causal, GOLDEN["scale"])
        ok &= np.allclose(o[0, 0, :, 0], GOLDEN[mode]["O"]["value"], rtol=0, atol=1e-15)
        ok &= np.allclose(lse[0, 0], GOLDEN[mode]["LSE"]["value"], rtol=0, atol=1e-15)
    rng = np.random.default_rng(0)
    for shape in ((1, 2, 17, 16), (1, 1, 40, 8)):
        q, k, v = (rng.standard_normal(shape) for _ in range(3))
        for causal in (False, True):
            o, lse = _run(lib, q, k, v, causal, 0.37)
            o2, lse2 = oracle.attention_naive(q, k, v, causal, 0.37)
            ok &= np.allclose(o, o2, rtol=0, atol=1e-12) and np.allclose(lse, lse2, rtol=0, atol=1e-12)
    # dominant key with a logit gap of ~1000
    N, d = 16, 4
    q = np.zeros((1, 1, N, d))
    q[..., 0] = 1.0
    k = rng.standard_normal((1, 1, N, d)) * 0.1
    k[0, 0, 5, 0] = 1000.0
    v = rng.standard_normal((1, 1, N, d))
    o, _ = _run(lib, q, k, v, False, 1.0)
    ok &= np.allclose(o[0, 0], np.broadcast_to(v[0, 0, 5], (N, d)), rtol=0, atol=1e-12)
    # fewer queries than keys, and key ranges, against the materialised routine
    q = rng.standard_normal((1, 2, 5, 8))
    k, v = rng.standard_normal((1, 2, 19, 8)), rng.standard_normal((1, 2, 19, 8))
    for causal in (False, True):
        for lo, hi in ((0, 19), (3, 11), (15, 19)):
            o, lse = _run_range(lib, q, k, v, causal, 0.45, lo, hi)
            o2, lse2 = oracle.attention_naive(q, k, v, causal, 0.45, key_range=(lo, hi))
            ok &= _same(o, lse, o2, lse2)
    return bool(ok)


def test_unmutated_copy_passes_the_pins(tmp_path):
    assert _pins_pass(_build(tmp_path, "clean", SRC))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_each_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTANTS[name]
    assert SRC.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    assert not _pins_pass(_build(tmp_path, name, SRC.replace(old, new)))


# ------------------------------------------------- rotation sign order --
# M = D H_d / sqrt(d) (signs first, "FlashAttention-3 (PT)", "Inovações
# técnicas do FlashAttention-3", subsection 3, step 1). The mistaken order
# H_d D / sqrt(d) is orthogonal and keeps Q Kᵀ too, so orthogonality and
# invariance pins cannot catch it; the hand-derived golden values must.
ROTATION_MUTANTS = {
    "signs_after_hadamard": ("return s[:, None] * h", "return h * s[None, :]"),
    "signs_ignored": ("return s[:, None] * h", "return h"),
    "unnormalised": ("h = sylvester_hadamard(d) / np.sqrt(d)", "h = sylvester_hadamard(d)"),
}


def _rotation_mutant(name):
    import inspect

    src = inspect.getsource(oracle.rotation_matrix)
    old, new = ROTATION_MUTANTS[name]
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    ns = {"np": np, "sylvester_hadamard": oracle.sylvester_hadamard, "_as_f64": oracle._as_f64}
    exec(src.replace(old, new), ns)
    return ns["rotation_matrix"]


def test_rotation_golden_accepts_the_oracle():
    from test_codec import rotation_golden_holds

    assert rotation_golden_holds(oracle.rotation_matrix)


@pytest.mark.parametrize("name", sorted(ROTATION_MUTANTS))
def test_each_planted_rotation_mistake_is_caught(name):
    from test_codec import rotation_golden_holds

    assert not rotation_golden_holds(_rotation_mutant(name))
