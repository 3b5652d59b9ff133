"""TEST INFRASTRUCTURE ONLY — the CPU oracle for the attention forward pass and
for the FP8 (e4m3) rotate-and-quantise step.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package. The CUDA
library never does, and this package imports nothing from the library.

Pieces, each citing the passage it follows:

* :func:`attention` — exact attention in fp64, row by row, in plain C
  (``attn_oracle.c``). Definition: "Flash Attention" glossary page, first two
  paragraphs (same result as standard attention; standard attention forms the
  N x N matrix).
  Queries may be fewer than keys (the queries are then the last positions of
  the sequence, for the causal mask), and a key range restricts the softmax to
  one block of keys: the partial result the glossary page's online softmax
  accumulates (second paragraph).
* :func:`attention_naive` — a second, independently written fp64 routine that
  materialises the whole N x N score and probability matrices, i.e. the
  "standard attention" of "FlashAttention-3 (PT)", section "O problema do
  mecanismo de atenção". Used to cross-check :func:`attention` on tiny inputs.
* :func:`lse_merge` — combines results over disjoint key blocks into the
  result over their union, from their LSEs: the online-softmax rescale of the
  glossary page (second paragraph) applied to whole partial results, as
  splitting the keys over several processors needs (same page, fourth
  paragraph, ring attention over several devices).
* :func:`attention_bwd` — the gradients dQ, dK, dV of a scalar loss through
  exact attention, given dO = dLoss/dO. The pages name training with the method
  ("FlashAttention-3 (PT)", opening paragraph and section "Desempenho e
  importância": faster training)
  but print no backward algorithm, so this is the chain rule through the plain
  definition, written out with the whole N x N probability matrix per head:
  dV = Pᵀ dO, dP = dO Vᵀ, dS = P ∘ (dP - rowsum(P ∘ dP)) (the softmax Jacobian),
  dQ = scale dS K, dK = scale dSᵀ Q. fp64 numpy.
* :func:`sylvester_hadamard`, :func:`rotation_matrix`, :func:`rotate` — the
  orthogonal transform of "FlashAttention-3 (PT)", section "Inovações técnicas",
  subsection 3 ("Baixa precisão (FP8)"), steps 1 and 4: Q and K multiplied by a
  random orthogonal (Hadamard) matrix, which leaves Q Kᵀ unchanged.
* :func:`e4m3_decode`, :func:`e4m3_encode` — the 8-bit e4m3 format (OCP 8-bit
  floating point, E4M3: bias 7, no infinities, one NaN pattern per sign, largest
  finite 448), encoded with round-to-nearest-even and saturation.
* :func:`quantize_per_tensor` — step 3 of the same subsection ("quantização para
  FP8") with one scale per tensor: descale = amax/448 after rotation.
* :func:`quantize_per_block` — the same step with one scale per block of 128
  consecutive rows of a head (the attention kernel's tile), so that a block's
  codes use the range its own values need. The pages name no block size; this is
  the finer-grained variant of the per-tensor step.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
_SRC = _HERE / "attn_oracle.c"
_LIB_PATH = _HERE / "liboracle.so"
_lib = None

E4M3_MAX = 448.0


def build(force: bool = False) -> Path:
    """Compile ``attn_oracle.c`` into ``liboracle.so`` next to it (gcc, -O2, IEEE math)."""
    if force or not _LIB_PATH.exists() or _LIB_PATH.stat().st_mtime < _SRC.stat().st_mtime:
        tmp = _LIB_PATH.with_suffix(".so.tmp")
        subprocess.run(
            ["gcc", "-std=c99", "-O2", "-fPIC", "-shared", "-pthread", "-o", str(tmp), str(_SRC), "-lm"],
            check=True,
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(str(_LIB_PATH))
        dp = ctypes.POINTER(ctypes.c_double)
        lib.oracle_attn_rows.argtypes = [
            dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_double,
            ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, dp, dp, ctypes.c_int,
        ]
        lib.oracle_attn_rows.restype = ctypes.c_int
        lib.oracle_attn_range_rows.argtypes = [
            dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
            ctypes.c_double, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int64), ctypes.c_int64, dp, dp,
            ctypes.c_int,
        ]
        lib.oracle_attn_range_rows.restype = ctypes.c_int
        _lib = lib
    return _lib


def default_threads() -> int:
    return len(os.sched_getaffinity(0))


def _as_f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor: widen exactly on the host
        x = x.detach().cpu().double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def attention(q, k, v, causal: bool, scale: float, rows=None, threads: int | None = None, key_range=None):
    """Exact attention in fp64 of ``q`` ``[B, H, Nq, d]`` over ``k``, ``v``
    ``[B, H, Nk, d]``.

    ``causal``: key j is visible to query i iff j <= i + (Nk - Nq) (the queries
    are the last Nq positions; for Nq = Nk, j <= i). ``key_range=(lo, hi)``:
    only keys lo <= j < hi take part (default: all); rows left with no key get
    O = 0 and LSE = -inf. ``rows``: optional flat row ids ``(b*H + h)*Nq + i``;
    if given, only those rows are computed and the result has shape
    ``[len(rows), d]`` / ``[len(rows)]``, otherwise ``[B, H, Nq, d]`` /
    ``[B, H, Nq]``. Returns ``(O, LSE)`` with the natural-log LSE.
    """
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    if q.ndim != 4 or k.shape != v.shape or k.ndim != 4 or q.shape[:2] != k.shape[:2] or q.shape[3] != k.shape[3]:
        raise ValueError("q must be [B, H, Nq, d] and k, v one [B, H, Nk, d] shape")
    B, H, Nq, d = q.shape
    Nk = k.shape[2]
    lo, hi = (0, Nk) if key_range is None else (int(key_range[0]), int(key_range[1]))
    lib = _load()
    dp = ctypes.POINTER(ctypes.c_double)
    if rows is None:
        nrows = B * H * Nq
        rows_arr = None
        rows_ptr = None
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        nrows = rows_arr.size
        rows_ptr = rows_arr.ctypes.data_as(ctypes.POINTER(ctypes.c_int64))
    o = np.zeros((nrows, d), dtype=np.float64)
    lse = np.zeros((nrows,), dtype=np.float64)
    rc = lib.oracle_attn_range_rows(
        q.ctypes.data_as(dp), k.ctypes.data_as(dp), v.ctypes.data_as(dp), B, H, Nq, Nk, d, int(bool(causal)),
        float(scale), lo, hi, rows_ptr, nrows, o.ctypes.data_as(dp), lse.ctypes.data_as(dp),
        int(threads or default_threads()),
    )
    if rc != 0:
        raise RuntimeError(f"oracle_attn_range_rows failed with code {rc}")
    if rows is None:
        return o.reshape(B, H, Nq, d), lse.reshape(B, H, Nq)
    return o, lse


def attention_naive(q, k, v, causal: bool, scale: float, return_probs: bool = False, key_range=None):
    """Standard attention: materialise S = scale*Q Kᵀ (Nq x Nk per head), mask,
    softmax along keys, then P V. fp64 numpy; for small sizes only.

    Masked scores are -inf: keys j > i + (Nk - Nq) when causal, and keys outside
    ``key_range = (lo, hi)``. A row with every key masked has P = 0, O = 0 and
    LSE = -inf."""
    q, k, v = _as_f64(q), _as_f64(k), _as_f64(v)
    Nq, Nk = q.shape[-2], k.shape[-2]
    s = scale * np.einsum("bhid,bhjd->bhij", q, k)
    i = np.arange(Nq)[:, None]
    j = np.arange(Nk)[None, :]
    hidden = np.zeros((Nq, Nk), dtype=bool)
    if causal:
        hidden |= j > i + (Nk - Nq)
    if key_range is not None:
        hidden |= (j < key_range[0]) | (j >= key_range[1])
    s = np.where(hidden, -np.inf, s)
    row_max = s.max(axis=-1, keepdims=True)
    empty = np.isneginf(row_max)
    w = np.where(empty, 0.0, np.exp(s - np.where(empty, 0.0, row_max)))
    denom = w.sum(axis=-1, keepdims=True)
    p = w / np.where(empty, 1.0, denom)
    o = np.einsum("bhij,bhjd->bhid", p, v)
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, row_max + np.log(denom))[..., 0]
    if return_probs:
        return o, lse, p
    return o, lse


def lse_merge(o_parts, lse_parts):
    """Result over the union of disjoint key blocks from the results over each.

    ``o_parts`` ``[S, ..., d]`` and ``lse_parts`` ``[S, ...]`` hold, for each
    block s, the normalised output O_s and the natural-log LSE_s (-inf for a row
    that saw no key of block s). With M = max_s LSE_s and w_s = exp(LSE_s - M):
    LSE = M + ln(sum_s w_s) and O = sum_s w_s O_s / sum_s w_s, since
    exp(LSE_s) is the softmax denominator of block s. Rows with no key in any
    block get O = 0 and LSE = -inf. fp64."""
    o_parts = _as_f64(o_parts)
    lse_parts = _as_f64(lse_parts)
    m = lse_parts.max(axis=0)
    empty = np.isneginf(m)
    w = np.where(empty[None], 0.0, np.exp(lse_parts - np.where(empty, 0.0, m)[None]))
    total = w.sum(axis=0)
    o = (w[..., None] * o_parts).sum(axis=0) / np.where(empty, 1.0, total)[..., None]
    with np.errstate(divide="ignore"):
        lse = np.where(empty, -np.inf, m + np.log(np.where(empty, 1.0, total)))
    return o, lse


def attention_bwd(q, k, v, do, causal: bool, scale: float, return_bounds: bool = False):
    """Gradients of a loss L through O = softmax(scale Q Kᵀ) V, per (batch, head),
    for square heads (N queries over the same N positions' keys).

    ``do`` is dL/dO ``[B, H, N, d]``; ``causal`` hides key j from query i when
    j > i. Per head, with S = scale Q Kᵀ (hidden entries -inf) and P its row
    softmax:

    * dV = Pᵀ dO;
    * dP = dO Vᵀ and, since dP_i·P_i = Σ_j P_ij dP_ij is the derivative of the
      softmax normaliser, dS = P ∘ (dP - rowsum(P ∘ dP));
    * dQ = scale dS K and dK = scale dSᵀ Q.

    Returns ``(dQ, dK, dV)``, each ``[B, H, N, d]``. With ``return_bounds`` it
    also returns ``(mQ, mK, mV)``: the same products taken over absolute values,
    with |dS| replaced by P (|dP| + A), A_i = Σ_c |dO_ic O_ic| — the envelope
    that bounds how far rounding the products' operands can move each entry.
    """
    q, k, v, do = _as_f64(q), _as_f64(k), _as_f64(v), _as_f64(do)
    if not (q.shape == k.shape == v.shape == do.shape) or q.ndim != 4:
        raise ValueError("q, k, v and do must share one [B, H, N, d] shape")
    B, H, N, d = q.shape
    dq, dk, dv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    if return_bounds:
        mq, mk, mv = np.zeros_like(q), np.zeros_like(q), np.zeros_like(q)
    hidden = np.triu(np.ones((N, N), dtype=bool), 1) if causal else np.zeros((N, N), dtype=bool)
    for b in range(B):
        for h in range(H):
            qh, kh, vh, doh = q[b, h], k[b, h], v[b, h], do[b, h]
            s = np.where(hidden, -np.inf, scale * (qh @ kh.T))
            w = np.exp(s - s.max(axis=1, keepdims=True))
            p = w / w.sum(axis=1, keepdims=True)
            dv[b, h] = p.T @ doh
            dp = doh @ vh.T
            ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
            dq[b, h] = scale * (ds @ kh)
            dk[b, h] = scale * (ds.T @ qh)
            if return_bounds:
                a = np.abs(doh * (p @ vh)).sum(axis=1, keepdims=True)
                e = p * (np.abs(dp) + a)
                mv[b, h] = p.T @ np.abs(doh)
                mq[b, h] = scale * (e @ np.abs(kh))
                mk[b, h] = scale * (e.T @ np.abs(qh))
    if return_bounds:
        return (dq, dk, dv), (mq, mk, mv)
    return dq, dk, dv


# ----------------------------------------------------------------- rotation --
def sylvester_hadamard(d: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix H_d (d a power of two):
    H_1 = [1], H_2n = [[H_n, H_n], [H_n, -H_n]]."""
    if d < 1 or d & (d - 1):
        raise ValueError("d must be a power of two")
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < d:
        h = np.block([[h, h], [h, -h]])
    return h


def rotation_matrix(d: int, signs=None) -> np.ndarray:
    """M = D H_d / sqrt(d), D = diag(signs) (identity if ``signs`` is None).
    Orthogonal: M Mᵀ = I. Applied to row vectors, x' = x M."""
    h = sylvester_hadamard(d) / np.sqrt(d)
    if signs is None:
        return h
    s = _as_f64(signs).reshape(d)
    return s[:, None] * h


def rotate(x, signs=None) -> np.ndarray:
    """x M along the last axis, in fp64."""
    x = _as_f64(x)
    return x @ rotation_matrix(x.shape[-1], signs)


# -------------------------------------------------------------------- e4m3 --
def e4m3_decode(codes) -> np.ndarray:
    """Value of each e4m3 code (uint8) as fp64; 0x7F / 0xFF decode to NaN."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c >> 7, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, np.ldexp(m / 8.0, -6), np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64)))
    out = sign * mag
    return np.where((c & 0x7F) == 0x7F, np.nan, out)


def e4m3_encode(x) -> np.ndarray:
    """Nearest e4m3 code to each finite fp64 value, ties to even, magnitudes
    above 448 saturated to 448. Negative values that round to zero give -0 (0x80)."""
    x = _as_f64(x)
    if not np.all(np.isfinite(x)):
        raise ValueError("e4m3_encode takes finite values only")
    neg = np.signbit(x)
    a = np.minimum(np.abs(x), E4M3_MAX)
    # Spacing of representable values around a: 2^(e-3) with e = floor(log2 a),
    # clamped to the subnormal spacing 2^-9 below the smallest normal 2^-6.
    _, ex = np.frexp(a)  # a = f * 2^ex, f in [0.5, 1)
    e = np.maximum(ex - 1, -6)
    quantum = np.ldexp(1.0, (e - 3).astype(np.int64))
    val = np.rint(a / quantum) * quantum  # np.rint rounds half to even
    # val is a representable magnitude (possibly the next binade's first value).
    _, vex = np.frexp(val)
    ve = vex - 1
    normal = val >= 2.0**-6
    e_field = np.where(normal, ve + 7, 0)
    m_field = np.where(
        normal,
        np.rint(val / np.ldexp(1.0, ve.astype(np.int64)) * 8.0 - 8.0),
        np.rint(val / 2.0**-9),
    )
    code = (e_field.astype(np.int64) << 3) | m_field.astype(np.int64)
    code = code | np.where(neg, 0x80, 0)
    return code.astype(np.uint8)


def quantize_per_tensor(x, rotate_qk: bool, signs=None, return_scaled: bool = False):
    """Rotate (optionally) then quantise a whole tensor to e4m3 with one scale.

    x' = x M (if ``rotate_qk``), amax = max |x'|, descale = amax / 448 (1 if
    amax = 0), codes = e4m3_encode(x' * 448 / amax). Returns ``(codes, descale)``
    and, with ``return_scaled``, also the unrounded ``x' * 448 / amax``.
    """
    xr = rotate(x, signs) if rotate_qk else _as_f64(x)
    amax = float(np.max(np.abs(xr))) if xr.size else 0.0
    if amax == 0.0:
        scaled = np.zeros_like(xr)
        descale = 1.0
    else:
        scaled = xr * (E4M3_MAX / amax)
        descale = amax / E4M3_MAX
    codes = e4m3_encode(scaled)
    if return_scaled:
        return codes, descale, scaled
    return codes, descale


def quantize_v_transposed(v, return_scaled: bool = False):
    """V's e4m3 codes with one scale per tensor, laid out ``[B, H, d, N]``.

    "FlashAttention-3 (PT)", section "Inovações técnicas", subsection 3
    quantises the FP8 operands with a scale and rotates only Q and K; the pages
    give neither V's scale granularity nor its layout. Reading: no rotation, one
    scale per tensor (amax over all of V, descale = amax / 448, 1 if amax = 0,
    codes = e4m3_encode(v * 448 / amax)), and the codes of head (b, h) stored
    with the keys along the last dimension: out[b, h, c, n] = code(v[b, h, n, c]).
    Returns ``(codes, descale)`` and, with ``return_scaled``, the unrounded scaled
    values in the same transposed layout.
    """
    vf = _as_f64(v)
    amax = float(np.max(np.abs(vf))) if vf.size else 0.0
    scaled = np.zeros_like(vf) if amax == 0.0 else vf * (E4M3_MAX / amax)
    descale = 1.0 if amax == 0.0 else amax / E4M3_MAX
    scaled_t = np.ascontiguousarray(np.swapaxes(scaled, -1, -2))
    codes = e4m3_encode(scaled_t)
    if return_scaled:
        return codes, descale, scaled_t
    return codes, descale


def quantize_per_block(x, rotate_qk: bool, signs=None, block_rows: int = 128):
    """Rotate (optionally) then quantise ``x`` ``[B, H, N, d]`` to e4m3 with one
    scale per block of ``block_rows`` rows of each head (the last block of a head
    holds the remaining N mod block_rows rows).

    Per block b: amax_b = max |x'| over its rows, descale_b = amax_b / 448 (1 if
    amax_b = 0), codes = e4m3_encode(x' * 448 / amax_b). Returns ``(codes,
    descales)`` with descales ``[B, H, ceil(N / block_rows)]``.
    """
    xr = rotate(x, signs) if rotate_qk else _as_f64(x)
    B, H, N, d = xr.shape
    nb = -(-N // block_rows)
    codes = np.zeros(xr.shape, dtype=np.uint8)
    descales = np.ones((B, H, nb), dtype=np.float64)
    for b in range(B):
        for h in range(H):
            for i in range(nb):
                rows = slice(i * block_rows, min(N, (i + 1) * block_rows))
                blk = xr[b, h, rows]
                amax = float(np.max(np.abs(blk)))
                if amax == 0.0:
                    codes[b, h, rows] = e4m3_encode(np.zeros_like(blk))
                    continue
                codes[b, h, rows] = e4m3_encode(blk * (E4M3_MAX / amax))
                descales[b, h, i] = amax / E4M3_MAX
    return codes, descales
