"""Helpers shared by the tests: code unpacking and the GPU-vs-oracle tolerance rules.

Tolerances (written here once, used by every parity test):
  * aligned values, float32 I/O: max |gpu - oracle| <= 1e-4 * max|x| per row;
  * aligned values, bf16 I/O: element by element, |gpu - oracle| <= 4e-3 * |oracle|
    + 1e-5 * max|oracle of the row| (the relative bound itself, plus a floor for
    elements near zero, where a relative error means nothing: the floor is far
    below the 4e-3 bound on every ordinary element of a row with outliers);
  * scales: relative error <= 1e-6 (both exactly 0 for an all-zero row); a
    scale below the float32 normal range cannot carry that relative precision,
    so the bound is 1e-6 * scale + 2^-149 (half the float32 subnormal spacing);
  * codes: equal, except +-1 where the oracle's pre-round value v/alpha lies
    within 1e-4 of a rounding tie (|frac(|v/alpha|) - 0.5| < 1e-4).  Such
    mismatches are added up over the whole test session together with the
    number of codes compared, and the session total may be at most 1e-5 of all
    codes (checked once at the end of the session, tests/conftest.py); a single
    check outside a session (smoke) applies the same fraction to its own codes,
    rounded down.
"""
from __future__ import annotations

import math

import numpy as np

ALIGN_F32_ABS = 1e-4
ALIGN_BF16_REL = 4e-3
ALIGN_BF16_FLOOR = 1e-5
SCALE_REL = 1e-6
TIE_BAND = 1e-4
TIE_FRACTION = 1e-5

# near-tie mismatches and codes compared, over the test session
TIE_TALLY = {"mismatches": 0, "codes": 0}


def tie_tally_check() -> None:
    """The session rule: near-tie mismatches <= 1e-5 of all codes compared."""
    m, n = TIE_TALLY["mismatches"], TIE_TALLY["codes"]
    assert m <= TIE_FRACTION * n, f"{m} near-tie code mismatches over {n} codes > {TIE_FRACTION:g} of them"


def unpack_int4(b: np.ndarray, n: int) -> np.ndarray:
    lo = (b & 0xF).astype(np.int16)
    hi = (b >> 4).astype(np.int16)
    out = np.empty(b.shape[:-1] + (n,), dtype=np.int16)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return np.where(out >= 8, out - 16, out).astype(np.int8)


def unpack_int3(b: np.ndarray, n: int) -> np.ndarray:
    b = b.astype(np.uint32).reshape(b.shape[:-1] + (n // 8, 3))
    word = b[..., 0] | (b[..., 1] << 8) | (b[..., 2] << 16)
    k = np.arange(8, dtype=np.uint32)
    c = ((word[..., None] >> (3 * k)) & 7).astype(np.int16)
    c = np.where(c >= 4, c - 8, c)
    return c.reshape(b.shape[:-2] + (n,)).astype(np.int8)


def unpack(b: np.ndarray, n: int, bits: int) -> np.ndarray:
    return unpack_int4(b, n) if bits == 4 else unpack_int3(b, n)


def check_codes(gpu_bytes: np.ndarray, ora_q: np.ndarray, ora_pre: np.ndarray, bits: int,
                label: str = "", session: bool = True) -> int:
    """Assert the code rule; returns the number of (allowed) near-tie mismatches.

    session=True adds the counts to the session tally (checked at the end of
    the session); session=False checks the fraction on this call's codes."""
    n = ora_q.shape[-1]
    g = unpack(np.asarray(gpu_bytes), n, bits)
    qmax = 2 ** (bits - 1) - 1
    assert g.size == 0 or (g.min() >= -qmax and g.max() <= qmax), f"{label}: code out of range"
    mism = g != ora_q
    if session:
        TIE_TALLY["codes"] += int(ora_q.size)
    if not mism.any():
        return 0
    a = np.abs(ora_pre)
    near = np.abs(a - np.floor(a) - 0.5) < TIE_BAND
    diff1 = np.abs(g.astype(np.int16) - ora_q.astype(np.int16)) == 1
    bad = mism & ~(near & diff1)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        info = [(tuple(i), int(g[tuple(i)]), int(ora_q[tuple(i)]), float(ora_pre[tuple(i)])) for i in idx]
        raise AssertionError(f"{label}: {int(bad.sum())} code mismatches outside the tie band, e.g. {info}")
    count = int(mism.sum())
    if session:
        TIE_TALLY["mismatches"] += count
    else:
        allowed = math.floor(TIE_FRACTION * ora_q.size)
        assert count <= allowed, f"{label}: {count} near-tie mismatches > {allowed} allowed"
    return count


def check_scales(gpu: np.ndarray, ora: np.ndarray, label: str = "") -> float:
    gpu = np.asarray(gpu, dtype=np.float64)
    zero = ora == 0
    assert np.all(gpu[zero] == 0), f"{label}: nonzero scale on an all-zero row"
    err = np.abs(gpu[~zero] - ora[~zero])
    ok = err <= SCALE_REL * ora[~zero] + 2.0 ** -149
    rel = err / ora[~zero]
    worst = float(rel.max()) if rel.size else 0.0
    assert ok.all(), f"{label}: scale rel err {float(rel[~ok].max()):.3e} > {SCALE_REL}"
    return worst


def check_aligned(gpu: np.ndarray, ora: np.ndarray, x: np.ndarray, dtype: str, label: str = "") -> float:
    """Assert the aligned-value rule; returns the largest error / bound ratio."""
    gpu = np.asarray(gpu, dtype=np.float64)
    ora = np.asarray(ora, dtype=np.float64)
    if gpu.size == 0:
        return 0.0
    err = np.abs(gpu - ora)
    if dtype == "f32":
        bound = ALIGN_F32_ABS * np.abs(np.asarray(x, dtype=np.float64)).max(axis=1, keepdims=True)
        err = err.max(axis=1, keepdims=True)
    else:
        bound = ALIGN_BF16_REL * np.abs(ora) + ALIGN_BF16_FLOOR * np.abs(ora).max(axis=1, keepdims=True)
    ok = err <= bound
    if not ok.all():
        i = np.unravel_index(np.argmax(np.where(ok, 0.0, err - bound)), err.shape)
        raise AssertionError(f"{label}: aligned-value error above bound at {int((~ok).sum())} places, "
                             f"e.g. {tuple(int(v) for v in i)}: err {float(err[i]):.3e} > {float(bound[i]):.3e}")
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, 0.0)
    return float(ratio.max())


GEMM_OUT_UNIT = {"f16": 2.0 ** -11, "bf16": 2.0 ** -8}


def check_gemm(y_gpu: np.ndarray, y_ora: np.ndarray, out: str, label: str = "") -> float:
    """16-bit GEMM outputs against the float64 oracle: one rounding to the output
    type (unit roundoff u: 2^-11 fp16, 2^-8 bf16) after three float32 operations
    (int32 -> float conversion, two scale products: <= 3 * 2^-24 relative), plus
    the output type's smallest subnormal spacing for results near zero."""
    y_gpu = np.asarray(y_gpu, dtype=np.float64)
    u = GEMM_OUT_UNIT[out]
    tiny = 2.0 ** -24 if out == "f16" else 2.0 ** -133
    bound = (u + 4 * 2.0 ** -24) * np.abs(y_ora) + tiny
    err = np.abs(y_gpu - y_ora)
    ok = err <= bound
    if not ok.all():
        i = np.unravel_index(np.argmax(np.where(ok, 0.0, err - bound)), err.shape)
        raise AssertionError(f"{label}: GEMM output error above bound at {int((~ok).sum())} places, e.g. "
                             f"{tuple(int(v) for v in i)}: gpu {float(y_gpu[i])!r} oracle {float(y_ora[i])!r}")
    return float((err / np.maximum(bound, 1e-300)).max()) if err.size else 0.0
