"""Helpers shared by the tests: code unpacking and the GPU-vs-oracle tolerance rules.

Tolerances (written here once, used by every parity test):
  * aligned values, float32 I/O: max |gpu - oracle| <= 1e-4 * max|x| per row;
  * aligned values, bf16 I/O:    max |gpu - oracle| <= 4e-3 * max|oracle| per row;
  * scales: relative error <= 1e-6 (both exactly 0 for an all-zero row); a
    scale below the float32 normal range cannot carry that relative precision,
    so the bound is 1e-6 * scale + 2^-149 (half the float32 subnormal spacing);
  * codes: equal, except +-1 where the oracle's pre-round value v/alpha lies
    within 1e-4 of a rounding tie (|frac(|v/alpha|) - 0.5| < 1e-4); such
    mismatches may number at most 1e-5 of all codes, rounded up to a whole code.
"""
from __future__ import annotations

import math

import numpy as np

ALIGN_F32_ABS = 1e-4
ALIGN_BF16_REL = 4e-3
SCALE_REL = 1e-6
TIE_BAND = 1e-4
TIE_FRACTION = 1e-5


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
                label: str = "") -> int:
    """Assert the code rule; returns the number of (allowed) near-tie mismatches."""
    n = ora_q.shape[-1]
    g = unpack(np.asarray(gpu_bytes), n, bits)
    qmax = 2 ** (bits - 1) - 1
    assert g.min() >= -qmax and g.max() <= qmax, f"{label}: code out of range"
    mism = g != ora_q
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
    allowed = math.ceil(TIE_FRACTION * ora_q.size)
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
    gpu = np.asarray(gpu, dtype=np.float64)
    err = np.abs(gpu - ora).max(axis=1)
    if dtype == "f32":
        bound = ALIGN_F32_ABS * np.abs(np.asarray(x, dtype=np.float64)).max(axis=1)
    else:
        bound = ALIGN_BF16_REL * np.abs(ora).max(axis=1)
    ok = err <= bound
    assert ok.all(), f"{label}: aligned-value error {err[~ok].max():.3e} above bound in {int((~ok).sum())} rows"
    with np.errstate(divide="ignore", invalid="ignore"):
        ratio = np.where(bound > 0, err / bound, 0.0)
    return float(ratio.max()) if ratio.size else 0.0
