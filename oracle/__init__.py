"""Float64 CPU oracle of the online activation path (ctypes wrapper of rsq_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the bench's CPU
baseline import this package; the product path never does, and this package
imports nothing from the product package.  Arrays go in as numpy (any float
dtype; widened to float64 exactly) and results come back as float64 / int8 /
uint8 numpy arrays.

Each function names the passage it follows in the C source's header comment.
"""
from __future__ import annotations

import ctypes
import os
import threading

import numpy as np

from .build import LIB_PATH, build

_lib = None
_lock = threading.Lock()

_D = ctypes.POINTER(ctypes.c_double)
_I8 = ctypes.POINTER(ctypes.c_int8)
_U8 = ctypes.POINTER(ctypes.c_uint8)


def lib():
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                build()
            L = ctypes.CDLL(LIB_PATH)
            i64, i32, f64 = ctypes.c_int64, ctypes.c_int, ctypes.c_double
            L.ora_set_threads.argtypes = [i32]
            L.ora_sylvester.argtypes = [i32, _D]
            L.ora_paley1.argtypes = [i32, _D]
            L.ora_fwht.argtypes = [i32, i64, _D]
            L.ora_fwht.restype = None
            L.ora_residual_align.argtypes = [i64, i32, i32, _D, _D, _D, _D]
            L.ora_rmsnorm.argtypes = [i64, i32, f64, _D, _D]
            L.ora_quant_sym.argtypes = [i64, i32, i32, _D, _I8, _D, _D]
            L.ora_rht.argtypes = [i64, i32, i32, _D, _D, _I8, _D]
            L.ora_pack.argtypes = [i64, i32, i32, _I8, _U8]
            L.ora_align_norm_quant.argtypes = [i64, i32, i32, i32, f64, _D, _D, _D, _D, _I8, _U8, _D, _D]
            L.ora_rht_quant.argtypes = [i64, i32, i32, i32, _D, _D, _I8, _I8, _U8, _D, _D]
            L.ora_silu_gate.argtypes = [i64, i32, _D, _D, _D]
            L.ora_head_rht.argtypes = [i64, i32, i32, _D, _I8, _D]
            L.ora_head_mix.argtypes = [i64, i32, i32, _D, _I8, _D]
            L.ora_head_rht_quant.argtypes = [i64, i32, i32, i32, _D, _I8, _I8, _U8, _D, _D]
            L.ora_head_mix_quant.argtypes = [i64, i32, i32, i32, _D, _I8, _I8, _U8, _D, _D]
            L.ora_w4a4_gemm.argtypes = [i64, i32, i32, _U8, _D, _U8, _D, ctypes.POINTER(ctypes.c_int32), _D]
            L.ora_rht_quant_gate.argtypes = [i64, i32, i32, i32, _D, _D, _D, _I8, _I8, _U8, _D, _D]
            L.ora_kron_affine.argtypes = [i64, i32, i32, _D, _D, _D, _D]
            L.ora_kron_affine_quant.argtypes = [i64, i32, i32, i32, _D, _D, _D, _I8, _U8, _D, _D]
            _lib = L
    return _lib


def _f64(a):
    return np.ascontiguousarray(a, dtype=np.float64)


def _p(a, t):
    return a.ctypes.data_as(t) if a is not None else None


def set_threads(n: int) -> int:
    """Set the OpenMP thread count (n <= 0 keeps it); returns the count in effect."""
    return int(lib().ora_set_threads(int(n)))


def sylvester(n: int) -> np.ndarray:
    """Sylvester Hadamard matrix of order n (entries +-1)."""
    H = np.empty((n, n), dtype=np.float64)
    if lib().ora_sylvester(n, _p(H, _D)) != 0:
        raise ValueError(f"order {n} is not a power of two")
    return H


def paley1(q: int = 11) -> np.ndarray:
    """Paley type-I Hadamard matrix of order q + 1 (entries +-1)."""
    H = np.empty((q + 1, q + 1), dtype=np.float64)
    if lib().ora_paley1(q, _p(H, _D)) != 0:
        raise ValueError(f"q={q} is not a prime = 3 mod 4")
    return H


def kron_factor(m: int) -> np.ndarray:
    """The order-m dense factor of H_{2^n} (x) H_m: [1] for m = 1, Paley I for m = q + 1."""
    if m == 1:
        return np.ones((1, 1))
    return paley1(m - 1)


def fwht(v: np.ndarray) -> np.ndarray:
    """Unnormalised Sylvester transform of each row of v (copy)."""
    out = _f64(v).copy()
    rows = out.reshape(-1, out.shape[-1])
    n = rows.shape[1]
    for t in range(rows.shape[0]):
        row = rows[t]
        lib().ora_fwht(n, 1, row.ctypes.data_as(_D))
    return out


def residual_align(x, Q, M) -> np.ndarray:
    x, Q, M = _f64(x), _f64(Q), _f64(M)
    T, D = x.shape
    r = Q.shape[1]
    xo = np.empty_like(x)
    rc = lib().ora_residual_align(T, D, r, _p(x, _D), _p(Q, _D), _p(M, _D), _p(xo, _D))
    if rc:
        raise MemoryError("oracle allocation failed")
    return xo


def rmsnorm(x, eps: float = 1e-5) -> np.ndarray:
    x = _f64(x)
    T, D = x.shape
    n = np.empty_like(x)
    lib().ora_rmsnorm(T, D, float(eps), _p(x, _D), _p(n, _D))
    return n


def quant_sym(v, bits: int):
    """Per-row symmetric absmax quantiser; returns (codes int8, scales, pre-round values)."""
    v = _f64(v)
    T, n = v.shape
    q = np.empty((T, n), dtype=np.int8)
    a = np.empty(T, dtype=np.float64)
    pre = np.empty_like(v)
    if lib().ora_quant_sym(T, n, bits, _p(v, _D), _p(q, _I8), _p(a, _D), _p(pre, _D)):
        raise ValueError(f"bits={bits}")
    return q, a, pre


def rht(x, signs, m: int = 1) -> np.ndarray:
    """v = (H_{2^n} (x) H_m) diag(s) x / sqrt(d) for each row."""
    x = _f64(x)
    T, d = x.shape
    s = np.ascontiguousarray(signs, dtype=np.int8)
    Hm = _f64(kron_factor(m))
    v = np.empty_like(x)
    if lib().ora_rht(T, d, m, _p(Hm, _D), _p(x, _D), _p(s, _I8), _p(v, _D)):
        raise ValueError(f"d={d}, m={m}")
    return v


def pack(q, bits: int) -> np.ndarray:
    q = np.ascontiguousarray(q, dtype=np.int8)
    T, n = q.shape
    out = np.empty((T, n * bits // 8), dtype=np.uint8)
    if lib().ora_pack(T, n, bits, _p(q, _I8), _p(out, _U8)):
        raise ValueError(f"bits={bits}, n={n}")
    return out


def align_norm_quant(x, Q, M, bits: int, eps: float = 1e-5, want_pre: bool = True) -> dict:
    """Residual alignment -> weight-free RMSNorm -> symmetric per-token quantisation -> pack."""
    x, Q, M = _f64(x), _f64(Q), _f64(M)
    T, D = x.shape
    r = Q.shape[1]
    xo = np.empty_like(x)
    q = np.empty((T, D), dtype=np.int8)
    codes = np.empty((T, D * bits // 8), dtype=np.uint8)
    scales = np.empty(T, dtype=np.float64)
    pre = np.empty_like(x) if want_pre else None
    rc = lib().ora_align_norm_quant(T, D, r, bits, float(eps), _p(x, _D), _p(Q, _D), _p(M, _D),
                                    _p(xo, _D), _p(q, _I8), _p(codes, _U8), _p(scales, _D),
                                    _p(pre, _D))
    if rc:
        raise ValueError(f"oracle rejected D={D}, bits={bits} (rc={rc})")
    return {"x_out": xo, "q": q, "codes": codes, "scales": scales, "pre": pre}


def rht_quant(x, signs, m: int, bits: int, want_pre: bool = True) -> dict:
    """Randomised Hadamard -> symmetric per-token quantisation -> pack (no normalisation)."""
    x = _f64(x)
    T, d = x.shape
    s = np.ascontiguousarray(signs, dtype=np.int8)
    Hm = _f64(kron_factor(m))
    q = np.empty((T, d), dtype=np.int8)
    codes = np.empty((T, d * bits // 8), dtype=np.uint8)
    scales = np.empty(T, dtype=np.float64)
    pre = np.empty_like(x) if want_pre else None
    rc = lib().ora_rht_quant(T, d, m, bits, _p(Hm, _D), _p(x, _D), _p(s, _I8), _p(q, _I8),
                             _p(codes, _U8), _p(scales, _D), _p(pre, _D))
    if rc:
        raise ValueError(f"oracle rejected d={d}, m={m}, bits={bits} (rc={rc})")
    return {"q": q, "codes": codes, "scales": scales, "pre": pre}


def silu_gate(a, b) -> np.ndarray:
    """g = SiLU(a) * b = a / (1 + exp(-a)) * b, element by element (the gated FFN product)."""
    a, b = _f64(a), _f64(b)
    T, d = a.shape
    g = np.empty_like(a)
    lib().ora_silu_gate(T, d, _p(a, _D), _p(b, _D), _p(g, _D))
    return g


def rht_quant_gate(a, b, signs, m: int, bits: int, want_pre: bool = True) -> dict:
    """SiLU(a) * b -> randomised Hadamard -> symmetric per-token quantisation -> pack."""
    a, b = _f64(a), _f64(b)
    T, d = a.shape
    s = np.ascontiguousarray(signs, dtype=np.int8)
    Hm = _f64(kron_factor(m))
    q = np.empty((T, d), dtype=np.int8)
    codes = np.empty((T, d * bits // 8), dtype=np.uint8)
    scales = np.empty(T, dtype=np.float64)
    pre = np.empty_like(a) if want_pre else None
    rc = lib().ora_rht_quant_gate(T, d, m, bits, _p(Hm, _D), _p(a, _D), _p(b, _D), _p(s, _I8), _p(q, _I8),
                                  _p(codes, _U8), _p(scales, _D), _p(pre, _D))
    if rc:
        raise ValueError(f"oracle rejected d={d}, m={m}, bits={bits} (rc={rc})")
    return {"q": q, "codes": codes, "scales": scales, "pre": pre}


def _signs_or_none(signs):
    return None if signs is None else np.ascontiguousarray(signs, dtype=np.int8)


def head_rht(x, signs, n_heads: int) -> np.ndarray:
    """Per-head randomised Hadamard (I_{n_h} (x) H_{d_h}) diag(s) x / sqrt(d_h) (signs may be None)."""
    x = _f64(x)
    T, d = x.shape
    s = _signs_or_none(signs)
    v = np.empty_like(x)
    if lib().ora_head_rht(T, d, n_heads, _p(x, _D), _p(s, _I8), _p(v, _D)):
        raise ValueError(f"d={d}, n_heads={n_heads}")
    return v


def head_mix(x, signs, n_heads: int) -> np.ndarray:
    """Head-mixing randomised Hadamard (H_{n_h} (x) I_{d_h}) diag(s) x / sqrt(n_h) (signs may be None)."""
    x = _f64(x)
    T, d = x.shape
    s = _signs_or_none(signs)
    v = np.empty_like(x)
    if lib().ora_head_mix(T, d, n_heads, _p(x, _D), _p(s, _I8), _p(v, _D)):
        raise ValueError(f"d={d}, n_heads={n_heads}")
    return v


def head_rht_quant(x, signs, n_heads: int, bits: int, want_pre: bool = True) -> dict:
    """Per-head rotation -> symmetric quantisation per (token, head) -> pack; scales T x n_heads."""
    x = _f64(x)
    T, d = x.shape
    s = _signs_or_none(signs)
    q = np.empty((T, d), dtype=np.int8)
    codes = np.empty((T, d * bits // 8), dtype=np.uint8)
    scales = np.empty((T, n_heads), dtype=np.float64)
    pre = np.empty_like(x) if want_pre else None
    rc = lib().ora_head_rht_quant(T, d, n_heads, bits, _p(x, _D), _p(s, _I8), _p(q, _I8), _p(codes, _U8),
                                  _p(scales, _D), _p(pre, _D))
    if rc:
        raise ValueError(f"oracle rejected d={d}, n_heads={n_heads}, bits={bits} (rc={rc})")
    return {"q": q, "codes": codes, "scales": scales, "pre": pre}


def head_mix_quant(x, signs, n_heads: int, bits: int, want_pre: bool = True) -> dict:
    """Head mixing -> symmetric per-token quantisation -> pack."""
    x = _f64(x)
    T, d = x.shape
    s = _signs_or_none(signs)
    q = np.empty((T, d), dtype=np.int8)
    codes = np.empty((T, d * bits // 8), dtype=np.uint8)
    scales = np.empty(T, dtype=np.float64)
    pre = np.empty_like(x) if want_pre else None
    rc = lib().ora_head_mix_quant(T, d, n_heads, bits, _p(x, _D), _p(s, _I8), _p(q, _I8), _p(codes, _U8),
                                  _p(scales, _D), _p(pre, _D))
    if rc:
        raise ValueError(f"oracle rejected d={d}, n_heads={n_heads}, bits={bits} (rc={rc})")
    return {"q": q, "codes": codes, "scales": scales, "pre": pre}


def kron_affine(x, P1, P2) -> np.ndarray:
    """FlatQuant's Kronecker affine transform of each row: x P with P = P1 (x) P2,
    computed as vec(P1^T X P2) with X the n1 x n2 row-major reshape of the row."""
    x, P1, P2 = _f64(x), _f64(P1), _f64(P2)
    T, n = x.shape
    n1, n2 = P1.shape[0], P2.shape[0]
    if n1 * n2 != n:
        raise ValueError(f"n1 * n2 = {n1 * n2} != row length {n}")
    v = np.empty_like(x)
    if lib().ora_kron_affine(T, n1, n2, _p(P1, _D), _p(P2, _D), _p(x, _D), _p(v, _D)):
        raise ValueError(f"n1={n1}, n2={n2}")
    return v


def kron_affine_quant(x, P1, P2, bits: int, want_pre: bool = True) -> dict:
    """Kronecker affine transform -> symmetric per-token quantisation -> pack."""
    x, P1, P2 = _f64(x), _f64(P1), _f64(P2)
    T, n = x.shape
    n1, n2 = P1.shape[0], P2.shape[0]
    if n1 * n2 != n:
        raise ValueError(f"n1 * n2 = {n1 * n2} != row length {n}")
    q = np.empty((T, n), dtype=np.int8)
    codes = np.empty((T, n * bits // 8), dtype=np.uint8)
    scales = np.empty(T, dtype=np.float64)
    pre = np.empty_like(x) if want_pre else None
    rc = lib().ora_kron_affine_quant(T, n1, n2, bits, _p(P1, _D), _p(P2, _D), _p(x, _D), _p(q, _I8),
                                     _p(codes, _U8), _p(scales, _D), _p(pre, _D))
    if rc:
        raise ValueError(f"oracle rejected n1={n1}, n2={n2}, bits={bits} (rc={rc})")
    return {"q": q, "codes": codes, "scales": scales, "pre": pre}


def w4a4_gemm(codes_a, scales_a, codes_w, scales_w) -> dict:
    """INT4 GEMM: acc = unpack(codes_a) unpack(codes_w)^T exactly (int32), y = acc * sa[t] * sw[n] (float64)."""
    ca = np.ascontiguousarray(codes_a, dtype=np.uint8)
    cw = np.ascontiguousarray(codes_w, dtype=np.uint8)
    T, kb = ca.shape
    N = cw.shape[0]
    K = 2 * kb
    sa, sw = _f64(scales_a), _f64(scales_w)
    acc = np.empty((T, N), dtype=np.int32)
    y = np.empty((T, N), dtype=np.float64)
    rc = lib().ora_w4a4_gemm(T, N, K, _p(ca, _U8), _p(sa, _D), _p(cw, _U8), _p(sw, _D),
                             acc.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)), _p(y, _D))
    if rc:
        raise ValueError(f"oracle rejected T={T}, N={N}, K={K} (rc={rc})")
    return {"acc": acc, "y": y}


def quant_weights_rtn(W, bits: int = 4) -> dict:
    """Per-output-channel symmetric round-to-nearest weight quantisation (the
    simple RTN option the pages name for QuaRot's weights): each row n of W
    (an output channel) gets scale max|W[n]| / qmax; codes packed like the
    activation codes."""
    q, a, _ = quant_sym(W, bits)
    return {"codes": pack(q, bits), "scales": a, "q": q}


def qm_construct(R_in, R_out, r: int) -> dict:
    """The offline (Q, M) construction of ReSpinQuant (paper notes, key design 2), in float64.

    T = R_out R_in^T is the transition matrix at a residual connection; its
    deviation dT = T - I is decomposed by SVD and Q takes the top-r left
    singular vectors; T_sub = Q^T T Q is the transition restricted to that
    subspace; the polar factor U V^T of T_sub (SVD T_sub = U S V^T), pulled
    back into SO(r) (when det(U V^T) = -1 the singular pair of the smallest
    singular value flips sign, the nearest rotation), is R_sub; M = R_sub - I.
    The low-rank approximation T_hat = I + Q M Q^T is then in SO(D).  numpy's
    SVD and matrix products are the library steps."""
    R_in = np.asarray(R_in, dtype=np.float64)
    R_out = np.asarray(R_out, dtype=np.float64)
    D = R_in.shape[0]
    T = R_out @ R_in.T
    U, S, _ = np.linalg.svd(T - np.eye(D))
    Q = U[:, :r]
    T_sub = Q.T @ T @ Q
    U2, S2, Vt2 = np.linalg.svd(T_sub)
    if np.linalg.det(U2 @ Vt2) < 0:
        U2 = U2.copy()
        U2[:, -1] = -U2[:, -1]
    R_sub = U2 @ Vt2
    return {"Q": Q, "R_sub": R_sub, "M": R_sub - np.eye(r), "T": T, "T_sub": T_sub, "sv": S}


def t_hat(Q, M) -> np.ndarray:
    """The dense D x D T_hat = I + Q M Q^T (tests only: the online path never forms it)."""
    Q = np.asarray(Q, dtype=np.float64)
    return np.eye(Q.shape[0]) + Q @ np.asarray(M, dtype=np.float64) @ Q.T
