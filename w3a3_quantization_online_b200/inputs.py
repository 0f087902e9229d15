"""Seeded synthetic inputs for the online activation path.

This module only draws random numbers and shapes them into the arrays that the
GPU path and the float64 oracle both read; it holds none of the method's
arithmetic (no projection, no Hadamard transform, no normalisation, no
quantisation).  Both sides receive exactly the same bits.

Recipe (numpy ``Generator(PCG64)``, one independent stream per array, keyed by
``SeedSequence([seed, stream])``):

* activations ``x``: float64 draws of the stated distribution, outlier channels
  (chosen once per seed, identical for every token) multiplied by a factor, then
  cast once to float32 and, for bf16 I/O, rounded to bf16 (round to nearest
  even).  ``x`` is always returned as a float32 array holding the exact I/O
  values;
* ``Q``: the orthonormal factor of the QR decomposition of a D x r standard
  Gaussian matrix, columns sign-fixed so that diag(R) > 0 (ReSpinQuant page,
  "key design 2": an orthonormal basis Q of the subspace);
* ``M = R_sub - I_r`` with ``R_sub = (I - A)^-1 (I + A)``, the Cayley map of a
  skew-symmetric A whose upper triangle is drawn N(0, 0.05^2); this stands in
  for the polar-decomposed rotation that calibration would produce
  (ReSpinQuant page, "key design 2" and "key design 3");
* ``signs``: int8 +-1 drawn uniformly (Infra Quant II page, QuaRot background:
  the randomised Hadamard H diag(s) with s drawn from {+1, -1});
* ``P1``, ``P2`` of FlatQuant's Kronecker affine transform (Infra Quant II page,
  FlatQuant: two small invertible matrices, learned by calibration): each is
  the orthonormal QR factor of a Gaussian matrix times a diagonal of
  exp(N(0, 0.25^2)) column scales, an invertible, well-conditioned, not
  orthogonal stand-in for a learned factor; handed over as float32.

Q and M are handed to the kernels as float32; the float64 originals are kept
for the pins that need exact orthogonality.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

# stream ids of SeedSequence([seed, stream])
_S_X, _S_OUTLIER, _S_Q, _S_A, _S_SIGNS, _S_GATE, _S_P1, _S_P2 = 0, 1, 2, 3, 4, 5, 6, 7

_CHUNK_ROWS = 2048


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([int(seed), int(stream)])))


def round_to_bf16(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a32 = np.ascontiguousarray(a, dtype=np.float32)
    u = a32.view(np.uint32).astype(np.uint64)
    u = (u + (((u >> 16) & 1) + 0x7FFF)) >> 16 << 16
    return u.astype(np.uint32).view(np.float32)


def _cast_io(a64: np.ndarray, dtype: str) -> np.ndarray:
    a32 = a64.astype(np.float32)
    if dtype == "bf16":
        return round_to_bf16(a32)
    if dtype == "f32":
        return a32
    raise ValueError(f"unknown I/O dtype {dtype!r}")


def activations(T: int, D: int, seed: int, dist: str = "normal", n_outliers: int = 0,
                outlier_scale: float = 1.0, dtype: str = "bf16") -> np.ndarray:
    """T x D activations: ``dist`` in {"normal", "student_t3", "silu_gate"}.

    ``silu_gate`` is the FFN down_proj input SiLU(a) * b with a, b ~ N(0, 1),
    computed in float64 here (it is input preparation, not part of the path).
    """
    rx = _rng(seed, _S_X)
    rg = _rng(seed, _S_GATE)
    out = np.empty((T, D), dtype=np.float32)
    ch = None
    if n_outliers:
        ch = _rng(seed, _S_OUTLIER).choice(D, size=n_outliers, replace=False)
    for r0 in range(0, T, _CHUNK_ROWS):
        n = min(_CHUNK_ROWS, T - r0)
        if dist == "normal":
            blk = rx.standard_normal((n, D))
        elif dist == "student_t3":
            blk = rx.standard_t(3.0, size=(n, D))
        elif dist == "silu_gate":
            a = rx.standard_normal((n, D))
            b = rg.standard_normal((n, D))
            blk = a / (1.0 + np.exp(-a)) * b
        else:
            raise ValueError(dist)
        if ch is not None:
            blk[:, ch] *= outlier_scale
        out[r0:r0 + n] = _cast_io(blk, dtype)
    return out


def outlier_channels(D: int, seed: int, n_outliers: int) -> np.ndarray:
    return np.sort(_rng(seed, _S_OUTLIER).choice(D, size=n_outliers, replace=False))


def subspace_basis(D: int, r: int, seed: int) -> np.ndarray:
    """D x r orthonormal Q (float64) from the QR of a seeded Gaussian matrix."""
    g = _rng(seed, _S_Q).standard_normal((D, r))
    q, rr = np.linalg.qr(g)
    sgn = np.sign(np.diag(rr))
    sgn[sgn == 0] = 1.0
    return q * sgn[None, :]


def cayley_rotation(r: int, seed: int, sigma: float = 0.05) -> np.ndarray:
    """r x r rotation (I - A)^-1 (I + A) of a seeded skew-symmetric A (float64)."""
    u = np.triu(_rng(seed, _S_A).normal(0.0, sigma, size=(r, r)), k=1)
    a = u - u.T
    eye = np.eye(r)
    return np.linalg.solve(eye - a, eye + a)


def random_signs(d: int, seed: int) -> np.ndarray:
    return np.where(_rng(seed, _S_SIGNS).integers(0, 2, size=d) == 1, 1, -1).astype(np.int8)


@dataclasses.dataclass
class AlignCase:
    """Inputs of one residual-alignment problem (float32 arrays as handed to the kernels)."""
    name: str
    x: np.ndarray          # T x D float32 holding the exact I/O values
    Q: np.ndarray          # D x r float32
    M: np.ndarray          # r x r float32, z_j = sum_k M[j,k] y_k
    Q64: np.ndarray        # float64 originals
    R64: np.ndarray        # r x r rotation, M64 = R64 - I
    dtype: str             # "f32" | "bf16"
    bits: int
    eps: float = 1e-5

    @property
    def T(self) -> int:
        return self.x.shape[0]

    @property
    def D(self) -> int:
        return self.x.shape[1]

    @property
    def r(self) -> int:
        return self.Q.shape[1]


@dataclasses.dataclass
class GateCase:
    """Inputs of one gated down_proj problem: SiLU(a) * b -> randomised Hadamard -> codes."""
    name: str
    a: np.ndarray          # T x d float32 holding the exact I/O values (gate projection)
    b: np.ndarray          # T x d float32 holding the exact I/O values (up projection)
    signs: np.ndarray      # d int8 +-1
    m: int
    dtype: str
    bits: int

    @property
    def T(self) -> int:
        return self.a.shape[0]

    @property
    def d(self) -> int:
        return self.a.shape[1]


@dataclasses.dataclass
class RhtCase:
    """Inputs of one randomised-Hadamard problem."""
    name: str
    x: np.ndarray          # T x d float32 holding the exact I/O values
    signs: np.ndarray      # d int8 +-1
    m: int                 # 1 (pure Sylvester) or 12 (Kronecker with the order-12 Paley matrix)
    dtype: str
    bits: int

    @property
    def T(self) -> int:
        return self.x.shape[0]

    @property
    def d(self) -> int:
        return self.x.shape[1]


def affine_factor(n: int, seed: int, stream: int) -> np.ndarray:
    """n x n invertible float32 matrix: orthonormal QR factor of a Gaussian matrix
    (columns sign-fixed) times exp(N(0, 0.25^2)) column scales."""
    rng = _rng(seed, stream)
    q, rr = np.linalg.qr(rng.standard_normal((n, n)))
    sgn = np.sign(np.diag(rr))
    sgn[sgn == 0] = 1.0
    c = np.exp(0.25 * rng.standard_normal(n))
    return (q * (sgn * c)[None, :]).astype(np.float32)


@dataclasses.dataclass
class KronAffineCase:
    """Inputs of one Kronecker affine transform + quantiser problem."""
    name: str
    x: np.ndarray          # T x (n1 n2) float32 holding the exact I/O values
    P1: np.ndarray         # n1 x n1 float32
    P2: np.ndarray         # n2 x n2 float32
    dtype: str
    bits: int

    @property
    def T(self) -> int:
        return self.x.shape[0]

    @property
    def d(self) -> int:
        return self.x.shape[1]

    @property
    def n1(self) -> int:
        return self.P1.shape[0]

    @property
    def n2(self) -> int:
        return self.P2.shape[0]


def kron_affine_case(T: int, n1: int, n2: int, seed: int, *, dtype: str = "bf16", bits: int = 4,
                     n_outliers: int = 8, outlier_scale: float = 20.0, name: str = "") -> KronAffineCase:
    d = n1 * n2
    x = activations(T, d, seed, "normal", min(n_outliers, d), outlier_scale, dtype)
    return KronAffineCase(name or f"affine_T{T}_{n1}x{n2}", x, affine_factor(n1, seed, _S_P1),
                          affine_factor(n2, seed, _S_P2), dtype, bits)


def align_case(T: int, D: int, r: int, seed: int, *, dtype: str = "bf16", bits: int = 4,
               dist: str = "normal", n_outliers: int = 0, outlier_scale: float = 1.0,
               qm_seed: Optional[int] = None, eps: float = 1e-5, name: str = "") -> AlignCase:
    qs = seed if qm_seed is None else qm_seed
    q64 = subspace_basis(D, r, qs)
    r64 = cayley_rotation(r, qs)
    x = activations(T, D, seed, dist, n_outliers, outlier_scale, dtype)
    return AlignCase(name or f"align_T{T}_D{D}_r{r}", x, q64.astype(np.float32),
                     (r64 - np.eye(r)).astype(np.float32), q64, r64, dtype, bits, eps)


def rht_case(T: int, d: int, m: int, seed: int, *, dtype: str = "bf16", bits: int = 4,
             dist: str = "normal", n_outliers: int = 0, outlier_scale: float = 1.0,
             name: str = "") -> RhtCase:
    x = activations(T, d, seed, dist, n_outliers, outlier_scale, dtype)
    return RhtCase(name or f"rht_T{T}_d{d}_m{m}", x, random_signs(d, seed), m, dtype, bits)


# ---------------------------------------------------------------------------
# The five workloads.  ``T`` may be overridden (the parity tests shrink it; the
# bench uses the full sizes).
# ---------------------------------------------------------------------------

def tiny_case(T: int = 64):
    """T=64, D=256, r=8, fp32 I/O, 4 outlier channels x50, INT4, order-256 RHT."""
    a = align_case(T, 256, 8, 0, dtype="f32", bits=4, n_outliers=4, outlier_scale=50.0, name="tiny")
    h = rht_case(T, 256, 1, 0, dtype="f32", bits=4, n_outliers=4, outlier_scale=50.0, name="tiny_rht")
    return a, h


def llama7b_case(T: int = 2048):
    """Llama-7B-like hidden stream: D=4096, r=32, bf16, 8 outlier channels x100, INT4; FWHT 2^12."""
    a = align_case(T, 4096, 32, 1, dtype="bf16", bits=4, n_outliers=8, outlier_scale=100.0,
                   name=f"hidden_T{T}_D4096")
    h = rht_case(T, 4096, 1, 1, dtype="bf16", bits=4, n_outliers=8, outlier_scale=100.0,
                 name=f"rht_T{T}_d4096")
    return a, h


def gate_inputs(T: int, d: int, seed: int, dtype: str = "bf16"):
    """The two FFN projections a (gate) and b (up), each N(0, 1), cast once to the
    I/O type; the same draws as the "silu_gate" activations of that seed."""
    rx = _rng(seed, _S_X)
    rg = _rng(seed, _S_GATE)
    a = np.empty((T, d), dtype=np.float32)
    b = np.empty((T, d), dtype=np.float32)
    for r0 in range(0, T, _CHUNK_ROWS):
        n = min(_CHUNK_ROWS, T - r0)
        a[r0:r0 + n] = _cast_io(rx.standard_normal((n, d)), dtype)
        b[r0:r0 + n] = _cast_io(rg.standard_normal((n, d)), dtype)
    return a, b


def gate_case(T: int, d: int, m: int, seed: int, *, dtype: str = "bf16", bits: int = 4, name: str = "") -> GateCase:
    a, b = gate_inputs(T, d, seed, dtype)
    return GateCase(name or f"gate_T{T}_d{d}_m{m}", a, b, random_signs(d, seed), m, dtype, bits)


def attention_case(T: int = 16384, n_heads: int = 32, d_head: int = 128, seed: int = 5, *, dtype: str = "bf16",
                   bits: int = 4) -> RhtCase:
    """Attention activations (queries / keys after the position transform, or the
    attention output), Llama-7B-like: n_heads x d_head = 32 x 128 columns, N(0, 1)
    with 8 outlier channels x20 (a key cache has a few large channels), random
    signs; INT4 per head / per token."""
    return rht_case(T, n_heads * d_head, 1, seed, dtype=dtype, bits=bits, n_outliers=8, outlier_scale=20.0,
                    name=f"attn_T{T}_h{n_heads}x{d_head}")


@dataclasses.dataclass
class GemmCase:
    """Inputs of one INT4 GEMM: packed activation and weight codes and their scales."""
    name: str
    codes_a: np.ndarray    # T x K/2 uint8 (two 4-bit codes per byte)
    scales_a: np.ndarray   # T float32
    codes_w: np.ndarray    # N x K/2 uint8
    scales_w: np.ndarray   # N float32

    @property
    def T(self) -> int:
        return self.codes_a.shape[0]

    @property
    def N(self) -> int:
        return self.codes_w.shape[0]

    @property
    def K(self) -> int:
        return 2 * self.codes_a.shape[1]


def gemm_case(T: int, N: int, K: int, seed: int) -> GemmCase:
    """Uniformly random bytes as packed 4-bit codes (every 4-bit two's complement
    value, -8 .. 7, equally likely), activation scales ~ U(0.01, 1) and weight
    scales ~ U(0.001, 0.02), float32 (the magnitudes of per-token activation
    steps and per-channel weight steps)."""
    r = _rng(seed, _S_X)
    ca = r.integers(0, 256, size=(T, K // 2), dtype=np.uint8)
    cw = _rng(seed, _S_Q).integers(0, 256, size=(N, K // 2), dtype=np.uint8)
    sa = _rng(seed, _S_A).uniform(0.01, 1.0, size=T).astype(np.float32)
    sw = _rng(seed, _S_SIGNS).uniform(0.001, 0.02, size=N).astype(np.float32)
    return GemmCase(f"gemm_T{T}_N{N}_K{K}", ca, sa, cw, sw)


def sylvester_signed(D: int, seed: int) -> np.ndarray:
    """Randomised Hadamard rotation H_D diag(s) / sqrt(D) (float64), the
    initialisation the pages' rotations start from; D a power of two."""
    H = np.ones((1, 1))
    while H.shape[0] < D:
        H = np.block([[H, H], [H, -H]])
    return H * random_signs(D, seed)[None, :].astype(np.float64) / np.sqrt(D)


def near_hadamard_pair(D: int, seed: int, n_planes: Optional[int] = None, theta0: float = 0.6,
                       decay: float = 0.85):
    """Two rotations R_in, R_out (float64 D x D) near the Hadamard start: R_in =
    H_D diag(s) / sqrt(D), R_out = R_in G with G a product of commuting plane
    rotations in the planes of an orthonormal D x 2m basis (QR of a Gaussian),
    angles theta0 * decay^i (i < m, m = D/4 unless given): T = R_out R_in^T =
    R_in G R_in^T deviates from I along few principal directions, with a
    decaying tail, as the pages observe for Cayley-trained rotations."""
    m = D // 4 if n_planes is None else n_planes
    g = _rng(seed, _S_Q).standard_normal((D, 2 * m))
    Ub, rr = np.linalg.qr(g)
    Ub = Ub * np.where(np.diag(rr) < 0, -1.0, 1.0)[None, :]
    th = theta0 * decay ** np.arange(m)
    c, s = np.cos(th), np.sin(th)
    u, v = Ub[:, 0::2], Ub[:, 1::2]
    # G = I + sum_i (c_i - 1)(u u^T + v v^T) + s_i (v u^T - u v^T)
    G = np.eye(D) + (u * (c - 1)) @ u.T + (v * (c - 1)) @ v.T + (v * s) @ u.T - (u * s) @ v.T
    R_in = sylvester_signed(D, seed)
    return R_in, R_in @ G


def down_proj_gate_case(T: int = 4096) -> GateCase:
    """FFN down_proj with the gate fused: a, b ~ N(0, 1) in bf16, d=12288=1024*12, INT4."""
    return gate_case(T, 12288, 12, 2, dtype="bf16", bits=4, name=f"downproj_gate_T{T}_d12288")


def down_proj_case(T: int = 4096):
    """FFN down_proj input SiLU(a)*b, d=12288=1024*12, bf16, H_1024 (x) H_12, INT4."""
    return rht_case(T, 12288, 12, 2, dtype="bf16", bits=4, dist="silu_gate", name=f"downproj_T{T}_d12288")


def flatquant_case(T: int = 16384) -> KronAffineCase:
    """FlatQuant's Kronecker affine transform on the hidden stream: d = 4096 =
    64 x 64 (n1 = n2 = 64, the split that minimises n1 + n2), bf16, 8 outlier
    channels x20, INT4."""
    return kron_affine_case(T, 64, 64, 11, dtype="bf16", bits=4, name=f"flatquant_T{T}_64x64")


def w3a3_case(T: int = 8192):
    """W3A3 large hidden: D=8192, r=32, bf16, Student-t(3) + 16 outlier channels x200, INT3; FWHT 2^13."""
    a = align_case(T, 8192, 32, 3, dtype="bf16", bits=3, dist="student_t3", n_outliers=16,
                   outlier_scale=200.0, name=f"w3a3_T{T}_D8192")
    h = rht_case(T, 8192, 1, 3, dtype="bf16", bits=3, dist="student_t3", n_outliers=16,
                 outlier_scale=200.0, name=f"w3a3_rht_T{T}_d8192")
    return a, h


CHAIN_LAYERS = 32


def chain_case(T: int = 16, layers: int = CHAIN_LAYERS):
    """32 independent (Q_i, M_i) pairs (seeds 1000+i) over one bf16 residual stream, D=4096, r=32."""
    x = activations(T, 4096, 4, "normal", 8, 100.0, "bf16")
    qs, ms, q64s, r64s = [], [], [], []
    for i in range(layers):
        q64 = subspace_basis(4096, 32, 1000 + i)
        r64 = cayley_rotation(32, 1000 + i)
        q64s.append(q64)
        r64s.append(r64)
        qs.append(q64.astype(np.float32))
        ms.append((r64 - np.eye(32)).astype(np.float32))
    return x, qs, ms, q64s, r64s

