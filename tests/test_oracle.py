"""Pins of the float64 oracle against facts fixed by the pages and by mathematics.

None of these tests needs a GPU.  Each pin is chosen so that a plausible slip in
the oracle (a dropped term, a wrong sign or index, a transposed operand, a wrong
row order, a wrong rounding or packing rule) makes at least one of them fail.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg

import oracle
from w3a3_quantization_online_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# Hadamard: worked example, order, orthogonality, FWHT == dense
# --------------------------------------------------------------------------

def test_worked_example_matrix_and_transform():
    g = _golden("hadamard4_worked_example.json")
    Hn = np.array(g["H_normalised"])
    np.testing.assert_array_equal(oracle.sylvester(4) / 2.0, Hn)  # row order of the printed H
    x = np.array([g["x"]])
    ones = np.ones(4, dtype=np.int8)
    np.testing.assert_array_equal(Hn.T @ x[0], g["HT_x"])  # the page's own arithmetic
    np.testing.assert_array_equal(oracle.rht(x, ones, 1)[0], g["HT_x"])
    np.testing.assert_array_equal(oracle.rht(np.array([g["x_back"]]), ones, 1)[0], g["H_x_back"])


def test_worked_example_quantisation():
    g = _golden("hadamard4_worked_example.json")
    ones = np.ones(4, dtype=np.int8)
    before = oracle.rht_quant(np.array([g["H_x_back"]]), ones, 1, 4)   # rht([20,0,0,0]) = [10]*4
    after = oracle.rht_quant(np.array([g["x_back"]]), ones, 1, 4)      # rht([10]*4) = [20,0,0,0]
    # rht maps [20,0,0,0] to [10,10,10,10] (step 10/7) and back (step 20/7)
    assert round(after["scales"][0], g["printed_decimals"]) == g["step_before_printed"]
    assert round(before["scales"][0], g["printed_decimals"]) == g["step_after_printed"]
    np.testing.assert_array_equal(after["q"][0], g["codes_before"])
    np.testing.assert_array_equal(before["q"][0], g["codes_after"])
    for res, v in ((before, [10.0] * 4), (after, [20.0, 0, 0, 0])):
        deq = res["scales"][0] * res["q"][0].astype(np.float64)
        assert np.max(np.abs(deq - np.array(v))) <= 1e-12 + g["dequant_error"]
    # the qmax of INT4 is the page's divisor 7
    assert g["qmax_int4"] == 2 ** (4 - 1) - 1


@pytest.mark.parametrize("n", [1, 2, 4, 8, 16, 64, 256, 1024])
def test_sylvester_matches_library_and_is_orthogonal(n):
    H = oracle.sylvester(n)
    np.testing.assert_array_equal(H, scipy.linalg.hadamard(n))  # textbook Sylvester construction
    np.testing.assert_array_equal(H.T @ H, n * np.eye(n))      # H^T H = I after 1/sqrt(n)


@pytest.mark.parametrize("n", [2, 4, 8, 16, 32, 64])
def test_fwht_equals_dense_bruteforce(n):
    rng = np.random.default_rng(n)
    v = rng.standard_normal((5, n))
    dense = v @ scipy.linalg.hadamard(n).T
    np.testing.assert_allclose(oracle.fwht(v), dense, rtol=0, atol=1e-12 * n)


@pytest.mark.parametrize("d", [4, 16, 64, 256])
def test_randomised_hadamard_equals_dense(d):
    rng = np.random.default_rng(d)
    x = rng.standard_normal((3, d))
    s = np.where(rng.integers(0, 2, d) == 1, 1, -1).astype(np.int8)
    Hs = scipy.linalg.hadamard(d) @ np.diag(s.astype(np.float64)) / math.sqrt(d)
    np.testing.assert_allclose(Hs @ Hs.T, np.eye(d), atol=1e-12)    # H diag(s) is orthogonal
    np.testing.assert_allclose(oracle.rht(x, s, 1), x @ Hs.T, atol=1e-12)
    # all-ones signs reduce to the plain normalised H
    np.testing.assert_allclose(oracle.rht(x, np.ones(d, np.int8), 1),
                               x @ scipy.linalg.hadamard(d).T / math.sqrt(d), atol=1e-12)


@pytest.mark.parametrize("d", [4096, 8192])
def test_randomised_hadamard_preserves_norm(d):
    case = inputs.rht_case(4, d, 1, 7, dtype="f32", n_outliers=4, outlier_scale=100.0)
    v = oracle.rht(case.x, case.signs, 1)
    np.testing.assert_allclose(np.linalg.norm(v, axis=1),
                               np.linalg.norm(case.x.astype(np.float64), axis=1), rtol=1e-13)
    # the outlier energy is spread: the largest coordinate shrinks for these inputs
    assert np.all(np.abs(v).max(axis=1) < np.abs(case.x).max(axis=1))


# --------------------------------------------------------------------------
# Paley order-12 matrix and the Kronecker transform
# --------------------------------------------------------------------------

def _quadratic_character(a, q):
    a %= q
    if a == 0:
        return 0
    return 1 if pow(a, (q - 1) // 2, q) == 1 else -1  # Euler's criterion


def test_paley12_is_hadamard_and_follows_the_textbook_construction():
    q = 11
    H = oracle.paley1(q)
    np.testing.assert_array_equal(H @ H.T, 12 * np.eye(12))
    S = H - np.eye(12)
    np.testing.assert_array_equal(S, -S.T)                  # Paley I: H - I is skew
    np.testing.assert_array_equal(H[0], np.ones(12))
    np.testing.assert_array_equal(H[1:, 0], -np.ones(11))
    for i in range(1, 12):
        for j in range(1, 12):
            if i != j:
                assert H[i, j] == _quadratic_character(j - i, q)


def test_paley_rejects_bad_orders():
    with pytest.raises(ValueError):
        oracle.paley1(13)   # 13 = 1 mod 4
    with pytest.raises(ValueError):
        oracle.paley1(15)   # not prime


@pytest.mark.parametrize("k", [0, 1, 2, 3])
def test_kronecker_transform_equals_dense_bruteforce(k):
    n2 = 2 ** k
    d = 12 * n2
    rng = np.random.default_rng(100 + k)
    x = rng.standard_normal((3, d))
    s = np.where(rng.integers(0, 2, d) == 1, 1, -1).astype(np.int8)
    Hd = np.kron(scipy.linalg.hadamard(n2), oracle.paley1(11)) / math.sqrt(d)
    np.testing.assert_allclose(Hd @ Hd.T, np.eye(d), atol=1e-12)
    want = x @ (Hd @ np.diag(s.astype(np.float64))).T
    np.testing.assert_allclose(oracle.rht(x, s, 12), want, atol=1e-12)


def test_kronecker_12288_preserves_norm():
    case = inputs.down_proj_case(T=3)
    v = oracle.rht(case.x, case.signs, 12)
    np.testing.assert_allclose(np.linalg.norm(v, axis=1),
                               np.linalg.norm(case.x.astype(np.float64), axis=1), rtol=1e-13)


# --------------------------------------------------------------------------
# Residual subspace alignment
# --------------------------------------------------------------------------

@pytest.mark.parametrize("D,r", [(64, 1), (128, 8), (256, 8), (256, 32)])
def test_low_rank_path_equals_dense_T_hat(D, r):
    case = inputs.align_case(9, D, r, 11, dtype="f32", n_outliers=2, outlier_scale=30.0)
    Q, R = case.Q64, case.R64
    T_hat = np.eye(D) + Q @ (R - np.eye(r)) @ Q.T
    np.testing.assert_allclose(T_hat.T @ T_hat, np.eye(D), atol=1e-10)   # T_hat orthogonal
    assert abs(np.linalg.det(T_hat) - 1.0) < 1e-9                       # ... and in SO(D)
    assert abs(np.linalg.det(R) - 1.0) < 1e-12                           # Cayley map is in SO(r)
    x = case.x.astype(np.float64)
    xo = oracle.residual_align(x, Q, R - np.eye(r))
    np.testing.assert_allclose(xo, x @ T_hat.T, atol=1e-11 * np.abs(x).max())
    np.testing.assert_allclose(np.linalg.norm(xo, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)


def test_zero_M_is_identity():
    case = inputs.align_case(5, 256, 8, 3, dtype="f32")
    xo = oracle.residual_align(case.x, case.Q64, np.zeros((8, 8)))
    np.testing.assert_array_equal(xo, case.x.astype(np.float64))


def test_full_rank_subspace_reproduces_the_rotation():
    # r = D: Q is a full orthogonal basis and T_hat = Q R Q^T exactly
    D = 16
    case = inputs.align_case(4, D, D, 5, dtype="f32")
    Q, R = case.Q64, case.R64
    xo = oracle.residual_align(case.x, Q, R - np.eye(D))
    np.testing.assert_allclose(xo, case.x.astype(np.float64) @ (Q @ R @ Q.T).T, atol=1e-12)


# --------------------------------------------------------------------------
# RMSNorm and the quantiser
# --------------------------------------------------------------------------

def test_rmsnorm_mean_square_and_rotation_commute():
    case = inputs.align_case(6, 128, 8, 4, dtype="f32", n_outliers=3, outlier_scale=20.0)
    eps = 1e-5
    x = case.x.astype(np.float64)
    n = oracle.rmsnorm(x, eps)
    ms = np.mean(x * x, axis=1)
    rs2 = 1.0 / (ms + eps)
    np.testing.assert_allclose(np.mean(n * n, axis=1), 1.0 - eps * rs2, rtol=0, atol=1e-14)
    T_hat = np.eye(128) + case.Q64 @ (case.R64 - np.eye(8)) @ case.Q64.T
    np.testing.assert_allclose(oracle.rmsnorm(x @ T_hat.T, eps), n @ T_hat.T, atol=1e-12)
    # eps = 0: invariant to a positive row factor
    np.testing.assert_allclose(oracle.rmsnorm(3.0 * x, 0.0), oracle.rmsnorm(x, 0.0), atol=1e-14)


@pytest.mark.parametrize("bits", [3, 4])
def test_quantiser_error_bound_range_and_absmax(bits):
    rng = np.random.default_rng(bits)
    v = rng.standard_t(3, size=(50, 96)) * rng.uniform(0.01, 100, size=(50, 1))
    q, a, pre = oracle.quant_sym(v, bits)
    qmax = 2 ** (bits - 1) - 1
    assert q.min() >= -qmax and q.max() <= qmax
    # dequantisation error at most half a step
    assert np.all(np.abs(a[:, None] * q - v) <= a[:, None] / 2 * (1 + 1e-12))
    # the absmax element lands on +-qmax
    am = np.argmax(np.abs(v), axis=1)
    assert np.all(np.abs(q[np.arange(50), am]) == qmax)
    np.testing.assert_allclose(a, np.abs(v).max(axis=1) / qmax, rtol=1e-15)
    # odd symmetry and invariance to power-of-two row factors (exact in binary)
    q2, _, _ = oracle.quant_sym(-v, bits)
    np.testing.assert_array_equal(q2, -q)
    for c in (0.25, 4.0):
        q3, a3, _ = oracle.quant_sym(c * v, bits)
        np.testing.assert_array_equal(q3, q)
        np.testing.assert_allclose(a3, c * a, rtol=1e-15)


def test_quantiser_rounds_half_to_even_and_handles_zero_rows():
    # qmax = 7: alpha = 1 exactly when the absmax is 7; ties at 0.5, 1.5, 2.5
    v = np.array([[7.0, 0.5, 1.5, 2.5, -0.5, -1.5, -2.5, 0.0],
                  [0.0] * 8])
    q, a, pre = oracle.quant_sym(v, 4)
    np.testing.assert_array_equal(q[0], [7, 0, 2, 2, 0, -2, -2, 0])
    assert a[1] == 0.0 and np.all(q[1] == 0) and np.all(pre[1] == 0)


# --------------------------------------------------------------------------
# Packing
# --------------------------------------------------------------------------

def _unpack_int4(b, n):
    lo = (b & 0xF).astype(np.int16)
    hi = (b >> 4).astype(np.int16)
    out = np.empty(b.shape[:-1] + (n,), dtype=np.int16)
    out[..., 0::2] = lo
    out[..., 1::2] = hi
    return np.where(out >= 8, out - 16, out).astype(np.int8)


def _unpack_int3(b, n):
    b = b.astype(np.uint32).reshape(b.shape[:-1] + (n // 8, 3))
    word = b[..., 0] | (b[..., 1] << 8) | (b[..., 2] << 16)
    k = np.arange(8, dtype=np.uint32)
    c = ((word[..., None] >> (3 * k)) & 7).astype(np.int16)
    c = np.where(c >= 4, c - 8, c)
    return c.reshape(b.shape[:-2] + (n,)).astype(np.int8)


def test_pack_int4_layout_and_exhaustive_round_trip():
    np.testing.assert_array_equal(oracle.pack(np.array([[1, -1, 7, -7]]), 4)[0], [0xF1, 0x97])
    vals = np.arange(-7, 8)
    pairs = np.array([[a, b] for a in vals for b in vals], dtype=np.int8)
    packed = oracle.pack(pairs, 4)
    np.testing.assert_array_equal(_unpack_int4(packed, 2), pairs)


def test_pack_int3_layout_and_exhaustive_round_trip():
    np.testing.assert_array_equal(oracle.pack(np.array([[1, 0, 0, 0, 0, 0, 0, 0]]), 3)[0], [1, 0, 0])
    np.testing.assert_array_equal(oracle.pack(np.array([[-1] * 8]), 3)[0], [0xFF, 0xFF, 0xFF])
    np.testing.assert_array_equal(oracle.pack(np.array([[0, 0, 0, 3, 0, 0, 0, -3]]), 3)[0],
                                  [0x00, 0x06, 0xA0])
    # every group of 8 codes in [-3, 3]: 7^8 = 5,764,801 groups
    idx = np.arange(7 ** 8, dtype=np.int64)
    groups = np.stack([(idx // 7 ** k) % 7 - 3 for k in range(8)], axis=1).astype(np.int8)
    packed = oracle.pack(groups, 3)
    np.testing.assert_array_equal(_unpack_int3(packed, 8), groups)


# --------------------------------------------------------------------------
# Pipelines and counts
# --------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [3, 4])
def test_align_norm_quant_is_the_composition_of_its_steps(bits):
    case = inputs.align_case(7, 256, 8, 21, dtype="bf16", bits=bits, n_outliers=4, outlier_scale=50.0)
    res = oracle.align_norm_quant(case.x, case.Q, case.M, bits, case.eps)
    xo = oracle.residual_align(case.x, case.Q, case.M)
    n = oracle.rmsnorm(xo, case.eps)
    q, a, pre = oracle.quant_sym(n, bits)
    np.testing.assert_array_equal(res["x_out"], xo)
    np.testing.assert_array_equal(res["q"], q)
    np.testing.assert_array_equal(res["scales"], a)
    np.testing.assert_array_equal(res["codes"], oracle.pack(q, bits))
    # scale invariance of the codes: RMSNorm output times a positive factor
    # (exact power of two) gives the same codes
    q4, _, _ = oracle.quant_sym(4.0 * n, bits)
    np.testing.assert_array_equal(q4, q)


def test_rht_quant_is_the_composition_of_its_steps():
    case = inputs.rht_case(5, 768, 12, 9, dtype="bf16", bits=4)
    res = oracle.rht_quant(case.x, case.signs, 12, 4)
    q, a, pre = oracle.quant_sym(oracle.rht(case.x, case.signs, 12), 4)
    np.testing.assert_array_equal(res["q"], q)
    np.testing.assert_array_equal(res["scales"], a)
    np.testing.assert_array_equal(res["codes"], oracle.pack(q, 4))


def test_online_parameter_count():
    g = _golden("online_param_count.json")
    case = inputs.align_case(1, g["D"], g["r"], 0, dtype="f32")
    per_module = case.Q.size + case.M.size
    total = g["modules_per_layer"] * g["layers"] * per_module
    assert math.floor(total / 1e5) / 10 == g["printed_millions"]


def test_inputs_are_deterministic_and_on_the_bf16_grid():
    a1, _ = inputs.llama7b_case(T=8)
    a2, _ = inputs.llama7b_case(T=8)
    np.testing.assert_array_equal(a1.x, a2.x)
    u = a1.x.view(np.uint32)
    assert np.all(u & 0xFFFF == 0)
    np.testing.assert_allclose(a1.Q64.T @ a1.Q64, np.eye(32), atol=1e-13)


# --------------------------------------------------------------------------
# The gated down_proj input: SiLU(a) * b fused in front of the Hadamard
# --------------------------------------------------------------------------

def test_silu_gate_matches_the_logistic_function_of_the_library():
    """g = a * sigmoid(a) * b against scipy's logistic sigmoid (an independent
    library routine); closed forms: sigmoid(0) = 1/2, sigmoid(ln 3) = 3/4."""
    import scipy.special
    rng = np.random.default_rng(5)
    a = rng.normal(0.0, 3.0, size=(7, 64))
    b = rng.normal(0.0, 1.0, size=(7, 64))
    np.testing.assert_allclose(oracle.silu_gate(a, b), a * scipy.special.expit(a) * b, rtol=1e-14, atol=1e-300)
    a2 = np.array([[0.0, math.log(3.0), -math.log(3.0), 1.0]])
    b2 = np.ones_like(a2)
    np.testing.assert_allclose(oracle.silu_gate(a2, b2)[0],
                               [0.0, 0.75 * math.log(3.0), -0.25 * math.log(3.0), 1.0 / (1.0 + math.exp(-1.0))],
                               rtol=1e-15)


def test_silu_gate_odd_part_and_limits():
    """SiLU(a) - SiLU(-a) = a for every a (sigmoid(a) + sigmoid(-a) = 1); SiLU
    tends to a for large a and to 0 for large negative a; b scales linearly."""
    a = np.linspace(-30.0, 30.0, 241)[None, :]
    one = np.ones_like(a)
    np.testing.assert_allclose(oracle.silu_gate(a, one) - oracle.silu_gate(-a, one), a, rtol=1e-14, atol=1e-13)
    big = np.array([[60.0, -60.0, 745.0, -745.0]])
    g = oracle.silu_gate(big, np.ones_like(big))[0]
    assert g[0] == 60.0 and abs(g[1]) < 1e-24 and g[2] == 745.0 and g[3] == 0.0
    np.testing.assert_array_equal(oracle.silu_gate(a, 2.0 * one), 2.0 * oracle.silu_gate(a, one))


def test_rht_quant_gate_is_the_rht_of_the_gated_product():
    """The fused path equals the randomised Hadamard quantiser applied to the
    gate values (no rounding in between); a zero up-projection row gives scale
    0 and all codes 0."""
    g = inputs.gate_case(5, 12 * 64, 12, 9, dtype="bf16", bits=4)
    g.b[2] = 0.0
    fused = oracle.rht_quant_gate(g.a, g.b, g.signs, 12, 4)
    plain = oracle.rht_quant(oracle.silu_gate(g.a, g.b), g.signs, 12, 4)
    np.testing.assert_array_equal(fused["codes"], plain["codes"])
    np.testing.assert_array_equal(fused["scales"], plain["scales"])
    assert fused["scales"][2] == 0.0 and np.all(fused["codes"][2] == 0)
    h = inputs.gate_case(3, 256, 1, 4, dtype="f32", bits=3)
    f3 = oracle.rht_quant_gate(h.a, h.b, h.signs, 1, 3)
    p3 = oracle.rht_quant(oracle.silu_gate(h.a, h.b), h.signs, 1, 3)
    np.testing.assert_array_equal(f3["codes"], p3["codes"])


def test_gate_inputs_match_the_down_proj_activations():
    """The two projections are the same seeded draws whose gated product the
    unfused down_proj workload stores: a from the activation stream, b from the
    gate stream of the same seed."""
    a, b = inputs.gate_inputs(4, 12288, 2, dtype="f32")
    ra = np.random.Generator(np.random.PCG64(np.random.SeedSequence([2, 0]))).standard_normal((4, 12288))
    rb = np.random.Generator(np.random.PCG64(np.random.SeedSequence([2, 5]))).standard_normal((4, 12288))
    np.testing.assert_array_equal(a, ra.astype(np.float32))
    np.testing.assert_array_equal(b, rb.astype(np.float32))


# --------------------------------------------------------------------------
# Attention: per-head Hadamard of queries and keys, head mixing of the output
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n_heads,dh", [(1, 16), (4, 8), (3, 32), (8, 4)])
def test_head_rht_equals_the_dense_block_diagonal_map(n_heads, dh):
    """(I_{n_h} (x) H_{d_h}) diag(s) / sqrt(d_h) built densely from the library
    Hadamard matrix and np.kron."""
    rng = np.random.default_rng(n_heads * 100 + dh)
    d = n_heads * dh
    x = rng.normal(size=(5, d))
    s = np.where(rng.integers(0, 2, size=d) == 1, 1, -1).astype(np.int8)
    dense = np.kron(np.eye(n_heads), scipy.linalg.hadamard(dh)) @ np.diag(s.astype(np.float64)) / math.sqrt(dh)
    np.testing.assert_allclose(oracle.head_rht(x, s, n_heads), x @ dense.T, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(oracle.head_rht(x, None, n_heads), oracle.head_rht(x, np.ones(d, np.int8), n_heads),
                               rtol=0, atol=0)


@pytest.mark.parametrize("n_heads,dh", [(2, 3), (4, 8), (8, 5), (16, 2)])
def test_head_mix_equals_the_dense_kronecker_map(n_heads, dh):
    """(H_{n_h} (x) I_{d_h}) diag(s) / sqrt(n_h) built densely; d_h need not be a
    power of two (it is only the stride)."""
    rng = np.random.default_rng(n_heads * 10 + dh)
    d = n_heads * dh
    x = rng.normal(size=(4, d))
    s = np.where(rng.integers(0, 2, size=d) == 1, 1, -1).astype(np.int8)
    dense = np.kron(scipy.linalg.hadamard(n_heads), np.eye(dh)) @ np.diag(s.astype(np.float64)) / math.sqrt(n_heads)
    np.testing.assert_allclose(oracle.head_mix(x, s, n_heads), x @ dense.T, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("n_heads,dh", [(4, 16), (32, 128), (8, 64)])
def test_head_mix_after_per_head_rotation_is_the_full_hadamard(n_heads, dh):
    """The identity the pages state for powers of two: (H_{n_h} (x) I)(I (x) H_{d_h})
    = H_{n_h d_h}, so mixing the heads of per-head-rotated activations equals
    the full Sylvester transform of order n_h d_h (normalised)."""
    rng = np.random.default_rng(dh)
    d = n_heads * dh
    x = rng.normal(size=(3, d))
    both = oracle.head_mix(oracle.head_rht(x, None, n_heads), None, n_heads)
    np.testing.assert_allclose(both, oracle.rht(x, np.ones(d, np.int8), 1), rtol=1e-11, atol=1e-11)


def test_per_head_rotation_keeps_the_attention_scores():
    """Rotating queries and keys with the same per-head Hadamard leaves every
    per-head dot product q_h . k_h unchanged (the pages: the scores P_1..P_{n_h}
    do not change), and every head keeps its norm."""
    rng = np.random.default_rng(3)
    n_heads, dh = 8, 64
    q = rng.normal(size=(6, n_heads * dh))
    k = rng.normal(size=(9, n_heads * dh))
    s = np.where(rng.integers(0, 2, size=n_heads * dh) == 1, 1, -1).astype(np.int8)
    qr, kr = oracle.head_rht(q, s, n_heads), oracle.head_rht(k, s, n_heads)
    for h in range(n_heads):
        sl = slice(h * dh, (h + 1) * dh)
        np.testing.assert_allclose(qr[:, sl] @ kr[:, sl].T, q[:, sl] @ k[:, sl].T, rtol=1e-12, atol=1e-11)
        np.testing.assert_allclose(np.linalg.norm(kr[:, sl], axis=1), np.linalg.norm(k[:, sl], axis=1), rtol=1e-13)


def test_head_rht_quant_is_per_head():
    """Each (token, head) group has its own step max|v_head| / qmax; a head of
    zeros gets scale 0 and zero codes while the other heads of the row do not;
    the worked example (20, 0, 0, 0) -> (10, 10, 10, 10), step 10/7, codes 7."""
    x = np.zeros((1, 3 * 4))
    x[0, 4] = 20.0                       # head 1: the worked example
    x[0, 8:12] = [1.0, -2.0, 3.0, 0.5]   # head 2: something else; head 0 stays zero
    r = oracle.head_rht_quant(x, None, 3, 4)
    np.testing.assert_array_equal(r["q"][0, 0:4], 0)
    assert r["scales"][0, 0] == 0.0
    np.testing.assert_array_equal(r["q"][0, 4:8], [7, 7, 7, 7])
    assert r["scales"][0, 1] == pytest.approx(10.0 / 7.0, rel=1e-15)
    v2 = oracle.head_rht(x, None, 3)[0, 8:12]
    assert r["scales"][0, 2] == pytest.approx(np.abs(v2).max() / 7.0, rel=1e-15)
    q, a, _ = oracle.quant_sym(v2[None, :], 4)
    np.testing.assert_array_equal(r["q"][0, 8:12], q[0])


def test_head_mix_quant_is_the_composition_of_its_steps():
    g = inputs.rht_case(5, 32 * 24, 1, 13, dtype="bf16", bits=3, n_outliers=4, outlier_scale=30.0)
    r = oracle.head_mix_quant(g.x, g.signs, 32, 3)
    v = oracle.head_mix(g.x, g.signs, 32)
    q, a, pre = oracle.quant_sym(v, 3)
    np.testing.assert_array_equal(r["q"], q)
    np.testing.assert_array_equal(r["scales"], a)
    np.testing.assert_array_equal(r["codes"], oracle.pack(q, 3))


# --------------------------------------------------------------------------
# The INT4 consumer GEMM: INT32 accumulation, then row scale x column scale
# --------------------------------------------------------------------------

def test_w4a4_gemm_integer_products_are_exact():
    """acc = qa qw^T over the full 4-bit two's complement range, against an
    independent unpacker and numpy's int64 matrix product; the extreme case
    K x (-8)(-8) stays exact."""
    from tests import helpers as H
    rng = np.random.default_rng(11)
    qa = rng.integers(-8, 8, size=(9, 256)).astype(np.int8)
    qw = rng.integers(-8, 8, size=(13, 256)).astype(np.int8)
    ca, cw = oracle.pack(qa, 4), oracle.pack(qw, 4)
    np.testing.assert_array_equal(H.unpack_int4(ca, 256), qa)
    r = oracle.w4a4_gemm(ca, np.ones(9), cw, np.ones(13))
    np.testing.assert_array_equal(r["acc"], qa.astype(np.int64) @ qw.astype(np.int64).T)
    big = np.full((1, 4096), -8, np.int8)
    rb = oracle.w4a4_gemm(oracle.pack(big, 4), [1.0], oracle.pack(big, 4), [1.0])
    assert rb["acc"][0, 0] == 64 * 4096


def test_w4a4_gemm_equals_the_product_of_the_dequantised_operands():
    """y[t][n] = (sa[t] qa[t]) . (sw[n] qw[n]): the same number as dequantising
    both operands first and multiplying them (a different order of the same
    exact arithmetic)."""
    rng = np.random.default_rng(12)
    qa = rng.integers(-7, 8, size=(6, 128)).astype(np.int8)
    qw = rng.integers(-7, 8, size=(5, 128)).astype(np.int8)
    sa, sw = rng.uniform(0.01, 2.0, 6), rng.uniform(0.001, 0.1, 5)
    r = oracle.w4a4_gemm(oracle.pack(qa, 4), sa, oracle.pack(qw, 4), sw)
    deq = (sa[:, None] * qa) @ (sw[:, None] * qw).T
    np.testing.assert_allclose(r["y"], deq, rtol=1e-13, atol=1e-13 * np.abs(deq).max())


def test_w4a4_gemm_stays_within_the_quantisation_error_bound():
    """Quantise real activations per token and weights per output channel
    (round to nearest, steps a and w); the GEMM of the codes approximates X W^T
    within sum_k (|x_k| w/2 + |w_k| a/2 + a w / 4)."""
    rng = np.random.default_rng(13)
    X = rng.normal(size=(8, 512))
    W = rng.normal(scale=0.05, size=(16, 512))
    qa, sa, _ = oracle.quant_sym(X, 4)
    qwt = oracle.quant_weights_rtn(W, 4)
    r = oracle.w4a4_gemm(oracle.pack(qa, 4), sa, qwt["codes"], qwt["scales"])
    exact = X @ W.T
    bound = (np.abs(X) @ np.ones((512, 16))) * (qwt["scales"][None, :] / 2) + \
            (np.ones((8, 512)) @ np.abs(W).T) * (sa[:, None] / 2) + 512 * sa[:, None] * qwt["scales"][None, :] / 4
    assert np.all(np.abs(r["y"] - exact) <= bound)
    assert np.abs(r["y"] - exact).max() < 0.5 * np.abs(exact).max()


# --------------------------------------------------------------------------
# The offline (Q, M) construction: SVD of T - I, subspace, polar factor
# --------------------------------------------------------------------------

def test_qm_reproduces_a_transition_whose_deviation_has_rank_r():
    """range(T - I) is invariant under an orthogonal T, so when T - I has rank k
    the top-k subspace captures all of it and T_hat = T exactly; r = D is the
    trivial case."""
    R_in, R_out = inputs.near_hadamard_pair(128, 5, n_planes=8)   # deviation of rank 16
    for r in (16, 128):
        c = oracle.qm_construct(R_in, R_out, r)
        np.testing.assert_allclose(oracle.t_hat(c["Q"], c["M"]), c["T"], rtol=0, atol=1e-12)
    assert np.linalg.norm(oracle.t_hat(*[oracle.qm_construct(R_in, R_out, 8)[k] for k in ("Q", "M")]) -
                          R_out @ R_in.T) > 0.1


@pytest.mark.parametrize("r", [2, 8, 32])
def test_qm_t_hat_is_a_rotation(r):
    """The pages: after the polar step T_hat = I + Q (R_sub - I) Q^T is in SO(D)."""
    R_in, R_out = inputs.near_hadamard_pair(256, 7)
    c = oracle.qm_construct(R_in, R_out, r)
    Th = oracle.t_hat(c["Q"], c["M"])
    np.testing.assert_allclose(Th.T @ Th, np.eye(256), rtol=0, atol=1e-10)
    sign, _ = np.linalg.slogdet(Th)
    assert sign == 1.0
    np.testing.assert_allclose(c["R_sub"].T @ c["R_sub"], np.eye(r), rtol=0, atol=1e-12)
    assert np.linalg.det(c["R_sub"]) > 0
    np.testing.assert_allclose(c["Q"].T @ c["Q"], np.eye(r), rtol=0, atol=1e-12)


def test_qm_error_does_not_grow_with_the_rank():
    """||T - T_hat||_F over r = 2, 4, ..., D (even r: the singular values of the
    deviation of a rotation come in pairs) is non-increasing, as in the pages'
    rank ablation, and zero at full rank."""
    R_in, R_out = inputs.near_hadamard_pair(256, 9)
    errs = []
    for r in (2, 4, 8, 16, 32, 64, 128, 256):
        c = oracle.qm_construct(R_in, R_out, r)
        errs.append(np.linalg.norm(oracle.t_hat(c["Q"], c["M"]) - c["T"]))
    assert all(b <= a + 1e-12 for a, b in zip(errs, errs[1:])), errs
    assert errs[-1] < 1e-12


def test_qm_polar_factor_is_the_nearest_rotation():
    """R_sub = U V^T is the rotation nearest to T_sub: R_sub^T T_sub is symmetric
    positive semidefinite, and small rotations of R_sub are farther from T_sub."""
    R_in, R_out = inputs.near_hadamard_pair(128, 11)
    c = oracle.qm_construct(R_in, R_out, 16)
    P = c["R_sub"].T @ c["T_sub"]
    np.testing.assert_allclose(P, P.T, rtol=0, atol=1e-12)
    assert np.linalg.eigvalsh((P + P.T) / 2).min() > -1e-12
    rng = np.random.default_rng(1)
    base = np.linalg.norm(c["R_sub"] - c["T_sub"])
    for _ in range(20):
        A = rng.normal(scale=0.01, size=(16, 16))
        A = A - A.T
        G = np.linalg.solve(np.eye(16) - A, np.eye(16) + A)
        assert np.linalg.norm(c["R_sub"] @ G - c["T_sub"]) >= base - 1e-12


def test_qm_feeds_the_online_path():
    """The constructed (Q, M) in the three-step online path equals the dense
    T_hat applied to the rows."""
    R_in, R_out = inputs.near_hadamard_pair(256, 13)
    c = oracle.qm_construct(R_in, R_out, 32)
    x = np.random.default_rng(2).normal(size=(7, 256))
    np.testing.assert_allclose(oracle.residual_align(x, c["Q"], c["M"]), x @ oracle.t_hat(c["Q"], c["M"]).T,
                               rtol=1e-12, atol=1e-12)


# --------------------------------------------------------------------------
# FlatQuant's Kronecker affine transform (Infra Quant II, FlatQuant):
# x P with P = P1 (x) P2 is vec(P1^T X P2), X the row-major n1 x n2 reshape
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n1,n2", [(4, 8), (8, 4), (3, 5), (12, 16)])
def test_kron_affine_equals_the_explicit_kronecker_product(n1, n2):
    # numpy's kron gives P[a n2 + b][i n2 + j] = P1[a][i] P2[b][j]; the factors are
    # not symmetric and the shapes not square, so a transposed factor, swapped
    # roles of n1 and n2 or a column-major reshape all fail
    rng = np.random.default_rng(100 * n1 + n2)
    P1, P2 = rng.standard_normal((n1, n1)), rng.standard_normal((n2, n2))
    x = rng.standard_normal((5, n1 * n2))
    ref = x @ np.kron(P1, P2)
    np.testing.assert_allclose(oracle.kron_affine(x, P1, P2), ref, rtol=0, atol=1e-12 * np.abs(ref).max())


def test_kron_affine_is_undone_by_the_inverse_factors():
    # (P1 (x) P2)^-1 = P1^-1 (x) P2^-1
    c = inputs.kron_affine_case(6, 8, 16, 2, dtype="f32")
    v = oracle.kron_affine(c.x, c.P1, c.P2)
    back = oracle.kron_affine(v, np.linalg.inv(c.P1.astype(np.float64)), np.linalg.inv(c.P2.astype(np.float64)))
    np.testing.assert_allclose(back, c.x, rtol=0, atol=1e-9 * np.abs(c.x).max())


@pytest.mark.parametrize("bits", [3, 4])
def test_kron_affine_quant_with_identity_factors_is_the_plain_quantiser(bits):
    c = inputs.kron_affine_case(7, 8, 16, 4, dtype="f32", bits=bits)
    r = oracle.kron_affine_quant(c.x, np.eye(8), np.eye(16), bits)
    q, a, _ = oracle.quant_sym(c.x, bits)
    np.testing.assert_array_equal(r["q"], q)
    np.testing.assert_array_equal(r["scales"], a)
    np.testing.assert_array_equal(r["codes"], oracle.pack(q, bits))


@pytest.mark.parametrize("bits", [3, 4])
def test_kron_affine_quant_with_sylvester_factors_is_the_hadamard_path(bits):
    # H_n1 (x) H_n2 = H_{n1 n2} (Sylvester, index a n2 + b): the codes are those of
    # the unrandomised Hadamard path, whose values carry the extra 1/sqrt(d)
    n1, n2 = 16, 32
    c = inputs.kron_affine_case(9, n1, n2, 5, dtype="f32", bits=bits)
    r = oracle.kron_affine_quant(c.x, oracle.sylvester(n1), oracle.sylvester(n2), bits)
    h = oracle.rht_quant(c.x, np.ones(n1 * n2, dtype=np.int8), 1, bits)
    np.testing.assert_array_equal(r["q"], h["q"])
    np.testing.assert_allclose(r["scales"], h["scales"] * math.sqrt(n1 * n2), rtol=1e-12)


def test_kron_affine_quant_zero_rows_and_step_bound():
    c = inputs.kron_affine_case(6, 8, 8, 6, dtype="f32", bits=4)
    x = c.x.copy()
    x[2] = 0.0
    r = oracle.kron_affine_quant(x, c.P1, c.P2, 4)
    assert r["scales"][2] == 0.0 and not r["q"][2].any()
    v = oracle.kron_affine(x, c.P1, c.P2)
    deq = r["q"].astype(np.float64) * r["scales"][:, None]
    assert np.all(np.abs(deq - v) <= 0.5 * r["scales"][:, None] * (1 + 1e-12))
