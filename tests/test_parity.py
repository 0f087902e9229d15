"""GPU parity: the CUDA path (through the C ABI) against the float64 oracle.

Small cases are compared element by element over whole outputs; full-size
workloads are run in the bench's launch configuration and compared on sampled
rows (token rows are independent, so the oracle recomputes just those rows).
Tolerances are the ones in tests/helpers.py.
"""
import numpy as np
import pytest
import torch

import oracle
from tests import helpers as H
from w3a3_quantization_online_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _rsq():
    from w3a3_quantization_online_b200 import rsq
    return rsq


def _to_dev(x: np.ndarray, dtype: str) -> torch.Tensor:
    t = torch.from_numpy(np.ascontiguousarray(x)).to(DEV)
    return t.to(torch.bfloat16) if dtype == "bf16" else t


def _host(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy() if t.dtype == torch.bfloat16 else t.cpu().numpy()


def run_align(case, x_dev=None, in_place=False):
    rsq = _rsq()
    x = _to_dev(case.x, case.dtype) if x_dev is None else x_dev
    Q = torch.from_numpy(case.Q).to(DEV)
    M = torch.from_numpy(case.M).to(DEV)
    xo = x if in_place else None
    xo, codes, scales = rsq.rsq_align_norm_quant(x, Q, M, x_out=xo, bits=case.bits, eps=case.eps)
    assert rsq.device_status() == 0
    return _host(xo), codes.cpu().numpy(), scales.cpu().numpy()


def run_rht(case):
    rsq = _rsq()
    x = _to_dev(case.x, case.dtype)
    s = torch.from_numpy(case.signs).to(DEV)
    codes, scales = rsq.rht_quant(x, s, case.m, bits=case.bits)
    assert rsq.device_status() == 0
    return codes.cpu().numpy(), scales.cpu().numpy()


def check_align(case, rows=None, label=""):
    xo, codes, scales = run_align(case)
    sel = slice(None) if rows is None else rows
    ref = oracle.align_norm_quant(case.x[sel], case.Q, case.M, case.bits, case.eps)
    H.check_aligned(xo[sel], ref["x_out"], case.x[sel], case.dtype, label)
    H.check_scales(scales[sel], ref["scales"], label)
    return H.check_codes(codes[sel], ref["q"], ref["pre"], case.bits, label)


def check_rht(case, rows=None, label=""):
    codes, scales = run_rht(case)
    sel = slice(None) if rows is None else rows
    ref = oracle.rht_quant(case.x[sel], case.signs, case.m, case.bits)
    H.check_scales(scales[sel], ref["scales"], label)
    return H.check_codes(codes[sel], ref["q"], ref["pre"], case.bits, label)


# --------------------------------------------------------------------------
# the five workloads at oracle-friendly sizes (several tiles plus a ragged tail)
# --------------------------------------------------------------------------

def test_tiny_config_full():
    a, h = inputs.tiny_case(T=64)
    check_align(a, label="tiny align")
    check_rht(h, label="tiny rht")


@pytest.mark.parametrize("T", [1, 131, 512])
def test_hidden_4096_align_int4(T):
    a, _ = inputs.llama7b_case(T=T)
    check_align(a, label=f"hidden T={T}")


@pytest.mark.parametrize("T", [1, 131, 512])
def test_hidden_4096_rht_int4(T):
    _, h = inputs.llama7b_case(T=T)
    check_rht(h, label=f"rht4096 T={T}")


@pytest.mark.parametrize("T", [3, 200])
def test_down_proj_kronecker_12288(T):
    check_rht(inputs.down_proj_case(T=T), label=f"kron T={T}")


@pytest.mark.parametrize("T", [2, 131])
def test_w3a3_8192_int3(T):
    a, h = inputs.w3a3_case(T=T)
    check_align(a, label=f"w3a3 align T={T}")
    check_rht(h, label=f"w3a3 rht T={T}")


@pytest.mark.parametrize("T", [16, 300])
def test_chain_32_layers_teacher_forced(T):
    """Each layer runs in place on the residual stream; the oracle layer i takes
    the GPU's bf16 stream before layer i as its input."""
    rsq = _rsq()
    x0, qs, ms, _, _ = inputs.chain_case(T=T)
    x = _to_dev(x0, "bf16")
    for i in range(len(qs)):
        x_in = _host(x).copy()
        Q = torch.from_numpy(qs[i]).to(DEV)
        M = torch.from_numpy(ms[i]).to(DEV)
        _, codes, scales = rsq.rsq_align_norm_quant(x, Q, M, x_out=x, bits=4)
        torch.cuda.synchronize()
        ref = oracle.align_norm_quant(x_in, qs[i], ms[i], 4, 1e-5)
        H.check_aligned(_host(x), ref["x_out"], x_in, "bf16", f"layer {i}")
        H.check_scales(scales.cpu().numpy(), ref["scales"], f"layer {i}")
        H.check_codes(codes.cpu().numpy(), ref["q"], ref["pre"], 4, f"layer {i}")
    assert rsq.device_status() == 0
    # End to end: every layer is orthogonal, so in float64 the stream keeps its
    # norm; storing it in bf16 between layers drifts the norm by a few percent
    # over 32 layers.  The GPU stream must follow the oracle chain that stores
    # the stream in bf16 between layers (independent of the GPU's values).
    xr = x0.astype(np.float64)
    for i in range(len(qs)):
        xr = inputs.round_to_bf16(oracle.residual_align(xr, qs[i], ms[i]).astype(np.float32)).astype(np.float64)
    n1 = np.linalg.norm(_host(x).astype(np.float64), axis=1)
    np.testing.assert_allclose(n1, np.linalg.norm(xr, axis=1), rtol=2e-3)


def test_chain_32_layers_prefill_16384_sampled():
    """The 32-layer chain at prefill size (T = 16384, in place, bench launch
    configuration): every layer runs on the whole stream on the GPU; before
    each layer the sampled rows of the GPU's bf16 stream are taken as that
    layer's oracle input (teacher forcing), and after it that layer's x_out,
    codes and scales of those rows are checked against the oracle."""
    rsq = _rsq()
    T = 16384
    x0, qs, ms, _, _ = inputs.chain_case(T=T)
    rows = _sample(T, 40, seed=4)
    rows_dev = torch.from_numpy(rows).to(DEV)
    x = _to_dev(x0, "bf16")
    codes = torch.empty((T, 2048), dtype=torch.uint8, device=DEV)
    scales = torch.empty((T,), dtype=torch.float32, device=DEV)
    for i in range(len(qs)):
        x_in = _host(x[rows_dev])
        Q = torch.from_numpy(qs[i]).to(DEV)
        M = torch.from_numpy(ms[i]).to(DEV)
        rsq.rsq_align_norm_quant(x, Q, M, x_out=x, codes=codes, scales=scales, bits=4)
        ref = oracle.align_norm_quant(x_in, qs[i], ms[i], 4, 1e-5)
        H.check_aligned(_host(x[rows_dev]), ref["x_out"], x_in, "bf16", f"prefill layer {i}")
        H.check_scales(scales[rows_dev].cpu().numpy(), ref["scales"], f"prefill layer {i}")
        H.check_codes(codes[rows_dev].cpu().numpy(), ref["q"], ref["pre"], 4, f"prefill layer {i}")
    assert rsq.device_status() == 0
    del x, codes, scales
    torch.cuda.empty_cache()


@pytest.mark.parametrize("T", [16, 300])
def test_back_to_back_layers_match_the_synchronised_run(T):
    """The default kernels may start before the previous kernel of the stream
    has finished (they stage Q and M first); every layer's input is the previous
    layer's in-place output, so the unsynchronised chain must reproduce the
    synchronised one bit for bit -- also when rht_quant reads the stream that
    the alignment just wrote."""
    rsq = _rsq()
    x0, qs, ms, _, _ = inputs.chain_case(T=T)
    signs = torch.from_numpy(inputs.rht_case(1, 4096, 1, 7).signs).to(DEV)
    Qd = [torch.from_numpy(q).to(DEV) for q in qs]
    Md = [torch.from_numpy(m).to(DEV) for m in ms]

    def run(sync):
        x = _to_dev(x0, "bf16")
        outs = []
        for i in range(len(qs)):
            codes = torch.empty((T, 2048), dtype=torch.uint8, device=DEV)
            scales = torch.empty((T,), dtype=torch.float32, device=DEV)
            rsq.rsq_align_norm_quant(x, Qd[i], Md[i], x_out=x, codes=codes, scales=scales, bits=4)
            if sync:
                torch.cuda.synchronize()
            hc, hs = rsq.rht_quant(x, signs, bits=4)
            if sync:
                torch.cuda.synchronize()
            outs.append((codes, scales, hc, hs))
        torch.cuda.synchronize()
        return _host(x), [tuple(t.cpu().numpy() for t in o) for o in outs]

    x_sync, o_sync = run(True)
    x_fast, o_fast = run(False)
    assert np.array_equal(x_sync.view(np.uint32), x_fast.view(np.uint32))
    for i, (a, b) in enumerate(zip(o_sync, o_fast)):
        for u, v in zip(a, b):
            assert np.array_equal(u, v), f"layer {i}"
    assert rsq.device_status() == 0


@pytest.mark.parametrize("T", [7, 17, 1000])
def test_repeated_back_to_back_launches_are_deterministic(T):
    """Hundreds of launches of the default kernels back to back on one stream
    (each may start before the previous one ends) reproduce the first outputs
    bit for bit and leave the device status word clean."""
    rsq = _rsq()
    a, h = inputs.llama7b_case(T=T)
    x = torch.from_numpy(a.x).to(DEV).to(torch.bfloat16)
    Q = torch.from_numpy(a.Q).to(DEV)
    M = torch.from_numpy(a.M).to(DEV)
    xh = torch.from_numpy(h.x).to(DEV).to(torch.bfloat16)
    sg = torch.from_numpy(h.signs).to(DEV)

    def run():
        xo, ca, sa = rsq.rsq_align_norm_quant(x, Q, M, bits=4)
        ch, sh = rsq.rht_quant(xh, sg, bits=4)
        return xo.view(torch.int16), ca, sa, ch, sh

    ref = [t.clone() for t in run()]
    for i in range(300):
        out = run()
        if i % 100 == 99:
            for u, v in zip(out, ref):
                assert torch.equal(u, v), f"launch {i}"
    assert rsq.device_status() == 0


@pytest.mark.parametrize("T", [1, 129, 3001])
def test_int3_at_4096_on_the_tensor_core_kernels(T):
    """INT3 at D = d = 4096 (cluster-of-8 alignment kernel with the deferred
    INT3 code stores; the RHT tensor-core kernel) against the oracle."""
    a = inputs.align_case(T, 4096, 32, 300 + T, dtype="bf16", bits=3, dist="student_t3", n_outliers=8,
                          outlier_scale=100.0)
    check_align(a, label=f"int3 align T={T}")
    h = inputs.rht_case(T, 4096, 1, 400 + T, dtype="bf16", bits=3, dist="student_t3", n_outliers=8,
                        outlier_scale=100.0)
    check_rht(h, label=f"int3 rht T={T}")


def test_bounded_wait_runs_out_and_reports():
    """The kernels' bounded wait, on an mbarrier that nothing arrives on, gives
    up after its limit; the kernel returns and sets the timeout bit of the
    device status word; the context stays usable (no fault, no hang)."""
    rsq = _rsq()
    assert rsq.device_status() == 0
    rsq.selftest_wait_timeout(20)
    assert rsq.device_status() == 1
    assert rsq.device_status() == 0  # read and cleared
    a, _ = inputs.llama7b_case(T=64)
    check_align(a, label="after the timeout self test")
    assert rsq.device_status() == 0


# --------------------------------------------------------------------------
# full sizes, sampled rows
# --------------------------------------------------------------------------

def _sample(T, n=48, seed=0):
    rng = np.random.default_rng(seed)
    rows = np.unique(np.concatenate([[0, T - 1], rng.choice(T, n, replace=False)]))
    return rows


def test_full_hidden_16384_sampled():
    a, h = inputs.llama7b_case(T=16384)
    rows = _sample(16384)
    check_align(a, rows, "hidden T=16384")
    check_rht(h, rows, "rht4096 T=16384")


def test_full_down_proj_sampled():
    h = inputs.down_proj_case(T=4096)
    check_rht(h, _sample(4096, 24), "kron T=4096")


def test_full_w3a3_sampled():
    a, h = inputs.w3a3_case(T=8192)
    rows = _sample(8192, 24)
    check_align(a, rows, "w3a3 T=8192")
    check_rht(h, rows, "w3a3 rht T=8192")


def test_batch_past_32_bit_byte_offsets():
    """T = 2^19 rows at D = 4096: 4 GiB of bf16 input, so x_out reaches past
    every 32-bit byte offset (codes up to 1 GiB).  The batch is one seeded
    8192-row block repeated 64 times on the device, so every block of every
    output must equal the first block bit for bit; sampled rows of the last
    block are also checked against the oracle on their source rows."""
    rsq = _rsq()
    blk, reps = 8192, 64
    a, h = inputs.llama7b_case(T=blk)
    x = _to_dev(a.x, "bf16").repeat(reps, 1)
    Q = torch.from_numpy(a.Q).to(DEV)
    M = torch.from_numpy(a.M).to(DEV)
    s = torch.from_numpy(h.signs).to(DEV)
    xo, codes, scales = rsq.rsq_align_norm_quant(x, Q, M, bits=4, eps=a.eps)
    hcodes, hscales = rsq.rht_quant(x, s, 1, bits=4)
    torch.cuda.synchronize()
    assert rsq.device_status() == 0
    for k in (1, reps // 2, reps - 1):
        sl = slice(k * blk, (k + 1) * blk)
        assert torch.equal(xo[sl].view(torch.int16), xo[:blk].view(torch.int16)), k
        assert torch.equal(codes[sl], codes[:blk]) and torch.equal(scales[sl], scales[:blk]), k
        assert torch.equal(hcodes[sl], hcodes[:blk]) and torch.equal(hscales[sl], hscales[:blk]), k
    rows = _sample(blk, 16)
    last = torch.from_numpy((reps - 1) * blk + rows).to(DEV)
    ref = oracle.align_norm_quant(a.x[rows], a.Q, a.M, 4, a.eps)
    H.check_aligned(_host(xo[last]), ref["x_out"], a.x[rows], "bf16", "T=2^19 align")
    H.check_scales(scales[last].cpu().numpy(), ref["scales"], "T=2^19 align")
    H.check_codes(codes[last].cpu().numpy(), ref["q"], ref["pre"], 4, "T=2^19 align")
    refh = oracle.rht_quant(a.x[rows], h.signs, 1, 4)
    H.check_scales(hscales[last].cpu().numpy(), refh["scales"], "T=2^19 rht")
    H.check_codes(hcodes[last].cpu().numpy(), refh["q"], refh["pre"], 4, "T=2^19 rht")
    del x, xo, codes, scales, hcodes, hscales
    torch.cuda.empty_cache()


# --------------------------------------------------------------------------
# edge cases
# --------------------------------------------------------------------------

def test_empty_batch_launches_nothing():
    rsq = _rsq()
    before = rsq.launch_count()
    x = torch.empty((0, 256), dtype=torch.bfloat16, device=DEV)
    Q = torch.zeros((256, 8), device=DEV)
    M = torch.zeros((8, 8), device=DEV)
    xo, codes, scales = rsq.rsq_align_norm_quant(x, Q, M)
    codes2, scales2 = rsq.rht_quant(x, torch.ones(256, dtype=torch.int8, device=DEV))
    assert xo.shape == (0, 256) and codes.shape == (0, 128) and codes2.shape == (0, 128)
    assert rsq.launch_count() == before


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_zero_rows_give_zero_scale_and_codes(dtype):
    a = inputs.align_case(9, 256, 8, 5, dtype=dtype)
    a.x[[0, 4, 8]] = 0.0
    xo, codes, scales = run_align(a)
    assert np.all(scales[[0, 4, 8]] == 0) and np.all(codes[[0, 4, 8]] == 0)
    assert np.all(xo[[0, 4, 8]] == 0)
    check_align(a, label="zero rows")
    h = inputs.rht_case(9, 256, 1, 5, dtype=dtype)
    h.x[[1, 7]] = 0.0
    codes, scales = run_rht(h)
    assert np.all(scales[[1, 7]] == 0) and np.all(codes[[1, 7]] == 0)
    check_rht(h, label="zero rows rht")


@pytest.fixture
def generic_align():
    rsq = _rsq()
    prev = rsq.select_align_kernel(rsq.ALIGN_GENERIC)
    yield
    rsq.select_align_kernel(prev)


@pytest.mark.parametrize("T", [1, 200])
def test_generic_kernel_at_the_tensor_core_shapes(generic_align, T):
    a, _ = inputs.llama7b_case(T=T)
    check_align(a, label=f"generic hidden T={T}")
    a, _ = inputs.w3a3_case(T=T)
    check_align(a, label=f"generic w3a3 T={T}")


@pytest.mark.parametrize("which", [2])
def test_tensor_core_kernel_serves_the_hot_shapes(which):
    rsq = _rsq()
    prev = rsq.select_align_kernel(which)
    try:
        for T in (1, 128, 129, 1000):
            a, _ = inputs.llama7b_case(T=T)
            check_align(a, label=f"tc hidden T={T}")
        a, _ = inputs.w3a3_case(T=257)
        check_align(a, label="tc w3a3 T=257")
        for r in (1, 7, 32):
            a = inputs.align_case(300, 4096, r, 40 + r, dtype="bf16", n_outliers=8, outlier_scale=100.0)
            check_align(a, label=f"tc r={r}")
        for T in (3000,):  # several tiles per cluster, ragged last tile
            a, _ = inputs.llama7b_case(T=T)
            check_align(a, rows=np.arange(0, T, 7), label=f"tc hidden T={T}")
        a = inputs.align_case(96, 4096, 32, 77, dtype="bf16", dist="student_t3")
        a.x[[0, 50, 95]] = 0.0
        xo, codes, scales = run_align(a)
        assert np.all(scales[[0, 50, 95]] == 0) and np.all(codes[[0, 50, 95]] == 0)
        check_align(a, label="tc zero rows")
        # codes buffer only 16-byte aligned: the kernel must not use 32-byte stores
        a, _ = inputs.llama7b_case(T=40)
        x = _to_dev(a.x, "bf16")
        Q = torch.from_numpy(a.Q).to(DEV)
        M = torch.from_numpy(a.M).to(DEV)
        big = torch.zeros(40 * 2048 + 16, dtype=torch.uint8, device=DEV)
        codes16 = big[16:].view(40, 2048)
        _, _, sc = rsq.rsq_align_norm_quant(x, Q, M, codes=codes16, bits=4)
        assert rsq.device_status() == 0
        ref = oracle.align_norm_quant(a.x, a.Q, a.M, 4, a.eps)
        H.check_codes(codes16.cpu().numpy(), ref["q"], ref["pre"], 4, "tc 16B-aligned codes")
        H.check_scales(sc.cpu().numpy(), ref["scales"], "tc 16B-aligned codes")
    finally:
        rsq.select_align_kernel(prev)


def test_decode_kernel_serves_small_batches():
    rsq = _rsq()
    prev = rsq.select_align_kernel(rsq.ALIGN_DECODE)
    try:
        for T in (1, 5, 16, 32):
            a, _ = inputs.llama7b_case(T=T)
            check_align(a, label=f"decode hidden T={T}")
        a, _ = inputs.w3a3_case(T=31)  # D = 8192, INT3
        check_align(a, label="decode w3a3 T=31")
        for r in (1, 7, 32):
            a = inputs.align_case(16, 4096, r, 50 + r, dtype="bf16", n_outliers=8, outlier_scale=100.0)
            check_align(a, label=f"decode r={r}")
        a = inputs.align_case(9, 2048, 16, 9, dtype="f32", n_outliers=2, outlier_scale=20.0)
        check_align(a, label="decode f32 D=2048")
        a = inputs.align_case(12, 4096, 32, 11, dtype="bf16", dist="student_t3")
        a.x[[0, 5]] = 0.0
        a.x[7] *= np.float32(2.0 ** -120)  # absmax far below 2^-64: rescaled path
        a.x = inputs.round_to_bf16(a.x)
        xo, codes, scales = run_align(a)
        assert np.all(scales[[0, 5]] == 0) and np.all(codes[[0, 5]] == 0)
        check_align(a, label="decode zero and tiny rows")
        # in place, as the chain runs it
        a, _ = inputs.llama7b_case(T=16)
        xo1, c1, s1 = run_align(a)
        x = _to_dev(a.x, "bf16")
        xo2, c2, s2 = run_align(a, x_dev=x, in_place=True)
        np.testing.assert_array_equal(xo1, xo2)
        np.testing.assert_array_equal(c1, c2)
        np.testing.assert_array_equal(s1, s2)
        # more rows than the decode kernel takes: refused, nothing launched
        a, _ = inputs.llama7b_case(T=33)
        with pytest.raises(rsq.RsqError):
            run_align(a)
    finally:
        rsq.select_align_kernel(prev)


def test_in_place_update_equals_out_of_place():
    a, _ = inputs.llama7b_case(T=77)
    xo1, c1, s1 = run_align(a)
    x = _to_dev(a.x, "bf16")
    xo2, c2, s2 = run_align(a, x_dev=x, in_place=True)
    np.testing.assert_array_equal(xo1, xo2)
    np.testing.assert_array_equal(c1, c2)
    np.testing.assert_array_equal(s1, s2)
    np.testing.assert_array_equal(_host(x), xo2)


@pytest.mark.parametrize("D,r", [(16, 1), (48, 3), (64, 64), (272, 17), (1024, 32), (12288, 32)])
@pytest.mark.parametrize("dtype,bits", [("f32", 4), ("bf16", 3)])
def test_odd_shapes(D, r, dtype, bits):
    a = inputs.align_case(37, D, r, D + r, dtype=dtype, bits=bits, n_outliers=2, outlier_scale=20.0)
    check_align(a, label=f"D={D} r={r}")


@pytest.mark.parametrize("d,m", [(16, 1), (64, 1), (2048, 1), (16384, 1),
                                 (192, 12), (24576, 12)])
@pytest.mark.parametrize("dtype,bits", [("f32", 4), ("bf16", 3)])
def test_rht_shapes(d, m, dtype, bits):
    h = inputs.rht_case(19, d, m, d + m, dtype=dtype, bits=bits, n_outliers=3, outlier_scale=40.0)
    check_rht(h, label=f"d={d} m={m}")


@pytest.mark.parametrize("d,kernels", [(4096, (3, 1)), (8192, (3, 1))])
def test_rht_kernels_agree_with_the_oracle(d, kernels):
    rsq = _rsq()
    for which in kernels:
        prev = rsq.select_rht_kernel(which)
        try:
            for T in (1, 7, 600):
                for bits in (4, 3):
                    h = inputs.rht_case(T, d, 1, 60 + T + bits + d, dtype="bf16", bits=bits, n_outliers=8,
                                        outlier_scale=100.0)
                    check_rht(h, label=f"rht d={d} kernel {which} T={T} bits={bits}")
        finally:
            rsq.select_rht_kernel(prev)


@pytest.mark.parametrize("which", [1, 4])
def test_kronecker_12288_kernels(which):
    rsq = _rsq()
    prev = rsq.select_rht_kernel(which)
    try:
        for T in (1, 7, 300):
            check_rht(inputs.down_proj_case(T=T), label=f"kron kernel {which} T={T}")
        h = inputs.rht_case(6, 12288, 12, 5, dtype="bf16", n_outliers=4, outlier_scale=50.0)
        h.x[1] = 0.0
        h.x[2] *= np.float32(2.0 ** -120)  # absmax far below 2^-64: rescaled path
        h.x = inputs.round_to_bf16(h.x)
        codes, scales = run_rht(h)
        assert scales[1] == 0 and np.all(codes[1] == 0)
        check_rht(h, label=f"kron kernel {which} zero and tiny rows")
    finally:
        rsq.select_rht_kernel(prev)


def check_gate(case, rows=None, label=""):
    rsq = _rsq()
    a = _to_dev(case.a, case.dtype)
    b = _to_dev(case.b, case.dtype)
    s = torch.from_numpy(case.signs).to(DEV)
    codes, scales = rsq.rht_quant_silu_gate(a, b, s, case.m, bits=case.bits)
    assert rsq.device_status() == 0
    codes, scales = codes.cpu().numpy(), scales.cpu().numpy()
    sel = slice(None) if rows is None else rows
    ref = oracle.rht_quant_gate(case.a[sel], case.b[sel], case.signs, case.m, case.bits)
    H.check_scales(scales[sel], ref["scales"], label)
    return H.check_codes(codes[sel], ref["q"], ref["pre"], case.bits, label)


@pytest.mark.parametrize("which", [0, 1, 4])
def test_silu_gate_down_proj_12288(which):
    """The gated down_proj input (SiLU(a) * b formed in fp32 in the kernel) at
    d = 12288 = 1024 * 12: the Kronecker kernel (default) and the radix-16 one."""
    rsq = _rsq()
    prev = rsq.select_rht_kernel(which)
    try:
        for T in (1, 7, 300):
            check_gate(inputs.down_proj_gate_case(T=T), label=f"gate kernel {which} T={T}")
        g = inputs.down_proj_gate_case(T=6)
        g.b[1] = 0.0                         # zero row
        g.a[2] = np.float32(-30.0)           # strongly negative gate: a row of tiny values
        g.a[3, :7] = np.float32(100.0)       # large gate: SiLU(a) -> a
        check_gate(g, label=f"gate kernel {which} edge rows")
    finally:
        rsq.select_rht_kernel(prev)


@pytest.mark.parametrize("d,m,dtype,bits", [(4096, 1, "bf16", 4), (8192, 1, "bf16", 3), (256, 1, "f32", 4),
                                             (192, 12, "f32", 3), (16, 1, "bf16", 4)])
def test_silu_gate_other_shapes(d, m, dtype, bits):
    check_gate(inputs.gate_case(37, d, m, d + m + bits, dtype=dtype, bits=bits), label=f"gate d={d} m={m}")


def test_silu_gate_full_down_proj_sampled():
    g = inputs.down_proj_gate_case(T=4096)
    check_gate(g, _sample(4096, 24), "gate T=4096")


def _signs_dev(case, use):
    return torch.from_numpy(case.signs).to(DEV) if use else None


@pytest.mark.parametrize("n_heads,d_head", [(32, 128), (1, 16), (7, 64), (3, 256), (64, 32)])
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_heads_rotation(n_heads, d_head, dtype):
    """Per-head rotation of queries / keys against the oracle (rotated values:
    the same tolerance as aligned values), with and without signs, and in place."""
    rsq = _rsq()
    c = inputs.rht_case(33, n_heads * d_head, 1, n_heads + d_head, dtype=dtype, n_outliers=3, outlier_scale=20.0)
    for use_signs in (True, False):
        x = _to_dev(c.x, dtype)
        out = rsq.rht_heads(x, _signs_dev(c, use_signs), n_heads)
        torch.cuda.synchronize()
        ref = oracle.head_rht(c.x, c.signs if use_signs else None, n_heads)
        H.check_aligned(_host(out), ref, c.x, dtype, f"heads {n_heads}x{d_head} {dtype} signs={use_signs}")
        rsq.rht_heads(x, _signs_dev(c, use_signs), n_heads, x_out=x)  # in place
        torch.cuda.synchronize()
        np.testing.assert_array_equal(_host(x), _host(out))
    assert rsq.device_status() == 0


def test_heads_rotation_keeps_the_scores():
    """Queries and keys rotated on the GPU (fp32 I/O) with the same signs give
    the same per-head dot products as the unrotated ones."""
    rsq = _rsq()
    n_heads, d_head = 32, 128
    q = inputs.rht_case(16, n_heads * d_head, 1, 61, dtype="f32", n_outliers=4, outlier_scale=20.0)
    k = inputs.rht_case(40, n_heads * d_head, 1, 62, dtype="f32", n_outliers=4, outlier_scale=20.0)
    s = torch.from_numpy(q.signs).to(DEV)
    qr = _host(rsq.rht_heads(_to_dev(q.x, "f32"), s, n_heads)).astype(np.float64)
    kr = _host(rsq.rht_heads(_to_dev(k.x, "f32"), s, n_heads)).astype(np.float64)
    for h in range(n_heads):
        sl = slice(h * d_head, (h + 1) * d_head)
        ref = q.x[:, sl].astype(np.float64) @ k.x[:, sl].astype(np.float64).T
        np.testing.assert_allclose(qr[:, sl] @ kr[:, sl].T, ref, rtol=1e-5, atol=1e-4 * np.abs(ref).max())


def check_heads_quant(case, n_heads, use_signs=True, rows=None, label=""):
    rsq = _rsq()
    codes, scales = rsq.rht_heads_quant(_to_dev(case.x, case.dtype), _signs_dev(case, use_signs), n_heads,
                                        bits=case.bits)
    assert rsq.device_status() == 0
    sel = slice(None) if rows is None else rows
    ref = oracle.head_rht_quant(case.x[sel], case.signs if use_signs else None, n_heads, case.bits)
    H.check_scales(scales.cpu().numpy()[sel].ravel(), ref["scales"].ravel(), label)
    return H.check_codes(codes.cpu().numpy()[sel], ref["q"], ref["pre"], case.bits, label)


def check_head_mix(case, n_heads, use_signs=True, rows=None, label=""):
    rsq = _rsq()
    codes, scales = rsq.rht_head_mix_quant(_to_dev(case.x, case.dtype), _signs_dev(case, use_signs), n_heads,
                                           bits=case.bits)
    assert rsq.device_status() == 0
    sel = slice(None) if rows is None else rows
    ref = oracle.head_mix_quant(case.x[sel], case.signs if use_signs else None, n_heads, case.bits)
    H.check_scales(scales.cpu().numpy()[sel], ref["scales"], label)
    return H.check_codes(codes.cpu().numpy()[sel], ref["q"], ref["pre"], case.bits, label)


@pytest.mark.parametrize("n_heads,d_head,dtype,bits", [(32, 128, "bf16", 4), (32, 128, "bf16", 3), (5, 16, "f32", 4),
                                                       (8, 256, "f32", 3), (64, 64, "bf16", 4)])
def test_heads_quant_per_head(n_heads, d_head, dtype, bits):
    c = inputs.rht_case(29, n_heads * d_head, 1, 7 + d_head, dtype=dtype, bits=bits, n_outliers=3,
                        outlier_scale=20.0)
    c.x[4] = 0.0                               # a zero row: every head scale 0
    c.x[5, :d_head] = 0.0                      # a zero head in an otherwise nonzero row
    check_heads_quant(c, n_heads, True, label=f"heads quant {n_heads}x{d_head}")
    check_heads_quant(c, n_heads, False, label=f"heads quant {n_heads}x{d_head} no signs")


@pytest.mark.parametrize("n_heads,d_head,dtype,bits", [(32, 128, "bf16", 4), (32, 128, "f32", 3), (2, 8, "bf16", 4),
                                                       (4, 96, "bf16", 3), (16, 512, "f32", 4), (64, 64, "bf16", 4),
                                                       (64, 256, "bf16", 3)])
def test_head_mix_quant(n_heads, d_head, dtype, bits):
    c = inputs.rht_case(23, n_heads * d_head, 1, 3 + n_heads, dtype=dtype, bits=bits, n_outliers=3,
                        outlier_scale=20.0)
    c.x[2] = 0.0
    check_head_mix(c, n_heads, True, label=f"head mix {n_heads}x{d_head}")
    check_head_mix(c, n_heads, False, label=f"head mix {n_heads}x{d_head} no signs")


@pytest.mark.parametrize("which", [3, 1])
@pytest.mark.parametrize("n_heads,d_head,T", [(32, 128, 600), (16, 64, 600), (32, 128, 1), (3, 128, 1000)])
def test_heads_tensor_core_and_cuda_core_kernels(which, n_heads, d_head, T):
    """rht_heads / rht_heads_quant through the tensor-core per-head kernel
    (which = 3; 128-token tiles, a ragged last tile, CTA ranges that cross a
    head boundary) and through the CUDA-core kernel (which = 1), bf16, each
    against the oracle."""
    rsq = _rsq()
    prev = rsq.select_rht_kernel(which)
    try:
        for bits in (4, 3):
            c = inputs.rht_case(T, n_heads * d_head, 1, T + n_heads + bits, dtype="bf16", bits=bits, n_outliers=3,
                                outlier_scale=20.0)
            if T > 7:
                c.x[7, d_head:2 * d_head] = 0.0  # a zero head
            x = _to_dev(c.x, "bf16")
            s = torch.from_numpy(c.signs).to(DEV)
            out = rsq.rht_heads(x, s, n_heads)
            torch.cuda.synchronize()
            H.check_aligned(_host(out), oracle.head_rht(c.x, c.signs, n_heads), c.x, "bf16",
                            f"heads kernel {which} {n_heads}x{d_head} T={T}")
            check_heads_quant(c, n_heads, True, label=f"heads quant kernel {which} {n_heads}x{d_head} T={T} b={bits}")
        assert rsq.device_status() == 0
    finally:
        rsq.select_rht_kernel(prev)


@pytest.mark.parametrize("which", [3, 1])
@pytest.mark.parametrize("T", [1, 3, 5, 600, 1001])
def test_head_mix_tensor_core_and_cuda_core_kernels(which, T):
    """rht_head_mix_quant at 32 heads x 128 through the tensor-core kernel
    (which = 3; groups of four tokens, a ragged last group when T % 4 != 0)
    and through the CUDA-core kernel (which = 1), bf16, INT4 and INT3, with
    and without signs, with a zero row and a row whose absmax is below 2^-64,
    each against the oracle."""
    rsq = _rsq()
    prev = rsq.select_rht_kernel(which)
    try:
        for bits in (4, 3):
            c = inputs.rht_case(T, 4096, 1, T + 11 * bits, dtype="bf16", bits=bits, n_outliers=3,
                                outlier_scale=20.0)
            if T > 2:
                c.x[1] = 0.0
                c.x[2] *= np.float32(2.0 ** -120)
                c.x = inputs.round_to_bf16(c.x)
            check_head_mix(c, 32, True, label=f"head mix kernel {which} T={T} b={bits}")
            check_head_mix(c, 32, False, label=f"head mix kernel {which} T={T} b={bits} no signs")
        assert rsq.device_status() == 0
    finally:
        rsq.select_rht_kernel(prev)


def test_heads_tensor_core_kernel_rejects_other_shapes():
    rsq = _rsq()
    prev = rsq.select_rht_kernel(3)
    try:
        x = torch.zeros((4, 3 * 256), dtype=torch.bfloat16, device=DEV)
        with pytest.raises(rsq.RsqError):
            rsq.rht_heads(x, None, 3)
    finally:
        rsq.select_rht_kernel(prev)


def test_attention_transforms_full_size_sampled():
    """T = 16384 tokens of 32 x 128 attention activations: per-head rotation,
    per-head key quantisation and head mixing with per-token quantisation, in
    the bench's launch configuration, sampled rows against the oracle."""
    rsq = _rsq()
    c = inputs.attention_case(T=16384)
    rows = _sample(16384, 32, seed=7)
    x = _to_dev(c.x, "bf16")
    s = torch.from_numpy(c.signs).to(DEV)
    out = rsq.rht_heads(x, s, 32)
    torch.cuda.synchronize()
    H.check_aligned(_host(out)[rows], oracle.head_rht(c.x[rows], c.signs, 32), c.x[rows], "bf16", "heads T=16384")
    check_heads_quant(c, 32, True, rows, "heads quant T=16384")
    check_head_mix(c, 32, True, rows, "head mix T=16384")


def unpack_int4_rows(codes: np.ndarray) -> np.ndarray:
    """Packed 4-bit two's complement codes (element 2i in the low nibble of
    byte i) -> int8 values, written out from the packing rule."""
    c = codes.astype(np.int16)
    lo, hi = c & 15, c >> 4
    out = np.empty((codes.shape[0], 2 * codes.shape[1]), dtype=np.int16)
    out[:, 0::2], out[:, 1::2] = lo, hi
    return np.where(out >= 8, out - 16, out).astype(np.int8)


def run_gemm(case, out="f16", with_acc=True, rows=None, prepared=False):
    rsq = _rsq()
    ca = torch.from_numpy(case.codes_a).to(DEV)
    cw = torch.from_numpy(case.codes_w).to(DEV)
    sa = torch.from_numpy(case.scales_a).to(DEV)
    sw = torch.from_numpy(case.scales_w).to(DEV)
    acc = torch.empty((case.T, case.N), dtype=torch.int32, device=DEV) if with_acc else None
    od = torch.float16 if out == "f16" else torch.bfloat16
    if prepared:
        w8 = rsq.w4a4_prepare_weights(cw)
        np.testing.assert_array_equal(w8.cpu().numpy(), unpack_int4_rows(case.codes_w))
        y = rsq.w4a4_gemm_s8w(ca, sa, w8, sw, acc=acc, out_dtype=od)
    else:
        y = rsq.w4a4_gemm(ca, sa, cw, sw, acc=acc, out_dtype=od)
    assert rsq.device_status() == 0
    sel = slice(None) if rows is None else rows
    ref = oracle.w4a4_gemm(case.codes_a[sel], case.scales_a[sel], case.codes_w, case.scales_w)
    if with_acc:
        np.testing.assert_array_equal(acc.cpu().numpy()[sel], ref["acc"])  # integer products: bit-exact
    H.check_gemm(y.float().cpu().numpy()[sel], ref["y"], out, case.name)
    return y


@pytest.mark.parametrize("T,N,K", [(1, 8, 128), (128, 256, 128), (127, 264, 256), (300, 512, 1024),
                                   (129, 4096, 4096), (515, 1000, 384)])
@pytest.mark.parametrize("out", ["f16", "bf16"])
@pytest.mark.parametrize("prepared", [False, True])
def test_w4a4_gemm(T, N, K, out, prepared):
    """The INT4 GEMM on tcgen05 (kind::i8): exact int32 products over the full
    4-bit range, then the scale epilogue, against the oracle; several tiles and
    ragged edges in both output dimensions.  With prepared = True the weights
    go through w4a4_prepare_weights (checked against the packing rule) and
    w4a4_gemm_s8w."""
    run_gemm(inputs.gemm_case(T, N, K, T + N + K), out, prepared=prepared)


def test_w4a4_gemm_without_accumulator_copy_matches():
    c = inputs.gemm_case(200, 768, 512, 3)
    y1 = run_gemm(c, "f16", with_acc=True)
    y2 = run_gemm(c, "f16", with_acc=False)
    assert torch.equal(y1, y2)


def test_w4a4_gemm_consumes_the_quantiser_codes():
    """The consumer of the path, both chains independent: on the GPU the
    alignment quantiser's INT4 codes and scales feed the GEMM; in the oracle
    its own codes feed its own GEMM.  The codes agree up to the tie rule, and
    on every row whose codes agree exactly the GEMM outputs agree within the
    output rounding."""
    rsq = _rsq()
    a, _ = inputs.llama7b_case(T=256)
    x = _to_dev(a.x, "bf16")
    _, codes, scales = rsq.rsq_align_norm_quant(x, torch.from_numpy(a.Q).to(DEV), torch.from_numpy(a.M).to(DEV), bits=4)
    W = np.random.default_rng(9).normal(scale=0.02, size=(512, 4096))
    wq = oracle.quant_weights_rtn(W, 4)
    sw = wq["scales"].astype(np.float32)
    y = rsq.w4a4_gemm(codes, scales, torch.from_numpy(wq["codes"]).to(DEV), torch.from_numpy(sw).to(DEV))
    ref_a = oracle.align_norm_quant(a.x, a.Q, a.M, 4, a.eps)
    c_gpu = codes.cpu().numpy()
    H.check_codes(c_gpu, ref_a["q"], ref_a["pre"], 4, "quantiser codes")
    H.check_scales(scales.cpu().numpy(), ref_a["scales"], "quantiser scales")
    ref = oracle.w4a4_gemm(ref_a["codes"], ref_a["scales"].astype(np.float32), wq["codes"], sw)
    same = np.all(c_gpu == ref_a["codes"], axis=1)
    assert same.sum() >= 250
    # the activation scales may differ by the scale tolerance (1e-6): two more
    # float32-sized terms in the bound
    yg = y.float().cpu().numpy()[same].astype(np.float64)
    bound = (2.0 ** -11 + 4 * 2.0 ** -24 + 2e-6) * np.abs(ref["y"][same]) + 2.0 ** -24
    assert np.all(np.abs(yg - ref["y"][same]) <= bound)


@pytest.mark.parametrize("prepared", [False, True])
def test_w4a4_gemm_full_size_sampled(prepared):
    """T = 16384, N = K = 4096 (the hidden stream through a 4096 x 4096 INT4
    projection), sampled rows against the oracle; packed and prepared weights
    give the same outputs bit for bit."""
    c = inputs.gemm_case(16384, 4096, 4096, 21)
    y = run_gemm(c, "f16", with_acc=True, rows=_sample(16384, 24, seed=3), prepared=prepared)
    if prepared:
        y0 = run_gemm(c, "f16", with_acc=False, rows=np.array([0]), prepared=False)
        assert torch.equal(y.view(torch.int16), y0.view(torch.int16))


def run_qm(D, r, seed, iters=16, **kw):
    rsq = _rsq()
    R_in, R_out = inputs.near_hadamard_pair(D, seed, **kw)
    Ri = torch.from_numpy(R_in.astype(np.float32)).to(DEV)
    Ro = torch.from_numpy(R_out.astype(np.float32)).to(DEV)
    Q, M = rsq.qm_build(Ri, Ro, r, iters=iters)
    torch.cuda.synchronize()
    assert rsq.device_status() == 0
    # the oracle on the same float32 rotations the GPU read
    ref = oracle.qm_construct(R_in.astype(np.float32), R_out.astype(np.float32), r)
    return Q.cpu().numpy().astype(np.float64), M.cpu().numpy().astype(np.float64), ref


# T_hat from the GPU's float32 (Q, M) against the oracle's float64 one: the
# outputs are rounded once to float32 (relative 2^-24 on Q entries ~ 1/sqrt(D)
# and on M entries <= 2), so T_hat entries differ by a few 1e-8; 2e-6 leaves
# room for the subspace iteration's residual after `iters` steps.
QM_TOL = 2e-6


@pytest.mark.parametrize("D,r", [(128, 2), (256, 8), (256, 32), (512, 16), (1024, 64)])
def test_qm_build_matches_the_oracle(D, r):
    Q, M, ref = run_qm(D, r, D + r)
    Th = oracle.t_hat(Q, M)
    Th_ref = oracle.t_hat(ref["Q"], ref["M"])
    np.testing.assert_allclose(Th, Th_ref, rtol=0, atol=QM_TOL)
    np.testing.assert_allclose(Q.T @ Q, np.eye(r), rtol=0, atol=1e-6)      # orthonormal basis
    np.testing.assert_allclose(Th.T @ Th, np.eye(D), rtol=0, atol=1e-5)    # a rotation (float32 outputs)
    e_gpu = np.linalg.norm(Th - ref["T"])
    e_ref = np.linalg.norm(Th_ref - ref["T"])
    assert e_gpu <= e_ref * (1 + 1e-4) + 1e-5


def test_qm_build_reproduces_an_exact_rank_deviation():
    Q, M, ref = run_qm(256, 16, 5, n_planes=8)     # T - I of rank 16
    np.testing.assert_allclose(oracle.t_hat(Q, M), ref["T"], rtol=0, atol=1e-5)


def test_qm_build_full_size_feeds_the_alignment_kernels():
    """D = 4096, r = 32 (the hidden stream's shape): T_hat against the oracle on
    random directions, then the constructed (Q, M) through the alignment path on
    the GPU against the oracle's path with the oracle's (Q, M)."""
    rsq = _rsq()
    Q, M, ref = run_qm(4096, 32, 77)
    rng = np.random.default_rng(4)
    V = rng.normal(size=(4096, 8))
    np.testing.assert_allclose(V + Q @ (M @ (Q.T @ V)), V + ref["Q"] @ (ref["M"] @ (ref["Q"].T @ V)),
                               rtol=0, atol=QM_TOL * np.abs(V).max() * 8)
    a, _ = inputs.llama7b_case(T=200)
    x = _to_dev(a.x, "bf16")
    xo, codes, scales = rsq.rsq_align_norm_quant(x, torch.from_numpy(Q.astype(np.float32)).to(DEV),
                                                 torch.from_numpy(M.astype(np.float32)).to(DEV), bits=4)
    torch.cuda.synchronize()
    r = oracle.align_norm_quant(a.x, ref["Q"].astype(np.float32), ref["M"].astype(np.float32), 4, a.eps)
    H.check_aligned(_host(xo), r["x_out"], a.x, "bf16", "qm -> align")
    H.check_codes(codes.cpu().numpy(), r["q"], r["pre"], 4, "qm -> align")


@pytest.mark.parametrize("d,which", [(4096, 1), (4096, 3), (8192, 3)])
def test_tiny_and_zero_rows_rht(d, which):
    rsq = _rsq()
    prev = rsq.select_rht_kernel(which)
    try:
        h = inputs.rht_case(6, d, 1, 3, dtype="bf16")
        h.x[1] = 0.0
        h.x[2] *= np.float32(2.0 ** -120)      # absmax far below 2^-64: rescaled path
        h.x[3, :] = 0.0
        h.x[3, 17] = np.float32(2.0 ** -130)   # a single subnormal-range value
        h.x = inputs.round_to_bf16(h.x)
        codes, scales = run_rht(h)
        assert scales[1] == 0 and np.all(codes[1] == 0)
        check_rht(h, label=f"tiny rows kernel {which}")
    finally:
        rsq.select_rht_kernel(prev)


def test_residual_align_only_matches_oracle():
    rsq = _rsq()
    for dtype in ("f32", "bf16"):
        a = inputs.align_case(50, 4096, 32, 8, dtype=dtype, n_outliers=8, outlier_scale=100.0)
        x = _to_dev(a.x, dtype)
        xo = rsq.rsq_residual_align(x, torch.from_numpy(a.Q).to(DEV), torch.from_numpy(a.M).to(DEV))
        torch.cuda.synchronize()
        H.check_aligned(_host(xo), oracle.residual_align(a.x, a.Q, a.M), a.x, dtype, f"align {dtype}")


@pytest.mark.parametrize("which", [0, 1, 2, 4])
def test_residual_align_kernels(which):
    """rsq_residual_align through the decode kernel (small T), the tensor-core
    kernel (bf16, D = 4096 / 8192) and the CUDA-core kernel, each without the
    norm and the codes; x_out must equal the alignment of rsq_align_norm_quant
    bit for bit where both use the same kernel."""
    rsq = _rsq()
    prev = rsq.select_align_kernel(which)
    try:
        shapes = {0: [(1, 4096), (16, 4096), (17, 4096), (1000, 4096), (300, 8192)],
                  1: [(16, 4096), (300, 4096)],
                  2: [(1, 4096), (200, 4096), (3001, 4096), (129, 8192)],
                  4: [(1, 4096), (16, 4096), (32, 2048), (31, 8192)]}[which]
        for T, D in shapes:
            a = inputs.align_case(T, D, 32, T + D, dtype="bf16", n_outliers=8, outlier_scale=100.0)
            x = _to_dev(a.x, "bf16")
            Q = torch.from_numpy(a.Q).to(DEV)
            M = torch.from_numpy(a.M).to(DEV)
            xo = rsq.rsq_residual_align(x, Q, M)
            torch.cuda.synchronize()
            H.check_aligned(_host(xo), oracle.residual_align(a.x, a.Q, a.M), a.x, "bf16", f"kernel {which} T={T} D={D}")
            xo2, _, _ = rsq.rsq_align_norm_quant(x, Q, M, bits=4)
            torch.cuda.synchronize()
            assert torch.equal(xo.view(torch.int16), xo2.view(torch.int16)), f"kernel {which} T={T} D={D}"
        if which == 4:  # decode kernel with fp32 I/O
            a = inputs.align_case(9, 2048, 16, 9, dtype="f32", n_outliers=2, outlier_scale=20.0)
            xo = rsq.rsq_residual_align(_to_dev(a.x, "f32"), torch.from_numpy(a.Q).to(DEV), torch.from_numpy(a.M).to(DEV))
            torch.cuda.synchronize()
            H.check_aligned(_host(xo), oracle.residual_align(a.x, a.Q, a.M), a.x, "f32", "decode f32")
        assert rsq.device_status() == 0
    finally:
        rsq.select_align_kernel(prev)


def test_exact_ties_round_half_to_even():
    """w = H x with small integers chosen so that v/alpha hits exact ties; both
    sides must round them to even with no exemption."""
    d = 16
    w = np.zeros((1, d))
    w[0, :7] = [14, 1, 3, 5, -1, -3, -5]
    Hd = oracle.sylvester(d)
    x = (w @ Hd) / d                       # H symmetric, H H = d I: H x = w exactly
    h = inputs.RhtCase("ties", x.astype(np.float32), np.ones(d, np.int8), 1, "f32", 4)
    codes, scales = run_rht(h)
    ref = oracle.rht_quant(h.x, h.signs, 1, 4)
    np.testing.assert_array_equal(H.unpack(codes, d, 4), ref["q"])
    np.testing.assert_array_equal(ref["q"][0, :7], [7, 0, 2, 2, 0, -2, -2])


def test_worked_example_on_gpu():
    """The 4x4 worked example, embedded in d = 16 (H_16 = H_4 (x) H_4 on a spike)."""
    d = 16
    x = np.zeros((2, d), np.float32)
    x[0, 0] = 20.0
    x[1, :] = 20.0 / 4.0        # H_16 maps a constant row to a spike
    h = inputs.RhtCase("worked", x, np.ones(d, np.int8), 1, "f32", 4)
    codes, scales = run_rht(h)
    q = H.unpack(codes, d, 4)
    np.testing.assert_array_equal(q[0], np.full(d, 7))
    np.testing.assert_array_equal(q[1], [7] + [0] * (d - 1))
    np.testing.assert_allclose(scales, [20.0 / 4.0 / 7.0, 20.0 / 7.0], rtol=1e-7)


def test_deterministic_repeat():
    a, h = inputs.llama7b_case(T=300)
    r1 = run_align(a)
    r2 = run_align(a)
    for u, v in zip(r1, r2):
        np.testing.assert_array_equal(u, v)
    c1 = run_rht(h)
    c2 = run_rht(h)
    for u, v in zip(c1, c2):
        np.testing.assert_array_equal(u, v)


# --------------------------------------------------------------------------
# FlatQuant's Kronecker affine transform vec(P1^T X P2) + quantiser
# --------------------------------------------------------------------------

def run_affine(case):
    rsq = _rsq()
    x = _to_dev(case.x, case.dtype)
    P1, P2 = torch.from_numpy(case.P1).to(DEV), torch.from_numpy(case.P2).to(DEV)
    codes, scales = rsq.kron_affine_quant(x, P1, P2, bits=case.bits)
    assert rsq.device_status() == 0
    return codes.cpu().numpy(), scales.cpu().numpy()


def check_affine(case, rows=None, label=""):
    codes, scales = run_affine(case)
    sel = slice(None) if rows is None else rows
    ref = oracle.kron_affine_quant(case.x[sel], case.P1, case.P2, case.bits)
    H.check_scales(scales[sel], ref["scales"], label)
    return H.check_codes(codes[sel], ref["q"], ref["pre"], case.bits, label)


@pytest.mark.parametrize("n1,n2,dtype,bits,T", [(64, 64, "bf16", 4, 300), (64, 64, "f32", 3, 149),
                                                 (32, 128, "bf16", 4, 97), (128, 32, "f32", 4, 5),
                                                 (4, 4, "bf16", 4, 1), (8, 16, "bf16", 3, 333),
                                                 (12, 20, "f32", 4, 37)])
def test_kron_affine_quant(n1, n2, dtype, bits, T):
    """Whole outputs of every token row: square and non-square factors (so a
    transposed factor or swapped roles of n1 and n2 would fail), fp32 and bf16
    input, INT4 and INT3, an all-zero row, more rows than SMs (each CTA walks
    several) and a single row."""
    c = inputs.kron_affine_case(T, n1, n2, 7 + n1, dtype=dtype, bits=bits)
    if T > 3:
        c.x[2] = 0.0
    check_affine(c, label=f"affine {n1}x{n2} {dtype} INT{bits} T={T}")


def test_kron_affine_quant_full_size_sampled():
    """The bench's workload (T = 16384, d = 4096 = 64 x 64, bf16, INT4) in its
    launch configuration, compared on sampled rows."""
    c = inputs.flatquant_case()
    rows = np.r_[0:64, 8000:8064, c.T - 64:c.T]
    check_affine(c, rows=rows, label="flatquant T=16384 sampled")
