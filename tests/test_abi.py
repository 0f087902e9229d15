"""C-ABI checks that need no GPU: the library loads, exports every declared
symbol, and rejects bad arguments on the host without launching anything.

Every rejected call below carries exactly one invalid property and fake (but
16-byte aligned) pointers; validation must return before any CUDA call, so
these tests are also safe on a GPU machine (nothing is ever launched).
"""
import ctypes
import os
import re
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "rsq.h")

from w3a3_quantization_online_b200 import rsq  # noqa: E402

L = rsq.library()
OK, NULL, SHAPE, DTYPE, BITS, ALIGN, ALIAS, UNSUP, CUDA, VALUE = range(10)
F32, BF16 = 0, 1

# fake device addresses, far apart and 16-byte aligned
X, Q, M, XO, C, S, SG, XB = (0x10_0000_0000 + i * 0x1_0000_0000 for i in range(8))


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w]+\s*\*?\s*(\w+)\s*\(", src, flags=re.M)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("rsq_residual_align", "rsq_align_norm_quant", "rht_quant", "rsq_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    for n in declared_functions():
        assert hasattr(L, n), f"librsq.so does not export {n}"
    nm = shutil.which("nm")
    if nm:
        out = subprocess.run([nm, "-D", "--defined-only", rsq.LIB_PATH], capture_output=True, text=True).stdout
        syms = set(line.split()[-1] for line in out.splitlines() if line.strip())
        for n in declared_functions():
            assert n in syms


def test_selftest_rejects_out_of_range_limits():
    # host-side validation: nothing is enqueued (no GPU needed)
    for bad in (0, -5, 1001):
        assert L.rsq_selftest_wait_timeout(bad, None) == 9  # RSQ_ERR_VALUE


def test_status_strings():
    for s in range(10):
        assert rsq.status_string(s)
    assert "unknown" in rsq.status_string(99)


def _anq(x=X, q=Q, m=M, xo=XO, c=C, s=S, T=4, D=256, r=8, bits=4, eps=1e-5, dt=BF16):
    return L.rsq_align_norm_quant(x, q, m, xo, c, s, T, D, r, bits, eps, dt, None)


def _ra(x=X, q=Q, m=M, xo=XO, T=4, D=256, r=8, dt=BF16):
    return L.rsq_residual_align(x, q, m, xo, T, D, r, dt, None)


def _rht(x=X, sg=SG, m=1, c=C, s=S, T=4, d=256, bits=4, dt=BF16):
    return L.rht_quant(x, sg, m, c, s, T, d, bits, dt, None)


@pytest.mark.parametrize("kw,want", [
    (dict(x=None), NULL), (dict(q=None), NULL), (dict(m=None), NULL), (dict(xo=None), NULL),
    (dict(c=None), NULL), (dict(s=None), NULL),
    (dict(T=-1), SHAPE), (dict(D=0), SHAPE), (dict(D=8), SHAPE), (dict(D=264 - 4), SHAPE),
    (dict(D=65536), SHAPE), (dict(r=0), SHAPE), (dict(r=65), SHAPE),
    (dict(bits=2), BITS), (dict(bits=8), BITS), (dict(dt=2), DTYPE),
    (dict(eps=-1.0), VALUE), (dict(eps=float("nan")), VALUE), (dict(eps=float("inf")), VALUE),
    (dict(x=X + 8), ALIGN), (dict(q=Q + 4), ALIGN), (dict(xo=XO + 2), ALIGN), (dict(c=C + 1), ALIGN),
    (dict(s=S + 4), ALIGN),
    (dict(xo=X + 16), ALIAS),            # partial overlap of x_out with x
    (dict(c=X + 256), ALIAS),            # codes inside x
    (dict(s=XO + 64), ALIAS),            # scales inside x_out
    (dict(c=Q), ALIAS),                  # codes over Q
    (dict(s=C + 16), ALIAS),             # scales inside codes
])
def test_align_norm_quant_rejects(kw, want):
    before = rsq.launch_count()
    assert _anq(**kw) == want
    assert rsq.launch_count() == before


@pytest.mark.parametrize("kw,want", [
    (dict(x=None), NULL), (dict(xo=None), NULL), (dict(T=-5), SHAPE), (dict(r=100), SHAPE),
    (dict(dt=7), DTYPE), (dict(m=M + 8), ALIGN), (dict(xo=X + 32), ALIAS), (dict(xo=Q + 16), ALIAS),
])
def test_residual_align_rejects(kw, want):
    before = rsq.launch_count()
    assert _ra(**kw) == want
    assert rsq.launch_count() == before


@pytest.mark.parametrize("kw,want", [
    (dict(x=None), NULL), (dict(sg=None), NULL), (dict(c=None), NULL), (dict(s=None), NULL),
    (dict(m=3), UNSUP), (dict(m=0), UNSUP), (dict(d=96, m=1), SHAPE), (dict(d=8), SHAPE),
    (dict(d=12 * 8, m=12), SHAPE), (dict(d=65536), SHAPE), (dict(d=12 * 48, m=12), SHAPE),
    (dict(T=-1), SHAPE), (dict(bits=5), BITS), (dict(dt=3), DTYPE),
    (dict(x=X + 4), ALIGN), (dict(sg=SG + 1), ALIGN), (dict(c=C + 8), ALIGN),
    (dict(c=X + 1024), ALIAS), (dict(s=SG), ALIAS), (dict(s=C + 64), ALIAS),
])
def test_rht_quant_rejects(kw, want):
    before = rsq.launch_count()
    assert _rht(**kw) == want
    assert rsq.launch_count() == before


def _gate(a=X, b=XB, sg=SG, m=12, c=C, s=S, T=4, d=12288, bits=4, dt=BF16):
    return L.rht_quant_silu_gate(a, b, sg, m, c, s, T, d, bits, dt, None)


@pytest.mark.parametrize("kw,want", [
    (dict(a=None), NULL), (dict(b=None), NULL), (dict(sg=None), NULL), (dict(c=None), NULL), (dict(s=None), NULL),
    (dict(m=3), UNSUP), (dict(d=12 * 48), SHAPE), (dict(d=96, m=1), SHAPE), (dict(T=-1), SHAPE),
    (dict(bits=2), BITS), (dict(dt=5), DTYPE),
    (dict(a=X + 4), ALIGN), (dict(b=XB + 8), ALIGN), (dict(s=S + 2), ALIGN),
    (dict(c=XB + 4096), ALIAS),          # codes inside b
    (dict(s=X + 64), ALIAS),             # scales inside a
    (dict(c=SG), ALIAS),                 # codes over the signs
    (dict(s=C + 32), ALIAS),             # scales inside codes
])
def test_rht_quant_silu_gate_rejects(kw, want):
    before = rsq.launch_count()
    assert _gate(**kw) == want
    assert rsq.launch_count() == before


def test_rht_quant_silu_gate_inputs_may_overlap():
    # a == b (SiLU(a) * a) passes validation; without a GPU the call then fails
    # at the first CUDA call (nothing launched); never run on fake pointers on a GPU
    import torch
    if torch.cuda.is_available():
        pytest.skip("would launch on fake pointers")
    assert _gate(b=X) == CUDA


def _heads(x=X, sg=SG, nh=32, xo=XO, T=4, d=4096, dt=BF16):
    return L.rht_heads(x, sg, nh, xo, T, d, dt, None)


def _heads_q(x=X, sg=SG, nh=32, c=C, s=S, T=4, d=4096, bits=4, dt=BF16):
    return L.rht_heads_quant(x, sg, nh, c, s, T, d, bits, dt, None)


def _mix_q(x=X, sg=SG, nh=32, c=C, s=S, T=4, d=4096, bits=4, dt=BF16):
    return L.rht_head_mix_quant(x, sg, nh, c, s, T, d, bits, dt, None)


@pytest.mark.parametrize("fn,kw,want", [
    (_heads, dict(x=None), NULL), (_heads, dict(xo=None), NULL), (_heads, dict(nh=0), SHAPE),
    (_heads, dict(nh=3), SHAPE),                      # d_h = 4096 / 3 is not whole
    (_heads, dict(nh=512), SHAPE),                    # d_h = 8 < 16
    (_heads, dict(nh=8), SHAPE),                      # d_h = 512 > 256
    (_heads, dict(d=96 * 32), SHAPE),                 # d_h = 96 is not a power of two
    (_heads, dict(dt=4), DTYPE), (_heads, dict(x=X + 2), ALIGN), (_heads, dict(sg=SG + 8), ALIGN),
    (_heads, dict(xo=X + 16), ALIAS), (_heads, dict(xo=SG - 64), ALIAS),
    (_heads_q, dict(c=None), NULL), (_heads_q, dict(s=None), NULL), (_heads_q, dict(bits=5), BITS),
    (_heads_q, dict(nh=64, d=4096 + 64), SHAPE), (_heads_q, dict(c=X + 512), ALIAS), (_heads_q, dict(s=C + 16), ALIAS),
    (_mix_q, dict(nh=3, d=48 * 3), SHAPE), (_mix_q, dict(nh=1), SHAPE), (_mix_q, dict(nh=128), SHAPE),
    (_mix_q, dict(nh=2, d=2 * 1024), SHAPE),          # d_h = 1024: more columns than threads per row
    (_mix_q, dict(d=4096 + 8), SHAPE), (_mix_q, dict(bits=1), BITS), (_mix_q, dict(c=C + 4), ALIGN),
    (_mix_q, dict(s=X + 32), ALIAS), (_mix_q, dict(c=SG), ALIAS),
])
def test_head_transforms_reject(fn, kw, want):
    before = rsq.launch_count()
    assert fn(**kw) == want
    assert rsq.launch_count() == before


def test_head_transforms_accept_null_signs():
    import torch
    if torch.cuda.is_available():
        pytest.skip("would launch on fake pointers")
    assert _heads(sg=None) == CUDA and _heads_q(sg=None) == CUDA and _mix_q(sg=None) == CUDA


def _aff(x=X, p1=Q, p2=M, n1=64, n2=64, c=C, s=S, T=4, bits=4, dt=BF16):
    return L.kron_affine_quant(x, p1, p2, n1, n2, c, s, T, bits, dt, None)


@pytest.mark.parametrize("kw,want", [
    (dict(x=None), NULL), (dict(p1=None), NULL), (dict(p2=None), NULL), (dict(c=None), NULL), (dict(s=None), NULL),
    (dict(bits=2), BITS), (dict(dt=2), DTYPE), (dict(T=-1), SHAPE),
    (dict(n1=2, n2=8), SHAPE),                        # below 4
    (dict(n1=6, n2=8), SHAPE),                        # not a multiple of 4
    (dict(n1=4, n2=256), SHAPE),                      # n2 > 128
    (dict(n1=128, n2=64), SHAPE),                     # d = 8192 > 4096
    (dict(x=X + 8), ALIGN), (dict(p1=Q + 4), ALIGN), (dict(p2=M + 2), ALIGN), (dict(c=C + 4), ALIGN),
    (dict(s=S + 8), ALIGN),
    (dict(c=X + 4096), ALIAS),                        # codes inside x
    (dict(s=Q + 256), ALIAS),                         # scales inside P1
    (dict(c=M), ALIAS),                               # codes over P2
    (dict(s=C + 16), ALIAS),                          # scales inside codes
])
def test_kron_affine_quant_rejects(kw, want):
    before = rsq.launch_count()
    assert _aff(**kw) == want
    assert rsq.launch_count() == before


def _gemm(ca=X, sa=S, cw=Q, sw=M, y=XO, acc=C, T=4, N=256, K=4096, dt=2):
    return L.w4a4_gemm(ca, sa, cw, sw, y, acc, T, N, K, dt, None)


@pytest.mark.parametrize("kw,want", [
    (dict(ca=None), NULL), (dict(sa=None), NULL), (dict(cw=None), NULL), (dict(sw=None), NULL), (dict(y=None), NULL),
    (dict(dt=0), DTYPE), (dict(dt=3), DTYPE), (dict(T=-1), SHAPE), (dict(N=4), SHAPE), (dict(N=260), SHAPE),
    (dict(K=64), SHAPE), (dict(K=4096 + 64), SHAPE), (dict(T=65536 * 128), SHAPE),
    (dict(ca=X + 1), ALIGN), (dict(y=XO + 2), ALIGN), (dict(acc=C + 8), ALIGN),
    (dict(y=X + 1024), ALIAS), (dict(acc=XO + 16), ALIAS), (dict(acc=Q), ALIAS), (dict(y=S), ALIAS),
])
def test_w4a4_gemm_rejects(kw, want):
    before = rsq.launch_count()
    assert _gemm(**kw) == want
    assert rsq.launch_count() == before


def _gemm_s8w(ca=X, sa=S, w=Q, sw=M, y=XO, acc=C, T=4, N=256, K=4096, dt=2):
    return L.w4a4_gemm_s8w(ca, sa, w, sw, y, acc, T, N, K, dt, None)


@pytest.mark.parametrize("kw,want", [
    (dict(ca=None), NULL), (dict(w=None), NULL), (dict(y=None), NULL), (dict(dt=0), DTYPE), (dict(N=4), SHAPE),
    (dict(K=64), SHAPE), (dict(w=Q + 8), ALIGN), (dict(y=Q + 512 * 1024), ALIAS), (dict(acc=Q + 1024 * 1024 - 16), ALIAS),
])
def test_w4a4_gemm_s8w_rejects(kw, want):
    """The prepared-weight GEMM checks the int8 weights as N x K bytes (a span
    twice that of the packed codes)."""
    before = rsq.launch_count()
    assert _gemm_s8w(**kw) == want
    assert rsq.launch_count() == before


@pytest.mark.parametrize("args,want", [
    ((Q, 256, 4096, XO), None), ((None, 256, 4096, XO), NULL), ((Q, 256, 4096, None), NULL),
    ((Q, 4, 4096, XO), SHAPE), ((Q, 256, 100, XO), SHAPE), ((Q + 4, 256, 4096, XO), ALIGN),
    ((Q, 256, 4096, Q + 256 * 2048 - 16), ALIAS), ((Q, 256, 4096, Q - 256 * 4096 + 16), ALIAS),
])
def test_w4a4_prepare_weights_rejects(args, want):
    import torch
    if want is None:
        if torch.cuda.is_available():
            pytest.skip("would launch on fake pointers")
        assert L.w4a4_prepare_weights(*args, None) == CUDA  # valid arguments reach the launch (no GPU here)
        return
    before = rsq.launch_count()
    assert L.w4a4_prepare_weights(*args, None) == want
    assert rsq.launch_count() == before


def _qm(ri=X, ro=XB, D=4096, r=32, it=16, q=Q, m=M, ws=C, wsb=1 << 30):
    return L.rsq_qm_build(ri, ro, D, r, it, q, m, ws, wsb, None)


@pytest.mark.parametrize("kw,want", [
    (dict(ri=None), NULL), (dict(ro=None), NULL), (dict(q=None), NULL), (dict(m=None), NULL), (dict(ws=None), NULL),
    (dict(D=4000), SHAPE), (dict(D=32), SHAPE), (dict(D=32768), SHAPE), (dict(r=0), SHAPE), (dict(r=65), SHAPE),
    (dict(D=64, r=33), SHAPE), (dict(it=0), VALUE), (dict(it=1001), VALUE), (dict(wsb=1024), VALUE),
    (dict(ri=X + 4), ALIGN), (dict(ws=C + 8), ALIGN), (dict(q=X + 4096), ALIAS), (dict(ws=XB + 64), ALIAS),
    (dict(m=Q + 256), ALIAS),
])
def test_qm_build_rejects(kw, want):
    before = rsq.launch_count()
    assert _qm(**kw) == want
    assert rsq.launch_count() == before


def test_qm_workspace_bytes():
    assert L.rsq_qm_workspace_bytes(4000, 32) == 0 and L.rsq_qm_workspace_bytes(4096, 65) == 0
    small, big = L.rsq_qm_workspace_bytes(256, 8), L.rsq_qm_workspace_bytes(4096, 32)
    assert 0 < small < big < 64 << 20                                # a few D x 64 float64 blocks
    assert L.rsq_qm_workspace_bytes(4096, 64) > big                  # 96 columns for r > 32


def test_empty_batch_is_a_no_op():
    before = rsq.launch_count()
    assert _anq(x=None, xo=None, c=None, s=None, T=0) == OK
    assert _ra(x=None, xo=None, T=0) == OK
    assert _rht(x=None, c=None, s=None, T=0) == OK
    assert _gate(a=None, b=None, c=None, s=None, T=0) == OK
    assert _heads(x=None, xo=None, T=0) == OK
    assert _heads_q(x=None, c=None, s=None, T=0) == OK
    assert _mix_q(x=None, c=None, s=None, T=0) == OK
    assert _aff(x=None, p1=None, p2=None, c=None, s=None, T=0) == OK
    assert _gemm(ca=None, sa=None, y=None, acc=None, T=0) == OK
    assert rsq.launch_count() == before


def test_in_place_alias_passes_validation_only_when_exact():
    # x_out == x is allowed: validation passes and the call reaches CUDA.  Only
    # run the accepted form where no GPU exists (no device => RSQ_ERR_CUDA,
    # nothing is launched), never with fake pointers on a GPU machine.
    import torch
    if torch.cuda.is_available():
        pytest.skip("would launch on fake pointers")
    assert _anq(xo=X) == CUDA


def test_binding_refuses_to_import_without_the_library(tmp_path):
    pkg = tmp_path / "w3a3_quantization_online_b200"
    pkg.mkdir()
    (pkg / "__init__.py").write_text("")
    shutil.copy(os.path.join(ROOT, "w3a3_quantization_online_b200", "rsq.py"), pkg / "rsq.py")
    r = subprocess.run([sys.executable, "-c", "import w3a3_quantization_online_b200.rsq"],
                       cwd=tmp_path, capture_output=True, text=True)
    assert r.returncode != 0 and "ImportError" in r.stderr and "no fallback" in r.stderr


def test_product_path_never_touches_the_oracle():
    pkg = os.path.join(ROOT, "w3a3_quantization_online_b200")
    pat = re.compile(r"^\s*(import\s+oracle|from\s+oracle\b|from\s+\.\.?\s*import\s+oracle)", re.M)
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h", ".cpp")):
                src = open(os.path.join(dirpath, f)).read()
                assert not pat.search(src), f"{f} imports the oracle"
                assert "rsq_oracle" not in src, f"{f} links the oracle"
