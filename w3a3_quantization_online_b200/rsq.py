"""Thin Python binding of librsq.so (include/rsq.h): argument marshalling only.

Every step of the path runs in the library's CUDA kernels.  PyTorch supplies
device memory and the current CUDA stream.  There is no CPU fallback: if the
library is missing, importing this module raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "librsq.so")

RSQ_F32, RSQ_BF16, RSQ_F16 = 0, 1, 2

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -c 'import __graft_entry__ as g; g.build()'` "
        "or `python w3a3_quantization_online_b200/build.py` (the CUDA path has no fallback)")

_lib = ctypes.CDLL(LIB_PATH)
_vp, _i64, _i32, _f32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float
_lib.rsq_residual_align.argtypes = [_vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _vp]
_lib.rsq_residual_align.restype = _i32
_lib.rsq_align_norm_quant.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _f32, _i32, _vp]
_lib.rsq_align_norm_quant.restype = _i32
_lib.rht_quant.argtypes = [_vp, _vp, _i32, _vp, _vp, _i64, _i32, _i32, _i32, _vp]
_lib.rht_quant.restype = _i32
_lib.rht_quant_silu_gate.argtypes = [_vp, _vp, _vp, _i32, _vp, _vp, _i64, _i32, _i32, _i32, _vp]
_lib.rht_quant_silu_gate.restype = _i32
_lib.rht_heads.argtypes = [_vp, _vp, _i32, _vp, _i64, _i32, _i32, _vp]
_lib.rht_heads.restype = _i32
_lib.rht_heads_quant.argtypes = [_vp, _vp, _i32, _vp, _vp, _i64, _i32, _i32, _i32, _vp]
_lib.rht_heads_quant.restype = _i32
_lib.rht_head_mix_quant.argtypes = [_vp, _vp, _i32, _vp, _vp, _i64, _i32, _i32, _i32, _vp]
_lib.rht_head_mix_quant.restype = _i32
_lib.kron_affine_quant.argtypes = [_vp, _vp, _vp, _i32, _i32, _vp, _vp, _i64, _i32, _i32, _vp]
_lib.kron_affine_quant.restype = _i32
_lib.w4a4_gemm.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _vp]
_lib.w4a4_gemm.restype = _i32
_lib.w4a4_prepare_weights.argtypes = [_vp, _i32, _i32, _vp, _vp]
_lib.w4a4_prepare_weights.restype = _i32
_lib.w4a4_gemm_s8w.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i64, _i32, _i32, _i32, _vp]
_lib.w4a4_gemm_s8w.restype = _i32
_lib.rsq_qm_build.argtypes = [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, ctypes.c_uint64, _vp]
_lib.rsq_qm_build.restype = _i32
_lib.rsq_qm_workspace_bytes.argtypes = [_i32, _i32]
_lib.rsq_qm_build_fixed_scratch.argtypes = [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp]
_lib.rsq_qm_build_fixed_scratch.restype = _i32
_lib.rsq_qm_workspace_bytes.restype = ctypes.c_uint64
_lib.rsq_status_string.argtypes = [_i32]
_lib.rsq_status_string.restype = ctypes.c_char_p
_lib.rsq_last_cuda_error.argtypes = []
_lib.rsq_last_cuda_error.restype = _i32
_lib.rsq_launch_count.argtypes = []
_lib.rsq_launch_count.restype = ctypes.c_uint64
_lib.rsq_select_align_kernel.argtypes = [_i32]
_lib.rsq_select_align_kernel.restype = _i32
_lib.rsq_select_rht_kernel.argtypes = [_i32]
_lib.rsq_select_rht_kernel.restype = _i32
_lib.rsq_device_status.argtypes = [_vp, ctypes.POINTER(_i32)]
_lib.rsq_device_status.restype = _i32
_lib.rsq_selftest_wait_timeout.argtypes = [_i32, _vp]
_lib.rsq_selftest_wait_timeout.restype = _i32

EXPORTED = ("rsq_residual_align", "rsq_align_norm_quant", "rht_quant", "rht_quant_silu_gate", "rht_heads",
            "rht_heads_quant", "rht_head_mix_quant", "kron_affine_quant", "w4a4_gemm", "w4a4_prepare_weights", "w4a4_gemm_s8w",
            "rsq_qm_build", "rsq_qm_workspace_bytes",
            "rsq_qm_build_fixed_scratch",
            "rsq_status_string",
            "rsq_last_cuda_error", "rsq_launch_count", "rsq_select_align_kernel", "rsq_select_rht_kernel", "rsq_device_status",
            "rsq_selftest_wait_timeout")

ALIGN_AUTO, ALIGN_GENERIC, ALIGN_TENSOR_CORE, ALIGN_DECODE = 0, 1, 2, 4
RHT_AUTO, RHT_GENERIC, RHT_TENSOR_CORE, RHT_KRONECKER = 0, 1, 3, 4


class RsqError(RuntimeError):
    def __init__(self, status: int):
        msg = _lib.rsq_status_string(status).decode()
        if status == 8:
            msg += f" (cudaError {int(_lib.rsq_last_cuda_error())})"
        super().__init__(msg)
        self.status = status


def library() -> ctypes.CDLL:
    return _lib


def launch_count() -> int:
    return int(_lib.rsq_launch_count())


def select_align_kernel(which: int) -> int:
    """0 auto, 1 CUDA-core, 2 tensor-core cluster kernel (one 128-row tile per CTA), 4 decode kernel;
    returns the previous setting."""
    prev = int(_lib.rsq_select_align_kernel(int(which)))
    if prev < 0:
        raise ValueError(which)
    return prev


def select_rht_kernel(which: int) -> int:
    """0 auto, 1 radix-16 SMEM kernel, 3 tensor-core kernel, 4 Kronecker kernel; returns the previous setting."""
    prev = int(_lib.rsq_select_rht_kernel(int(which)))
    if prev < 0:
        raise ValueError(which)
    return prev


def device_status(stream=None) -> int:
    """Take (and clear) the device status word on the stream, after the work
    queued on it; returns it (0 = healthy).  The word is per device and shared
    by all streams."""
    out = _i32(0)
    _check(_lib.rsq_device_status(_stream(stream), ctypes.byref(out)))
    return int(out.value)


def selftest_wait_timeout(limit_ms: int = 20, stream=None) -> None:
    """Enqueue the bounded-wait self test (a wait that runs out after limit_ms
    and sets the timeout bit of the device status word)."""
    _check(_lib.rsq_selftest_wait_timeout(int(limit_ms), _stream(stream)))


def status_string(status: int) -> str:
    return _lib.rsq_status_string(status).decode()


def _check(status: int) -> None:
    if status != 0:
        raise RsqError(status)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return RSQ_F32
    if t.dtype == torch.bfloat16:
        return RSQ_BF16
    raise TypeError(f"activations must be float32 or bfloat16, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor]) -> Optional[int]:
    return None if t is None else t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream if isinstance(stream, torch.cuda.Stream) else int(stream)


def _need(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def rsq_residual_align(x: torch.Tensor, Q: torch.Tensor, M: torch.Tensor,
                       x_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """x_out = x + Q (M (Q^T x)) per row of the T x D activations x (in place if x_out is x)."""
    _need(x, "x"); _need(Q, "Q", torch.float32); _need(M, "M", torch.float32)
    T, D = x.shape
    r = Q.shape[1]
    if x_out is None:
        x_out = torch.empty_like(x)
    _need(x_out, "x_out", x.dtype)
    _check(_lib.rsq_residual_align(_ptr(x), _ptr(Q), _ptr(M), _ptr(x_out), T, D, r,
                                   _dtype_code(x), _stream(stream)))
    return x_out


def rsq_align_norm_quant(x: torch.Tensor, Q: torch.Tensor, M: torch.Tensor,
                         x_out: Optional[torch.Tensor] = None, codes: Optional[torch.Tensor] = None,
                         scales: Optional[torch.Tensor] = None, bits: int = 4, eps: float = 1e-5,
                         stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Alignment -> weight-free RMSNorm -> per-token symmetric INT{bits} codes.

    Returns (x_out, codes uint8 T x D*bits/8, scales float32 T)."""
    _need(x, "x"); _need(Q, "Q", torch.float32); _need(M, "M", torch.float32)
    T, D = x.shape
    r = Q.shape[1]
    if x_out is None:
        x_out = torch.empty_like(x)
    if codes is None:
        codes = torch.empty((T, D * bits // 8), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((T,), dtype=torch.float32, device=x.device)
    _need(x_out, "x_out", x.dtype); _need(codes, "codes", torch.uint8); _need(scales, "scales", torch.float32)
    _check(_lib.rsq_align_norm_quant(_ptr(x), _ptr(Q), _ptr(M), _ptr(x_out), _ptr(codes), _ptr(scales),
                                     T, D, r, bits, float(eps), _dtype_code(x), _stream(stream)))
    return x_out, codes, scales


def rht_quant(x: torch.Tensor, signs: torch.Tensor, m: int = 1, codes: Optional[torch.Tensor] = None,
              scales: Optional[torch.Tensor] = None, bits: int = 4,
              stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Randomised Hadamard H_d diag(signs) x / sqrt(d) -> per-token symmetric INT{bits} codes.

    Returns (codes uint8 T x d*bits/8, scales float32 T)."""
    _need(x, "x"); _need(signs, "signs", torch.int8)
    T, d = x.shape
    if codes is None:
        codes = torch.empty((T, d * bits // 8), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((T,), dtype=torch.float32, device=x.device)
    _need(codes, "codes", torch.uint8); _need(scales, "scales", torch.float32)
    _check(_lib.rht_quant(_ptr(x), _ptr(signs), m, _ptr(codes), _ptr(scales), T, d, bits,
                          _dtype_code(x), _stream(stream)))
    return codes, scales


def rht_quant_silu_gate(a: torch.Tensor, b: torch.Tensor, signs: torch.Tensor, m: int = 1,
                        codes: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None,
                        bits: int = 4, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """SiLU(a) * b -> randomised Hadamard H_d diag(signs) / sqrt(d) -> per-token INT{bits} codes.

    Returns (codes uint8 T x d*bits/8, scales float32 T)."""
    _need(a, "a"); _need(b, "b", a.dtype); _need(signs, "signs", torch.int8)
    T, d = a.shape
    if tuple(b.shape) != (T, d):
        raise ValueError(f"b has shape {tuple(b.shape)}, expected {(T, d)}")
    if codes is None:
        codes = torch.empty((T, d * bits // 8), dtype=torch.uint8, device=a.device)
    if scales is None:
        scales = torch.empty((T,), dtype=torch.float32, device=a.device)
    _need(codes, "codes", torch.uint8); _need(scales, "scales", torch.float32)
    _check(_lib.rht_quant_silu_gate(_ptr(a), _ptr(b), _ptr(signs), m, _ptr(codes), _ptr(scales), T, d, bits,
                                    _dtype_code(a), _stream(stream)))
    return codes, scales


def _signs_ptr(signs: Optional[torch.Tensor]) -> Optional[int]:
    if signs is None:
        return None
    _need(signs, "signs", torch.int8)
    return signs.data_ptr()


def rht_heads(x: torch.Tensor, signs: Optional[torch.Tensor], n_heads: int,
              x_out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Per-head rotation (I (x) H_{d_h}) diag(signs) x / sqrt(d_h) of queries or keys (in place if x_out is x)."""
    _need(x, "x")
    T, d = x.shape
    if x_out is None:
        x_out = torch.empty_like(x)
    _need(x_out, "x_out", x.dtype)
    _check(_lib.rht_heads(_ptr(x), _signs_ptr(signs), n_heads, _ptr(x_out), T, d, _dtype_code(x), _stream(stream)))
    return x_out


def rht_heads_quant(x: torch.Tensor, signs: Optional[torch.Tensor], n_heads: int, codes: Optional[torch.Tensor] = None,
                    scales: Optional[torch.Tensor] = None, bits: int = 4,
                    stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Per-head rotation, then per-(token, head) INT{bits} codes.  Returns (codes T x d*bits/8, scales T x n_heads)."""
    _need(x, "x")
    T, d = x.shape
    if codes is None:
        codes = torch.empty((T, d * bits // 8), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((T, n_heads), dtype=torch.float32, device=x.device)
    _need(codes, "codes", torch.uint8); _need(scales, "scales", torch.float32)
    _check(_lib.rht_heads_quant(_ptr(x), _signs_ptr(signs), n_heads, _ptr(codes), _ptr(scales), T, d, bits,
                                _dtype_code(x), _stream(stream)))
    return codes, scales


def rht_head_mix_quant(x: torch.Tensor, signs: Optional[torch.Tensor], n_heads: int,
                       codes: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None, bits: int = 4,
                       stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Head mixing (H_{n_h} (x) I) diag(signs) x / sqrt(n_h), then per-token INT{bits} codes."""
    _need(x, "x")
    T, d = x.shape
    if codes is None:
        codes = torch.empty((T, d * bits // 8), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((T,), dtype=torch.float32, device=x.device)
    _need(codes, "codes", torch.uint8); _need(scales, "scales", torch.float32)
    _check(_lib.rht_head_mix_quant(_ptr(x), _signs_ptr(signs), n_heads, _ptr(codes), _ptr(scales), T, d, bits,
                                   _dtype_code(x), _stream(stream)))
    return codes, scales


def kron_affine_quant(x: torch.Tensor, P1: torch.Tensor, P2: torch.Tensor,
                      codes: Optional[torch.Tensor] = None, scales: Optional[torch.Tensor] = None, bits: int = 4,
                      stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """FlatQuant's Kronecker affine transform vec(P1^T X P2) of each row, then per-token INT{bits} codes."""
    _need(x, "x")
    _need(P1, "P1", torch.float32); _need(P2, "P2", torch.float32)
    T, d = x.shape
    n1, n2 = P1.shape[0], P2.shape[0]
    if P1.shape != (n1, n1) or P2.shape != (n2, n2) or n1 * n2 != d:
        raise ValueError(f"P1 {tuple(P1.shape)} and P2 {tuple(P2.shape)} do not factor a row of {d}")
    if codes is None:
        codes = torch.empty((T, d * bits // 8), dtype=torch.uint8, device=x.device)
    if scales is None:
        scales = torch.empty((T,), dtype=torch.float32, device=x.device)
    _need(codes, "codes", torch.uint8); _need(scales, "scales", torch.float32)
    _check(_lib.kron_affine_quant(_ptr(x), _ptr(P1), _ptr(P2), n1, n2, _ptr(codes), _ptr(scales), T, bits,
                                  _dtype_code(x), _stream(stream)))
    return codes, scales


def w4a4_gemm(codes_a: torch.Tensor, scales_a: torch.Tensor, codes_w: torch.Tensor, scales_w: torch.Tensor,
              y: Optional[torch.Tensor] = None, acc: Optional[torch.Tensor] = None, out_dtype=torch.float16,
              stream=None) -> torch.Tensor:
    """Y = (INT4 codes_a @ INT4 codes_w^T) * scales_a[:, None] * scales_w[None, :] in fp16 / bf16.

    codes_a: T x K/2 uint8, codes_w: N x K/2 uint8 (packed INT4); acc (optional) receives the int32 products."""
    _need(codes_a, "codes_a", torch.uint8); _need(codes_w, "codes_w", torch.uint8)
    _need(scales_a, "scales_a", torch.float32); _need(scales_w, "scales_w", torch.float32)
    T, kb = codes_a.shape
    N = codes_w.shape[0]
    if codes_w.shape[1] != kb:
        raise ValueError("codes_a and codes_w disagree on K")
    if out_dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("out_dtype must be float16 or bfloat16")
    if y is None:
        y = torch.empty((T, N), dtype=out_dtype, device=codes_a.device)
    _need(y, "y", out_dtype)
    if acc is not None:
        _need(acc, "acc", torch.int32)
    code = RSQ_F16 if out_dtype == torch.float16 else RSQ_BF16
    _check(_lib.w4a4_gemm(_ptr(codes_a), _ptr(scales_a), _ptr(codes_w), _ptr(scales_w), _ptr(y), _ptr(acc), T, N,
                          2 * kb, code, _stream(stream)))
    return y


def w4a4_prepare_weights(codes_w: torch.Tensor, w_s8: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """The packed INT4 weight codes (N x K/2 uint8) unpacked once to int8 (N x K) for w4a4_gemm_s8w."""
    _need(codes_w, "codes_w", torch.uint8)
    N, kb = codes_w.shape
    if w_s8 is None:
        w_s8 = torch.empty((N, 2 * kb), dtype=torch.int8, device=codes_w.device)
    _need(w_s8, "w_s8", torch.int8)
    if tuple(w_s8.shape) != (N, 2 * kb):
        raise ValueError("w_s8 must be N x K")
    _check(_lib.w4a4_prepare_weights(_ptr(codes_w), N, 2 * kb, _ptr(w_s8), _stream(stream)))
    return w_s8


def w4a4_gemm_s8w(codes_a: torch.Tensor, scales_a: torch.Tensor, w_s8: torch.Tensor, scales_w: torch.Tensor,
                  y: Optional[torch.Tensor] = None, acc: Optional[torch.Tensor] = None, out_dtype=torch.float16,
                  stream=None) -> torch.Tensor:
    """w4a4_gemm with the weights prepared by w4a4_prepare_weights (N x K int8)."""
    _need(codes_a, "codes_a", torch.uint8); _need(w_s8, "w_s8", torch.int8)
    _need(scales_a, "scales_a", torch.float32); _need(scales_w, "scales_w", torch.float32)
    T, kb = codes_a.shape
    N = w_s8.shape[0]
    if w_s8.shape[1] != 2 * kb:
        raise ValueError("codes_a and w_s8 disagree on K")
    if out_dtype not in (torch.float16, torch.bfloat16):
        raise TypeError("out_dtype must be float16 or bfloat16")
    if y is None:
        y = torch.empty((T, N), dtype=out_dtype, device=codes_a.device)
    _need(y, "y", out_dtype)
    if acc is not None:
        _need(acc, "acc", torch.int32)
    code = RSQ_F16 if out_dtype == torch.float16 else RSQ_BF16
    _check(_lib.w4a4_gemm_s8w(_ptr(codes_a), _ptr(scales_a), _ptr(w_s8), _ptr(scales_w), _ptr(y), _ptr(acc), T, N,
                              2 * kb, code, _stream(stream)))
    return y


def qm_workspace_bytes(D: int, r: int) -> int:
    return int(_lib.rsq_qm_workspace_bytes(D, r))


def qm_build(R_in: torch.Tensor, R_out: torch.Tensor, r: int, iters: int = 16,
             workspace: Optional[torch.Tensor] = None, stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """Offline (Q, M) of the alignment from the rotations on both sides of a residual connection.

    Returns (Q D x r float32, M r x r float32).  workspace: a uint8 CUDA tensor of at
    least qm_workspace_bytes(D, r) bytes (allocated here when None)."""
    _need(R_in, "R_in", torch.float32); _need(R_out, "R_out", torch.float32)
    D = R_in.shape[0]
    need = qm_workspace_bytes(D, r)
    if need == 0:
        raise RsqError(2)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=R_in.device)
    _need(workspace, "workspace", torch.uint8)
    Q = torch.empty((D, r), dtype=torch.float32, device=R_in.device)
    M = torch.empty((r, r), dtype=torch.float32, device=R_in.device)
    _check(_lib.rsq_qm_build(_ptr(R_in), _ptr(R_out), D, r, iters, _ptr(Q), _ptr(M), _ptr(workspace),
                             workspace.numel(), _stream(stream)))
    return Q, M


def qm_build_fixed_scratch(R_in: torch.Tensor, R_out: torch.Tensor, r: int, iters: int = 16,
                           stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """qm_build on the library's own fixed scratch array (no workspace argument).

    Shapes whose workspace exceeds the array are rejected; calls whose work
    overlaps on the GPU share the array and must be serialised."""
    _need(R_in, "R_in", torch.float32); _need(R_out, "R_out", torch.float32)
    D = R_in.shape[0]
    Q = torch.empty((D, r), dtype=torch.float32, device=R_in.device)
    M = torch.empty((r, r), dtype=torch.float32, device=R_in.device)
    _check(_lib.rsq_qm_build_fixed_scratch(_ptr(R_in), _ptr(R_out), D, r, iters, _ptr(Q), _ptr(M), _stream(stream)))
    return Q, M
