"""The (Q, M) construction through the entry point that allocates nothing.

Some callers cannot allocate device memory (a plugin inside an application
whose memory pool owns the device, or a latency-critical path that cannot
afford cudaMalloc's device-wide synchronisation).  rsq_qm_build_fixed_scratch
serves them from a scratch array inside the library.  This file runs last
(pytest collects it last), so a failure here cannot hide another test; it also
passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from w3a3_quantization_online_b200 import inputs

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
QM_TOL = 2e-6  # the same tolerance as the construction's parity tests


def _lib():
    from w3a3_quantization_online_b200 import rsq
    return rsq, rsq.library()


def test_fixed_scratch_construction_matches_the_workspace_entry_point():
    """Two calls in a row through the C ABI (the array keeps the first call's
    contents when the second starts) against rsq_qm_build with a caller
    workspace, on T_hat within the construction's tolerance."""
    rsq, L = _lib()
    D, r = 1024, 32
    R_in, R_out = inputs.near_hadamard_pair(D, 31)
    Ri = torch.from_numpy(R_in.astype(np.float32)).to(DEV)
    Ro = torch.from_numpy(R_out.astype(np.float32)).to(DEV)
    Q_ref, M_ref = rsq.qm_build(Ri, Ro, r, iters=16)
    torch.cuda.synchronize()
    assert rsq.device_status() == 0
    T_ref = oracle.t_hat(Q_ref.cpu().numpy(), M_ref.cpu().numpy())
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        Q = torch.empty((D, r), dtype=torch.float32, device=DEV)
        M = torch.empty((r, r), dtype=torch.float32, device=DEV)
        rc = L.rsq_qm_build_fixed_scratch(ctypes.c_void_p(Ri.data_ptr()), ctypes.c_void_p(Ro.data_ptr()), D, r, 16,
                                          ctypes.c_void_p(Q.data_ptr()), ctypes.c_void_p(M.data_ptr()),
                                          ctypes.c_void_p(stream))
        assert rc == 0, rsq.status_string(rc)
        torch.cuda.synchronize()
        assert rsq.device_status() == 0
        np.testing.assert_allclose(oracle.t_hat(Q.cpu().numpy(), M.cpu().numpy()), T_ref, rtol=0, atol=QM_TOL,
                                   err_msg=f"call {call}")


def test_fixed_scratch_rejects_shapes_beyond_the_array():
    rsq, L = _lib()
    before = rsq.launch_count()
    fake = ctypes.c_void_p(0x10_0000_0000)
    assert L.rsq_qm_build_fixed_scratch(fake, ctypes.c_void_p(0x20_0000_0000), 8192, 32, 16, ctypes.c_void_p(0x30_0000_0000),
                                        ctypes.c_void_p(0x40_0000_0000), None) == 2  # RSQ_ERR_SHAPE
    assert L.rsq_qm_build_fixed_scratch(fake, ctypes.c_void_p(0x20_0000_0000), 4096, 64, 16, ctypes.c_void_p(0x30_0000_0000),
                                        ctypes.c_void_p(0x40_0000_0000), None) == 2
    assert rsq.launch_count() == before
