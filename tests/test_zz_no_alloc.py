"""ret_chunkwise_gate_static: the chunkwise forward with the fused
GroupNorm + swish gate for callers that may not allocate device memory
(memory reserved up front by a host framework, or a fixed budget once
serving starts).  Its scratch is the library's fixed device array.  The
tests call it through the C ABI, twice in a row (the calls share the
array), and check Y and the final state against the fp64 oracle and against
the allocating entry point ret_chunkwise on the same inputs: on the CUDA-core
path, which uses the array, and on the tensor-core path, which needs none.
A problem too large for the array is refused.  The file sits on its own,
collected last, and must pass alone in a fresh process as well."""
import ctypes

import numpy as np
import pytest
import torch

from oracle import oracle as orc
from parity import normwise, rel_l2, TOL_BF16, TOL_F32
from retentive_network_scale_b200 import build
from retentive_network_scale_b200 import retention as R
from retentive_network_scale_b200.synth import random_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def lib():
    build.build()
    return R.load_library()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _call_static(lib, Q, K, V, G, Y, g, chunk, rotate, S_in=None, S_out=None):
    B, H, L, dk = Q.shape
    dv = V.shape[-1]
    code = R.RET_F32 if Q.dtype == torch.float32 else R.RET_BF16
    d = R.make_desc(B, H, L, dk, dv, code, code, g, rotate)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.ret_chunkwise_gate_static(ctypes.byref(d), chunk, _ptr(Q), _ptr(K), _ptr(V),
                                         _ptr(S_in), _ptr(S_out), _ptr(G), ctypes.c_float(1e-5),
                                         _ptr(Y), stream)


@pytest.mark.parametrize("dtype,dk,dv,chunk,rotate,with_state,scratch", [
    (torch.float32, 32, 48, 32, True, False, True),     # CUDA-core path: uses the array
    (torch.bfloat16, 64, 64, 32, False, True, True),    # CUDA-core path: uses the array
    (torch.bfloat16, 128, 128, 128, True, True, False),  # tensor-core path: no scratch
])
def test_static_scratch_matches_oracle_and_allocating_entry(lib, dtype, dk, dv, chunk, rotate,
                                                            with_state, scratch):
    B, H, L = 2, 3, 150
    Q = random_tensor((B, H, L, dk), 61, dk ** -0.5).to(dtype)
    K = random_tensor((B, H, L, dk), 62, dk ** -0.5).to(dtype)
    V = random_tensor((B, H, L, dv), 63).to(dtype)
    G = random_tensor((B, L, H * dv), 64).to(dtype)
    S0 = random_tensor((B, H, dk, dv), 65, 0.2) if with_state else None
    g = [0.9, 0.96875, 0.999]
    need = R.ret_workspace_size(B, H, L, dk, dv, R._dtype_code(Q), R._dtype_code(Q), g, chunk,
                                want_O=False, want_Y=True, rotate=rotate)
    assert (need > 0) == scratch
    O_ref, S_ref = orc.recurrent(Q, K, V, g, rotate=rotate, state_in=S0)
    Y_ref = orc.gate_groupnorm(O_ref, G)
    Qd, Kd, Vd, Gd = Q.cuda(), K.cuda(), V.cuda(), G.cuda()
    S0d = None if S0 is None else S0.cuda()
    # the allocating entry point, with its workspace (or the prep workspace
    # of the tensor-core path)
    Y_alloc = torch.empty(B, L, H * dv, device="cuda", dtype=dtype)
    S_alloc = torch.empty(B, H, dk, dv, device="cuda")
    R.ret_chunkwise(Qd, Kd, Vd, g, chunk, G=Gd, Y=Y_alloc, rotate=rotate, state_in=S0d,
                    state_out=S_alloc, prep=not scratch)
    metric, tol = (normwise, TOL_F32) if dtype == torch.float32 else (rel_l2, TOL_BF16)
    for _ in range(2):  # two calls in a row share the array
        Y = torch.full((B, L, H * dv), float("nan"), device="cuda", dtype=dtype)
        S = torch.full((B, H, dk, dv), float("nan"), device="cuda")
        assert _call_static(lib, Qd, Kd, Vd, Gd, Y, g, chunk, rotate, S0d, S) == 0
        torch.cuda.synchronize()
        assert R.ret_last_device_status() == 0
        assert metric(Y, Y_ref) <= tol
        assert metric(S, S_ref) <= tol
        assert metric(Y, Y_alloc) <= tol
        assert metric(S, S_alloc) <= tol
        assert np.isfinite(Y.float().cpu().numpy()).all()


def test_static_scratch_refuses_oversized_problem(lib):
    # B*H*L*d_v floats beyond the fixed array: refused before anything runs
    B, H, dk, dv = 1, 1, 16, 64
    L = R.RET_STATIC_SCRATCH_FLOATS // dv + 1
    Q = torch.zeros(1, device="cuda")
    d = R.make_desc(B, H, L, dk, dv, R.RET_F32, R.RET_F32, [0.9])
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    rc = lib.ret_chunkwise_gate_static(ctypes.byref(d), 16, _ptr(Q), _ptr(Q), _ptr(Q), None, None,
                                       _ptr(Q), ctypes.c_float(1e-5), _ptr(Q), stream)
    assert rc == R.STATUS_NAMES.index("RET_ERR_WORKSPACE")
