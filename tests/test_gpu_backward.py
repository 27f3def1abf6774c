"""ret_backward: dQ, dK, dV of the retention output against the fp64
backward oracle (itself pinned to finite differences of the forward
oracle), for d_v with one and two column blocks of the dO . V contraction,
with and without rotation, fp32 and bf16 gradients, a ragged length; and
one full-size (b, h) slice of the RetNet-1.3B shape."""
import pytest
import torch

from oracle import oracle as orc
from parity import rel_l2, TOL_BF16
from retentive_network_scale_b200 import retention as R
from retentive_network_scale_b200.synth import WORKLOADS, make_inputs, random_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from retentive_network_scale_b200 import build
    build.build()
    R.load_library()
    yield
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0


@pytest.mark.parametrize("dk,dv,rotate,out", [
    (128, 128, True, torch.float32),
    (256, 384, False, torch.float32),
    (128, 512, True, torch.bfloat16),
    (256, 512, True, torch.float32),   # the second column block folds the sums and the turn in
])
def test_backward_matches_oracle(dk, dv, rotate, out):
    B, H, L = 2, 2, 300
    g = [0.96875, 0.999]
    Q = random_tensor((B, H, L, dk), 800, dk ** -0.5).bfloat16()
    K = random_tensor((B, H, L, dk), 801, dk ** -0.5).bfloat16()
    V = random_tensor((B, H, L, dv), 802).bfloat16()
    dO = random_tensor((B, H, L, dv), 803).bfloat16()
    rQ, rK, rV = orc.retention_backward(Q, K, V, dO, g, rotate=rotate, pos_offset=7)
    dQ, dK, dV = R.ret_backward(Q.cuda(), K.cuda(), V.cuda(), dO.cuda(), g, 128, out_dtype=out,
                                rotate=rotate, pos_offset=7)
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    for b in range(B):
        for h in range(H):
            assert rel_l2(dQ[b, h], rQ[b, h]) <= TOL_BF16, ("dQ", b, h)
            assert rel_l2(dK[b, h], rK[b, h]) <= TOL_BF16, ("dK", b, h)
            assert rel_l2(dV[b, h], rV[b, h]) <= TOL_BF16, ("dV", b, h)


def test_backward_msr_1p3b_sampled():
    w = WORKLOADS["msr_1p3b"]
    x = make_inputs(w)
    dO = random_tensor((w.B, w.H, w.L, w.d_v), 804).bfloat16()
    g = R.msr_gammas(w.H)
    dQ, dK, dV = R.ret_backward(x["Q"].cuda(), x["K"].cuda(), x["V"].cuda(), dO.cuda(), g, w.chunk,
                                rotate=w.rotate)
    torch.cuda.synchronize()
    b, h = 5, 3
    gam = orc.gammas(w.H)
    sl = lambda t: t[b:b + 1, h:h + 1]  # noqa: E731
    rQ, rK, rV = orc.retention_backward(sl(x["Q"]), sl(x["K"]), sl(x["V"]), sl(dO), [gam[h]],
                                        rotate=w.rotate)
    assert rel_l2(dQ[b, h], rQ[0, 0]) <= TOL_BF16
    assert rel_l2(dK[b, h], rK[0, 0]) <= TOL_BF16
    assert rel_l2(dV[b, h], rV[0, 0]) <= TOL_BF16


def test_backward_on_a_user_stream_matches_default_stream():
    """The weighting passes run on the library's side stream, joined to the
    caller's stream by events: called on a non-blocking stream of the
    caller's own, with that stream's earlier work (the inputs' copies)
    still queued, the gradients equal those of a call on the default
    stream bit for bit, and a second call in a row reuses the buffers
    correctly."""
    B, H, L, dk, dv = 2, 4, 700, 256, 512
    g = [0.96875, 0.99, 0.999, 1.0]
    Q = random_tensor((B, H, L, dk), 810, dk ** -0.5).bfloat16()
    K = random_tensor((B, H, L, dk), 811, dk ** -0.5).bfloat16()
    V = random_tensor((B, H, L, dv), 812).bfloat16()
    dO = random_tensor((B, H, L, dv), 813).bfloat16()
    ref = R.ret_backward(Q.cuda(), K.cuda(), V.cuda(), dO.cuda(), g, 128, rotate=True)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        d = [t.pin_memory().to("cuda", non_blocking=True) for t in (Q, K, V, dO)]
        for _ in range(2):
            got = R.ret_backward(*d, g, 128, rotate=True, stream=s)
    s.synchronize()
    assert R.ret_last_device_status() == 0
    for a, b in zip(got, ref):
        assert torch.equal(a, b)
