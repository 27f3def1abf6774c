"""Failure detection without a GPU fault: a bounded wait that runs out.

A kernel waits, through the same bounded mbarrier wait every tensor-core
kernel uses, on a barrier that nothing completes, with a limit of about a
millisecond.  The wait must give up, latch RET_ERR_TIMEOUT in the device
status word, end normally, and leave the device usable: the status read
clears it, and a full chunkwise call afterwards still matches the oracle."""
import time

import pytest
import torch

from oracle import oracle as orc
from parity import rel_l2, TOL_BF16
from retentive_network_scale_b200 import retention as R
from retentive_network_scale_b200.synth import random_tensor

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    from retentive_network_scale_b200 import build
    build.build()
    R.load_library()
    yield


def test_bounded_wait_times_out_and_device_stays_usable():
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    t0 = time.perf_counter()
    R.ret_selftest_wait_timeout(2_000_000)       # ~1 ms at the boost clock
    assert R.ret_last_device_status() == R.STATUS_NAMES.index("RET_ERR_TIMEOUT")
    assert time.perf_counter() - t0 < 30.0
    assert R.ret_last_device_status() == 0       # the read cleared it
    # the context is intact: a tensor-core chunkwise call still matches
    B, H, L, dk, dv = 1, 2, 200, 128, 128
    Q = random_tensor((B, H, L, dk), 91, dk ** -0.5).bfloat16()
    K = random_tensor((B, H, L, dk), 92, dk ** -0.5).bfloat16()
    V = random_tensor((B, H, L, dv), 93).bfloat16()
    g = [0.96875, 0.999]
    O = torch.empty(B, H, L, dv, device="cuda")
    R.ret_chunkwise(Q.cuda(), K.cuda(), V.cuda(), g, 128, O=O, rotate=True)
    O_ref, _ = orc.recurrent(Q, K, V, g, rotate=True)
    torch.cuda.synchronize()
    assert R.ret_last_device_status() == 0
    assert rel_l2(O, O_ref) <= TOL_BF16
