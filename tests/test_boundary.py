"""C-ABI boundary checks that need no GPU: the library loads, exports every
symbol ``include/retention.h`` declares, and rejects invalid arguments with
the documented status before any device work.  Only invalid calls are made
here (they return before the library touches CUDA), plus one valid call on a
machine without an sm_100 device, which must refuse rather than fall back."""
import ctypes
import os
import re

import pytest
import torch

from retentive_network_scale_b200 import build as rbuild
from retentive_network_scale_b200 import retention as R

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "retention.h")

# A 16-byte aligned address that is never dereferenced: every call below is
# rejected by argument checks that run before any pointer is used.
FAKE = 0x10000
MISALIGNED = 0x10008


@pytest.fixture(scope="module")
def lib():
    rbuild.build()
    return R.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ret_[a-z0-9_]+)\s*\(", text)))


def test_header_lists_the_entry_points():
    assert declared_functions() == sorted(R.EXPORTS)


def test_library_exports_every_declared_symbol(lib):
    for name in declared_functions():
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(len(R.STATUS_NAMES)):
        s = lib.ret_status_string(code)
        assert s and len(s) >= 2
    assert lib.ret_status_string(0) == b"ok"


def desc(**kw):
    base = dict(B=2, H=2, L=8, d_k=16, d_v=16, in_dtype=R.RET_BF16, out_dtype=R.RET_BF16,
                gamma=[0.9, 0.99], rotate=True)
    base.update(kw)
    return R.make_desc(**base)


def call_parallel(lib, d, Q=FAKE, K=FAKE, V=FAKE, O=FAKE, ws=None, ws_bytes=0):
    return lib.ret_parallel(ctypes.byref(d), Q, K, V, O, ws, ws_bytes, None)


def call_chunkwise(lib, d, chunk=4, Q=FAKE, K=FAKE, V=FAKE, s_in=None, s_out=None, O=FAKE,
                   G=None, eps=1e-5, Y=None, ws=None, ws_bytes=0):
    return lib.ret_chunkwise(ctypes.byref(d), chunk, Q, K, V, s_in, s_out, O, G, eps, Y, ws,
                             ws_bytes, None)


@pytest.mark.parametrize("kw,status", [
    (dict(B=-1), "RET_ERR_SHAPE"), (dict(L=-2), "RET_ERR_SHAPE"), (dict(H=0, gamma=[]), "RET_ERR_SHAPE"),
    (dict(H=R.RET_MAX_HEADS + 1, gamma=[0.5] * (R.RET_MAX_HEADS + 1)), "RET_ERR_SHAPE"),
    (dict(d_k=258), "RET_ERR_SHAPE"), (dict(d_v=516), "RET_ERR_SHAPE"),
    (dict(d_v=18), "RET_ERR_SHAPE"), (dict(d_k=0), "RET_ERR_SHAPE"),
    (dict(in_dtype=7), "RET_ERR_DTYPE"), (dict(out_dtype=-1), "RET_ERR_DTYPE"),
    (dict(gamma=[1.5, 0.9]), "RET_ERR_ARG"), (dict(gamma=[-0.1, 0.9]), "RET_ERR_ARG"),
    (dict(gamma=[float("nan"), 0.9]), "RET_ERR_ARG"),
    (dict(d_k=15), "RET_ERR_ARG"), (dict(theta_base=0.0), "RET_ERR_ARG"),
    (dict(pos_offset=-1), "RET_ERR_ARG"), (dict(raw_rotate=2), "RET_ERR_ARG"),
])
def test_bad_descriptions(lib, kw, status):
    raw_rotate = kw.pop("raw_rotate", None)
    d = desc(**kw)
    if raw_rotate is not None:
        d.rotate = raw_rotate
    want = R.STATUS_NAMES.index(status)
    assert call_parallel(lib, d) == want
    assert call_chunkwise(lib, d) == want
    assert lib.ret_workspace_size(ctypes.byref(d), 4, 0, 1) == 0


def test_null_description(lib):
    assert lib.ret_parallel(None, FAKE, FAKE, FAKE, FAKE, None, 0, None) == R.STATUS_NAMES.index("RET_ERR_NULL")


def test_bad_pointers(lib):
    d = desc()
    NULL, ALIGN = R.STATUS_NAMES.index("RET_ERR_NULL"), R.STATUS_NAMES.index("RET_ERR_ALIGN")
    assert call_parallel(lib, d, Q=None) == NULL
    assert call_parallel(lib, d, O=None) == NULL
    assert call_parallel(lib, d, V=MISALIGNED) == ALIGN
    # the tensor-core parallel form with rotation needs workspace for the turned Q, K
    dp = desc(d_k=128, d_v=128, gamma=[0.9, 0.99])
    need = lib.ret_parallel_workspace_size(ctypes.byref(dp))
    assert need == 2 * 2 * 2 * 8 * 128 * 2
    assert call_parallel(lib, dp) == R.STATUS_NAMES.index("RET_ERR_WORKSPACE")
    assert call_parallel(lib, desc(d_k=128, d_v=128, rotate=False)) != R.STATUS_NAMES.index("RET_ERR_WORKSPACE")
    assert call_chunkwise(lib, d, O=None) == NULL                      # nothing requested
    assert call_chunkwise(lib, d, G=FAKE, Y=None) == NULL              # G without Y
    assert call_chunkwise(lib, d, s_out=MISALIGNED) == ALIGN
    assert call_chunkwise(lib, d, chunk=0) == R.STATUS_NAMES.index("RET_ERR_ARG")
    assert call_chunkwise(lib, d, G=FAKE, Y=FAKE, eps=-1.0) == R.STATUS_NAMES.index("RET_ERR_ARG")
    # Y without O needs workspace for the fp32 O it normalises
    need = lib.ret_workspace_size(ctypes.byref(d), 4, 0, 1)
    assert need == 4 * 2 * 2 * 8 * 16
    assert call_chunkwise(lib, d, O=None, G=FAKE, Y=FAKE) == R.STATUS_NAMES.index("RET_ERR_WORKSPACE")
    assert call_chunkwise(lib, d, O=None, G=FAKE, Y=FAKE, ws=FAKE, ws_bytes=need - 1) == \
        R.STATUS_NAMES.index("RET_ERR_WORKSPACE")


def test_chunkwise_prep_size(lib):
    """Optional workspace of the tensor-core chunkwise path: the rotated Q
    and the decay-weighted K in bf16 (only K without rotation); 0 wherever
    that path does not apply."""
    size = lambda d, chunk=128: lib.ret_chunkwise_prep_size(ctypes.byref(d), chunk)
    bf = R.RET_BF16
    base = dict(B=2, H=2, L=300, d_k=256, d_v=512, in_dtype=bf, out_dtype=bf, gamma=[0.9, 0.99])
    assert size(desc(**base)) == 2 * (2 * 2 * 300 * 256) * 2
    assert size(desc(**{**base, "rotate": False})) == (2 * 2 * 300 * 256) * 2
    assert size(desc(**{**base, "d_k": 128})) == 2 * (2 * 2 * 300 * 128) * 2
    assert size(desc(**base), chunk=64) == size(desc(**base))           # blocks of 128 rows
    assert size(desc(**base), chunk=192) == size(desc(**base))
    assert size(desc(**base), chunk=256) == size(desc(**base))
    assert size(desc(**base), chunk=96) == 0                            # not a multiple of 64
    assert size(desc(**{**base, "in_dtype": R.RET_F32})) == 0            # fp32 inputs
    assert size(desc(**{**base, "d_k": 64})) == 2 * (2 * 2 * 300 * 64) * 2
    assert size(desc(**{**base, "d_v": 64})) == size(desc(**base))
    assert size(desc(**{**base, "d_k": 32})) == 0
    assert size(desc(**{**base, "d_v": 192})) == 0                       # neither 64 nor 128 m
    assert size(desc(**{**base, "d_v": 640})) == 0                       # more than 4 column tiles
    assert size(desc(**{**base, "gamma": [0.5, 0.99]})) == 0             # 0.5^128 < 2^-60
    assert size(desc(**{**base, "gamma": [1.5, 0.99]})) == 0             # rejected description
    assert size(desc(**base), chunk=0) == 0
    assert lib.ret_chunkwise_prep_size(None, 128) == 0


def test_recurrent_step_arguments(lib):
    for L in (0, R.RET_MAX_DECODE_STEPS + 1):   # tokens per call: 1..RET_MAX_DECODE_STEPS
        d = desc(L=L)
        assert lib.ret_recurrent_step(ctypes.byref(d), FAKE, FAKE, FAKE, FAKE, FAKE, None) == \
            R.STATUS_NAMES.index("RET_ERR_SHAPE")
    d = desc(L=R.RET_MAX_DECODE_STEPS)
    assert lib.ret_recurrent_step(ctypes.byref(d), FAKE, FAKE, None, FAKE, FAKE, None) == \
        R.STATUS_NAMES.index("RET_ERR_NULL")
    d = desc(L=1)
    assert lib.ret_recurrent_step(ctypes.byref(d), FAKE, FAKE, None, FAKE, FAKE, None) == \
        R.STATUS_NAMES.index("RET_ERR_NULL")
    assert lib.ret_recurrent_step(ctypes.byref(d), FAKE, FAKE, FAKE, MISALIGNED, FAKE, None) == \
        R.STATUS_NAMES.index("RET_ERR_ALIGN")


def test_gate_norm_arguments(lib):
    SHAPE, DT = R.STATUS_NAMES.index("RET_ERR_SHAPE"), R.STATUS_NAMES.index("RET_ERR_DTYPE")
    assert lib.ret_gate_norm(1, 4, 2, 18, 0, FAKE, 0, FAKE, 1e-5, 0, FAKE, None) == SHAPE
    assert lib.ret_gate_norm(1, 4, 0, 16, 0, FAKE, 0, FAKE, 1e-5, 0, FAKE, None) == SHAPE
    assert lib.ret_gate_norm(1, 4, 2, 16, 3, FAKE, 0, FAKE, 1e-5, 0, FAKE, None) == DT
    assert lib.ret_gate_norm(1, 4, 2, 16, 0, FAKE, 0, FAKE, -1.0, 0, FAKE, None) == \
        R.STATUS_NAMES.index("RET_ERR_ARG")
    assert lib.ret_gate_norm(1, 4, 2, 16, 0, None, 0, FAKE, 1e-5, 0, FAKE, None) == \
        R.STATUS_NAMES.index("RET_ERR_NULL")


def test_msr_gammas_schedule(lib):
    """ret_msr_gammas (a host function) against the hand-worked binary
    fractions of section 2.2's schedule, and its refusals."""
    import os
    from fractions import Fraction
    want = {}
    with open(os.path.join(os.path.dirname(__file__), "golden", "gamma_schedule.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                h, frac = line.split()
                want[int(h)] = Fraction(frac)
    got = R.msr_gammas(16)
    assert len(got) == 16
    for h, fr in want.items():
        assert Fraction(got[h]) == fr, (h, got[h], fr)
    out = (ctypes.c_double * 4)()
    assert lib.ret_msr_gammas(0, out) == R.STATUS_NAMES.index("RET_ERR_SHAPE")
    assert lib.ret_msr_gammas(R.RET_MAX_HEADS + 1, out) == R.STATUS_NAMES.index("RET_ERR_SHAPE")
    assert lib.ret_msr_gammas(4, None) == R.STATUS_NAMES.index("RET_ERR_NULL")


def test_gate_norm_backward_arguments(lib):
    SHAPE, DT = R.STATUS_NAMES.index("RET_ERR_SHAPE"), R.STATUS_NAMES.index("RET_ERR_DTYPE")
    f = lib.ret_gate_norm_backward
    assert f(1, 4, 2, 18, 0, FAKE, 0, FAKE, FAKE, 1e-5, FAKE, FAKE, None) == SHAPE
    assert f(1, 4, 2, 16, 0, FAKE, 2, FAKE, FAKE, 1e-5, FAKE, FAKE, None) == DT
    assert f(1, 4, 2, 16, 0, FAKE, 0, FAKE, FAKE, float("nan"), FAKE, FAKE, None) == \
        R.STATUS_NAMES.index("RET_ERR_ARG")
    assert f(1, 4, 2, 16, 0, FAKE, 0, FAKE, None, 1e-5, FAKE, FAKE, None) == \
        R.STATUS_NAMES.index("RET_ERR_NULL")
    assert f(1, 4, 2, 16, 0, FAKE, 0, FAKE, FAKE, 1e-5, FAKE, MISALIGNED, None) == \
        R.STATUS_NAMES.index("RET_ERR_ALIGN")


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the refusal on a machine without sm_100")
def test_valid_call_without_sm100_refuses(lib):
    # zero-length problem: valid arguments, nothing would be read
    d = desc(L=0)
    assert call_parallel(lib, d) == R.STATUS_NAMES.index("RET_ERR_UNSUPPORTED")


def test_binding_rejects_host_tensors():
    q = torch.zeros(1, 1, 4, 8)
    with pytest.raises(TypeError):
        R.ret_parallel(q, q, q, q, [0.5])


def test_host_pipeline_arguments(lib):
    """ret_chunkwise_host rejects bad calls before any CUDA call (so these
    run without a GPU), and its workspace contract."""
    d = desc(B=4, L=8)
    call = lambda **kw: lib.ret_chunkwise_host(
        ctypes.byref(kw.get("d", d)), kw.get("chunk", 4), kw.get("Q", FAKE), FAKE, FAKE,
        kw.get("O", FAKE), kw.get("G", None), ctypes.c_float(1e-5), kw.get("Y", None),
        kw.get("slices", 2), kw.get("ws", None), kw.get("ws_bytes", 0), None)
    S = R.STATUS_NAMES.index
    assert call(slices=0) == S("RET_ERR_ARG")
    assert call(chunk=0) == S("RET_ERR_ARG")
    assert call(Q=None) == S("RET_ERR_NULL")
    assert call(O=None) == S("RET_ERR_NULL")                     # nothing requested
    assert call(G=FAKE) == S("RET_ERR_NULL")                     # G without Y
    assert call() == S("RET_ERR_WORKSPACE")
    assert call(d=desc(B=0, L=8)) == S("RET_OK")                 # empty: nothing queued
    size = lambda slices, O=1, Y=0, dd=d: lib.ret_chunkwise_host_workspace_size(
        ctypes.byref(dd), 4, O, Y, slices)
    assert size(1) > 0 and size(2) == size(1)                    # 1 slot of 4, or 2 slots of 2
    assert size(4) < size(2)                                     # 2 slots of 1 batch element
    assert size(64) == size(4)                                   # clamped to B slices
    assert size(0) == 0 and size(2, O=0, Y=0) == 0
    assert size(2, dd=desc(gamma=[2.0, 0.5])) == 0              # rejected description
    assert call(ws=FAKE, ws_bytes=size(2) - 1) == S("RET_ERR_WORKSPACE")


def test_gemm_arguments(lib):
    """ret_gemm_bf16 checks its sizes, leading dimensions, pointers and
    alignment before any CUDA call, and refuses a machine without sm_100."""
    S = R.STATUS_NAMES.index
    g = lambda M=256, N=256, K=64, A=FAKE, lda=64, B=FAKE, ldb=256, C=FAKE, ldc=256: \
        lib.ret_gemm_bf16(M, N, K, A, lda, B, ldb, C, ldc, None)  # noqa: E731
    assert g(M=-1) == S("RET_ERR_ARG")
    assert g(M=0) == S("RET_OK") and g(N=0) == S("RET_OK")        # empty: nothing launched
    assert g(N=12, ldb=16, ldc=16) == S("RET_ERR_SHAPE")           # N not a multiple of 8
    assert g(K=0) == S("RET_ERR_SHAPE")
    assert g(lda=32) == S("RET_ERR_SHAPE")                          # lda < K
    assert g(ldb=260) == S("RET_ERR_SHAPE")                         # not a multiple of 8
    assert g(A=None) == S("RET_ERR_NULL")
    assert g(C=FAKE + 2) == S("RET_ERR_ALIGN")
    if not torch.cuda.is_available():
        assert g() == S("RET_ERR_UNSUPPORTED")


def test_selftest_wait_timeout_arguments(lib):
    S = R.STATUS_NAMES.index
    assert lib.ret_selftest_wait_timeout(999, None) == S("RET_ERR_ARG")
    assert lib.ret_selftest_wait_timeout(4000000001, None) == S("RET_ERR_ARG")
    if not torch.cuda.is_available():
        assert lib.ret_selftest_wait_timeout(2000000, None) == S("RET_ERR_UNSUPPORTED")


def test_header_constants_match_binding():
    import re
    text = open(HEADER).read()
    for name in ("RET_MAX_HEADS", "RET_MAX_DECODE_STEPS", "RET_MAX_SEGMENTS"):
        m = re.search(r"#define\s+%s\s+(\d+)" % name, text)
        assert m and int(m.group(1)) == getattr(R, name), name


def test_segment_state_arguments(lib):
    """ret_segment_state / ret_state_scan reject bad calls before any CUDA
    call, and the workspace contract of the segment state."""
    S = R.STATUS_NAMES.index
    d = desc(B=2, L=300, d_k=16, d_v=8, in_dtype=R.RET_BF16)
    seg = lambda **kw: lib.ret_segment_state(
        ctypes.byref(kw.get("d", d)), kw.get("K", FAKE), FAKE, kw.get("U", FAKE),
        kw.get("ws", None), kw.get("ws_bytes", 0), None)
    assert seg(d=desc(B=2, L=300, d_k=16, d_v=8, in_dtype=R.RET_F32)) == S("RET_ERR_DTYPE")
    assert seg(d=desc(B=2, L=300, d_k=12, d_v=8, in_dtype=R.RET_BF16)) == S("RET_ERR_SHAPE")
    assert seg(U=None) == S("RET_ERR_NULL")
    assert seg(U=MISALIGNED) == S("RET_ERR_ALIGN")
    assert seg(d=desc(B=0, L=300, d_k=16, d_v=8, in_dtype=R.RET_BF16)) == S("RET_OK")
    size = lib.ret_segment_state_workspace_size(ctypes.byref(d))
    assert size >= 2 * 300 * 16 * 2          # the weighted keys, and cuBLAS room
    assert lib.ret_segment_state_workspace_size(ctypes.byref(desc(B=0))) == 0
    if not torch.cuda.is_available():
        assert seg() == S("RET_ERR_UNSUPPORTED")
    lens = (ctypes.c_int * 3)(4, 5, 6)
    scan = lambda n=3, rank=1, L=lens, U=FAKE, R_=FAKE, s0=None: lib.ret_state_scan(
        ctypes.byref(d), n, L, rank, U, s0, R_, None)
    assert scan(n=0) == S("RET_ERR_SHAPE")
    assert scan(n=R.RET_MAX_SEGMENTS + 1) == S("RET_ERR_SHAPE")
    assert scan(rank=4) == S("RET_ERR_SHAPE")
    assert scan(rank=-1) == S("RET_ERR_SHAPE")
    assert scan(L=(ctypes.c_int * 3)(4, 0, 6)) == S("RET_ERR_SHAPE")
    assert scan(L=None) == S("RET_ERR_NULL")
    assert scan(U=None) == S("RET_ERR_NULL")      # segment 0 must be read for rank 1
    assert scan(R_=None) == S("RET_ERR_NULL")
    assert scan(s0=MISALIGNED) == S("RET_ERR_ALIGN")
    if not torch.cuda.is_available():
        assert scan(rank=0, U=None) == S("RET_ERR_UNSUPPORTED")


def test_chunkwise_prepared_arguments(lib):
    """ret_chunkwise_prepared rejects bad calls before any CUDA call."""
    S = R.STATUS_NAMES.index
    d = desc(B=2, L=300, d_k=128, d_v=128, gamma=[0.9, 0.99])
    call = lambda dd=d, chunk=128, Qh=FAKE, Kt=FAKE, V=FAKE, O=FAKE, G=None, Y=None: \
        lib.ret_chunkwise_prepared(ctypes.byref(dd), chunk, Qh, Kt, V, None, None, O, G,
                                   ctypes.c_float(1e-5), Y, None)
    assert call(chunk=0) == S("RET_ERR_ARG")
    assert call(dd=desc(B=0, L=300, d_k=128, d_v=128)) == S("RET_ERR_SHAPE")   # nothing prepared
    assert call(dd=desc(B=2, L=300, d_k=32, d_v=128)) == S("RET_ERR_SHAPE")    # not a tensor-core shape
    assert call(chunk=96) == S("RET_ERR_SHAPE")
    assert call(Kt=None) == S("RET_ERR_NULL")
    assert call(O=None) == S("RET_ERR_NULL")                                   # nothing requested
    assert call(G=FAKE) == S("RET_ERR_NULL")                                   # G without Y
    assert call(V=MISALIGNED) == S("RET_ERR_ALIGN")
    if not torch.cuda.is_available():
        assert call() == S("RET_ERR_UNSUPPORTED")


def test_chunkwise_segmented_arguments(lib):
    """ret_chunkwise_segmented rejects bad calls before any CUDA call, and
    its workspace size is 0 for the calls it would reject."""
    S = R.STATUS_NAMES.index
    d = desc(B=1, H=4, L=1024, d_k=128, d_v=256, gamma=[0.9, 0.95, 0.99, 0.999])
    call = lambda dd=d, chunk=128, seg=4, Q=FAKE, O=FAKE, ws=None, nb=0: \
        lib.ret_chunkwise_segmented(ctypes.byref(dd), chunk, seg, Q, FAKE, FAKE, None, None, O,
                                    ws, nb, None)
    size = lambda dd=d, chunk=128, seg=4: lib.ret_chunkwise_segmented_workspace_size(
        ctypes.byref(dd), chunk, seg)
    assert call(seg=0) == S("RET_ERR_ARG") and size(seg=0) == 0
    assert call(seg=3) == S("RET_ERR_SHAPE") and size(seg=3) == 0          # L % segments
    assert call(seg=64) == S("RET_ERR_SHAPE")                                # H * segments > 128
    assert call(chunk=96) == S("RET_ERR_SHAPE")                              # not a tensor-core chunk
    assert call(dd=desc(B=1, H=4, L=1024, d_k=32, d_v=256,
                        gamma=[0.9] * 4)) == S("RET_ERR_SHAPE")              # not a tensor-core d_k
    assert call(dd=desc(B=1, H=4, L=1024, d_k=128, d_v=256, in_dtype=R.RET_F32,
                        gamma=[0.9] * 4)) == S("RET_ERR_DTYPE")
    assert call(O=None) == S("RET_ERR_NULL")
    assert call(Q=MISALIGNED) == S("RET_ERR_ALIGN")
    assert size() > 0
    assert call() == S("RET_ERR_WORKSPACE")
    if not torch.cuda.is_available():
        assert call(ws=FAKE, nb=size()) == S("RET_ERR_UNSUPPORTED")


def test_static_entry_checks_arguments_before_its_scratch_limit(lib):
    """ret_chunkwise_gate_static reports the errors ret_chunkwise would
    before it compares the problem with its fixed scratch: a missing Y on a
    shape far beyond the array is a NULL error, not a workspace one."""
    S = lambda n: R.STATUS_NAMES.index(n)  # noqa: E731
    big_L = R.RET_STATIC_SCRATCH_FLOATS  # B*H*L*d_v floats far beyond the array
    d = desc(B=1, H=1, L=big_L, d_k=16, d_v=64, in_dtype=R.RET_F32, out_dtype=R.RET_F32,
             gamma=[0.9])
    call = lambda dd, chunk=16, G=FAKE, Y=FAKE: lib.ret_chunkwise_gate_static(  # noqa: E731
        ctypes.byref(dd), chunk, FAKE, FAKE, FAKE, None, None, G, ctypes.c_float(1e-5), Y, None)
    assert call(d, Y=None) == S("RET_ERR_NULL")
    assert call(d, G=None) == S("RET_ERR_NULL")
    assert call(d, chunk=0) == S("RET_ERR_ARG")
    assert call(desc(gamma=[1.5, 0.9])) == S("RET_ERR_ARG")
    assert call(d) == S("RET_ERR_WORKSPACE")


def test_fast_size(lib):
    """ret_chunkwise_fast_size: the streaming pass's room for shapes with
    enough heads, the segmented layout (segments keeping one wave of CTAs,
    at least 512 rows each) for few heads, or the one-launch path's block
    sums where they are larger, 0 off the tensor-core path."""
    bf = R.RET_BF16
    fast = lambda d, chunk=128: lib.ret_chunkwise_fast_size(ctypes.byref(d), chunk)  # noqa: E731
    prep = lambda d, chunk=128: lib.ret_chunkwise_prep_size(ctypes.byref(d), chunk)  # noqa: E731
    seg = lambda d, n, chunk=128: lib.ret_chunkwise_segmented_workspace_size(  # noqa: E731
        ctypes.byref(d), chunk, n)
    many = desc(B=8, H=8, L=1024, d_k=256, d_v=512, in_dtype=bf, out_dtype=bf, gamma=[0.9] * 8)
    assert fast(many) == prep(many) > 0                                  # 256 CTAs: no segments
    # 2 heads x 1 value tile: 8 segments of 256 rows would be too short, 4 of 512 qualify
    few = desc(B=1, H=2, L=2048, d_k=128, d_v=128, in_dtype=bf, out_dtype=bf, gamma=[0.9, 0.99])
    assert fast(few) == seg(few, 4) > prep(few) > 0
    # msr_small's shape: 32 heads of d_v 64, no rotation: room for the
    # one-launch path's block sums (B*H*16 blocks of a 64 x 64 fp32 sum, then
    # a flag per block) or for 4 segments of 512 rows, whichever is larger
    small = desc(B=4, H=8, L=2048, d_k=64, d_v=64, in_dtype=bf, out_dtype=bf,
                 gamma=[0.9] * 8, rotate=False)
    onepass = 4 * 8 * 16 * 64 * 64 * 4 + 4 * 8 * 16 * 4
    assert fast(small, 64) == max(seg(small, 4, 64), onepass) > 0
    # the same with rotation: the segments only
    small_rot = desc(B=4, H=8, L=2048, d_k=64, d_v=64, in_dtype=bf, out_dtype=bf,
                     gamma=[0.9] * 8, rotate=True)
    assert fast(small_rot, 64) == seg(small_rot, 4, 64) > 0
    # rows that do not split into segments of 512: the streaming pass only
    odd = desc(B=1, H=2, L=1000, d_k=128, d_v=128, in_dtype=bf, out_dtype=bf, gamma=[0.9, 0.99])
    assert fast(odd) == prep(odd) > 0
    f32 = desc(B=1, H=2, L=2048, d_k=128, d_v=128, in_dtype=R.RET_F32, out_dtype=R.RET_F32,
               gamma=[0.9, 0.99])
    assert fast(f32) == 0


def test_workspace_size_of_tensor_core_shapes(lib):
    """The tensor-core path needs no workspace, except for rotated shapes
    of d_k 64, which only the prepared-rows loop serves (the loop turns
    tiles of d_k 128 and 256 itself): there ret_workspace_size asks for the
    streaming pass's room."""
    bf = R.RET_BF16
    ws = lambda d, chunk=128, o=0, y=1: lib.ret_workspace_size(ctypes.byref(d), chunk, o, y)  # noqa: E731
    prep = lambda d, chunk=128: lib.ret_chunkwise_prep_size(ctypes.byref(d), chunk)  # noqa: E731
    big = dict(B=1, H=2, L=300, d_k=256, d_v=512, in_dtype=bf, out_dtype=bf, gamma=[0.9, 0.99])
    assert ws(desc(**big)) == 0 and ws(desc(**big), chunk=256) == 0
    assert ws(desc(**big), chunk=64) == 0 and prep(desc(**big), chunk=64) > 0
    small = {**big, "d_k": 64, "d_v": 64}
    assert ws(desc(**small), chunk=64) == prep(desc(**small), chunk=64) > 0
    assert ws(desc(**small), chunk=64, o=1, y=0) == prep(desc(**small), chunk=64)
    assert ws(desc(**{**small, "rotate": False}), chunk=64) == 0
    # fp32 inputs take the CUDA-core path: an fp32 O to normalise for Y alone
    f32 = {**small, "in_dtype": R.RET_F32, "out_dtype": R.RET_F32}
    assert ws(desc(**f32), chunk=64) == 1 * 2 * 300 * 64 * 4
    assert ws(desc(**f32), chunk=64, o=1, y=1) == 0
