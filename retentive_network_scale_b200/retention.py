"""ctypes binding of ``libretention.so`` (declared in ``include/retention.h``).

Argument marshalling only: every step of the computation runs in the CUDA
library.  The functions take torch CUDA tensors (torch provides device
memory and streams), check that they are contiguous CUDA tensors of the
expected shapes -- a host pointer handed to a kernel would fault -- build the
``ret_desc``, call the C entry point of the same name on the current (or
given) stream and raise ``RetentionError`` on any non-zero status.

The library is required: if it is missing or cannot be loaded, every call
raises; nothing falls back to another implementation.
"""
from __future__ import annotations

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libretention.so")

RET_F32, RET_BF16 = 0, 1
RET_MAX_HEADS = 128
STATUS_NAMES = ["RET_OK", "RET_ERR_NULL", "RET_ERR_SHAPE", "RET_ERR_DTYPE", "RET_ERR_ALIGN",
                "RET_ERR_ARG", "RET_ERR_WORKSPACE", "RET_ERR_UNSUPPORTED", "RET_ERR_CUDA",
                "RET_ERR_TIMEOUT"]

# every symbol include/retention.h declares
EXPORTS = ("ret_parallel", "ret_parallel_workspace_size", "ret_chunkwise",
           "ret_chunkwise_gate_static", "ret_workspace_size", "ret_chunkwise_prep_size",
           "ret_chunkwise_fast_size",
           "ret_chunkwise_prepare", "ret_chunkwise_prepared", "ret_chunkwise_host", "ret_chunkwise_host_workspace_size",
           "ret_selftest_wait_timeout", "ret_msr_layer", "ret_msr_layer_workspace_size",
           "ret_gemm_bf16",
           "ret_backward", "ret_backward_workspace_size",
           "ret_segment_state", "ret_segment_state_workspace_size", "ret_state_scan",
           "ret_chunkwise_segmented", "ret_chunkwise_segmented_workspace_size",
           "ret_recurrent_step", "ret_gate_norm", "ret_gate_norm_backward", "ret_last_device_status",
           "ret_kernel_launches", "ret_status_string", "ret_msr_gammas")
RET_STATIC_SCRATCH_FLOATS = 4 << 20
RET_MAX_DECODE_STEPS = 16
RET_MAX_SEGMENTS = 64


class RetentionError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        super().__init__(f"{what}: {name} ({_status_text(status)})")


class RetDesc(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int),
        ("d_k", ctypes.c_int), ("d_v", ctypes.c_int),
        ("in_dtype", ctypes.c_int), ("out_dtype", ctypes.c_int),
        ("gamma", ctypes.POINTER(ctypes.c_double)),
        ("rotate", ctypes.c_int), ("theta_base", ctypes.c_double),
        ("pos_offset", ctypes.c_longlong),
    ]


_lib = None


def load_library(path: str = LIB_PATH):
    """Load the CUDA library (once).  Raises if it is missing."""
    global _lib
    if _lib is not None and path == LIB_PATH:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m retentive_network_scale_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    vp, st, D = ctypes.c_void_p, ctypes.c_size_t, ctypes.POINTER(RetDesc)
    lib.ret_parallel.argtypes = [D, vp, vp, vp, vp, vp, st, vp]
    lib.ret_parallel_workspace_size.argtypes = [D]
    lib.ret_parallel_workspace_size.restype = st
    lib.ret_chunkwise.argtypes = [D, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp,
                                  ctypes.c_float, vp, vp, st, vp]
    lib.ret_chunkwise_gate_static.argtypes = [D, ctypes.c_int, vp, vp, vp, vp, vp, vp,
                                              ctypes.c_float, vp, vp]
    lib.ret_workspace_size.argtypes = [D, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.ret_workspace_size.restype = st
    lib.ret_chunkwise_fast_size.argtypes = [D, ctypes.c_int]
    lib.ret_chunkwise_fast_size.restype = st
    lib.ret_chunkwise_prep_size.argtypes = [D, ctypes.c_int]
    lib.ret_chunkwise_prep_size.restype = st
    lib.ret_chunkwise_prepare.argtypes = [D, ctypes.c_int, vp, vp, vp, st, vp]
    lib.ret_chunkwise_prepared.argtypes = [D, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp,
                                           ctypes.c_float, vp, vp]
    lib.ret_chunkwise_host.argtypes = [D, ctypes.c_int, vp, vp, vp, vp, vp, ctypes.c_float, vp,
                                       ctypes.c_int, vp, st, vp]
    lib.ret_chunkwise_host_workspace_size.argtypes = [D, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                                      ctypes.c_int]
    lib.ret_chunkwise_host_workspace_size.restype = st
    lib.ret_selftest_wait_timeout.argtypes = [ctypes.c_longlong, vp]
    lib.ret_msr_layer.argtypes = [D, ctypes.c_int, ctypes.c_int, vp, vp, vp, ctypes.c_float, vp, vp,
                                  st, vp]
    lib.ret_msr_layer_workspace_size.argtypes = [D, ctypes.c_int, ctypes.c_int]
    lib.ret_msr_layer_workspace_size.restype = st
    ll = ctypes.c_longlong
    lib.ret_gemm_bf16.argtypes = [ll, ll, ll, vp, ll, vp, ll, vp, ll, vp]
    lib.ret_backward.argtypes = [D, ctypes.c_int, vp, vp, vp, vp, vp, vp, vp, vp, st, vp]
    lib.ret_backward_workspace_size.argtypes = [D, ctypes.c_int]
    lib.ret_backward_workspace_size.restype = st
    lib.ret_segment_state.argtypes = [D, vp, vp, vp, vp, st, vp]
    lib.ret_segment_state_workspace_size.argtypes = [D]
    lib.ret_segment_state_workspace_size.restype = st
    lib.ret_state_scan.argtypes = [D, ctypes.c_int, ctypes.POINTER(ctypes.c_int), ctypes.c_int, vp,
                                   vp, vp, vp]
    lib.ret_chunkwise_segmented.argtypes = [D, ctypes.c_int, ctypes.c_int, vp, vp, vp, vp, vp, vp,
                                            vp, st, vp]
    lib.ret_chunkwise_segmented_workspace_size.argtypes = [D, ctypes.c_int, ctypes.c_int]
    lib.ret_chunkwise_segmented_workspace_size.restype = st
    lib.ret_recurrent_step.argtypes = [D, vp, vp, vp, vp, vp, vp]
    lib.ret_gate_norm.argtypes = [ctypes.c_int] * 5 + [vp, ctypes.c_int, vp, ctypes.c_float,
                                                       ctypes.c_int, vp, vp]
    lib.ret_gate_norm_backward.argtypes = [ctypes.c_int] * 5 + [vp, ctypes.c_int, vp, vp,
                                                                ctypes.c_float, vp, vp, vp]
    lib.ret_last_device_status.argtypes = [vp]
    lib.ret_msr_gammas.argtypes = [ctypes.c_int, ctypes.POINTER(ctypes.c_double)]
    lib.ret_msr_gammas.restype = ctypes.c_int
    lib.ret_kernel_launches.argtypes = []
    lib.ret_kernel_launches.restype = ctypes.c_ulonglong
    lib.ret_status_string.argtypes = [ctypes.c_int]
    lib.ret_status_string.restype = ctypes.c_char_p
    for f in ("ret_parallel", "ret_chunkwise", "ret_chunkwise_gate_static", "ret_recurrent_step",
              "ret_gate_norm", "ret_gate_norm_backward", "ret_last_device_status"):
        getattr(lib, f).restype = ctypes.c_int
    if path == LIB_PATH:
        _lib = lib
    return lib


def _status_text(status: int) -> str:
    try:
        return load_library().ret_status_string(status).decode()
    except Exception:  # the library itself failed to load
        return "?"


def msr_gammas(H: int) -> list:
    """Decay schedule gamma_h = 1 - 2^(-5-h) of the multi-scale retention
    layer ("Retentive Network" paper summary, section 2.2), from the
    library's ret_msr_gammas."""
    out = (ctypes.c_double * max(int(H), 1))()
    _check(load_library().ret_msr_gammas(int(H), out), "ret_msr_gammas")
    return list(out)[:H]


# ---------------------------------------------------------------- marshalling
def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return RET_F32
    if t.dtype == torch.bfloat16:
        return RET_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _dev(t, name, shape=None, dtype=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return t


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def make_desc(B, H, L, d_k, d_v, in_dtype, out_dtype, gamma, rotate=False,
              theta_base=10000.0, pos_offset=0):
    if len(gamma) != H:
        raise ValueError("gamma needs one value per head")
    g = (ctypes.c_double * H)(*[float(x) for x in gamma])
    d = RetDesc(B, H, L, d_k, d_v, in_dtype, out_dtype,
                ctypes.cast(g, ctypes.POINTER(ctypes.c_double)), int(bool(rotate)),
                float(theta_base), int(pos_offset))
    d._keep = g  # keep the host gamma array alive with the struct
    return d


def _check(status, what):
    if status != 0:
        raise RetentionError(status, what)


# ---------------------------------------------------------------- entry points
def ret_parallel(Q, K, V, O, gamma, rotate=False, theta_base=10000.0, pos_offset=0,
                 workspace=None, stream=None):
    """Parallel form: O = (Q^ K^^T (.) D) V.  Q, K [B,H,L,dk], V, O [B,H,L,dv].
    Allocates the workspace with torch when the call needs one and none is
    given."""
    lib = load_library()
    B, H, L, dk = Q.shape
    dv = V.shape[-1]
    _dev(Q, "Q"); _dev(K, "K", Q.shape, Q.dtype); _dev(V, "V", (B, H, L, dv), Q.dtype)
    _dev(O, "O", (B, H, L, dv))
    d = make_desc(B, H, L, dk, dv, _dtype_code(Q), _dtype_code(O), gamma, rotate,
                  theta_base, pos_offset)
    need = int(lib.ret_parallel_workspace_size(ctypes.byref(d)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ret_parallel(ctypes.byref(d), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                            _ptr(workspace), ws_bytes, _stream(stream)), "ret_parallel")
    return O


def ret_chunkwise_prep_size(B, H, L, d_k, d_v, in_dtype, out_dtype, gamma, chunk, rotate=False,
                            theta_base=10000.0, pos_offset=0):
    """Optional workspace bytes for the prepared operands of the
    tensor-core chunkwise path (0 where that path does not apply)."""
    lib = load_library()
    d = make_desc(B, H, L, d_k, d_v, in_dtype, out_dtype, gamma, rotate, theta_base, pos_offset)
    return int(lib.ret_chunkwise_prep_size(ctypes.byref(d), int(chunk)))


def ret_chunkwise_fast_size(B, H, L, d_k, d_v, in_dtype, out_dtype, gamma, chunk, rotate=False,
                            theta_base=10000.0, pos_offset=0):
    """Optional workspace bytes with which ret_chunkwise takes its fastest
    path (the prepared operands; for few heads, the segmented layout)."""
    lib = load_library()
    d = make_desc(B, H, L, d_k, d_v, in_dtype, out_dtype, gamma, rotate, theta_base, pos_offset)
    return int(lib.ret_chunkwise_fast_size(ctypes.byref(d), int(chunk)))


def ret_chunkwise_prepare(Q, K, gamma, chunk, workspace, rotate=False, theta_base=10000.0,
                          pos_offset=0, stream=None):
    """The streaming pass alone: rotated Q (with rotation) then the
    decay-weighted rotated K, bf16, into `workspace` (a uint8 device tensor
    of at least ret_chunkwise_prep_size bytes).  Returns (Q^ or None, K~)
    as views of the workspace."""
    lib = load_library()
    B, H, L, dk = Q.shape
    _dev(Q, "Q"); _dev(K, "K", Q.shape, Q.dtype); _dev(workspace, "workspace")
    d = make_desc(B, H, L, dk, dk, _dtype_code(Q), _dtype_code(Q), gamma, rotate, theta_base,
                  pos_offset)
    ws_bytes = workspace.numel() * workspace.element_size()
    _check(lib.ret_chunkwise_prepare(ctypes.byref(d), int(chunk), _ptr(Q), _ptr(K),
                                     _ptr(workspace), ws_bytes, _stream(stream)),
           "ret_chunkwise_prepare")
    n = B * H * L * dk
    flat = workspace.view(torch.bfloat16)
    if rotate:
        return flat[:n].view(B, H, L, dk), flat[n:2 * n].view(B, H, L, dk)
    return None, flat[:n].view(B, H, L, dk)


def ret_chunkwise_prepared(Qh, Kt, V, gamma, chunk, O=None, state_in=None, state_out=None,
                           G=None, Y=None, gn_eps=1e-5, rotate=False, theta_base=10000.0,
                           pos_offset=0, stream=None):
    """The chunk loop alone on rows ret_chunkwise_prepare wrote (its views;
    Q itself for Qh without rotation).  Returns (O, Y, state_out)."""
    lib = load_library()
    B, H, L, dk = Qh.shape
    dv = V.shape[-1]
    _dev(Qh, "Qh", dtype=torch.bfloat16); _dev(Kt, "Kt", Qh.shape, torch.bfloat16)
    _dev(V, "V", (B, H, L, dv), torch.bfloat16)
    _dev(O, "O", (B, H, L, dv)); _dev(G, "G", (B, L, H * dv)); _dev(Y, "Y", (B, L, H * dv))
    _dev(state_in, "state_in", (B, H, dk, dv), torch.float32)
    _dev(state_out, "state_out", (B, H, dk, dv), torch.float32)
    out = O if O is not None else Y
    if out is None:
        raise ValueError("ret_chunkwise_prepared needs O or Y")
    d = make_desc(B, H, L, dk, dv, RET_BF16, _dtype_code(out), gamma, rotate, theta_base,
                  pos_offset)
    _check(lib.ret_chunkwise_prepared(ctypes.byref(d), int(chunk), _ptr(Qh), _ptr(Kt), _ptr(V),
                                      _ptr(state_in), _ptr(state_out), _ptr(O), _ptr(G),
                                      ctypes.c_float(gn_eps), _ptr(Y), _stream(stream)),
           "ret_chunkwise_prepared")
    return O, Y, state_out


def _host(t, name, shape=None, dtype=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor) or t.is_cuda:
        raise TypeError(f"{name} must be a host (CPU) tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    return t


def ret_chunkwise_host(Q, K, V, gamma, chunk, O=None, G=None, Y=None, gn_eps=1e-5, rotate=False,
                       theta_base=10000.0, pos_offset=0, slices=None, workspace=None, stream=None):
    """Chunkwise form from host tensors to host tensors (page-locked for
    overlap), pipelined over batch slices on the device.  Allocates the
    device workspace with torch when none is given.  Returns (O, Y)."""
    lib = load_library()
    B, H, L, dk = Q.shape
    dv = V.shape[-1]
    _host(Q, "Q"); _host(K, "K", Q.shape, Q.dtype); _host(V, "V", (B, H, L, dv), Q.dtype)
    _host(O, "O", (B, H, L, dv)); _host(G, "G", (B, L, H * dv), Q.dtype); _host(Y, "Y", (B, L, H * dv))
    out_t = O if O is not None else Y
    if out_t is None:
        raise ValueError("request O, Y or both")
    if O is not None and Y is not None and O.dtype != Y.dtype:
        raise TypeError("O and Y must share a dtype")
    slices = min(B, 8) if slices is None else int(slices)
    d = make_desc(B, H, L, dk, dv, _dtype_code(Q), _dtype_code(out_t), gamma, rotate,
                  theta_base, pos_offset)
    need = int(lib.ret_chunkwise_host_workspace_size(ctypes.byref(d), int(chunk), int(O is not None),
                                                     int(Y is not None), max(slices, 1)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device="cuda")
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ret_chunkwise_host(ctypes.byref(d), int(chunk), _ptr(Q), _ptr(K), _ptr(V), _ptr(O),
                                  _ptr(G), float(gn_eps), _ptr(Y), slices, _ptr(workspace), ws_bytes,
                                  _stream(stream)), "ret_chunkwise_host")
    return O, Y


def ret_chunkwise_host_workspace_size(B, H, L, d_k, d_v, in_dtype, out_dtype, gamma, chunk, slices,
                                      want_O=False, want_Y=True, rotate=False, theta_base=10000.0,
                                      pos_offset=0) -> int:
    lib = load_library()
    d = make_desc(B, H, L, d_k, d_v, in_dtype, out_dtype, gamma, rotate, theta_base, pos_offset)
    return int(lib.ret_chunkwise_host_workspace_size(ctypes.byref(d), int(chunk), int(bool(want_O)),
                                                     int(bool(want_Y)), int(slices)))


def ret_msr_layer(X, W_qkvg, W_o, gamma, chunk, d_k, d_v, out=None, gn_eps=1e-5, rotate=False,
                  theta_base=10000.0, pos_offset=0, workspace=None, stream=None):
    """The multi-scale retention layer: X [B,L,d_model] bf16, W_qkvg
    [d_model, H*(2 d_k + 2 d_v)], W_o [H*d_v, d_model]; returns out
    [B,L,d_model] bf16.  Allocates the workspace with torch when none is
    given."""
    lib = load_library()
    B, L, dm = X.shape
    H = len(gamma)
    n_proj = H * (2 * d_k + 2 * d_v)
    _dev(X, "X", dtype=torch.bfloat16); _dev(W_qkvg, "W_qkvg", (dm, n_proj), torch.bfloat16)
    _dev(W_o, "W_o", (H * d_v, dm), torch.bfloat16)
    if out is None:
        out = torch.empty(B, L, dm, device=X.device, dtype=torch.bfloat16)
    _dev(out, "out", (B, L, dm), torch.bfloat16)
    d = make_desc(B, H, L, d_k, d_v, RET_BF16, RET_BF16, gamma, rotate, theta_base, pos_offset)
    need = int(lib.ret_msr_layer_workspace_size(ctypes.byref(d), int(dm), int(chunk)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=X.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ret_msr_layer(ctypes.byref(d), int(dm), int(chunk), _ptr(X), _ptr(W_qkvg), _ptr(W_o),
                             float(gn_eps), _ptr(out), _ptr(workspace), ws_bytes, _stream(stream)),
           "ret_msr_layer")
    return out


def ret_gemm_bf16(A, B, C=None, stream=None):
    """C = A B (bf16 [M, K] times bf16 [K, N], fp32 accumulation, bf16 C
    [M, N]) on the library's tensor-core product; 2-D tensors whose rows
    may be strided (unit stride along a row).  Returns C."""
    lib = load_library()
    for t, n in ((A, "A"), (B, "B")):
        if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dim() != 2 or t.stride(1) != 1 \
                or t.dtype != torch.bfloat16:
            raise ValueError(f"{n} must be a 2-D bf16 CUDA tensor with unit row stride")
    M, K = A.shape
    K2, N = B.shape
    if K2 != K:
        raise ValueError("inner sizes differ")
    if C is None:
        C = torch.empty(M, N, device=A.device, dtype=torch.bfloat16)
    if not C.is_cuda or C.dim() != 2 or C.stride(1) != 1 or tuple(C.shape) != (M, N) \
            or C.dtype != torch.bfloat16:
        raise ValueError("C must be a 2-D bf16 CUDA tensor [M, N] with unit row stride")
    _check(lib.ret_gemm_bf16(M, N, K, _ptr(A), A.stride(0), _ptr(B), B.stride(0), _ptr(C),
                             C.stride(0), _stream(stream)), "ret_gemm_bf16")
    return C


def lib_msr_layer_workspace_size(B, H, L, d_k, d_v, gamma, d_model, chunk, rotate=False):
    """Device workspace bytes of ret_msr_layer for these sizes."""
    lib = load_library()
    d = make_desc(B, H, L, d_k, d_v, RET_BF16, RET_BF16, gamma, rotate)
    return int(lib.ret_msr_layer_workspace_size(ctypes.byref(d), int(d_model), int(chunk)))


def ret_backward(Q, K, V, dO, gamma, chunk, dQ=None, dK=None, dV=None, out_dtype=torch.float32,
                 rotate=False, theta_base=10000.0, pos_offset=0, workspace=None, stream=None):
    """Gradients of the retention output with respect to Q, K, V given dO
    (bf16 inputs); returns (dQ, dK, dV), allocated in `out_dtype` when not
    given.  Allocates the workspace with torch when none is given."""
    lib = load_library()
    B, H, L, dk = Q.shape
    dv = V.shape[-1]
    _dev(Q, "Q", dtype=torch.bfloat16); _dev(K, "K", Q.shape, torch.bfloat16)
    _dev(V, "V", (B, H, L, dv), torch.bfloat16); _dev(dO, "dO", (B, H, L, dv), torch.bfloat16)
    mk = lambda t, shape: t if t is not None else torch.empty(shape, device=Q.device, dtype=out_dtype)  # noqa: E731
    dQ, dK, dV = mk(dQ, (B, H, L, dk)), mk(dK, (B, H, L, dk)), mk(dV, (B, H, L, dv))
    _dev(dQ, "dQ", (B, H, L, dk)); _dev(dK, "dK", (B, H, L, dk), dQ.dtype)
    _dev(dV, "dV", (B, H, L, dv), dQ.dtype)
    d = make_desc(B, H, L, dk, dv, RET_BF16, _dtype_code(dQ), gamma, rotate, theta_base, pos_offset)
    need = int(lib.ret_backward_workspace_size(ctypes.byref(d), int(chunk)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ret_backward(ctypes.byref(d), int(chunk), _ptr(Q), _ptr(K), _ptr(V), _ptr(dO), _ptr(dQ),
                            _ptr(dK), _ptr(dV), _ptr(workspace), ws_bytes, _stream(stream)),
           "ret_backward")
    return dQ, dK, dV


def lib_backward_workspace_size(B, H, L, d_k, d_v, gamma, chunk, rotate=False):
    """Device workspace bytes of ret_backward for these sizes."""
    lib = load_library()
    d = make_desc(B, H, L, d_k, d_v, RET_BF16, RET_F32, gamma, rotate)
    return int(lib.ret_backward_workspace_size(ctypes.byref(d), int(chunk)))


def ret_segment_state(K, V, gamma, U=None, rotate=False, theta_base=10000.0, pos_offset=0,
                      workspace=None, stream=None):
    """The state a segment of rows leaves behind from a zero state (bf16
    K, V), fp32 [B][H][d_k][d_v]; allocated when not given, as is the
    workspace."""
    lib = load_library()
    B, H, L, dk = K.shape
    dv = V.shape[-1]
    _dev(K, "K", dtype=torch.bfloat16); _dev(V, "V", (B, H, L, dv), torch.bfloat16)
    if U is None:
        U = torch.empty(B, H, dk, dv, device=K.device, dtype=torch.float32)
    _dev(U, "U", (B, H, dk, dv), torch.float32)
    d = make_desc(B, H, L, dk, dv, RET_BF16, RET_F32, gamma, rotate, theta_base, pos_offset)
    need = int(lib.ret_segment_state_workspace_size(ctypes.byref(d)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=K.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ret_segment_state(ctypes.byref(d), _ptr(K), _ptr(V), _ptr(U), _ptr(workspace),
                                 ws_bytes, _stream(stream)), "ret_segment_state")
    return U


def lib_segment_state_workspace_size(B, H, L, d_k, d_v, gamma, rotate=False):
    """Device workspace bytes of ret_segment_state for these sizes."""
    lib = load_library()
    d = make_desc(B, H, L, d_k, d_v, RET_BF16, RET_F32, gamma, rotate)
    return int(lib.ret_segment_state_workspace_size(ctypes.byref(d)))


def ret_state_scan(U_all, seg_lens, rank, gamma, state_in=None, R=None, stream=None):
    """The state entering segment `rank` of consecutive segments of
    seg_lens rows, from the segments' own states U_all [n_seg][B][H][d_k][d_v]
    (fp32, device) and the state before the first segment."""
    lib = load_library()
    n_seg, B, H, dk, dv = U_all.shape
    _dev(U_all, "U_all", dtype=torch.float32)
    if state_in is not None:
        _dev(state_in, "state_in", (B, H, dk, dv), torch.float32)
    if R is None:
        R = torch.empty(B, H, dk, dv, device=U_all.device, dtype=torch.float32)
    _dev(R, "R", (B, H, dk, dv), torch.float32)
    lens = (ctypes.c_int * len(seg_lens))(*[int(x) for x in seg_lens])
    d = make_desc(B, H, 0, dk, dv, RET_F32, RET_F32, gamma)
    _check(lib.ret_state_scan(ctypes.byref(d), len(seg_lens), lens, int(rank), _ptr(U_all),
                              _ptr(state_in), _ptr(R), _stream(stream)), "ret_state_scan")
    return R


def ret_chunkwise_segmented(Q, K, V, gamma, chunk, segments, O=None, state_in=None,
                            state_out=None, rotate=False, theta_base=10000.0, pos_offset=0,
                            workspace=None, out_dtype=torch.bfloat16, stream=None):
    """ret_chunkwise for few long sequences: each cut into `segments` equal
    segments that run at once, joined through their states.  Returns
    (O, state_out); O is allocated in `out_dtype` when not given, as is the
    workspace."""
    lib = load_library()
    B, H, L, dk = Q.shape
    dv = V.shape[-1]
    _dev(Q, "Q", dtype=torch.bfloat16); _dev(K, "K", Q.shape, torch.bfloat16)
    _dev(V, "V", (B, H, L, dv), torch.bfloat16)
    if O is None:
        O = torch.empty(B, H, L, dv, device=Q.device, dtype=out_dtype)
    _dev(O, "O", (B, H, L, dv))
    _dev(state_in, "state_in", (B, H, dk, dv), torch.float32)
    _dev(state_out, "state_out", (B, H, dk, dv), torch.float32)
    d = make_desc(B, H, L, dk, dv, RET_BF16, _dtype_code(O), gamma, rotate, theta_base, pos_offset)
    need = int(lib.ret_chunkwise_segmented_workspace_size(ctypes.byref(d), int(chunk), int(segments)))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ret_chunkwise_segmented(ctypes.byref(d), int(chunk), int(segments), _ptr(Q), _ptr(K),
                                       _ptr(V), _ptr(state_in), _ptr(state_out), _ptr(O),
                                       _ptr(workspace), ws_bytes, _stream(stream)),
           "ret_chunkwise_segmented")
    return O, state_out


def lib_segmented_workspace_size(B, H, L, d_k, d_v, gamma, chunk, segments, rotate=False):
    """Device workspace bytes of ret_chunkwise_segmented for these sizes."""
    lib = load_library()
    d = make_desc(B, H, L, d_k, d_v, RET_BF16, RET_BF16, gamma, rotate)
    return int(lib.ret_chunkwise_segmented_workspace_size(ctypes.byref(d), int(chunk), int(segments)))


def ret_selftest_wait_timeout(cycles, stream=None):
    """Diagnostic: a bounded wait that runs out (see the header); afterwards
    ret_last_device_status() reports RET_ERR_TIMEOUT."""
    lib = load_library()
    _check(lib.ret_selftest_wait_timeout(int(cycles), _stream(stream)), "ret_selftest_wait_timeout")


def ret_workspace_size(B, H, L, d_k, d_v, in_dtype, out_dtype, gamma, chunk,
                       want_O=True, want_Y=False, rotate=False, theta_base=10000.0,
                       pos_offset=0) -> int:
    lib = load_library()
    d = make_desc(B, H, L, d_k, d_v, in_dtype, out_dtype, gamma, rotate, theta_base, pos_offset)
    return int(lib.ret_workspace_size(ctypes.byref(d), int(chunk), int(bool(want_O)),
                                      int(bool(want_Y))))


def ret_chunkwise(Q, K, V, gamma, chunk, O=None, state_in=None, state_out=None, G=None,
                  Y=None, gn_eps=1e-5, rotate=False, theta_base=10000.0, pos_offset=0,
                  workspace=None, stream=None, prep=True):
    """Chunkwise recurrent form with optional state in/out and the fused
    GroupNorm + swish gate (Y).  Allocates the workspace with torch when the
    call needs one and none is given; with `prep` it also makes room for
    the operands the tensor-core path prepares ahead of the chunk loop
    (ret_chunkwise_prep_size), else that path prepares them in the loop.
    Returns (O, Y, state_out)."""
    lib = load_library()
    B, H, L, dk = Q.shape
    dv = V.shape[-1]
    _dev(Q, "Q"); _dev(K, "K", Q.shape, Q.dtype); _dev(V, "V", (B, H, L, dv), Q.dtype)
    _dev(O, "O", (B, H, L, dv))
    _dev(state_in, "state_in", (B, H, dk, dv), torch.float32)
    _dev(state_out, "state_out", (B, H, dk, dv), torch.float32)
    _dev(G, "G", (B, L, H * dv), Q.dtype)
    _dev(Y, "Y", (B, L, H * dv))
    if O is not None and Y is not None and O.dtype != Y.dtype:
        raise TypeError("O and Y must share a dtype")
    out_t = O if O is not None else Y
    if out_t is None:
        raise ValueError("request O, Y or both")
    d = make_desc(B, H, L, dk, dv, _dtype_code(Q), _dtype_code(out_t), gamma, rotate,
                  theta_base, pos_offset)
    need = int(lib.ret_workspace_size(ctypes.byref(d), int(chunk), int(O is not None),
                                      int(Y is not None)))
    if prep:
        need = max(need, int(lib.ret_chunkwise_fast_size(ctypes.byref(d), int(chunk))))
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=Q.device)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.ret_chunkwise(ctypes.byref(d), int(chunk), _ptr(Q), _ptr(K), _ptr(V),
                             _ptr(state_in), _ptr(state_out), _ptr(O), _ptr(G),
                             float(gn_eps), _ptr(Y), _ptr(workspace), ws_bytes,
                             _stream(stream)), "ret_chunkwise")
    return O, Y, state_out


def ret_chunkwise_gate_static(Q, K, V, gamma, chunk, G, Y, state_in=None, state_out=None,
                              gn_eps=1e-5, rotate=False, theta_base=10000.0, pos_offset=0,
                              stream=None):
    """Chunkwise form with the fused GroupNorm + swish gate (Y only) whose
    scratch is the library's fixed device array: nothing is allocated."""
    lib = load_library()
    B, H, L, dk = Q.shape
    dv = V.shape[-1]
    _dev(Q, "Q"); _dev(K, "K", Q.shape, Q.dtype); _dev(V, "V", (B, H, L, dv), Q.dtype)
    _dev(G, "G", (B, L, H * dv), Q.dtype); _dev(Y, "Y", (B, L, H * dv))
    _dev(state_in, "state_in", (B, H, dk, dv), torch.float32)
    _dev(state_out, "state_out", (B, H, dk, dv), torch.float32)
    d = make_desc(B, H, L, dk, dv, _dtype_code(Q), _dtype_code(Y), gamma, rotate, theta_base,
                  pos_offset)
    _check(lib.ret_chunkwise_gate_static(ctypes.byref(d), int(chunk), _ptr(Q), _ptr(K), _ptr(V),
                                         _ptr(state_in), _ptr(state_out), _ptr(G), float(gn_eps),
                                         _ptr(Y), _stream(stream)), "ret_chunkwise_gate_static")
    return Y


def ret_recurrent_step(q, k, v, state, o, gamma, pos, rotate=False, theta_base=10000.0,
                       stream=None):
    """Recurrent steps starting at absolute position ``pos``: one token with
    q, k [B,H,dk] and v, o [B,H,dv], or T tokens (T <= RET_MAX_DECODE_STEPS)
    with q, k [B,H,T,dk] and v, o [B,H,T,dv]; state [B,H,dk,dv] fp32 is
    updated in place (read and written once for all T)."""
    lib = load_library()
    if q.dim() == 3:
        B, H, dk = q.shape
        T = 1
    else:
        B, H, T, dk = q.shape
    dv = v.shape[-1]
    lead = tuple(q.shape[:-1])
    _dev(q, "q"); _dev(k, "k", q.shape, q.dtype); _dev(v, "v", lead + (dv,), q.dtype)
    _dev(state, "state", (B, H, dk, dv), torch.float32); _dev(o, "o", lead + (dv,))
    d = make_desc(B, H, T, dk, dv, _dtype_code(q), _dtype_code(o), gamma, rotate,
                  theta_base, pos)
    _check(lib.ret_recurrent_step(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(state),
                                  _ptr(o), _stream(stream)), "ret_recurrent_step")
    return o


def ret_gate_norm(O, G, Y, eps=1e-5, stream=None):
    """Y = swish(G) (.) GroupNorm_h(O): O [B,H,L,dv]; G, Y [B,L,H*dv]."""
    lib = load_library()
    B, H, L, dv = O.shape
    _dev(O, "O"); _dev(G, "G", (B, L, H * dv)); _dev(Y, "Y", (B, L, H * dv))
    _check(lib.ret_gate_norm(B, L, H, dv, _dtype_code(O), _ptr(O), _dtype_code(G), _ptr(G),
                             float(eps), _dtype_code(Y), _ptr(Y), _stream(stream)),
           "ret_gate_norm")
    return Y


def ret_gate_norm_backward(O, G, dY, dO, dG, eps=1e-5, stream=None):
    """dO, dG of Y = swish(G) (.) GroupNorm_h(O) given dY: O, dO [B,H,L,dv]
    (O's dtype); G, dY, dG [B,L,H*dv] (G's dtype)."""
    lib = load_library()
    B, H, L, dv = O.shape
    _dev(O, "O"); _dev(dO, "dO", (B, H, L, dv)); _dev(G, "G", (B, L, H * dv))
    _dev(dY, "dY", (B, L, H * dv)); _dev(dG, "dG", (B, L, H * dv))
    if dO.dtype != O.dtype or dY.dtype != G.dtype or dG.dtype != G.dtype:
        raise TypeError("dO takes O's dtype; dY and dG take G's")
    _check(lib.ret_gate_norm_backward(B, L, H, dv, _dtype_code(O), _ptr(O), _dtype_code(G),
                                      _ptr(G), _ptr(dY), float(eps), _ptr(dO), _ptr(dG),
                                      _stream(stream)), "ret_gate_norm_backward")
    return dO, dG


def ret_last_device_status(stream=None) -> int:
    return int(load_library().ret_last_device_status(_stream(stream)))


def ret_kernel_launches() -> int:
    """Kernels the library has launched in this process so far."""
    return int(load_library().ret_kernel_launches())


def ret_status_string(status: int) -> str:
    return load_library().ret_status_string(int(status)).decode()
