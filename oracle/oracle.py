"""ctypes front end of the fp64 CPU oracle (``retention_oracle.c``).

TEST INFRASTRUCTURE ONLY.  The product path never imports this module; only
the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` do.  Arrays go in as anything numpy can turn into float64 and
come back as float64 numpy arrays.  The arithmetic lives in the C file; this
module only marshals arguments.

Layouts: Q, K ``[B, H, L, dk]``; V, O ``[B, H, L, dv]``; G, Y ``[B, L, H*dv]``;
state ``[B, H, dk, dv]``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "retention_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


class _Problem(ctypes.Structure):
    _fields_ = [
        ("B", ctypes.c_int), ("H", ctypes.c_int), ("L", ctypes.c_int),
        ("dk", ctypes.c_int), ("dv", ctypes.c_int),
        ("gamma", ctypes.POINTER(ctypes.c_double)),
        ("rotate", ctypes.c_int), ("theta_base", ctypes.c_double),
        ("pos_offset", ctypes.c_longlong), ("nthreads", ctypes.c_int),
    ]


def build(src: str = _SRC, out: str = _LIB_PATH, extra_flags=()) -> str:
    """Compile the oracle with gcc (IEEE arithmetic: no fast-math)."""
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
           *extra_flags, src, "-o", out, "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def _stale() -> bool:
    return (not os.path.exists(_LIB_PATH)
            or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))


def load(path: str | None = None):
    """Load (building first if missing or older than the source)."""
    global _lib
    if path is not None:
        return _bind(ctypes.CDLL(path))
    with _lock:
        if _lib is None:
            if _stale():
                build()
            _lib = _bind(ctypes.CDLL(_LIB_PATH))
    return _lib


def _bind(lib):
    P = ctypes.POINTER(_Problem)
    d = ctypes.POINTER(ctypes.c_double)
    lib.oracle_msr_gammas.argtypes = [ctypes.c_int, d]
    lib.oracle_xpos_rotate.argtypes = [d, ctypes.c_int, ctypes.c_double,
                                       ctypes.c_double, d]
    lib.oracle_retention_parallel.argtypes = [P, d, d, d, d]
    lib.oracle_retention_recurrent.argtypes = [P, d, d, d, d, d, d]
    lib.oracle_retention_chunkwise.argtypes = [P, ctypes.c_int, d, d, d, d, d, d]
    lib.oracle_retention_rows.argtypes = [
        ctypes.c_int, ctypes.c_int, ctypes.c_int, d, d, d, ctypes.c_double,
        ctypes.c_int, ctypes.c_double, ctypes.c_longlong, d, ctypes.c_int,
        ctypes.POINTER(ctypes.c_longlong), d]
    lib.oracle_gate_groupnorm.argtypes = [ctypes.c_int] * 4 + [
        d, d, ctypes.c_double, d]
    lib.oracle_gate_groupnorm_backward.argtypes = [ctypes.c_int] * 4 + [
        d, d, d, ctypes.c_double, d, d]
    for f in ("oracle_retention_parallel", "oracle_retention_recurrent",
              "oracle_retention_chunkwise", "oracle_retention_rows",
              "oracle_gate_groupnorm", "oracle_gate_groupnorm_backward"):
        getattr(lib, f).restype = ctypes.c_int
    return lib


def _f64(x) -> np.ndarray:
    if hasattr(x, "detach"):  # a torch tensor: exact upcast on the host
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _problem(Q, V, gamma, rotate, theta_base, pos_offset, nthreads):
    B, H, L, dk = Q.shape
    dv = V.shape[-1]
    g = _f64(gamma).reshape(-1)
    if g.shape[0] != H:
        raise ValueError("gamma must have one entry per head")
    p = _Problem(B, H, L, dk, dv, _ptr(g), int(bool(rotate)), float(theta_base),
                 int(pos_offset), int(nthreads))
    return p, g  # keep g alive


def _check(rc, what):
    if rc != 0:
        raise ValueError(f"oracle {what} rejected its arguments (code {rc})")


def gammas(H: int, lib=None) -> np.ndarray:
    lib = lib or load()
    g = np.zeros(H, dtype=np.float64)
    lib.oracle_msr_gammas(H, _ptr(g))
    return g


def xpos_rotate(x, pos: float, theta_base: float = 10000.0, lib=None) -> np.ndarray:
    lib = lib or load()
    x = _f64(x).reshape(-1)
    out = np.zeros_like(x)
    lib.oracle_xpos_rotate(_ptr(x), x.shape[0], float(pos), float(theta_base), _ptr(out))
    return out


def parallel(Q, K, V, gamma, rotate=False, theta_base=10000.0, pos_offset=0,
             nthreads=0, lib=None) -> np.ndarray:
    lib = lib or load()
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    p, _g = _problem(Q, V, gamma, rotate, theta_base, pos_offset, nthreads)
    O = np.zeros(Q.shape[:3] + (V.shape[-1],))
    _check(lib.oracle_retention_parallel(ctypes.byref(p), _ptr(Q), _ptr(K),
                                         _ptr(V), _ptr(O)), "parallel")
    return O


def recurrent(Q, K, V, gamma, rotate=False, theta_base=10000.0, pos_offset=0,
              state_in=None, nthreads=0, lib=None):
    """Returns (O, state_out)."""
    lib = lib or load()
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    p, _g = _problem(Q, V, gamma, rotate, theta_base, pos_offset, nthreads)
    B, H, L, dk = Q.shape
    dv = V.shape[-1]
    S_in = None if state_in is None else _f64(state_in)
    S_out = np.zeros((B, H, dk, dv))
    O = np.zeros((B, H, L, dv))
    _check(lib.oracle_retention_recurrent(ctypes.byref(p), _ptr(Q), _ptr(K), _ptr(V),
                                          _ptr(S_in), _ptr(S_out), _ptr(O)),
           "recurrent")
    return O, S_out


def chunkwise(Q, K, V, gamma, chunk, rotate=False, theta_base=10000.0,
              pos_offset=0, state_in=None, nthreads=0, lib=None):
    """Returns (O, state_out)."""
    lib = lib or load()
    Q, K, V = _f64(Q), _f64(K), _f64(V)
    p, _g = _problem(Q, V, gamma, rotate, theta_base, pos_offset, nthreads)
    B, H, L, dk = Q.shape
    dv = V.shape[-1]
    S_in = None if state_in is None else _f64(state_in)
    S_out = np.zeros((B, H, dk, dv))
    O = np.zeros((B, H, L, dv))
    _check(lib.oracle_retention_chunkwise(ctypes.byref(p), int(chunk), _ptr(Q), _ptr(K),
                                          _ptr(V), _ptr(S_in), _ptr(S_out), _ptr(O)),
           "chunkwise")
    return O, S_out


def rows(q, k, v, gamma: float, rows, rotate=False, theta_base=10000.0,
         pos_offset=0, state0=None, lib=None) -> np.ndarray:
    """Outputs of selected rows of ONE (b,h) slice: q, k [L, dk], v [L, dv]."""
    lib = lib or load()
    q, k, v = _f64(q), _f64(k), _f64(v)
    L, dk = q.shape
    dv = v.shape[-1]
    r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64).reshape(-1))
    out = np.zeros((r.shape[0], dv))
    s0 = None if state0 is None else _f64(state0)
    _check(lib.oracle_retention_rows(
        L, dk, dv, _ptr(q), _ptr(k), _ptr(v), float(gamma), int(bool(rotate)),
        float(theta_base), int(pos_offset), _ptr(s0), r.shape[0],
        r.ctypes.data_as(ctypes.POINTER(ctypes.c_longlong)), _ptr(out)), "rows")
    return out


def segment_state(K, V, gamma, rotate=False, theta_base=10000.0, pos_offset=0,
                  nthreads=0, lib=None) -> np.ndarray:
    """The state a segment of rows (K, V at positions pos_offset ..) leaves
    behind from a zero state: the recurrent form's state after its last row
    ("Retentive Network" paper summary, section 2.1, form (2)).  The query
    rows do not enter the state, so K stands in for them."""
    return recurrent(K, K, V, gamma, rotate=rotate, theta_base=theta_base,
                     pos_offset=pos_offset, nthreads=nthreads, lib=lib)[1]


def state_scan(U, seg_lens, gamma, state_in=None) -> np.ndarray:
    """States entering each of n consecutive segments of seg_lens rows, from
    the segments' own states U [n, B, H, dk, dv] (each the state its segment
    leaves from a zero start) and the state before the first segment:
    R_0 = state_in (zero if None), R_{s+1} = gamma_h^{seg_lens[s]} R_s + U_s,
    the chunkwise form's state recurrence ("Retentive Network" paper
    summary, section 2.1, form (3)) applied between segments.  Returns
    R [n + 1, B, H, dk, dv]; R[n] is the state after the last segment."""
    U = _f64(U)
    g = np.asarray(gamma, dtype=np.float64)
    n = U.shape[0]
    R = np.zeros((n + 1,) + U.shape[1:])
    if state_in is not None:
        R[0] = _f64(state_in)
    for s in range(n):
        decay = g ** int(seg_lens[s])
        R[s + 1] = decay[None, :, None, None] * R[s] + U[s]
    return R


def gate_groupnorm(O, G, eps=1e-5, lib=None) -> np.ndarray:
    """O [B, H, L, dv], G [B, L, H*dv] -> Y [B, L, H*dv]."""
    lib = lib or load()
    O, G = _f64(O), _f64(G)
    B, H, L, dv = O.shape
    Y = np.zeros((B, L, H * dv))
    _check(lib.oracle_gate_groupnorm(B, L, H, dv, _ptr(O), _ptr(G), float(eps), _ptr(Y)),
           "gate_groupnorm")
    return Y


def gate_groupnorm_backward(O, G, dY, eps=1e-5, lib=None):
    """Gradients (dO, dG) of Y = gate_groupnorm(O, G) given dY.  O, dO
    [B, H, L, dv]; G, dY, dG [B, L, H*dv]."""
    lib = lib or load()
    O, G, dY = _f64(O), _f64(G), _f64(dY)
    B, H, L, dv = O.shape
    dO, dG = np.zeros_like(O), np.zeros_like(G)
    _check(lib.oracle_gate_groupnorm_backward(B, L, H, dv, _ptr(O), _ptr(G), _ptr(dY), float(eps),
                                              _ptr(dO), _ptr(dG)), "gate_groupnorm_backward")
    return dO, dG


def msr_layer(X, W_qkvg, W_o, gamma, d_k, d_v, rotate=False, theta_base=10000.0, pos_offset=0,
              eps=1e-5, lib=None) -> np.ndarray:
    """The multi-scale retention layer, fp64 ("Retentive Network" paper
    summary, section 2.1: Q = (X W_Q) (.) Theta, K = (X W_K) (.) conj(Theta),
    V = X W_V, one decay per head; section 2.2: Y = GroupNorm_h(Concat of
    the heads), MSR(X) = (swish(X W_G) (.) Y) W_O).  X [B, L, d_model];
    W_qkvg [d_model, H*(2 d_k + 2 d_v)] with the column blocks Q, K, V, G
    (head h at h*d_k or h*d_v inside its block); W_o [H*d_v, d_model].
    The projections are plain matrix products; the retention and the
    GroupNorm + gate are this module's recurrent form and gate_groupnorm."""
    X, W, Wo = _f64(X), _f64(W_qkvg), _f64(W_o)
    B, L, _ = X.shape
    H = len(gamma)
    P = X @ W
    heads = lambda a, d: a.reshape(B, L, H, d).transpose(0, 2, 1, 3)  # noqa: E731
    Q = heads(P[..., :H * d_k], d_k)
    K = heads(P[..., H * d_k:2 * H * d_k], d_k)
    V = heads(P[..., 2 * H * d_k:2 * H * d_k + H * d_v], d_v)
    G = P[..., 2 * H * d_k + H * d_v:]
    O, _ = recurrent(np.ascontiguousarray(Q), np.ascontiguousarray(K), np.ascontiguousarray(V),
                     gamma, rotate=rotate, theta_base=theta_base, pos_offset=pos_offset, lib=lib)
    Y = gate_groupnorm(O, np.ascontiguousarray(G), eps=eps, lib=lib)
    return Y @ Wo


def retention_backward(Q, K, V, dO, gamma, rotate=False, theta_base=10000.0, pos_offset=0,
                       lib=None):
    """Gradients (dQ, dK, dV) of O = Retention(Q, K, V) from a zero state,
    given dO, fp64 ("Retentive Network" paper summary, section 2.1: the
    parallel form (Q^ K^T (.) D) V with q^_t = Theta_t q_t, k^_m = Theta_m
    k_m, D_tm = gamma^{t-m} for m <= t).  Written from that definition in
    matrix form, per (b, h):
        A = (Q^ K^^T) (.) D,  dV = A^T dO,
        dA = (dO V^T) (.) D,  dQ^ = dA K^,  dK^ = dA^T Q^,
        dq_t = Theta_t^T dq^_t = Theta_{-t} dq^_t  (and the same for dk)."""
    lib = lib or load()
    Q, K, V, dO = _f64(Q), _f64(K), _f64(V), _f64(dO)
    B, H, L, dk = Q.shape
    t = np.arange(L)

    def turn(x, sign):
        if not rotate:
            return x.copy()
        return np.stack([xpos_rotate(x[i], sign * (pos_offset + i), theta_base, lib=lib)
                         for i in range(L)])

    dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
    for b in range(B):
        for h in range(H):
            g = float(gamma[h])
            diff = t[:, None] - t[None, :]
            D = np.where(diff >= 0, np.power(g, np.maximum(diff, 0)), 0.0)
            D[np.arange(L), np.arange(L)] = 1.0
            qh, kh = turn(Q[b, h], 1), turn(K[b, h], 1)
            A = (qh @ kh.T) * D
            dV[b, h] = A.T @ dO[b, h]
            dA = (dO[b, h] @ V[b, h].T) * D
            dQ[b, h] = turn(dA @ kh, -1)
            dK[b, h] = turn(dA.T @ qh, -1)
    return dQ, dK, dV
