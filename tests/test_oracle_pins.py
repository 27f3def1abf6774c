"""Pins for the fp64 CPU oracle: each checks it against something other than
itself -- closed forms, textbook special cases, a library routine, or an
identity between two independently written forms.

Sources: "Retentive Network: A Successor to Transformer for Large Language
Models" paper summary (blog.csdn.net 132817411) section 2.1 (scalar-gamma
retention, parallel form (1), recurrent form (2), chunkwise form (3)) and
section 2.2 (gamma schedule, GroupNorm, swish gate); "RetNet dual-mode
hands-on manual" section 3.1 (unrolled state S_t = sum gamma^{t-i} K_i^T V_i).

Every ``pin_*`` function takes the loaded oracle library so that the mutation
test can run the same pins against a copy of the oracle with a planted
mistake.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch

from oracle import oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rng(seed):
    return np.random.default_rng(seed)


def _normwise(x, r):
    return float(np.abs(x - r).max() / max(np.abs(r).max(), 1e-300))


# --------------------------------------------------------------------------
def pin_gamma_schedule(lib):
    """Section 2.2: gamma_h = 1 - 2^(-5-h), against hand-worked fractions."""
    want = {}
    with open(os.path.join(GOLDEN, "gamma_schedule.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                h, frac = line.split()
                want[int(h)] = Fraction(frac)
    got = orc.gammas(16, lib=lib)
    for h, fr in want.items():
        assert Fraction(float(got[h])) == fr, (h, got[h], fr)


def pin_three_forms_agree(lib):
    """Parallel (1), recurrent (2) and chunkwise (3) reach the same result
    (section 2.1); chunk sizes cover 1, ragged tails and chunk >= L."""
    rng = _rng(1)
    B, H, L, dk, dv = 2, 3, 37, 8, 6
    Q, K, V = (rng.normal(size=(B, H, L, d)) for d in (dk, dk, dv))
    g = np.array([0.5, 0.87, 0.999])
    kw = dict(rotate=True, theta_base=10000.0, pos_offset=7, lib=lib)
    P = orc.parallel(Q, K, V, g, **kw)
    R, S = orc.recurrent(Q, K, V, g, **kw)
    assert _normwise(R, P) < 1e-10
    for C in (1, 2, 3, 16, 36, 37, 50):
        Cw, Sc = orc.chunkwise(Q, K, V, g, C, **kw)
        assert _normwise(Cw, P) < 1e-10, C
        assert _normwise(Sc, S) < 1e-10, C


def pin_linear_attention(lib):
    """gamma = 1 without rotation is causal, unnormalised linear attention:
    O = tril(Q K^T) V, computed here with numpy matrix products."""
    rng = _rng(2)
    B, H, L, dk, dv = 1, 2, 29, 5, 4
    Q, K, V = (rng.normal(size=(B, H, L, d)) for d in (dk, dk, dv))
    ref = np.tril(Q @ np.swapaxes(K, -1, -2)) @ V
    g = np.ones(H)
    assert _normwise(orc.parallel(Q, K, V, g, lib=lib), ref) < 1e-12
    assert _normwise(orc.recurrent(Q, K, V, g, lib=lib)[0], ref) < 1e-12
    assert _normwise(orc.chunkwise(Q, K, V, g, 4, lib=lib)[0], ref) < 1e-12


def pin_gamma_zero(lib):
    """gamma = 0 keeps only n = m (D_nn = gamma^0 = 1): o_t = (q_t.k_t) v_t;
    both rows turn by the same angle, so the rotation drops out."""
    rng = _rng(3)
    B, H, L, dk, dv = 2, 1, 19, 6, 3
    Q, K, V = (rng.normal(size=(B, H, L, d)) for d in (dk, dk, dv))
    ref = np.einsum("bhtd,bhtd->bht", Q, K)[..., None] * V
    g = np.zeros(H)
    kw = dict(rotate=True, pos_offset=3, lib=lib)
    assert _normwise(orc.parallel(Q, K, V, g, **kw), ref) < 1e-12
    assert _normwise(orc.recurrent(Q, K, V, g, **kw)[0], ref) < 1e-12
    assert _normwise(orc.chunkwise(Q, K, V, g, 5, **kw)[0], ref) < 1e-12


def pin_single_token(lib):
    """L = 1: o = (q.k) v at any absolute position."""
    rng = _rng(4)
    q, k, v = rng.normal(size=(1, 1, 1, 8)), rng.normal(size=(1, 1, 1, 8)), rng.normal(size=(1, 1, 1, 5))
    ref = float((q * k).sum()) * v
    for pos in (0, 1, 123456):
        for gam in (0.0, 0.3, 1.0):
            o = orc.parallel(q, k, v, [gam], rotate=True, pos_offset=pos, lib=lib)
            assert _normwise(o, ref) < 1e-12
            o, s = orc.recurrent(q, k, v, [gam], rotate=True, pos_offset=pos, lib=lib)
            assert _normwise(o, ref) < 1e-12


def _sum_cos(t, a):
    # sum_{k=0}^{t} cos(k a) = sin((t+1)a/2) cos(t a/2) / sin(a/2)
    return math.sin((t + 1) * a / 2) * math.cos(t * a / 2) / math.sin(a / 2)


def _sum_sin(t, a):
    # sum_{k=0}^{t} sin(k a) = sin((t+1)a/2) sin(t a/2) / sin(a/2)
    return math.sin((t + 1) * a / 2) * math.sin(t * a / 2) / math.sin(a / 2)


def pin_rotation_closed_forms(lib):
    """Section 2.1: Q_n e^{in theta}, K_m e^{im theta}, theta_j =
    base^(-2j/dk), score Re[(q e^{in theta})(k e^{im theta})^dagger].
    With gamma = 1 and v = 1 the output is a sum of cosines (or sines) with
    the trigonometric closed forms above.  Pair 0 has theta = 1; pair 1 of
    dk = 4 has theta = base^(-1/2) = 1/100 for base 10000."""
    L = 40
    t = np.arange(L)
    one = np.ones((1, 1, L, 1))
    # pair 0, q = (1,0), k = (1,0): cos((t-m) * 1)
    q = np.zeros((1, 1, L, 2)); q[..., 0] = 1
    k = np.zeros((1, 1, L, 2)); k[..., 0] = 1
    want = np.array([_sum_cos(i, 1.0) for i in t])
    for fn in ("parallel", "recurrent", "chunkwise"):
        args = (q, k, one, [1.0]) + ((7,) if fn == "chunkwise" else ())
        out = getattr(orc, fn)(*args, rotate=True, pos_offset=11, lib=lib)
        out = out[0] if isinstance(out, tuple) else out
        assert np.abs(out[0, 0, :, 0] - want).max() < 1e-9, fn
    # pair 0, q = (1,0), k = (0,1): sin((t-m) * 1) -- fixes the direction
    k2 = np.zeros((1, 1, L, 2)); k2[..., 1] = 1
    want = np.array([_sum_sin(i, 1.0) for i in t])
    out = orc.parallel(q, k2, one, [1.0], rotate=True, lib=lib)
    assert np.abs(out[0, 0, :, 0] - want).max() < 1e-9
    # pair 1 of dk = 4: frequency base^(-2/4)
    q4 = np.zeros((1, 1, L, 4)); q4[..., 2] = 1
    want = np.array([_sum_cos(i, 0.01) for i in t])
    out = orc.parallel(q4, q4, one, [1.0], rotate=True, theta_base=10000.0, lib=lib)
    assert np.abs(out[0, 0, :, 0] - want).max() < 1e-9
    # the rotation itself: (1, 0) at position p becomes (cos p, sin p)
    r = orc.xpos_rotate([1.0, 0.0], 2.5, lib=lib)
    assert abs(r[0] - math.cos(2.5)) < 1e-15 and abs(r[1] - math.sin(2.5)) < 1e-15


def pin_offset_invariance(lib):
    """Scores depend only on n - m, so shifting every position leaves the
    parallel output unchanged."""
    rng = _rng(5)
    Q, K, V = (rng.normal(size=(1, 2, 23, d)) for d in (8, 8, 3))
    g = [0.9, 0.99]
    a = orc.parallel(Q, K, V, g, rotate=True, pos_offset=0, lib=lib)
    b = orc.parallel(Q, K, V, g, rotate=True, pos_offset=12345, lib=lib)
    assert _normwise(a, b) < 1e-10


def pin_state_closed_form(lib):
    """Dual-mode manual 3.1: unrolled, S_t = sum_i gamma^{t-i} K_i^T V_i (plus
    gamma^L times a starting state)."""
    rng = _rng(6)
    B, H, L, dk, dv = 1, 2, 17, 4, 3
    Q, K, V = (rng.normal(size=(B, H, L, d)) for d in (dk, dk, dv))
    S0 = rng.normal(size=(B, H, dk, dv))
    g = np.array([0.8, 0.95])
    w = g[None, :, None] ** (L - 1 - np.arange(L))[None, None, :]
    want = np.einsum("bht,bhti,bhtj->bhij", w, K, V) + (g ** L)[None, :, None, None] * S0
    _, S = orc.recurrent(Q, K, V, g, state_in=S0, lib=lib)
    assert _normwise(S, want) < 1e-12
    _, S = orc.chunkwise(Q, K, V, g, 5, state_in=S0, lib=lib)
    assert _normwise(S, want) < 1e-12


def pin_state_handoff(lib):
    """A long call equals two calls joined by the state (positions continue)."""
    rng = _rng(7)
    B, H, L1, L2, dk, dv = 1, 2, 21, 14, 6, 5
    Q, K, V = (rng.normal(size=(B, H, L1 + L2, d)) for d in (dk, dk, dv))
    g = [0.7, 0.97]
    kw = dict(rotate=True, lib=lib)
    full, Sf = orc.chunkwise(Q, K, V, g, 8, **kw)
    a, Sa = orc.chunkwise(Q[:, :, :L1], K[:, :, :L1], V[:, :, :L1], g, 8, **kw)
    b, Sb = orc.chunkwise(Q[:, :, L1:], K[:, :, L1:], V[:, :, L1:], g, 8,
                          pos_offset=L1, state_in=Sa, **kw)
    assert _normwise(np.concatenate([a, b], axis=2), full) < 1e-12
    assert _normwise(Sb, Sf) < 1e-12
    r, Sr = orc.recurrent(Q[:, :, L1:], K[:, :, L1:], V[:, :, L1:], g,
                          pos_offset=L1, state_in=Sa, **kw)
    assert _normwise(r, full[:, :, L1:]) < 1e-12
    # selected rows from the definition, with the state before row 0
    rows = [0, 5, 13]
    got = orc.rows(Q[0, 1, L1:], K[0, 1, L1:], V[0, 1, L1:], g[1], rows,
                   rotate=True, pos_offset=L1, state0=Sa[0, 1], lib=lib)
    assert _normwise(got, full[0, 1, L1:][rows]) < 1e-12


def pin_gate_groupnorm(lib):
    """Section 2.2: GroupNorm over each head's channels then swish(G) gate,
    against torch's group_norm and silu in fp64; plus the invariants."""
    rng = _rng(8)
    B, H, L, dv = 2, 3, 5, 8
    O = rng.normal(size=(B, H, L, dv)) * 3 + 1
    G = rng.normal(size=(B, L, H * dv))
    eps = 1e-5
    Y = orc.gate_groupnorm(O, G, eps, lib=lib)
    o = torch.from_numpy(O).permute(0, 2, 1, 3).reshape(B * L, H * dv)
    ref = torch.nn.functional.group_norm(o, H, eps=eps).reshape(B, L, H * dv)
    ref = torch.nn.functional.silu(torch.from_numpy(G)) * ref
    assert _normwise(Y, ref.numpy()) < 1e-12
    # G = 0 gives 0; a constant head row normalises to 0
    assert np.abs(orc.gate_groupnorm(O, np.zeros_like(G), eps, lib=lib)).max() == 0
    Oc = np.broadcast_to(rng.normal(size=(B, H, L, 1)), O.shape).copy()
    assert np.abs(orc.gate_groupnorm(Oc, G, eps, lib=lib)).max() < 1e-9
    # normalised rows: mean 0, variance sigma^2/(sigma^2+eps)
    Y1 = orc.gate_groupnorm(O, np.full_like(G, 50.0), eps, lib=lib)  # swish(50) = 50
    Yn = (Y1 / 50.0).reshape(B, L, H, dv)
    var = O.var(axis=-1).transpose(0, 2, 1)
    assert np.abs(Yn.mean(-1)).max() < 1e-12
    assert np.abs(Yn.var(-1) - var / (var + eps)).max() < 1e-10


def pin_gate_groupnorm_backward(lib):
    """Gradients of section 2.2's GroupNorm + swish gate against central
    finite differences of the forward oracle along random directions:
    d/de <dY, Y(O + e U, G + e W)> at 0 equals <dO, U> + <dG, W>.  This only
    runs the forward, so it is independent of the gradient formulas.  Plus
    what the mathematics fixes: every dO row sums to 0 (adding a constant to
    a row leaves its normalisation unchanged), and at G = 0 dO is 0 and dG is
    dY times the normalised row over 2 (swish'(0) = 1/2)."""
    rng = _rng(21)
    B, H, L, dv = 2, 3, 4, 8
    O = rng.normal(size=(B, H, L, dv)) * 2 + 0.5
    G = rng.normal(size=(B, L, H * dv)) * 1.5
    dY = rng.normal(size=(B, L, H * dv))
    eps = 1e-3
    dO, dG = orc.gate_groupnorm_backward(O, G, dY, eps, lib=lib)
    f = lambda o, g: float(np.sum(dY * orc.gate_groupnorm(o, g, eps, lib=lib)))  # noqa: E731
    h = 1e-6
    for _ in range(3):
        U = rng.normal(size=O.shape)
        W = rng.normal(size=G.shape)
        for u, w in ((U, 0 * W), (0 * U, W), (U, W)):
            fd = (f(O + h * u, G + h * w) - f(O - h * u, G - h * w)) / (2 * h)
            an = float(np.sum(dO * u) + np.sum(dG * w))
            assert abs(fd - an) <= 1e-7 * max(1.0, abs(fd)), (fd, an)
    assert np.abs(dO.sum(-1)).max() < 1e-12
    dO0, dG0 = orc.gate_groupnorm_backward(O, np.zeros_like(G), dY, eps, lib=lib)
    assert np.abs(dO0).max() == 0
    mu = O.mean(-1, keepdims=True)
    n = ((O - mu) / np.sqrt(O.var(-1, keepdims=True) + eps)).transpose(0, 2, 1, 3)
    assert _normwise(dG0, 0.5 * dY * n.reshape(B, L, H * dv)) < 1e-13


PINS = [pin_gamma_schedule, pin_three_forms_agree, pin_linear_attention,
        pin_gamma_zero, pin_single_token, pin_rotation_closed_forms,
        pin_offset_invariance, pin_state_closed_form, pin_state_handoff,
        pin_gate_groupnorm, pin_gate_groupnorm_backward]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin, olib):
    pin(olib)


def test_rejects_bad_arguments(olib):
    Q = np.zeros((1, 1, 4, 3))
    with pytest.raises(ValueError):
        orc.parallel(Q, Q, Q, [0.5], rotate=True, lib=olib)  # odd dk with rotation
    with pytest.raises(ValueError):
        orc.chunkwise(Q, Q, Q, [0.5], 0, lib=olib)  # chunk < 1


def test_empty_sequence(olib):
    Q = np.zeros((1, 2, 0, 4))
    O = orc.parallel(Q, Q, Q, [0.5, 0.6], lib=olib)
    assert O.shape == (1, 2, 0, 4)
    S0 = np.ones((1, 2, 4, 4))
    O, S = orc.chunkwise(Q, Q, Q, [0.5, 0.6], 4, state_in=S0, lib=olib)
    assert np.array_equal(S, S0)


def test_msr_layer_identity_projections(olib):
    """With identity projections the layer is the retention + GroupNorm +
    gate of the blocks of X (summary, sections 2.1-2.2): X holds, for every
    (b, t), the heads' q, k, v and the gate side by side; W_qkvg = I selects
    them, and W_o = [I | 0] hands Y back.  Pins the block order, the head
    slicing and the transposes of the layer oracle."""
    rng = np.random.default_rng(7)
    B, L, H, dk, dv = 2, 9, 3, 4, 6
    gam = [0.5, 0.9, 1.0]
    Q = rng.standard_normal((B, H, L, dk)) * 0.5
    K = rng.standard_normal((B, H, L, dk)) * 0.5
    V = rng.standard_normal((B, H, L, dv))
    G = rng.standard_normal((B, L, H * dv))
    flat = lambda a: a.transpose(0, 2, 1, 3).reshape(B, L, -1)  # noqa: E731
    X = np.concatenate([flat(Q), flat(K), flat(V), G], axis=-1)
    n = X.shape[-1]
    W_o = np.zeros((H * dv, n))
    W_o[:, :H * dv] = np.eye(H * dv)
    out = orc.msr_layer(X, np.eye(n), W_o, gam, dk, dv, rotate=True, pos_offset=3, lib=olib)
    O, _ = orc.recurrent(Q, K, V, gam, rotate=True, pos_offset=3, lib=olib)
    Y = orc.gate_groupnorm(O, G, lib=olib)
    assert np.allclose(out[..., :H * dv], Y, rtol=0, atol=1e-12)
    assert np.all(out[..., H * dv:] == 0)
    # a projection that swaps two heads' value blocks swaps their outputs
    P = np.eye(n)
    v0 = 2 * H * dk
    P[:, v0:v0 + dv], P[:, v0 + dv:v0 + 2 * dv] = np.eye(n)[:, v0 + dv:v0 + 2 * dv], np.eye(n)[:, v0:v0 + dv]
    out2 = orc.msr_layer(X, P, W_o, [0.7, 0.7, 1.0], dk, dv, lib=olib)
    O2, _ = orc.recurrent(Q, K, V[:, [1, 0, 2]], [0.7, 0.7, 1.0], lib=olib)
    assert np.allclose(out2[..., :H * dv], orc.gate_groupnorm(O2, G, lib=olib), atol=1e-12)


@pytest.mark.parametrize("rotate", [False, True])
def test_backward_matches_finite_differences(olib, rotate):
    """The backward oracle against central finite differences of the
    forward oracle along random directions: d/de <dO, O(X + e dX)> at 0
    equals <grad_X, dX> for X = Q, K, V (independent of the gradient
    formulas: it only runs the forward recurrence)."""
    rng = np.random.default_rng(11)
    B, H, L, dk, dv = 1, 2, 7, 4, 6
    gam = [0.8, 1.0]
    Q = rng.standard_normal((B, H, L, dk)) * 0.5
    K = rng.standard_normal((B, H, L, dk)) * 0.5
    V = rng.standard_normal((B, H, L, dv))
    dO = rng.standard_normal((B, H, L, dv))
    dQ, dK, dV = orc.retention_backward(Q, K, V, dO, gam, rotate=rotate, pos_offset=5, lib=olib)
    f = lambda q, k, v: float(np.sum(dO * orc.recurrent(q, k, v, gam, rotate=rotate,  # noqa: E731
                                                        pos_offset=5, lib=olib)[0]))
    eps = 1e-5
    for grad, which in ((dQ, 0), (dK, 1), (dV, 2)):
        for _ in range(3):
            args = [Q, K, V]
            d = rng.standard_normal(args[which].shape)
            plus = list(args); plus[which] = args[which] + eps * d
            minus = list(args); minus[which] = args[which] - eps * d
            fd = (f(*plus) - f(*minus)) / (2 * eps)
            assert abs(fd - float(np.sum(grad * d))) <= 1e-6 * max(1.0, abs(fd)), which


@pytest.mark.parametrize("rotate", [False, True])
def test_state_scan_joins_segments(olib, rotate):
    """The segment state and the scan against the recurrent form over the
    whole sequence: a sequence cut into unequal segments, each run from the
    state the scan gives it (at its own absolute positions), reproduces the
    outputs and the final state of one uncut run.  A wrong decay exponent,
    segment order or position offset fails it."""
    rng = np.random.default_rng(23)
    B, H, dk, dv = 1, 3, 4, 6
    lens = [5, 9, 3, 7]
    L = sum(lens)
    gam = [0.6, 0.93, 1.0]
    Q = rng.standard_normal((B, H, L, dk)) * 0.5
    K = rng.standard_normal((B, H, L, dk)) * 0.5
    V = rng.standard_normal((B, H, L, dv))
    S0 = rng.standard_normal((B, H, dk, dv))
    O_ref, S_ref = orc.recurrent(Q, K, V, gam, rotate=rotate, pos_offset=11, state_in=S0, lib=olib)
    starts = np.cumsum([0] + lens[:-1])
    U = np.stack([orc.segment_state(K[:, :, a:a + n], V[:, :, a:a + n], gam, rotate=rotate,
                                    pos_offset=11 + a, lib=olib) for a, n in zip(starts, lens)])
    R = orc.state_scan(U, lens, gam, state_in=S0)
    assert _normwise(R[-1], S_ref) <= 1e-12
    for s, (a, n) in enumerate(zip(starts, lens)):
        O_s, S_s = orc.recurrent(Q[:, :, a:a + n], K[:, :, a:a + n], V[:, :, a:a + n], gam,
                                 rotate=rotate, pos_offset=11 + a, state_in=R[s], lib=olib)
        assert _normwise(O_s, O_ref[:, :, a:a + n]) <= 1e-12
        assert _normwise(S_s, R[s + 1]) <= 1e-12
