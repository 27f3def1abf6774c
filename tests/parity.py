"""Shared helpers for the GPU parity tests: error metrics, tolerances and
oracle runs on sampled (b, h) slices.

Tolerances (fixed by the problem statement): fp32 inputs -- normwise
max|x - r| / max|r| <= 1e-5; bf16 inputs with fp32 accumulation -- relative
L2 error ||x - r|| / ||r|| <= 1e-2.  The same metrics apply to states."""
import numpy as np
import torch

from oracle import oracle as orc

TOL_F32 = 1e-5
TOL_BF16 = 1e-2


def to64(t):
    return t.detach().to("cpu").double().numpy() if isinstance(t, torch.Tensor) else np.asarray(t, np.float64)


def normwise(x, r):
    x, r = to64(x), to64(r)
    return float(np.abs(x - r).max() / max(np.abs(r).max(), 1e-300))


def rel_l2(x, r):
    x, r = to64(x), to64(r)
    return float(np.linalg.norm((x - r).ravel()) / max(np.linalg.norm(r.ravel()), 1e-300))


def within(x, r, dtype):
    """(ok, err) under the tolerance of the input dtype."""
    if dtype == torch.float32:
        e = normwise(x, r)
        return e <= TOL_F32, e
    e = rel_l2(x, r)
    return e <= TOL_BF16, e


def oracle_gammas(H):
    return orc.gammas(H)


def oracle_slices(Q, K, V, pairs, gamma, rotate, theta_base=10000.0, pos_offset=0,
                  state_in=None):
    """Recurrent-form oracle on the (b, h) slices in ``pairs``; returns
    (O [n, L, dv], S [n, dk, dv]) in fp64.  Inputs are host or device
    tensors; only the sampled slices are copied to the host."""
    q = np.stack([to64(Q[b, h]) for b, h in pairs])[None]
    k = np.stack([to64(K[b, h]) for b, h in pairs])[None]
    v = np.stack([to64(V[b, h]) for b, h in pairs])[None]
    g = np.array([gamma[h] for _, h in pairs])
    s0 = None
    if state_in is not None:
        s0 = np.stack([to64(state_in[b, h]) for b, h in pairs])[None]
    O, S = orc.recurrent(q, k, v, g, rotate=rotate, theta_base=theta_base,
                         pos_offset=pos_offset, state_in=s0)
    return O[0], S[0]


def oracle_gate_slices(O_sl, G, pairs, eps=1e-5):
    """Y of the sampled slices: O_sl [n, L, dv] (oracle), G [B, L, H*dv]."""
    n, L, dv = O_sl.shape
    g = np.concatenate([to64(G[b, :, h * dv:(h + 1) * dv]) for b, h in pairs], axis=-1)
    return orc.gate_groupnorm(O_sl[None], g[None], eps)[0].reshape(L, n, dv).transpose(1, 0, 2)


def y_slices(Y, pairs, dv):
    return np.stack([to64(Y[b, :, h * dv:(h + 1) * dv]) for b, h in pairs])
