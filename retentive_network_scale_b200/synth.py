"""Seeded synthetic inputs for retention workloads.

This module only draws random numbers and names workload shapes.  It holds
none of the retention arithmetic (no decay, rotation or normalisation), so
both the CUDA path and the CPU oracle may use it.

Recipe: fp32 standard normals from a ``torch.Generator`` seeded with
``seed``, drawn in the order Q, K, V, G, each scaled by its standard
deviation and then rounded once to the workload dtype (round-to-nearest-even
for bf16).  Both sides see the same rounded values.  Workloads too large to
draw on the host are drawn on the device with a device generator; the values
then differ from a host draw of the same seed but are identical from run to
run.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    """One retention workload: shapes, dtypes and input distributions."""
    name: str
    B: int
    H: int
    L: int
    d_k: int
    d_v: int
    chunk: int
    dtype: torch.dtype          # dtype of Q, K, V (and G)
    rotate: bool                # xPos rotation on/off
    std_qk: float               # standard deviation of Q and K entries
    std_v: float                # standard deviation of V entries
    gate: bool = False          # G present (GroupNorm + swish gate epilogue)
    std_g: float = 1.0
    seed: int = 20260
    decode_steps: int = 0       # recurrent steps after an L-token prefill
    theta_base: float = 10000.0
    notes: str = field(default="", compare=False)

    @property
    def tokens(self) -> int:
        return self.B * self.L


def _w(name, **kw) -> Workload:
    return Workload(name=name, **kw)


# The five workloads the pages' problem statement is measured on.  Index i
# uses seed 20260 + i.
WORKLOADS = {
    "tiny_fp32": _w("tiny_fp32", B=1, H=2, L=64, d_k=16, d_v=16, chunk=16,
                    dtype=torch.float32, rotate=True, std_qk=1 / math.sqrt(16),
                    std_v=1 / math.sqrt(16), seed=20260),
    "msr_small": _w("msr_small", B=4, H=8, L=2048, d_k=64, d_v=64, chunk=64,
                    dtype=torch.bfloat16, rotate=False, std_qk=1 / 8.0, std_v=1 / 8.0,
                    gate=True, std_g=1.0, seed=20261),
    "msr_1p3b": _w("msr_1p3b", B=8, H=8, L=4096, d_k=256, d_v=512, chunk=128,
                   dtype=torch.bfloat16, rotate=True, std_qk=1 / 16.0, std_v=1.0,
                   gate=True, std_g=1.0, seed=20262),
    "decode": _w("decode", B=64, H=16, L=8192, d_k=256, d_v=512, chunk=128,
                 dtype=torch.bfloat16, rotate=False, std_qk=1 / 16.0, std_v=1 / 16.0,
                 decode_steps=256, seed=20263),
    "long_ctx": _w("long_ctx", B=1, H=16, L=65536, d_k=128, d_v=256, chunk=256,
                   dtype=torch.bfloat16, rotate=True, std_qk=1 / math.sqrt(128),
                   std_v=1 / math.sqrt(128), seed=20264),
}


def _draw(gen, shape, std, dtype, device):
    x = torch.randn(shape, generator=gen, dtype=torch.float32, device=device)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def make_inputs(w: Workload, device="cpu", gen_device=None, L=None, B=None, shard=0):
    """Draw Q, K, V (and G) for workload ``w``.

    Returns a dict with ``Q``, ``K`` ``[B,H,L,d_k]``, ``V`` ``[B,H,L,d_v]``
    and, when the workload has a gate, ``G`` ``[B,L,H*d_v]``.  ``L``/``B``
    override the workload's sizes (same recipe, smaller draw).  ``shard``
    selects an independent draw of the same recipe (one per data-parallel
    replica); shard 0 is the workload's own draw.
    """
    B = w.B if B is None else B
    L = w.L if L is None else L
    gen_device = device if gen_device is None else gen_device
    gen = torch.Generator(device=gen_device)
    gen.manual_seed(shard_seed(w.seed, shard))
    out = {
        "Q": _draw(gen, (B, w.H, L, w.d_k), w.std_qk, w.dtype, gen_device),
        "K": _draw(gen, (B, w.H, L, w.d_k), w.std_qk, w.dtype, gen_device),
        "V": _draw(gen, (B, w.H, L, w.d_v), w.std_v, w.dtype, gen_device),
    }
    if w.gate:
        out["G"] = _draw(gen, (B, L, w.H * w.d_v), w.std_g, w.dtype, gen_device)
    return {k: v.to(device) for k, v in out.items()}


def shard_seed(seed: int, shard: int) -> int:
    """Seed of data-parallel shard ``shard`` of a workload seeded ``seed``
    (shard 0 keeps the workload's own seed)."""
    if shard < 0:
        raise ValueError("shard must be >= 0")
    return seed + 1_000_003 * shard


def make_decode_inputs(w: Workload, steps=None, device="cpu", gen_device=None, B=None):
    """Per-step q, k ``[steps,B,H,d_k]`` and v ``[steps,B,H,d_v]``."""
    steps = w.decode_steps if steps is None else steps
    B = w.B if B is None else B
    gen_device = device if gen_device is None else gen_device
    gen = torch.Generator(device=gen_device)
    gen.manual_seed(w.seed * 7919 + 1)
    out = {
        "q": _draw(gen, (steps, B, w.H, w.d_k), w.std_qk, w.dtype, gen_device),
        "k": _draw(gen, (steps, B, w.H, w.d_k), w.std_qk, w.dtype, gen_device),
        "v": _draw(gen, (steps, B, w.H, w.d_v), w.std_v, w.dtype, gen_device),
    }
    return {k: v.to(device) for k, v in out.items()}


def random_tensor(shape, seed, std=1.0, dtype=torch.float32, device="cpu"):
    """A standalone seeded draw (edge-case tests)."""
    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    return _draw(gen, shape, std, dtype, device)
