"""Seeded synthetic inputs shared by the tests, the benchmark and the smoke check.

This module draws random tensors and nothing else: it holds none of the
attention arithmetic, so the GPU path and the CPU oracle can both be fed from
it without sharing any of the method's code.

Recipe (the same for every workload): a ``torch.Generator`` on the target
device seeded with the workload's seed draws float32 standard normals with
``torch.randn`` in the order Q, K, V, dO, each of shape [B, H, N, D].  Q, K
and V are multiplied by 1/sqrt(D) unless the workload says ``scaled=False``;
dO is never scaled.  The float32 values are then cast to the workload dtype.
Decode inputs continue with their own generator (seed + 1000) and draw q, k,
v of shape [steps, B, H, D] in that order, scaled by 1/sqrt(D).

The shapes are the head sizes and sequence lengths the linear-attention pages
discuss (heads of D = 64-128, sequences from 2K to 128K tokens, and the layer
shape of a 1.4B-parameter language model: width 2048 = 16 heads x 128).
"""
from __future__ import annotations

import dataclasses
import math

import torch

PHI_ELU1 = 0
PHI_RELU_EPS = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    H: int
    N: int
    D: int
    dtype: torch.dtype
    causal: bool
    phi: int
    seed: int
    scaled: bool = True
    backward: bool = False

    @property
    def tokens(self) -> int:
        return self.B * self.N


WORKLOADS = {
    # small fp32 case: causal forward, unscaled N(0,1) inputs
    "causal_fwd_b1h1n256d32_f32": Workload(
        "causal_fwd_b1h1n256d32_f32", 1, 1, 256, 32, torch.float32, True, PHI_ELU1, 0,
        scaled=False),
    # short-sequence forward, both modes
    "fwd_b4h8n2048d64_bf16": Workload(
        "fwd_b4h8n2048d64_bf16", 4, 8, 2048, 64, torch.bfloat16, True, PHI_ELU1, 1),
    "ncfwd_b4h8n2048d64_bf16": Workload(
        "ncfwd_b4h8n2048d64_bf16", 4, 8, 2048, 64, torch.bfloat16, False, PHI_ELU1, 1),
    # the timed training step: causal forward + backward, 8K tokens, D = 64
    "causal_fwdbwd_b8h16n8192d64_bf16": Workload(
        "causal_fwdbwd_b8h16n8192d64_bf16", 8, 16, 8192, 64, torch.bfloat16, True, PHI_ELU1,
        2, backward=True),
    # 1.4B-parameter LM layer shape (width 2048 = 16 heads x 128), both maps
    "causal_fwdbwd_b4h16n4096d128_relu_bf16": Workload(
        "causal_fwdbwd_b4h16n4096d128_relu_bf16", 4, 16, 4096, 128, torch.bfloat16, True,
        PHI_RELU_EPS, 3, backward=True),
    "causal_fwdbwd_b4h16n4096d128_elu_bf16": Workload(
        "causal_fwdbwd_b4h16n4096d128_elu_bf16", 4, 16, 4096, 128, torch.bfloat16, True,
        PHI_ELU1, 3, backward=True),
    # long context forward
    "causal_fwd_b1h32n131072d128_bf16": Workload(
        "causal_fwd_b1h32n131072d128_bf16", 1, 32, 131072, 128, torch.bfloat16, True,
        PHI_ELU1, 4),
}

# decayed (gated) training step on the timed shape: one decay factor per
# head, gamma_h = 1 - 2^-(5 + 7 h / (H - 1)) (0.969 ... 0.99976), the fixed
# per-head decays of retention-style linear attention
DECAY_TRAIN = Workload("decay_causal_fwdbwd_b8h16n8192d64_bf16", 8, 16, 8192, 64, torch.bfloat16,
                       True, PHI_ELU1, 6, backward=True)


def decay_factors(H: int) -> list:
    """Per-head decay factors 1 - 2^-(5 + 7 h / (H - 1)), h = 0..H-1."""
    return [1.0 - 2.0 ** -(5.0 + 7.0 * h / max(H - 1, 1)) for h in range(H)]


# recurrent decode: batch 256, 32 heads of 128, fp32 state updated in place
DECODE = dict(B=256, H=32, D=128, steps=1024, seed=4, dtype=torch.bfloat16, phi=PHI_ELU1)
# the same decode with grouped-query attention: 8 key/value heads, each
# shared by 4 query heads (the state is 4x smaller)
DECODE_GQA = dict(B=256, H=32, Hkv=8, D=128, steps=1024, seed=5, dtype=torch.bfloat16,
                  phi=PHI_ELU1)


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_inputs(w: Workload, device="cpu", with_grad_out: bool | None = None):
    """Q, K, V (and dO when the workload has a backward) for workload ``w``."""
    if with_grad_out is None:
        with_grad_out = w.backward
    return make_tensors(w.B, w.H, w.N, w.D, w.dtype, w.seed, device=device,
                        scaled=w.scaled, with_grad_out=with_grad_out)


def make_tensors(B, H, N, D, dtype, seed, device="cpu", scaled=True, with_grad_out=False):
    g = _gen(device, seed)
    shape = (B, H, N, D)
    scale = 1.0 / math.sqrt(D) if scaled else 1.0
    out = []
    names = ["q", "k", "v"] + (["dO"] if with_grad_out else [])
    for name in names:
        t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if name != "dO" and scale != 1.0:
            t.mul_(scale)
        out.append(t.to(dtype).contiguous())
    return tuple(out)


def make_gqa_tensors(B, H, Hkv, N, D, dtype, seed, device="cpu", with_grad_out=False):
    """Grouped key/value heads: q [B, H, N, D], k, v [B, Hkv, N, D] (and dO
    [B, H, N, D]), drawn in that order from one generator seeded with
    ``seed``; q, k, v scaled by 1/sqrt(D), dO not; then cast to ``dtype``."""
    g = _gen(device, seed)
    scale = 1.0 / math.sqrt(D)
    shapes = [(B, H, N, D), (B, Hkv, N, D), (B, Hkv, N, D)] + (
        [(B, H, N, D)] if with_grad_out else [])
    out = []
    for i, shape in enumerate(shapes):
        t = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
        if i < 3:
            t.mul_(scale)
        out.append(t.to(dtype).contiguous())
    return tuple(out)


def make_decode_gqa_inputs(B, H, Hkv, D, steps, seed, dtype=torch.bfloat16, device="cpu"):
    """q [steps, B, H, D] and k, v [steps, B, Hkv, D] for grouped decode
    steps (generator seed + 1000, scaled by 1/sqrt(D))."""
    g = _gen(device, seed + 1000)
    scale = 1.0 / math.sqrt(D)
    out = []
    for heads in (H, Hkv, Hkv):
        t = torch.randn((steps, B, heads, D), generator=g, device=device, dtype=torch.float32)
        out.append(t.mul_(scale).to(dtype).contiguous())
    return tuple(out)


def make_favor_directions(m, D, seed, dtype=torch.bfloat16, device="cpu"):
    """The Performer's random directions omega [m, D]: independent N(0, 1)
    entries (generator seed + 2000), cast to ``dtype``."""
    g = _gen(device, seed + 2000)
    return torch.randn((m, D), generator=g, device=device, dtype=torch.float32).to(dtype)


def make_decode_inputs(B, H, D, steps, seed, dtype=torch.bfloat16, device="cpu"):
    """q, k, v of shape [steps, B, H, D] for ``steps`` recurrent decode steps."""
    g = _gen(device, seed + 1000)
    scale = 1.0 / math.sqrt(D)
    out = []
    for _ in range(3):
        t = torch.randn((steps, B, H, D), generator=g, device=device, dtype=torch.float32)
        out.append(t.mul_(scale).to(dtype).contiguous())
    return tuple(out)
