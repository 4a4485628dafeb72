"""Seeded synthetic inputs for the decode hot path.

This module only draws random numbers.  It holds none of the method's
arithmetic (no quantisation, routing or GEMV): the tests, the benchmark and the
CPU oracle all take their inputs from here, and each side then quantises and
computes on its own.

Every tensor comes from its own ``torch.Generator`` whose seed is a hash of the
run seed and a tag naming the tensor (``"L0/e17/gate"``, ``"x/3"``...).  So one
expert of one layer can be drawn alone, and the oracle can regenerate only the
experts a token selects, bit for bit, without drawing the other 511.

Recipe (the shapes and value distributions of the workload the pages time:
batch-1 decode of a Ling-shaped MoE with hidden 2,560, 512 routed experts of
intermediate 768, top-8, one shared expert, and a 157,184 x 2,560 LM head):

- hidden states: bf16, N(0, 1);
- router weight: fp32, N(0, 0.02), kept in fp32;
- skewed router regime: a per-expert fp32 logit bias drawn from N(0, 2^2);
- expert weights (gate, up: [I, H]; down: [H, I]): N(0, 0.02) rounded to
  bf16, as a bf16 checkpoint would hold them before MXFP4 quantisation;
- LM head: bf16 [V, H], N(0, 0.02); embedding table: bf16 [V, H], N(0, 1).

On a CPU generator the draws are reproducible across runs and machines with
the same torch build.  Draws on a CUDA generator are faster but differ from
the CPU ones; only timing runs use them.
"""
from __future__ import annotations

import hashlib
from dataclasses import dataclass

import torch

WEIGHT_STD = 0.02
HIDDEN_STD = 1.0
SKEW_BIAS_STD = 2.0


@dataclass(frozen=True)
class MoEShape:
    """Shapes of one MoE layer: hidden H, expert intermediate I, routed
    experts E, experts per token k (plus one shared expert of width I)."""
    hidden: int
    inter: int
    experts: int
    top_k: int


@dataclass(frozen=True)
class HeadShape:
    vocab: int
    hidden: int


# The small case the oracle finishes in seconds, and the Ling-shaped case.
TINY_MOE = MoEShape(hidden=256, inter=64, experts=16, top_k=2)
LING_MOE = MoEShape(hidden=2560, inter=768, experts=512, top_k=8)
TINY_HEAD = HeadShape(vocab=4096, hidden=256)
LING_HEAD = HeadShape(vocab=157184, hidden=2560)


def derive_seed(seed: int, tag: str) -> int:
    h = hashlib.sha256(f"{int(seed)}/{tag}".encode()).digest()
    return int.from_bytes(h[:8], "little") & ((1 << 63) - 1)


def _gen(seed: int, tag: str, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(derive_seed(seed, tag))
    return g


def normal(seed: int, tag: str, shape, std: float, dtype=torch.bfloat16, device="cpu") -> torch.Tensor:
    """N(0, std^2) drawn in fp32, scaled, then cast to ``dtype`` (RNE for bf16)."""
    g = _gen(seed, tag, device)
    t = torch.randn(tuple(shape), generator=g, dtype=torch.float32, device=device)
    if std != 1.0:
        t.mul_(std)
    return t if dtype == torch.float32 else t.to(dtype)


def hidden_states(seed: int, M: int, H: int, tag: str = "x", device="cpu") -> torch.Tensor:
    return normal(seed, f"hidden/{tag}", (M, H), HIDDEN_STD, device=device)


def router_weight(seed: int, E: int, H: int, layer: int = 0, device="cpu") -> torch.Tensor:
    return normal(seed, f"L{layer}/router", (E, H), WEIGHT_STD, dtype=torch.float32, device=device)


def router_bias(seed: int, E: int, layer: int = 0, device="cpu") -> torch.Tensor:
    return normal(seed, f"L{layer}/router_bias", (E,), SKEW_BIAS_STD, dtype=torch.float32, device=device)


def expert_matrix(seed: int, shape: MoEShape, expert, which: str, layer: int = 0, device="cpu") -> torch.Tensor:
    """bf16 weights of one expert matrix.  ``expert`` is an int or "shared";
    ``which`` is "gate", "up" ([I, H]) or "down" ([H, I])."""
    rows, cols = (shape.inter, shape.hidden) if which in ("gate", "up") else (shape.hidden, shape.inter)
    return normal(seed, f"L{layer}/e{expert}/{which}", (rows, cols), WEIGHT_STD, device=device)


def expert_bank(seed: int, shape: MoEShape, which: str, layer: int = 0, experts=None, device="cpu") -> torch.Tensor:
    """Stack of one matrix kind over experts: [len(experts), rows, cols] bf16."""
    ids = range(shape.experts) if experts is None else experts
    return torch.stack([expert_matrix(seed, shape, e, which, layer, device) for e in ids])


def lmhead_weight(seed: int, shape: HeadShape, device="cpu", rows_per_draw: int = 8192) -> torch.Tensor:
    """bf16 [V, H], drawn in row slabs so any slab can be regenerated alone."""
    out = torch.empty((shape.vocab, shape.hidden), dtype=torch.bfloat16, device=device)
    for r0 in range(0, shape.vocab, rows_per_draw):
        r1 = min(shape.vocab, r0 + rows_per_draw)
        out[r0:r1] = normal(seed, f"lmhead/{r0}", (r1 - r0, shape.hidden), WEIGHT_STD, device=device)
    return out


def embedding_table(seed: int, shape: HeadShape, device="cpu", rows_per_draw: int = 8192) -> torch.Tensor:
    out = torch.empty((shape.vocab, shape.hidden), dtype=torch.bfloat16, device=device)
    for r0 in range(0, shape.vocab, rows_per_draw):
        r1 = min(shape.vocab, r0 + rows_per_draw)
        out[r0:r1] = normal(seed, f"embed/{r0}", (r1 - r0, shape.hidden), HIDDEN_STD, device=device)
    return out
