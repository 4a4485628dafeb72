"""Algorithmic byte counts of the decode hot path (the roofline numerators).

Only bytes the method must move count: the router matrix, each distinct
selected expert once per step plus the shared expert (packed E2M1 codes and
their E8M0 scales), and the whole FP8 LM head with its fp32 row scales.
Activations (a few KB per token) are left out.  Never the 512-expert total,
never a dense equivalent.
"""
from __future__ import annotations

from .inputs import HeadShape, MoEShape


def mxfp4_row_bytes(K: int) -> int:
    """One MXFP4 row of K elements: K/2 bytes of E2M1 codes + K/32 E8M0 scales."""
    assert K % 32 == 0
    return K // 2 + K // 32


def expert_bytes(s: MoEShape) -> int:
    """gate [I,H] + up [I,H] + down [H,I], all MXFP4."""
    return 2 * s.inter * mxfp4_row_bytes(s.hidden) + s.hidden * mxfp4_row_bytes(s.inter)


def router_bytes(s: MoEShape) -> int:
    """fp32 router matrix [E, H]."""
    return 4 * s.experts * s.hidden


def moe_layer_bytes(s: MoEShape, distinct_routed: int) -> int:
    """Router + every distinct routed expert the step selects + the shared expert."""
    return router_bytes(s) + (distinct_routed + 1) * expert_bytes(s)


def lmhead_fp8_bytes(h: HeadShape) -> int:
    """E4M3 [V, H] + fp32 row scales [V]."""
    return h.vocab * h.hidden + 4 * h.vocab


def lmhead_bf16_bytes(h: HeadShape) -> int:
    return 2 * h.vocab * h.hidden


def moe_layer_flops(s: MoEShape, token_expert_pairs: int, M: int) -> int:
    """Multiply-adds x 2: router for M tokens, plus one expert MLP per
    (token, expert) pair, shared expert included in the count of pairs."""
    per_expert = 2 * (2 * s.inter * s.hidden + s.hidden * s.inter)
    return 2 * M * s.experts * s.hidden + token_expert_pairs * per_expert
