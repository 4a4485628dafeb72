"""The seeded input generators that the oracle, the parity tests and the
benchmark share: reproducible per tag, independent across tags, able to
regenerate one expert or one head slab alone, and drawing the stated
distributions (bf16 N(0,1) hidden states, fp32 N(0,0.02) router, N(0,2^2)
skew bias, bf16 N(0,0.02) expert and head weights).  CPU only."""
import math

import torch

from moe_decode_gemv_b200 import inputs as I


def test_same_seed_and_tag_give_the_same_bits():
    a = I.hidden_states(3, 4, 256, tag="t")
    b = I.hidden_states(3, 4, 256, tag="t")
    assert a.dtype == torch.bfloat16 and a.shape == (4, 256)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_tags_and_seeds_give_independent_streams():
    base = I.hidden_states(0, 1, 4096, tag="a").float()
    for other in (I.hidden_states(0, 1, 4096, tag="b"), I.hidden_states(1, 1, 4096, tag="a")):
        o = other.float()
        assert not torch.equal(base, o)
        # independent N(0,1) draws: the sample correlation is O(1/sqrt(n))
        r = torch.corrcoef(torch.stack([base[0], o[0]]))[0, 1].item()
        assert abs(r) < 0.06
    assert I.derive_seed(0, "x") != I.derive_seed(0, "y") and 0 <= I.derive_seed(7, "x") < 2 ** 63


def test_one_expert_regenerates_alone():
    s = I.TINY_MOE
    bank = I.expert_bank(5, s, "down")
    assert bank.shape == (s.experts, s.hidden, s.inter)
    e = I.expert_matrix(5, s, 11, "down")
    assert torch.equal(bank[11].view(torch.int16), e.view(torch.int16))
    sub = I.expert_bank(5, s, "gate", experts=[3, 9])
    assert torch.equal(sub[1].view(torch.int16), I.expert_matrix(5, s, 9, "gate").view(torch.int16))
    # layers and the shared expert draw their own weights
    assert not torch.equal(I.expert_matrix(5, s, 11, "down", layer=1), e)
    assert not torch.equal(I.expert_matrix(5, s, "shared", "down"), e)


def test_head_slabs_regenerate_alone():
    shape = I.HeadShape(vocab=3000, hidden=64)
    w = I.lmhead_weight(2, shape, rows_per_draw=1024)
    assert w.shape == (3000, 64) and w.dtype == torch.bfloat16
    slab = I.normal(2, "lmhead/2048", (3000 - 2048, 64), I.WEIGHT_STD)
    assert torch.equal(w[2048:].view(torch.int16), slab.view(torch.int16))


def _close(x: float, want: float, tol: float) -> bool:
    return abs(x - want) <= tol


def test_distributions_match_the_recipe():
    n = 1 << 16
    x = I.hidden_states(0, 1, n).double()
    assert _close(x.mean().item(), 0.0, 5 / math.sqrt(n)) and _close(x.std().item(), 1.0, 0.02)
    r = I.router_weight(0, 64, 1024)
    assert r.dtype == torch.float32
    assert _close(r.double().std().item(), 0.02, 0.02 * 0.02)
    b = I.router_bias(0, 4096)
    assert b.dtype == torch.float32 and _close(b.double().std().item(), 2.0, 0.1)
    w = I.expert_matrix(0, I.TINY_MOE, 0, "up").double()
    assert w.shape == (64, 256) and _close(w.std().item(), 0.02, 0.02 * 0.03)
    # a bf16 draw is the fp32 draw of the same tag, rounded to bf16
    f = I.normal(9, "probe", (4096,), I.WEIGHT_STD, dtype=torch.float32)
    h = I.normal(9, "probe", (4096,), I.WEIGHT_STD)
    assert torch.equal(h, f.to(torch.bfloat16))
