"""GPU parity of the MoE layer (router GEMV + top-k softmax routing, MXFP4
gate/up GEMV + SiLU, down GEMV, shared expert, combine) at M = 1 and at the
M = 4 verify step, against the fp64 CPU oracle on the same quantised bytes.

Routing reading: softmax over the routed logits, top-k, renormalised; 8 of
512 routed experts plus one shared expert (saipien.org essay, "Why one user
waits on weights"); four verify positions wake up to 32 experts (same essay,
"Draft three tokens, verify four")."""
import numpy as np
import pytest
import torch

import oracle
from gpu_support import Layer, check_moe, u16
from moe_decode_gemv_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from moe_decode_gemv_b200 import build
    build.build()
    from moe_decode_gemv_b200 import binding
    return binding


@pytest.fixture(scope="module")
def O():
    return oracle.load()


@pytest.fixture(scope="module")
def tiny(B):
    return Layer(B, 0, I.TINY_MOE)


@pytest.fixture(scope="module")
def tiny_skewed(B):
    return Layer(B, 1, I.TINY_MOE, skewed=True)


def test_tiny_bank_matches_oracle_quantisation(B, O, tiny):
    for kind, bank in zip(Layer.KINDS, tiny.bank):
        for e in (0, 7, 15):
            d, s = O.mxfp4_quantize(u16(I.expert_matrix(0, I.TINY_MOE, e, kind)))
            assert np.array_equal(bank.data[e].cpu().numpy(), d) and np.array_equal(bank.scales[e].cpu().numpy(), s)


@pytest.mark.parametrize("M", [1, 2, 3, 4])
def test_tiny_layer(B, O, tiny, M):
    for seed in range(5):
        x = I.hidden_states(seed, M, I.TINY_MOE.hidden, tag=f"moe{M}")
        y, ids, w = tiny.run_gpu(x.cuda())
        rep = check_moe(tiny, O, x, y, ids, w)
        assert rep["skipped_tokens"] == 0, rep


@pytest.mark.parametrize("M", [1, 4])
def test_tiny_layer_skewed(B, O, tiny_skewed, M):
    for seed in range(5):
        x = I.hidden_states(seed, M, I.TINY_MOE.hidden, tag=f"skew{M}")
        y, ids, w = tiny_skewed.run_gpu(x.cuda())
        check_moe(tiny_skewed, O, x, y, ids, w)


def test_identical_tokens_share_experts(B, O, tiny):
    """Four copies of one token: the union holds top_k experts, each streamed
    once, and every token's output equals the single-token output."""
    x1 = I.hidden_states(9, 1, I.TINY_MOE.hidden)
    y1, ids1, w1 = tiny.run_gpu(x1.cuda())
    x4 = x1.repeat(4, 1)
    y4, ids4, w4 = tiny.run_gpu(x4.cuda())
    for m in range(4):
        assert np.array_equal(ids4[m], ids1[0]) and np.array_equal(w4[m], w1[0])
        assert np.array_equal(y4[m], y1[0])
    check_moe(tiny, O, x4, y4, ids4, w4)


def test_degenerate_router_ties(B, O):
    """A zero router makes every logit 0: experts 0..k-1 win (lower id first)
    with equal weights 1/k."""
    layer = Layer(B, 2, I.TINY_MOE)
    layer.router_w = torch.zeros_like(layer.router_w)
    layer.router_w_dev = layer.router_w.cuda()
    x = I.hidden_states(2, 4, I.TINY_MOE.hidden)
    y, ids, w = layer.run_gpu(x.cuda())
    assert (ids == np.arange(I.TINY_MOE.top_k)).all() and np.allclose(w, 1.0 / I.TINY_MOE.top_k)
    check_moe(layer, O, x, y, ids, w)


def test_every_expert_selected_and_top1(B, O):
    """E = top_k = 8 (all experts active) and top_k = 1."""
    s8 = I.MoEShape(hidden=256, inter=64, experts=8, top_k=8)
    layer = Layer(B, 4, s8)
    x = I.hidden_states(4, 4, 256)
    y, ids, w = layer.run_gpu(x.cuda())
    check_moe(layer, O, x, y, ids, w)
    s1 = I.MoEShape(hidden=256, inter=64, experts=16, top_k=1)
    layer = Layer(B, 5, s1)
    x = I.hidden_states(5, 2, 256)
    y, ids, w = layer.run_gpu(x.cuda())
    assert np.allclose(w, 1.0)
    check_moe(layer, O, x, y, ids, w)


@pytest.mark.parametrize("H,Inter,E,k,M", [(192, 192, 24, 3, 3), (96, 32, 5, 2, 4), (32, 96, 9, 8, 2)])
def test_odd_sizes(B, O, H, Inter, E, k, M):
    """H and I multiples of 32 that are not powers of two (down to one K block
    and one pair of 16-row slices), E not a multiple of the CTA count."""
    s = I.MoEShape(hidden=H, inter=Inter, experts=E, top_k=k)
    layer = Layer(B, 6, s)
    x = I.hidden_states(6, M, H)
    y, ids, w = layer.run_gpu(x.cuda())
    check_moe(layer, O, x, y, ids, w)


def test_repeat_calls_deterministic(B, tiny):
    x = I.hidden_states(8, 4, I.TINY_MOE.hidden).cuda()
    ws = B.new_workspace(B.moe_workspace_bytes(4, 2, 16, 256, 64))
    runs = [tiny.run_gpu(x, workspace=ws) for _ in range(3)]
    assert B.moe_workspace_status(ws) == B.Status.OK
    for r in runs[1:]:
        for a, b in zip(r, runs[0]):
            assert np.array_equal(a, b)


@pytest.fixture(scope="module")
def ling(B):
    return Layer(B, 0, I.LING_MOE)


@pytest.fixture(scope="module")
def ling_skewed(B):
    return Layer(B, 1, I.LING_MOE, skewed=True)


@pytest.mark.parametrize("M", [1, 4])
def test_ling_layer(B, O, ling, M):
    """The Ling-shaped layer (512 experts, top-8, intermediate 768, hidden
    2560) in the launch configuration the benchmark times."""
    for seed in range(2):
        x = I.hidden_states(seed, M, I.LING_MOE.hidden, tag=f"ling{M}")
        y, ids, w = ling.run_gpu(x.cuda())
        rep = check_moe(ling, O, x, y, ids, w)
        print(f"ling layer M={M} seed={seed}: rel-L2 {rep['rel_l2']:.2e}, max-abs {rep['max_abs']:.2e}")
        assert rep["skipped_tokens"] == 0, rep
        if M == 4:
            assert len(set(ids.reshape(-1).tolist())) <= 32


@pytest.mark.parametrize("M", [1, 4])
def test_ling_layer_back_to_back_calls_identical(B, ling, M):
    """24 calls of the Ling layer queued back to back on one stream, sharing
    one workspace (each call's CTAs start as the previous call's leave): every
    call's output, ids and weights bit-identical to the first."""
    k, H = ling.shape.top_k, ling.shape.hidden
    x = I.hidden_states(6, M, H, tag="back2back").cuda()
    ws = B.new_workspace(B.moe_workspace_bytes(M, k, ling.shape.experts, H, ling.shape.inter))
    outs = [(torch.full((M, H), float("nan"), dtype=torch.float32, device="cuda"),
             torch.empty((M, k), dtype=torch.int32, device="cuda"), torch.empty((M, k), dtype=torch.float32, device="cuda"))
            for _ in range(24)]
    for y, ids, w in outs:
        B.moe_decode(x, ling.router_w_dev, ling.router_bias_dev, ling.packed, ling.packed_shared, k, y, ids, w,
                     workspace=ws)
    torch.cuda.synchronize()
    assert B.moe_workspace_status(ws) == B.Status.OK
    first = [t.cpu().numpy() for t in outs[0]]
    assert np.isfinite(first[0]).all()
    for c, o in enumerate(outs[1:], 1):
        for a, b in zip(o, first):
            assert np.array_equal(a.cpu().numpy(), b), f"call {c} differs"


def test_ling_layer_skewed_m4(B, O, ling_skewed):
    """Skewed router (per-expert logit bias N(0, 2^2)): tokens share experts."""
    x = I.hidden_states(0, 4, I.LING_MOE.hidden, tag="skew")
    y, ids, w = ling_skewed.run_gpu(x.cuda())
    check_moe(ling_skewed, O, x, y, ids, w)
    assert len(set(ids.reshape(-1).tolist())) < 32


# ---------------------------------------------------------------------------
# Inputs that stress the GPU path's own number handling: activations are
# carried as E4M3 parts per 32-element block (x) and as f16 parts per
# 16-value slice (h), and E8M0 scales are decoded by exponent placement.
# The bar is the same as everywhere: rel-L2 <= 2e-3, max-abs <= 1e-2 against
# the fp64 oracle on the same quantised bytes, ids exact outside the margin.
# ---------------------------------------------------------------------------

def outlier_tokens(M, H, seed=0):
    """Token 0: one element at 1e3, the rest 1e-3 N(0, 1); token 1: N(0, 1);
    token 2: one element at -1e3 among 1e-3 N(0, 1); token 3: 8 N(0, 1)."""
    base = I.hidden_states(seed, 4, H, tag="outlier").float()
    x = torch.empty((4, H))
    x[0] = base[0] * 1e-3
    x[0, 1234 % H] = 1e3
    x[1] = base[1]
    x[2] = base[2] * 1e-3
    x[2, 77 % H] = -1e3
    x[3] = base[3] * 8
    return x[:M].to(torch.bfloat16)


@pytest.mark.parametrize("M", [1, 4])
def test_ling_layer_outlier_tokens(B, O, ling, M):
    """A token with one 1e3 element among 1e-3 values: the block holding the
    outlier spans 2^20, the other blocks are tiny."""
    x = outlier_tokens(M, I.LING_MOE.hidden)
    y, ids, w = ling.run_gpu(x.cuda())
    rep = check_moe(ling, O, x, y, ids, w)
    print(f"outlier tokens M={M}: rel-L2 {rep['rel_l2']:.2e}, max-abs {rep['max_abs']:.2e}, "
          f"|y|max {np.abs(y).max():.1f}")
    assert rep["skipped_tokens"] == 0, rep


LING_WIDTH = I.MoEShape(hidden=2560, inter=768, experts=64, top_k=8)


def test_ling_width_h_spans_2_20_per_slice(B, O):
    """Gate and up rows 16j of every expert scaled by 2^4, the other rows by
    2^-6: within each 16-row slice h spans about 2^20."""
    def wfn(kind, e, w):
        if kind == "down":
            return w
        f = torch.full((w.shape[0], 1), 2.0 ** -6)
        f[::16] = 2.0 ** 4
        return (w.float() * f).to(torch.bfloat16)

    layer = Layer(B, 12, LING_WIDTH, wfn=wfn)
    for M in (1, 3):
        x = I.hidden_states(12, M, LING_WIDTH.hidden, tag="hrange")
        y, ids, w = layer.run_gpu(x.cuda())
        rep = check_moe(layer, O, x, y, ids, w)
        print(f"h range M={M}: rel-L2 {rep['rel_l2']:.2e}, max-abs {rep['max_abs']:.2e}")
        assert rep["skipped_tokens"] == 0, rep


def test_ling_width_e8m0_extremes(B, O):
    """Every gate and up row's block 0 carries E8M0 code 254 (2^127) and block
    1 code 1 (2^-126); the activations' block 0 is bf16-subnormal (about
    2^-128) and block 1 about 2^118, so the products stay finite.  The router
    ignores block 1 (its columns are zero)."""
    def sfn(kind, sc):
        if kind != "down":
            sc = sc.copy()
            sc[..., 0] = 254
            sc[..., 1] = 1
        return sc

    layer = Layer(B, 13, LING_WIDTH, sfn=sfn)
    layer.router_w[:, 32:64] = 0.0
    layer.router_w_dev = layer.router_w.cuda()
    M = 2
    x = I.hidden_states(13, M, LING_WIDTH.hidden, tag="e8m0").float()
    x[:, :32] *= 2.0 ** -128
    x[:, 32:64] *= 2.0 ** 118
    x = x.to(torch.bfloat16)
    assert (x[:, :32].float().abs() < 2.0 ** -126).any()  # subnormal bf16 values are present
    y, ids, w = layer.run_gpu(x.cuda())
    assert np.isfinite(y).all()
    rep = check_moe(layer, O, x, y, ids, w)
    print(f"E8M0 extremes: rel-L2 {rep['rel_l2']:.2e}, max-abs {rep['max_abs']:.2e}, |y|max {np.abs(y).max():.1f}")
    assert rep["skipped_tokens"] == 0, rep
