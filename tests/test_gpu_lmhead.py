"""GPU parity of the FP8 LM head (GEMV + per-row scale + top-k) and of the
BF16 comparator head, against the fp64 CPU oracle on the same quantised
bytes.  Greedy argmax is top_k = 1; the sampled workload's top_k is 29
(ncijnetwork.com summary, "What happens on a real workload?")."""
import numpy as np
import pytest
import torch

import oracle
from gpu_support import check_head, run_head_gpu, u16
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


def _head(B, O, seed, shape):
    w = I.lmhead_weight(seed, shape)
    canon = B.lmhead_quantize_fp8(w.cuda(), tiled=False)
    q, s = O.fp8_rowquant(u16(w))
    torch.cuda.synchronize()
    assert np.array_equal(canon.q.cpu().numpy(), q)
    head = B.lmhead_tile_fp8(canon)
    return w, head, q, s


@pytest.fixture(scope="module")
def tiny(B, O):
    return _head(B, O, 0, I.TINY_HEAD)


@pytest.mark.parametrize("M", [1, 2, 4])
@pytest.mark.parametrize("k", [1, 29])
def test_tiny_head(B, O, tiny, M, k):
    w, head, q, s = tiny
    for seed in range(3):
        x = I.hidden_states(seed, M, I.TINY_HEAD.hidden, tag=f"head{M}")
        ids, vals, logits = run_head_gpu(B, head, x.cuda(), k)
        ref = O.lmhead_fp8(u16(x), q, s)
        check_head(ids, vals, logits, ref)
        # without the logits write the top-k is the same
        ids2, vals2, _ = run_head_gpu(B, head, x.cuda(), k, with_logits=False)
        assert np.array_equal(ids, ids2) and np.array_equal(vals, vals2)


def test_ragged_head(B, O):
    """V not a multiple of the 16-row tile, H = 320 (64 mod 128), top_k = 64."""
    shape = I.HeadShape(vocab=4099, hidden=320)
    w, head, q, s = _head(B, O, 7, shape)
    x = I.hidden_states(7, 3, 320)
    ids, vals, logits = run_head_gpu(B, head, x.cuda(), 64)
    check_head(ids, vals, logits, O.lmhead_fp8(u16(x), q, s))


def test_small_vocab_fewer_rows_than_ctas(B, O):
    shape = I.HeadShape(vocab=40, hidden=128)
    w, head, q, s = _head(B, O, 8, shape)
    x = I.hidden_states(8, 4, 128)
    ids, vals, logits = run_head_gpu(B, head, x.cuda(), 40)
    check_head(ids, vals, logits, O.lmhead_fp8(u16(x), q, s))


def test_degenerate_ties(B, O, tiny):
    """All-zero activations: every logit is exactly 0, so the top-k must be
    token ids 0..k-1 (ties go to the lower id)."""
    w, head, q, s = tiny
    x = torch.zeros((2, I.TINY_HEAD.hidden), dtype=torch.bfloat16)
    ids, vals, logits = run_head_gpu(B, head, x.cuda(), 29)
    assert (ids == np.arange(29)).all() and (vals == 0).all() and (logits == 0).all()
    # identical rows tie exactly; the lower id must win
    w2 = w.clone()
    w2[100] = w2[3000]
    h2 = B.lmhead_quantize_fp8(w2.cuda())
    x = I.hidden_states(1, 1, I.TINY_HEAD.hidden)
    ref = O.lmhead_fp8(u16(x), *O.fp8_rowquant(u16(w2)))
    top = int(np.argmax(ref[0]))
    w2[top + 1 if top < 4095 else top - 1] = w2[top]
    h3 = B.lmhead_quantize_fp8(w2.cuda())
    ids, vals, logits = run_head_gpu(B, h3, x.cuda(), 2)
    pair = sorted([top, top + 1 if top < 4095 else top - 1])
    assert ids[0].tolist() == pair, (ids, pair)
    assert vals[0, 0] == vals[0, 1]


def test_bf16_comparator_tiny(B, O, tiny):
    w, head, q, s = tiny
    x = I.hidden_states(11, 4, I.TINY_HEAD.hidden)
    ids, vals, logits = run_head_gpu(B, None, x.cuda(), 29, bf16_w=w.cuda())
    check_head(ids, vals, logits, O.lmhead_bf16(u16(x), u16(w)))


@pytest.fixture(scope="module")
def ling(B, O):
    return _head(B, O, 0, I.LING_HEAD)


@pytest.mark.parametrize("M,k", [(1, 1), (1, 29), (4, 29)])
def test_ling_head(B, O, ling, M, k):
    """The 157,184 x 2,560 head in the launch configuration the benchmark times."""
    w, head, q, s = ling
    x = I.hidden_states(0, M, I.LING_HEAD.hidden, tag="lmhead")
    ids, vals, logits = run_head_gpu(B, head, x.cuda(), k)
    ref = O.lmhead_fp8(u16(x), q, s)
    check_head(ids, vals, logits, ref)


def test_ling_bf16_comparator(B, O, ling):
    w, head, q, s = ling
    x = I.hidden_states(1, 1, I.LING_HEAD.hidden, tag="lmhead")
    ids, vals, logits = run_head_gpu(B, None, x.cuda(), 29, bf16_w=w.cuda())
    check_head(ids, vals, logits, O.lmhead_bf16(u16(x), u16(w)))


def test_repeat_calls_identical(B, tiny):
    w, head, q, s = tiny
    x = I.hidden_states(3, 4, I.TINY_HEAD.hidden).cuda()
    ws = B.new_workspace(B.lmhead_workspace_bytes(4, 29, 4096, 256))
    outs = []
    for _ in range(3):
        ids = torch.empty((4, 29), dtype=torch.int32, device="cuda")
        vals = torch.empty((4, 29), dtype=torch.float32, device="cuda")
        B.lmhead_decode(x, head, 29, ids, vals, None, workspace=ws)
        outs.append((ids.cpu().numpy(), vals.cpu().numpy()))
    assert B.moe_workspace_status(ws) == B.Status.OK
    for o in outs[1:]:
        assert np.array_equal(o[0], outs[0][0]) and np.array_equal(o[1], outs[0][1])


@pytest.mark.parametrize("M", [1, 4])
def test_ling_head_back_to_back_calls_identical(B, ling, M):
    """The full head, 24 calls queued back to back on one stream (each call's
    CTAs start as the previous call's leave): every call's logits and top-k
    bit-identical to the first.  A ring whose stages alternated between the
    two consumer groups once let a group compute the other group's tile and
    leave rows of the logits unwritten; this catches that class of race."""
    w, head, q, s = ling
    x = I.hidden_states(5, M, I.LING_HEAD.hidden, tag="lmhead").cuda()
    ws = B.new_workspace(B.lmhead_workspace_bytes(M, 29, I.LING_HEAD.vocab, I.LING_HEAD.hidden))
    outs = [(torch.empty((M, 29), dtype=torch.int32, device="cuda"), torch.empty((M, 29), dtype=torch.float32, device="cuda"),
             torch.full((M, I.LING_HEAD.vocab), float("nan"), dtype=torch.float32, device="cuda")) for _ in range(24)]
    for ids, vals, logits in outs:
        B.lmhead_decode(x, head, 29, ids, vals, logits, workspace=ws)
    torch.cuda.synchronize()
    assert B.moe_workspace_status(ws) == B.Status.OK
    ids0, vals0, lg0 = (t.cpu().numpy() for t in outs[0])
    assert np.isfinite(lg0).all()
    for c, (ids, vals, logits) in enumerate(outs[1:], 1):
        assert np.array_equal(ids.cpu().numpy(), ids0), f"call {c}: ids differ"
        assert np.array_equal(vals.cpu().numpy(), vals0), f"call {c}: values differ"
        assert np.array_equal(logits.cpu().numpy(), lg0), f"call {c}: logits differ"


@pytest.mark.parametrize("M", [1, 4])
def test_ling_head_outlier_tokens(B, O, ling, M):
    """A token with one element at 1e3 among 1e-3 values (and, at M = 4, a
    plain token, a negative outlier and a scaled token beside it)."""
    w, head, q, s = ling
    base = I.hidden_states(0, 4, I.LING_HEAD.hidden, tag="outlier").float()
    x = torch.empty((4, I.LING_HEAD.hidden))
    x[0] = base[0] * 1e-3
    x[0, 1234] = 1e3
    x[1] = base[1]
    x[2] = base[2] * 1e-3
    x[2, 77] = -1e3
    x[3] = base[3] * 8
    x = x[:M].to(torch.bfloat16)
    ids, vals, logits = run_head_gpu(B, head, x.cuda(), 29)
    ref = O.lmhead_fp8(u16(x), q, s)
    near = check_head(ids, vals, logits, ref)
    err = max(float(np.abs(logits[m] - ref[m]).max()) for m in range(M))
    print(f"head outlier tokens M={M}: max-abs {err:.2e}, near ties {near}")
