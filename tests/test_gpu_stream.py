"""GPU parity of the decode-step stream: embedding of the previous greedy
token -> a stack of MoE layers, each re-routed from the previous layer's
RMS-normalised output -> the FP8 LM head -> argmax -> next step.

The GPU and the oracle each run their own chain from the same first tokens
(the oracle never consumes a GPU result).  At every step the greedy tokens
must agree as long as the oracle's own decisions are safe: every routing
choice and the head's argmax clear the selection margin.  After the first
unsafe step the chains may legitimately part, and the comparison stops."""
import numpy as np
import pytest
import torch

import oracle
from gpu_support import Layer, margin_ok, u16
from moe_decode_gemv_b200 import inputs as I

pytestmark = pytest.mark.gpu
EPS = 1e-6


@pytest.fixture(scope="module")
def B():
    from moe_decode_gemv_b200 import build
    build.build()
    from moe_decode_gemv_b200 import binding
    return binding


@pytest.fixture(scope="module")
def O():
    return oracle.load()


class Stack:
    def __init__(self, B, O, seed, moe: I.MoEShape, head: I.HeadShape, n_layers: int):
        self.B, self.O, self.moe, self.head_shape = B, O, moe, head
        self.layers = [Layer(B, seed, moe, layer=l) for l in range(n_layers)]
        w = I.lmhead_weight(seed, head)
        self.head = B.lmhead_quantize_fp8(w.cuda())
        self.q, self.s = O.fp8_rowquant(u16(w))
        self.table = I.embedding_table(seed, head)
        self.table_dev = self.table.cuda()
        self.banks = [None] * n_layers

    def gpu(self, tokens, steps):
        B, M, H = self.B, len(tokens), self.moe.hidden
        ids = torch.tensor(tokens, dtype=torch.int32, device="cuda").view(M, 1)
        x = torch.empty((M, H), dtype=torch.bfloat16, device="cuda")
        y = torch.empty((M, H), dtype=torch.float32, device="cuda")
        tk = torch.empty((M, 1), dtype=torch.int32, device="cuda")
        tv = torch.empty((M, 1), dtype=torch.float32, device="cuda")
        out = []
        for _ in range(steps):
            B.moe_embed_gather(self.table_dev, ids, x, ids_stride=1)
            for layer in self.layers:
                B.moe_decode(x, layer.router_w_dev, None, layer.packed, layer.packed_shared, self.moe.top_k, y)
                B.moe_rmsnorm_bf16(y, x, EPS)
            B.lmhead_decode(x, self.head, 1, tk, tv)
            ids = tk.clone()
            out.append(tk.cpu().numpy()[:, 0].copy())
        torch.cuda.synchronize()
        return np.array(out)  # [steps, M]

    def oracle(self, tokens, steps):
        O, M = self.O, len(tokens)
        table = u16(self.table)
        toks = np.array(tokens)
        out, safe = [], []
        for _ in range(steps):
            x = np.ascontiguousarray(table[toks])
            ok = True
            for l, layer in enumerate(self.layers):
                logits, rid, rw = O.router(x, layer.router_w.numpy(), None, self.moe.top_k)
                ok &= all(margin_ok(logits[m], self.moe.top_k) for m in range(M))
                bank, shared = layer.oracle_banks(O, rid.reshape(-1))
                y = O.moe_layer(x, rid, rw, bank, shared)
                x = np.stack([O.rmsnorm_bf16(y[m], EPS) for m in range(M)])
            lg = O.lmhead_fp8(x, self.q, self.s)
            ok &= all(margin_ok(lg[m], 1) for m in range(M))
            toks = np.argmax(lg, axis=1)  # first maximum: the lower id on a tie
            out.append(toks.copy())
            safe.append(ok)
        return np.array(out), safe


def _compare(gpu_tokens, ref_tokens, safe):
    checked = 0
    for t in range(len(safe)):
        assert np.array_equal(gpu_tokens[t], ref_tokens[t]), f"step {t}: gpu {gpu_tokens[t]} oracle {ref_tokens[t]}"
        checked += 1
        if not safe[t]:
            break
    return checked


def test_tiny_stack_stream(B, O):
    st = Stack(B, O, 0, I.TINY_MOE, I.TINY_HEAD, n_layers=3)
    for tokens in ([7], [1, 2, 3, 4]):
        g = st.gpu(tokens, steps=6)
        r, safe = st.oracle(tokens, steps=6)
        assert _compare(g, r, safe) >= 2


def test_ling_stack_stream(B, O):
    """Two Ling-shaped layers and the 157,184 x 2,560 head, three steps."""
    st = Stack(B, O, 1, I.LING_MOE, I.LING_HEAD, n_layers=2)
    g = st.gpu([11], steps=3)
    r, safe = st.oracle([11], steps=3)
    assert _compare(g, r, safe) >= 1


def test_rmsnorm_and_gather_kernels(B, O):
    g = torch.Generator().manual_seed(3)
    y = torch.randn(4, 2560, generator=g) * 3.0
    out = torch.empty((4, 2560), dtype=torch.bfloat16, device="cuda")
    B.moe_rmsnorm_bf16(y.cuda(), out, EPS)
    got = out.cpu().float().numpy()
    for m in range(4):
        ref = O.rmsnorm_bf16(y[m].double().numpy(), EPS).view(np.int16)
        ref = torch.from_numpy(ref.copy()).view(torch.bfloat16).float().numpy()
        # each element is the oracle's bf16 or one of its neighbours (fp32 vs fp64 rounding)
        assert np.all(np.abs(got[m] - ref) <= np.abs(ref) * 2.0 ** -7 + 1e-30)
        assert (got[m] == ref).mean() > 0.99
    table = I.embedding_table(0, I.TINY_HEAD).cuda()
    ids = torch.tensor([[5, 0], [4095, 0], [-1, 0], [4096, 0]], dtype=torch.int32, device="cuda")
    rows = torch.empty((4, 256), dtype=torch.bfloat16, device="cuda")
    B.moe_embed_gather(table, ids, rows, ids_stride=2)
    assert torch.equal(rows[0], table[5]) and torch.equal(rows[1], table[4095])
    assert (rows[2] == 0).all() and (rows[3] == 0).all()  # out-of-range ids give zero rows
