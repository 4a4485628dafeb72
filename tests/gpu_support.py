"""Helpers for the GPU parity tests: seeded layers and heads on the device,
the same inputs handed to the CPU oracle, and the comparison rules.

Comparison rules (floating point decides integers here, so both sides are
compared only where the decision is robust):
- outputs: relative L2 error <= 2e-3 and max-abs error <= 1e-2 against the
  oracle's fp64 result on the same quantised bytes;
- ids (experts, tokens): where the oracle's scores on both sides of rank r are
  separated by more than delta = 1e-4 * (1 + |score|), the GPU's id at rank r
  must equal the oracle's; inside a near tie, the GPU's choice must score
  within delta of the oracle's choice.  delta sits far above the fp32
  reduction error of these dot products (about 1e-6 for unit-scale logits)
  and far below the typical gap between neighbouring top scores.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from moe_decode_gemv_b200 import inputs as I

REL_L2_TOL = 2e-3
MAX_ABS_TOL = 1e-2


def delta(v):
    return 1e-4 * (1.0 + np.abs(v))


def u16(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().view(torch.int16).numpy().view(np.uint16)


def rel_l2(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))


def assert_close(got, ref, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    r, m = rel_l2(got, ref), float(np.max(np.abs(got - ref))) if ref.size else 0.0
    assert r <= REL_L2_TOL and m <= MAX_ABS_TOL, f"{what}: rel-L2 {r:.3e}, max-abs {m:.3e}"
    return r, m


def ranked(scores: np.ndarray) -> np.ndarray:
    """Indices by descending score, ties to the lower index."""
    return np.lexsort((np.arange(scores.shape[0]), -scores))


def margin_ok(scores: np.ndarray, k: int) -> bool:
    """True if the k-th and (k+1)-th best scores are more than delta apart."""
    if k >= scores.shape[0]:
        return True
    o = ranked(scores)
    a, b = scores[o[k - 1]], scores[o[k]]
    return (a - b) > delta(a)


def check_ranked_ids(gpu_ids, scores: np.ndarray, k: int) -> int:
    """Check a GPU top-k list against oracle scores; returns the number of
    ranks that fell inside a near tie (and were checked by score)."""
    gpu_ids = np.asarray(gpu_ids).astype(np.int64)
    assert len(set(gpu_ids.tolist())) == k, f"duplicate ids {gpu_ids}"
    assert ((gpu_ids >= 0) & (gpu_ids < scores.shape[0])).all()
    o = ranked(scores)
    ref = o[:k]
    ext = scores[o[: k + 1]] if k < scores.shape[0] else np.append(scores[o[:k]], -np.inf)
    near = 0
    for r in range(k):
        v = ext[r]
        sep_above = r == 0 or ext[r - 1] - v > delta(v)
        sep_below = v - ext[r + 1] > delta(v)
        if sep_above and sep_below:
            assert gpu_ids[r] == ref[r], f"rank {r}: gpu {gpu_ids[r]} oracle {ref[r]}"
        else:
            near += 1
            assert abs(scores[gpu_ids[r]] - v) <= 2 * delta(v), f"rank {r}: gpu id {gpu_ids[r]} off the tie"
    return near


# ---------------------------------------------------------------------------
# MoE layers
# ---------------------------------------------------------------------------

class Layer:
    """A seeded MoE layer: bf16 weights drawn per expert on the CPU, copied to
    the GPU and quantised there by the library; the oracle redraws and
    quantises only the experts it needs."""

    KINDS = ("gate", "up", "down")

    def __init__(self, B, seed: int, shape: I.MoEShape, layer: int = 0, skewed: bool = False,
                 wfn=None, sfn=None):
        """wfn(kind, expert, w_bf16) -> w_bf16 changes an expert's weights before
        quantisation; sfn(kind, scales_uint8) -> scales_uint8 patches the E8M0
        codes after it.  Both sides (GPU and oracle) apply the same hooks."""
        self.B, self.seed, self.shape, self.layer = B, seed, shape, layer
        self.wfn = wfn or (lambda kind, e, w: w)
        self.sfn = sfn or (lambda kind, sc: sc)
        self.router_w = I.router_weight(seed, shape.experts, shape.hidden, layer)
        self.router_bias = I.router_bias(seed, shape.experts, layer) if skewed else None
        self.router_w_dev = self.router_w.cuda()
        self.router_bias_dev = None if self.router_bias is None else self.router_bias.cuda()
        self.bank = tuple(self._quantize_bank(k, range(shape.experts)) for k in self.KINDS)
        self.shared = tuple(self._quantize_bank(k, ["shared"]) for k in self.KINDS)
        # the layout moe_decode reads (same bytes, regrouped)
        self.packed = B.moe_pack_experts(self.bank)
        self.packed_shared = B.moe_pack_experts(self.shared)

    def _quantize_bank(self, kind, experts):
        s = self.shape
        rows, cols = (s.inter, s.hidden) if kind != "down" else (s.hidden, s.inter)
        experts = list(experts)
        staging = torch.empty((len(experts), rows, cols), dtype=torch.bfloat16, device="cuda")
        for i, e in enumerate(experts):
            staging[i].copy_(self.wfn(kind, e, I.expert_matrix(self.seed, s, e, kind, self.layer)), non_blocking=False)
        bank = self.B.moe_quantize_mxfp4(staging)
        del staging
        patched = self.sfn(kind, bank.scales.cpu().numpy())
        bank.scales.copy_(torch.from_numpy(np.ascontiguousarray(patched)))
        return bank

    def _oracle_quantize(self, kind, e):
        w = self.wfn(kind, e, I.expert_matrix(self.seed, self.shape, e, kind, self.layer))
        d, sc = oracle.load().mxfp4_quantize(u16(w))
        return d, self.sfn(kind, sc)

    def oracle_banks(self, O, experts):
        """Stacked numpy banks holding the oracle's own quantisation of the
        given experts (zeros elsewhere; the oracle reads only routed ids)."""
        s = self.shape
        out = {}
        for kind in self.KINDS:
            rows, cols = (s.inter, s.hidden) if kind != "down" else (s.hidden, s.inter)
            d = np.zeros((s.experts, rows, cols // 2), np.uint8)
            sc = np.zeros((s.experts, rows, cols // 32), np.uint8)
            for e in sorted(set(int(v) for v in experts)):
                d[e], sc[e] = self._oracle_quantize(kind, e)
            out[kind] = (d, sc)
        shared = {k: self._oracle_quantize(k, "shared") for k in self.KINDS}
        shared = {k: (v[0][None], v[1][None]) for k, v in shared.items()}
        return out, shared

    def run_gpu(self, x_dev: torch.Tensor, workspace=None):
        M, k = x_dev.shape[0], self.shape.top_k
        out = torch.empty((M, self.shape.hidden), dtype=torch.float32, device="cuda")
        ids = torch.empty((M, k), dtype=torch.int32, device="cuda")
        w = torch.empty((M, k), dtype=torch.float32, device="cuda")
        self.B.moe_decode(x_dev, self.router_w_dev, self.router_bias_dev, self.packed, self.packed_shared, k, out, ids, w,
                          workspace=workspace)
        torch.cuda.synchronize()
        return out.cpu().numpy(), ids.cpu().numpy(), w.cpu().numpy()

    def run_oracle(self, O, x: torch.Tensor):
        xb = u16(x)
        logits, ids, w = O.router(xb, self.router_w.numpy(),
                                  None if self.router_bias is None else self.router_bias.numpy(), self.shape.top_k)
        bank, shared = self.oracle_banks(O, ids.reshape(-1))
        y = O.moe_layer(xb, ids, w, bank, shared)
        return logits, ids, w, y


def check_moe(layer: Layer, O, x: torch.Tensor, y_gpu, ids_gpu, w_gpu):
    """Parity of one MoE call; returns a small report."""
    logits, ids, w, y = layer.run_oracle(O, x)
    k = layer.shape.top_k
    report = {"near_ties": 0, "skipped_tokens": 0, "rel_l2": 0.0, "max_abs": 0.0}
    for m in range(x.shape[0]):
        report["near_ties"] += check_ranked_ids(ids_gpu[m], logits[m], k)
        if not margin_ok(logits[m], k):
            report["skipped_tokens"] += 1  # selection itself is a near tie: outputs may differ legitimately
            continue
        assert sorted(ids_gpu[m].tolist()) == sorted(ids[m].tolist())
        # weights: compare per expert id
        ref_w = dict(zip(ids[m].tolist(), w[m].tolist()))
        got_w = dict(zip(ids_gpu[m].tolist(), w_gpu[m].tolist()))
        for e in ref_w:
            assert abs(got_w[e] - ref_w[e]) <= 1e-5, (m, e, got_w[e], ref_w[e])
        r, a = assert_close(y_gpu[m], y[m], f"token {m}")
        report["rel_l2"] = max(report["rel_l2"], r)
        report["max_abs"] = max(report["max_abs"], a)
    return report


# ---------------------------------------------------------------------------
# LM head
# ---------------------------------------------------------------------------

def head_weights(seed: int, shape: I.HeadShape) -> torch.Tensor:
    return I.lmhead_weight(seed, shape)


def run_head_gpu(B, head, x_dev, k, with_logits=True, bf16_w=None):
    M = x_dev.shape[0]
    V = bf16_w.shape[0] if bf16_w is not None else head.vocab
    ids = torch.empty((M, k), dtype=torch.int32, device="cuda")
    vals = torch.empty((M, k), dtype=torch.float32, device="cuda")
    logits = torch.empty((M, V), dtype=torch.float32, device="cuda") if with_logits else None
    if bf16_w is None:
        B.lmhead_decode(x_dev, head, k, ids, vals, logits)
    else:
        B.lmhead_decode_bf16(x_dev, bf16_w, k, ids, vals, logits)
    torch.cuda.synchronize()
    return ids.cpu().numpy(), vals.cpu().numpy(), None if logits is None else logits.cpu().numpy()


def check_head(ids_gpu, vals_gpu, logits_gpu, ref_logits):
    near = 0
    for m in range(ref_logits.shape[0]):
        k = ids_gpu.shape[1]
        near += check_ranked_ids(ids_gpu[m], ref_logits[m], k)
        # the value reported with each id is that id's logit
        assert np.allclose(vals_gpu[m], ref_logits[m][ids_gpu[m]], rtol=0, atol=MAX_ABS_TOL)
        if logits_gpu is not None:
            assert_close(logits_gpu[m], ref_logits[m], f"logits of token {m}")
            # the top-k list is the top-k of the logits the kernel wrote
            o = ranked(logits_gpu[m].astype(np.float64))[:k]
            assert np.array_equal(o, ids_gpu[m]), "top-k list disagrees with the kernel's own logits"
    return near
