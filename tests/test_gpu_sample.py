"""GPU parity of the decode-step tail: one draw from the head's top-k with
temperature and top-p, and greedy acceptance of draft tokens.  Inputs are
seeded and synthetic (sorted logit lists, token ids); the oracle never sees a
GPU result."""
import numpy as np
import pytest
import torch

import oracle

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


def _near_boundary(vals, T, top_p, u, tol=1e-9):
    """True when u * (kept mass) lies within tol of a cumulative boundary: a
    draw there may legitimately differ between two fp64 evaluations."""
    v = np.asarray(vals, np.float64)
    p = np.exp((v - v[0]) / T)
    c = np.cumsum(p)
    n = int(np.searchsorted(c, top_p * c[-1]) + 1)
    r = u * c[n - 1]
    return np.min(np.abs(c[:n] - r)) <= tol * c[n - 1] or abs(c[n - 2 if n > 1 else 0] - top_p * c[-1]) <= tol * c[-1]


@pytest.mark.parametrize("k,T,top_p", [(29, 0.6, 0.95), (1, 0.6, 0.95), (64, 1.0, 1.0), (8, 0.05, 0.5), (29, 2.0, 0.3)])
def test_sample_matches_oracle(B, O, k, T, top_p):
    rng = np.random.default_rng(k * 100 + int(T * 10))
    M = 512
    vals = -np.sort(-rng.normal(0, 2.0, (M, k)), axis=1).astype(np.float32)
    ids = rng.integers(0, 157184, (M, k)).astype(np.int32)
    u = rng.random(M).astype(np.float32)
    out = B.lmhead_sample(torch.from_numpy(ids).cuda(), torch.from_numpy(vals).cuda(), T, top_p,
                          torch.from_numpy(u).cuda())
    got = out.cpu().numpy()
    mism = 0
    for m in range(M):
        want = ids[m, O.sample_topk(vals[m].astype(np.float64), T, top_p, float(u[m]))]
        if got[m] != want:
            assert _near_boundary(vals[m], T, top_p, float(u[m])), (m, got[m], want)
            mism += 1
    assert mism <= 1


def test_sample_edges(B, O):
    # equal logits: the draw is floor(u * k); a tiny top_p keeps only the first
    k = 29
    vals = np.zeros((4, k), np.float32)
    ids = np.arange(4 * k, dtype=np.int32).reshape(4, k)
    u = np.array([0.0, 0.5, 0.999, 0.26], np.float32)
    got = B.lmhead_sample(torch.from_numpy(ids).cuda(), torch.from_numpy(vals).cuda(), 0.6, 1.0,
                          torch.from_numpy(u).cuda()).cpu().numpy()
    assert got.tolist() == [ids[m, min(int(float(u[m]) * k), k - 1)] for m in range(4)]
    got = B.lmhead_sample(torch.from_numpy(ids).cuda(), torch.from_numpy(vals).cuda(), 0.6, 1e-6,
                          torch.from_numpy(u).cuda()).cpu().numpy()
    assert got.tolist() == ids[:, 0].tolist()


def test_sample_rejects_bad_arguments(B):
    ids = torch.zeros((2, 4), dtype=torch.int32, device="cuda")
    vals = torch.zeros((2, 4), dtype=torch.float32, device="cuda")
    u = torch.zeros((2,), dtype=torch.float32, device="cuda")
    for T, p in ((0.0, 0.9), (-1.0, 0.9), (0.6, 0.0), (0.6, 1.5), (float("nan"), 0.9)):
        with pytest.raises(B.MoEError):
            B.lmhead_sample(ids, vals, T, p, u)


def test_mtp_accept_matches_oracle(B, O):
    rng = np.random.default_rng(9)
    for D in (1, 3, 7):
        for _ in range(50):
            draft = rng.integers(0, 3, D).astype(np.int32)       # a small vocabulary makes matches common
            verify = rng.integers(0, 3, D + 1).astype(np.int32)
            emitted, n = B.moe_mtp_accept(torch.from_numpy(draft).cuda(), torch.from_numpy(verify).cuda())
            n = int(n.cpu().item())
            assert emitted.cpu().numpy()[:n].tolist() == O.mtp_accept(draft, verify).tolist()
