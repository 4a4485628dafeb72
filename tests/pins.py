"""Pins for the CPU oracle: checks against what the format specifications,
library routines, brute force and the pages fix -- never against the oracle
itself.

Each ``pin_*`` takes an ``oracle.Oracle`` and raises ``AssertionError`` when
the oracle disagrees.  The oracle tests call them on the oracle as built; the
mutation test calls them on copies of the oracle with a planted mistake and
expects at least one pin to fail for each mistake.

Independent references used here:
- ml_dtypes ``float4_e2m1fn`` (E2M1 decode and its RNE, saturating cast);
- torch ``float8_e4m3fn`` / ``float8_e8m0fnu`` (E4M3 / E8M0 decode, E4M3 RNE cast);
- torch float64 matmul, softmax, silu, and numpy sorting;
- brute force over all k-subsets / all bf16 neighbours;
- the text fixtures in tests/golden/ (spec tables, RNE ties, page facts).
"""
from __future__ import annotations

import itertools
import math
import os

import ml_dtypes
import numpy as np
import torch

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def read_golden(name: str) -> list[list[str]]:
    rows = []
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append(line.split())
    return rows


def _same(a: float, b: float) -> bool:
    """Equal including the sign of zero and NaN == NaN."""
    if math.isnan(a) or math.isnan(b):
        return math.isnan(a) and math.isnan(b)
    return a == b and math.copysign(1.0, a) == math.copysign(1.0, b)


# ---------------------------------------------------------------------------
# independent decoders
# ---------------------------------------------------------------------------

def lib_e2m1(codes: np.ndarray) -> np.ndarray:
    return np.asarray(codes, np.uint8).view(ml_dtypes.float4_e2m1fn).astype(np.float64)


def lib_e8m0(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e8m0fnu)
    return t.to(torch.float64).numpy()


def lib_e4m3(codes: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn)
    return t.to(torch.float64).numpy()


def lib_bf16(bits: np.ndarray) -> np.ndarray:
    t = torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16)).view(torch.bfloat16)
    return t.to(torch.float64).numpy()


def lib_mxfp4_dequant(data: np.ndarray, scales: np.ndarray) -> np.ndarray:
    """[..., K/2] codes + [..., K/32] scales -> [..., K] float64, by library decoders.
    Element 2j is the low nibble of byte j."""
    lo = data & 15
    hi = data >> 4
    codes = np.stack([lo, hi], axis=-1).reshape(data.shape[:-1] + (data.shape[-1] * 2,))
    vals = lib_e2m1(codes)
    sc = np.repeat(lib_e8m0(scales), 32, axis=-1)
    return vals * sc


# ---------------------------------------------------------------------------
# formats
# ---------------------------------------------------------------------------

def pin_e2m1_table(O) -> None:
    for code, val in read_golden("e2m1_code_points.txt"):
        assert _same(O.e2m1(int(code)), float(val)), (code, O.e2m1(int(code)), val)
    ref = lib_e2m1(np.arange(16))
    for c in range(16):
        assert _same(O.e2m1(c), float(ref[c])), c


def pin_e8m0_table(O) -> None:
    ref = lib_e8m0(np.arange(256))
    for c in range(256):
        assert _same(O.e8m0(c), float(ref[c])), (c, O.e8m0(c), ref[c])
    assert O.e8m0(127) == 1.0 and O.e8m0(0) == 2.0 ** -127 and O.e8m0(254) == 2.0 ** 127
    assert math.isnan(O.e8m0(255))


def pin_e4m3_table(O) -> None:
    for code, val in read_golden("e4m3_code_points.txt"):
        got = O.e4m3(int(code, 16))
        assert _same(got, float(val)), (code, got, val)
    ref = lib_e4m3(np.arange(256))
    for c in range(256):
        assert _same(O.e4m3(c), float(ref[c])), (hex(c), O.e4m3(c), ref[c])


def pin_e2m1_encode(O) -> None:
    for v, want in read_golden("e2m1_rne_ties.txt"):
        got = O.e2m1(O.e2m1_encode(float(v)))
        assert _same(got, float(want)), (v, got, want)
    # dense sweep, every midpoint and both neighbours of it, against ml_dtypes
    mags = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]
    pts = set(np.linspace(-9.0, 9.0, 7201).tolist())
    for a, b in zip(mags, mags[1:]):
        mid = (a + b) / 2
        for d in (-1e-9, 0.0, 1e-9):
            pts.add(mid + d)
            pts.add(-(mid + d))
    pts = np.array(sorted(pts), np.float32)
    ref = pts.astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    for v, c in zip(pts.tolist(), ref.tolist()):
        assert O.e2m1_encode(v) == c, (v, O.e2m1_encode(v), c)


def pin_e4m3_encode(O) -> None:
    rng = np.random.default_rng(1234)
    # every code's value, every midpoint between neighbours (ties), their
    # neighbours, and a log-uniform sample, all below the max normal
    finite = [c for c in range(0x7F)]
    vals = lib_e4m3(np.array(finite, np.uint8))
    pts = list(vals)
    for a, b in zip(vals[:-1], vals[1:]):
        m = (a + b) / 2
        pts += [m, np.nextafter(np.float32(m), np.float32(0)), np.nextafter(np.float32(m), np.float32(1e9))]
    pts += list(np.exp(rng.uniform(np.log(1e-4), np.log(447.9), 20000)))
    pts = np.array(pts, np.float32)
    pts = np.concatenate([pts, -pts])
    ref = torch.from_numpy(pts).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    for v, c in zip(pts.tolist(), ref.tolist()):
        assert O.e4m3_encode(v) == c, (v, hex(O.e4m3_encode(v)), hex(c))
    # satfinite: beyond the max normal the code is +-448, never NaN
    for v in (448.0, 449.0, 464.0, 480.0, 1e6, 3.4e38):
        assert O.e4m3_encode(v) == 0x7E and O.e4m3_encode(-v) == 0xFE, v


def _bf16_neighbours(v: float) -> tuple[float, float]:
    f = np.float32(v)
    b = (np.array([f], np.float32).view(np.uint32)[0] >> 16).astype(np.uint32)
    cands = []
    for d in (-1, 0, 1, 2):
        bits = np.uint32(((int(b) + d) & 0xFFFF) << 16)
        cands.append(float(np.array([bits], np.uint32).view(np.float32)[0]))
    lo = max(c for c in cands if c <= v)
    hi = min(c for c in cands if c >= v)
    return lo, hi


def pin_bf16_round(O) -> None:
    rng = np.random.default_rng(7)
    xs = list(rng.normal(0, 3, 4000)) + [1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, -(1.0 + 2.0 ** -8), 0.0]
    for v in xs:
        bits = O.double_to_bf16(float(v))
        got = float(lib_bf16(np.array([bits], np.uint16))[0])
        lo, hi = _bf16_neighbours(abs(v))
        lo, hi = (lo, hi) if v >= 0 else (-hi, -lo)
        assert got in (lo, hi), (v, got, lo, hi)
        dl, dh = abs(v - lo), abs(hi - v)
        if dl != dh:
            assert got == (lo if dl < dh else hi), (v, got)
        else:  # tie: the even significand (last bit 0) wins
            assert (bits & 1) == 0, (v, hex(bits))


# ---------------------------------------------------------------------------
# quantisers
# ---------------------------------------------------------------------------

def _bf16_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def pin_mxfp4_quantize(O) -> None:
    g = torch.Generator().manual_seed(11)
    w = (torch.randn(24, 128, generator=g) * 0.02)
    w[0, :32] = 0.0                          # all-zero block
    w[1, :32] = 0.0
    w[1, 0] = 7.0                            # amax in the saturating band [6, 8)
    w[2, :32] = 0.0
    w[2, 5] = -0.1                           # one element: scale 2^-6, |v|/X = 6.4 -> 6
    w[3, 32:64] = torch.linspace(-1, 1, 32)  # symmetric block
    w[4, :32] = 0.0
    w[4, 0] = 1.0                            # layout: only element 0 is nonzero
    wb = w.to(torch.bfloat16)
    bits = _bf16_bits(wb)
    data, scales = O.mxfp4_quantize(bits)
    assert data.shape == (24, 64) and scales.shape == (24, 4)

    # nibble order: element 0 sits in the low nibble of byte 0
    assert data[4, 0] & 15 != 0 and data[4, 0] >> 4 == 0 and (data[4, 1:16] == 0).all()

    v = wb.to(torch.float64).numpy().reshape(24, 4, 32)
    amax = np.abs(v).max(axis=-1)
    X = lib_e8m0(scales)
    nz = amax > 0
    # the scale puts the block's largest element in E2M1's top binade [4, 8)
    assert ((amax[nz] / X[nz] >= 4) & (amax[nz] / X[nz] < 8)).all()
    assert (scales[~nz] == 0).all()
    # the elements are V/X cast to E2M1 by an independent converter
    ref_codes = (v / X[..., None]).astype(np.float32).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 15
    ref_codes = ref_codes.reshape(24, 128)
    got_codes = np.stack([data & 15, data >> 4], -1).reshape(24, 128)
    assert (got_codes == ref_codes).all(), np.argwhere(got_codes != ref_codes)[:5]
    # special cases by hand
    assert scales[1, 0] == 127 and got_codes[1, 0] == 7      # 7.0 saturates to 6.0 * 2^0
    assert scales[2, 0] == 127 - 6 and got_codes[2, 5] == 15  # -0.1 -> -6 * 2^-6

    # a non-finite input survives quantisation as NaN: under OCP MX a NaN
    # scale makes every element of its block NaN when decoded (here by the
    # library's E8M0 decoder); the row's other blocks stay finite
    nf = (torch.randn(3, 64, generator=g) * 0.02).to(torch.bfloat16)
    nf[0, 3] = float("inf")
    nf[1, 40] = float("-inf")
    nf[2, 7] = float("nan")
    d2, s2 = O.mxfp4_quantize(_bf16_bits(nf))
    deq2 = lib_mxfp4_dequant(d2, s2).reshape(3, 2, 32)
    bad = np.array([[True, False], [False, True], [True, False]])
    assert np.isnan(deq2[bad]).all() and np.isfinite(deq2[~bad]).all()


def pin_mxfp4_roundtrip(O) -> None:
    g = torch.Generator().manual_seed(12)
    wb = (torch.randn(64, 256, generator=g) * 0.02).to(torch.bfloat16)
    data, scales = O.mxfp4_quantize(_bf16_bits(wb))
    deq = lib_mxfp4_dequant(data, scales).reshape(64, 8, 32)
    v = wb.to(torch.float64).numpy().reshape(64, 8, 32)
    X = lib_e8m0(scales)[..., None]
    r = np.abs(v) / X
    # half a grid step of E2M1 at each magnitude: 0.25 below 2, 0.5 in [2,4), 1 in [4,6]
    half_ulp = np.where(r < 2, 0.25, np.where(r < 4, 0.5, 1.0)) * X
    err = np.abs(deq - v)
    sat = r > 6
    assert (err[~sat] <= half_ulp[~sat] + 1e-30).all()
    Xb = np.broadcast_to(X, v.shape)
    assert (np.abs(deq[sat]) == 6 * Xb[sat]).all()
    # the slow element-wise dequantiser agrees with the library decode
    assert np.array_equal(O.mxfp4_dequantize(data[:2], scales[:2]), deq.reshape(64, 256)[:2])


def pin_fp8_rowquant(O) -> None:
    g = torch.Generator().manual_seed(13)
    w = torch.randn(40, 96, generator=g) * 0.02
    w[3] = 0.0                       # all-zero row
    w[5, 7] = 3.0                    # a large outlier
    wb = w.to(torch.bfloat16)
    q, s = O.fp8_rowquant(_bf16_bits(wb))
    wf = wb.float()
    amax = wf.abs().amax(dim=1)
    s_ref = torch.where(amax == 0, torch.ones_like(amax), amax / 448.0)  # fp32 division
    assert np.array_equal(s, s_ref.numpy())
    q_ref = (wf / s_ref[:, None]).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(q, q_ref), np.argwhere(q != q_ref)[:5]
    # the row maximum maps to +-448
    deq = lib_e4m3(q)
    arg = wf.abs().argmax(dim=1).numpy()
    for r in range(40):
        if r != 3:
            assert abs(deq[r, arg[r]]) == 448.0, (r, deq[r, arg[r]])
    assert (q[3] == 0).all() and s[3] == 1.0


# ---------------------------------------------------------------------------
# router, experts, layer
# ---------------------------------------------------------------------------

def _tiny_router_inputs(seed: int, M: int = 3, E: int = 16, H: int = 64):
    g = torch.Generator().manual_seed(seed)
    x = torch.randn(M, H, generator=g).to(torch.bfloat16)
    Wr = torch.randn(E, H, generator=g) * 0.02
    bias = torch.randn(E, generator=g) * 2.0
    return x, Wr, bias


def pin_router(O) -> None:
    for use_bias in (False, True):
        x, Wr, bias = _tiny_router_inputs(21)
        k = 2
        logits, ids, w = O.router(_bf16_bits(x), Wr.numpy(), bias.numpy() if use_bias else None, k)
        ref_logits = x.double() @ Wr.double().T + (bias.double() if use_bias else 0.0)
        assert np.allclose(logits, ref_logits.numpy(), rtol=1e-12, atol=1e-12)
        for m in range(x.shape[0]):
            best = max(itertools.combinations(range(16), k), key=lambda c: sum(ref_logits[m, list(c)]))
            assert sorted(ids[m].tolist()) == sorted(best)
            assert ref_logits[m, ids[m, 0]] >= ref_logits[m, ids[m, 1]]
            p = torch.softmax(ref_logits[m], dim=0)[ids[m].tolist()]
            assert np.allclose(w[m], (p / p.sum()).numpy(), rtol=1e-12)
            assert abs(w[m].sum() - 1.0) < 1e-12
    # equal logits: the lower expert id comes first
    xz = torch.zeros(1, 64, dtype=torch.bfloat16)
    _, ids, w = O.router(_bf16_bits(xz), np.zeros((16, 64), np.float32), None, 4)
    assert ids[0].tolist() == [0, 1, 2, 3] and np.allclose(w, 0.25)


def _quant_pair(O, t: torch.Tensor):
    return O.mxfp4_quantize(_bf16_bits(t.to(torch.bfloat16)))


def pin_expert_special_case(O) -> None:
    H, I = 64, 32
    x = torch.zeros(H)
    x[3], x[40] = 1.5, -2.0
    xb = x.to(torch.bfloat16)
    gate = torch.zeros(I, H)
    up = torch.zeros(I, H)
    down = torch.zeros(H, I)
    gate[7, 3] = 0.25      # 4 * 2^-4: exact in MXFP4
    up[7, 40] = 0.5        # 4 * 2^-3
    down[11, 7] = -0.75    # 6 * 2^-3
    out, h = O.expert_mlp(_bf16_bits(xb), _quant_pair(O, gate), _quant_pair(O, up), _quant_pair(O, down))
    g, u = 0.25 * 1.5, 0.5 * -2.0
    h7 = g / (1.0 + math.exp(-g)) * u
    assert abs(h[7] - h7) < 1e-15 and np.count_nonzero(h) == 1
    assert abs(out[11] - (-0.75 * h7)) < 1e-15 and np.count_nonzero(out) == 1


def pin_expert_vs_torch(O) -> None:
    g = torch.Generator().manual_seed(31)
    H, I = 128, 64
    x = torch.randn(H, generator=g).to(torch.bfloat16)
    mats = [torch.randn(I, H, generator=g) * 0.02, torch.randn(I, H, generator=g) * 0.02,
            torch.randn(H, I, generator=g) * 0.02]
    q = [_quant_pair(O, t) for t in mats]
    out, h = O.expert_mlp(_bf16_bits(x), *q)
    Wg, Wu, Wd = [torch.from_numpy(lib_mxfp4_dequant(*p)) for p in q]
    xd = x.double()
    h_ref = torch.nn.functional.silu(Wg @ xd) * (Wu @ xd)
    out_ref = Wd @ h_ref
    assert np.allclose(h, h_ref.numpy(), rtol=1e-12, atol=1e-15)
    assert np.allclose(out, out_ref.numpy(), rtol=1e-12, atol=1e-15)


def pin_moe_layer(O) -> None:
    """A whole tiny layer against a dense torch fp64 restatement that routes
    with torch.topk and applies every expert through library dequantisation."""
    g = torch.Generator().manual_seed(41)
    M, H, I, E, k = 3, 64, 32, 8, 2
    x = torch.randn(M, H, generator=g).to(torch.bfloat16)
    Wr = torch.randn(E, H, generator=g) * 0.02
    banks = {n: torch.randn(E, *((I, H) if n != "down" else (H, I)), generator=g) * 0.02
             for n in ("gate", "up", "down")}
    shared_w = {n: torch.randn(*((I, H) if n != "down" else (H, I)), generator=g) * 0.02
                for n in ("gate", "up", "down")}
    bank = {n: _quant_pair(O, t) for n, t in banks.items()}
    shared = {n: _quant_pair(O, t) for n, t in shared_w.items()}
    _, ids, w = O.router(_bf16_bits(x), Wr.numpy(), None, k)
    y = O.moe_layer(_bf16_bits(x), ids, w, bank, shared)

    deq = {n: torch.from_numpy(lib_mxfp4_dequant(*bank[n])) for n in bank}
    sdeq = {n: torch.from_numpy(lib_mxfp4_dequant(*shared[n])) for n in shared}
    xd = x.double()
    logits = xd @ Wr.double().T
    vals, sel = torch.topk(logits, k, dim=1)
    wt = torch.softmax(vals, dim=1)

    def expert(Wg, Wu, Wd, v):
        return Wd @ (torch.nn.functional.silu(Wg @ v) * (Wu @ v))

    for m in range(M):
        ref = expert(sdeq["gate"], sdeq["up"], sdeq["down"], xd[m])
        for i in range(k):
            e = int(sel[m, i])
            ref = ref + wt[m, i] * expert(deq["gate"][e], deq["up"][e], deq["down"][e], xd[m])
        assert np.allclose(y[m], ref.numpy(), rtol=1e-11, atol=1e-14), m


# ---------------------------------------------------------------------------
# LM head, top-k, RMSNorm
# ---------------------------------------------------------------------------

def pin_lmhead(O) -> None:
    g = torch.Generator().manual_seed(51)
    V, H, M = 300, 96, 2
    wb = (torch.randn(V, H, generator=g) * 0.02).to(torch.bfloat16)
    x = torch.randn(M, H, generator=g).to(torch.bfloat16)
    q, s = O.fp8_rowquant(_bf16_bits(wb))
    logits, abss = O.lmhead_fp8(_bf16_bits(x), q, s, want_abssum=True)
    Wq = torch.from_numpy(lib_e4m3(q)) * torch.from_numpy(s.astype(np.float64))[:, None]
    ref = x.double() @ Wq.T
    assert np.allclose(logits, ref.numpy(), rtol=1e-12, atol=1e-15)
    ref_abs = x.double().abs() @ Wq.abs().T
    assert np.allclose(abss, ref_abs.numpy(), rtol=1e-12)
    lb = O.lmhead_bf16(_bf16_bits(x), _bf16_bits(wb))
    assert np.allclose(lb, (x.double() @ wb.double().T).numpy(), rtol=1e-12, atol=1e-15)


def pin_topk(O) -> None:
    rng = np.random.default_rng(61)
    v = rng.normal(size=1000)
    ids, vals = O.topk(v, 29)
    order = np.lexsort((np.arange(1000), -v))[:29]  # descending value, then ascending index
    assert ids.tolist() == order.tolist() and np.array_equal(vals, v[order])
    t = np.array([1.0, 3.0, 3.0, 2.0, 3.0, -1.0])
    ids, vals = O.topk(t, 4)
    assert ids.tolist() == [1, 2, 4, 3] and vals.tolist() == [3.0, 3.0, 3.0, 2.0]


def pin_rmsnorm(O) -> None:
    rng = np.random.default_rng(71)
    # unit-scale values, and values small enough that eps (inside the square
    # root) changes the result by several bf16 steps
    for sd, eps in ((5.0, 1e-6), (1e-3, 1e-6)):
        y = rng.normal(0, sd, 256)
        got = lib_bf16(O.rmsnorm_bf16(y, eps))
        r = torch.nn.functional.rms_norm(torch.from_numpy(y), (256,), eps=eps).numpy()
        # each output is one of the two bf16 neighbours of the exact value, the nearer one
        for a, b in zip(got.tolist(), r.tolist()):
            lo, hi = _bf16_neighbours(abs(b))
            lo, hi = (lo, hi) if b >= 0 else (-hi, -lo)
            assert a in (lo, hi) and abs(a - b) <= abs((hi if a == lo else lo) - b) + 1e-300, (a, b)


def pin_sample_topk(O) -> None:
    """Closed forms of top-k / top-p / temperature sampling."""
    # equal logits, no nucleus cut: the draw is floor(u * k)
    for k in (1, 4, 29):
        for u in (0.0, 0.2, 0.26, 0.5, 0.74, 0.999):
            assert O.sample_topk([1.5] * k, 0.6, 1.0, u) == min(int(u * k), k - 1), (k, u)
    # equal logits and a nucleus: the kept prefix is the smallest whose mass reaches top_p
    assert all(O.sample_topk([0.0] * 4, 1.0, 0.5, u) == int(u * 2) for u in (0.1, 0.49, 0.51, 0.99))
    assert all(O.sample_topk([0.0] * 4, 1.0, 0.51, u) == int(u * 3) for u in (0.1, 0.34, 0.67, 0.99))
    # two candidates, gap d at temperature T: P(first) = 1 / (1 + exp(-d / T))
    for d, T in ((1.0, 0.6), (0.3, 1.0), (2.0, 2.5)):
        p0 = 1.0 / (1.0 + math.exp(-d / T))
        assert O.sample_topk([d, 0.0], T, 1.0, p0 - 1e-9) == 0
        assert O.sample_topk([d, 0.0], T, 1.0, p0 + 1e-9) == 1
        # a nucleus below the first probability keeps only the first
        assert O.sample_topk([d, 0.0], T, p0 * 0.999, 0.999) == 0
    # a near-zero temperature is greedy
    assert all(O.sample_topk([3.0, 2.9, 1.0, -2.0], 1e-3, 0.95, u) == 0 for u in (0.0, 0.5, 0.9999))
    # stratified draws reproduce the nucleus distribution of scipy's softmax
    from scipy.special import softmax
    rng = np.random.default_rng(5)
    v = np.sort(rng.normal(0, 1.5, 29))[::-1].copy()
    T, top_p, N = 0.6, 0.95, 20000
    p = softmax(v / T)
    n = int(np.searchsorted(np.cumsum(p), top_p) + 1)  # first prefix whose mass reaches top_p
    q = p[:n] / p[:n].sum()
    counts = np.bincount([O.sample_topk(v, T, top_p, (i + 0.5) / N) for i in range(N)], minlength=29)
    assert counts[n:].sum() == 0
    assert np.all(np.abs(counts[:n] - q * N) <= 1.0 + 1e-6), (counts[:n], q * N)


def pin_mtp_accept(O) -> None:
    """Greedy acceptance, enumerated from its definition."""
    cases = [
        ([5, 6, 7], [5, 6, 7, 8], [5, 6, 7, 8]),    # all drafts accepted, plus the verify step's next token
        ([5, 6, 7], [4, 6, 7, 8], [4]),             # the first draft rejected: only the verify token
        ([5, 6, 7], [5, 9, 7, 8], [5, 9]),          # a later match after a mismatch does not count
        ([5, 6, 7], [5, 6, 1, 8], [5, 6, 1]),
        ([3], [3, 2], [3, 2]),
        ([3], [2, 3], [2]),
    ]
    for draft, verify, want in cases:
        assert O.mtp_accept(draft, verify).tolist() == want, (draft, verify)


ALL_PINS = [
    pin_e2m1_table, pin_e8m0_table, pin_e4m3_table, pin_e2m1_encode, pin_e4m3_encode,
    pin_bf16_round, pin_mxfp4_quantize, pin_mxfp4_roundtrip, pin_fp8_rowquant, pin_router,
    pin_expert_special_case, pin_expert_vs_torch, pin_moe_layer, pin_lmhead, pin_topk,
    pin_rmsnorm, pin_sample_topk, pin_mtp_accept,
]
