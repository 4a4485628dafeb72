"""GPU parity of the load-time quantisers: bit-exact with the CPU oracle.

MXFP4 (OCP MX E2M1 + E8M0 per 32) for expert weights and the per-row FP8
E4M3 quantisation of the LM head (ncijnetwork.com summary, "What are the 3
optimizations?", item 2).  Integer and byte work: every byte must match.
"""
import numpy as np
import pytest
import torch

import oracle
from gpu_support import u16
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


def adversarial_bf16(rows: int, K: int) -> torch.Tensor:
    """Rows that hit every branch of the rounding rules."""
    g = torch.Generator().manual_seed(99)
    w = torch.randn(rows, K, generator=g) * 0.02
    grid = torch.tensor([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])
    mids = (grid[:-1] + grid[1:]) / 2
    r = 0
    w[r] = 0.0; r += 1                                               # all zero
    w[r] = -0.0; r += 1                                              # negative zeros
    w[r, :32] = 0.0; w[r, 0] = 4.0; w[r, 1:8] = mids; w[r, 8:15] = -mids; r += 1   # ties at scale 1
    w[r, :32] = 7.5; w[r, 1] = 6.5; w[r, 2] = -7.9; r += 1           # saturating band [6, 8)
    w[r, :32] = 1e-39; w[r, 1] = -3e-39; r += 1                      # bf16 subnormals
    w[r, :32] = 3e38; w[r, 5] = -1e38; r += 1                        # near the top of the range
    w[r, :32] = torch.linspace(-1e-3, 1e-3, 32); r += 1
    w[r, :32] = 2.0 ** -130; r += 1                                  # exponent clamp at -127
    w[r, 32:64] = float("inf"); r += 1                               # non-finite block
    w[r, 64:96] = float("nan"); r += 1
    w[r] = torch.randn(K, generator=g) * 100.0; r += 1
    return w.to(torch.bfloat16)


@pytest.mark.parametrize("shape", [(3, 64, 256), (1, 2560, 768), (2, 768, 2560)])
def test_mxfp4_random_bit_exact(B, O, shape):
    g = torch.Generator().manual_seed(sum(shape))
    w = (torch.randn(*shape, generator=g) * 0.02).to(torch.bfloat16)
    bank = B.moe_quantize_mxfp4(w.cuda())
    torch.cuda.synchronize()
    d_ref, s_ref = O.mxfp4_quantize(u16(w))
    assert bank.fmt == B.Format.MXFP4_E2M1_E8M0_32
    assert np.array_equal(bank.scales.cpu().numpy(), s_ref)
    d = bank.data.cpu().numpy()
    bad = np.argwhere(d != d_ref)
    assert bad.size == 0, bad[:8]


def test_mxfp4_adversarial_bit_exact(B, O):
    w = adversarial_bf16(16, 256)
    bank = B.moe_quantize_mxfp4(w.cuda())
    torch.cuda.synchronize()
    d_ref, s_ref = O.mxfp4_quantize(u16(w))
    s = bank.scales.cpu().numpy()[0]
    d = bank.data.cpu().numpy()[0]
    assert np.array_equal(s, s_ref), np.argwhere(s != s_ref)[:8]
    assert np.array_equal(d, d_ref), np.argwhere(d != d_ref)[:8]
    assert s[8, 1] == 0xFF and s[9, 2] == 0xFF  # the Inf and NaN blocks


def test_mxfp4_ling_expert_bank_sampled(B, O):
    """Full Ling-shaped gate bank (512 x 768 x 2560) on the GPU; the oracle
    re-quantises a sample of experts and every byte must match."""
    s = I.LING_MOE
    staging = torch.empty((s.experts, s.inter, s.hidden), dtype=torch.bfloat16, device="cuda")
    for e in range(s.experts):
        staging[e].copy_(I.expert_matrix(3, s, e, "gate"))
    bank = B.moe_quantize_mxfp4(staging)
    torch.cuda.synchronize()
    for e in (0, 1, 255, 511):
        d_ref, s_ref = O.mxfp4_quantize(u16(I.expert_matrix(3, s, e, "gate")))
        assert np.array_equal(bank.data[e].cpu().numpy(), d_ref), e
        assert np.array_equal(bank.scales[e].cpu().numpy(), s_ref), e


def test_fp8_rowquant_random_and_adversarial(B, O):
    g = torch.Generator().manual_seed(5)
    w = torch.randn(512, 320, generator=g) * 0.02
    w[0] = 0.0
    w[1, 3] = 5.0                      # outlier row
    w[2] = -0.0
    w[3, :] = 1e-39                    # subnormal row
    w[4, :] = torch.linspace(-3, 3, 320)
    w[5, :] = 448.0 * 3                # amax / 448 exactly representable
    wb = w.to(torch.bfloat16)
    head = B.lmhead_quantize_fp8(wb.cuda(), tiled=False)
    torch.cuda.synchronize()
    q_ref, s_ref = O.fp8_rowquant(u16(wb))
    assert head.fmt == B.Format.FP8_E4M3_ROWSCALE_F32
    assert np.array_equal(head.row_scale.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    q = head.q.cpu().numpy()
    assert np.array_equal(q, q_ref), np.argwhere(q != q_ref)[:8]


def test_fp8_rowquant_full_head(B, O):
    """The 157,184 x 2,560 head: every scale and every byte against the oracle."""
    w = I.lmhead_weight(0, I.LING_HEAD)
    head = B.lmhead_quantize_fp8(w.cuda(), tiled=False)
    torch.cuda.synchronize()
    q_ref, s_ref = O.fp8_rowquant(u16(w))
    assert np.array_equal(head.row_scale.cpu().numpy().view(np.uint32), s_ref.view(np.uint32))
    assert np.array_equal(head.q.cpu().numpy(), q_ref)
    # bytes read per token halve against the bf16 head (ncijnetwork.com summary, item 2)
    assert head.q.numel() * 2 == w.numel() * w.element_size()
