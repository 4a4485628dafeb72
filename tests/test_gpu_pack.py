"""The sliced expert-bank layout, byte for byte, against a numpy statement of
the layout that moe_gemv.h documents for moe_packed_bank (packing moves
bytes and bits only, so the comparison is exact)."""
import numpy as np
import pytest
import torch

from moe_decode_gemv_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from moe_decode_gemv_b200 import build
    build.build()
    from moe_decode_gemv_b200 import binding
    return binding


def relayout(b):
    """The documented bit placement of one packed data byte: element 2j (low
    nibble) sign|e1 e0 m -> bits 7|3 2 1, element 2j+1 (high nibble) -> 0|6 5 4."""
    b = b.astype(np.uint8)
    lo, hi = b & 0xF, b >> 4
    out = ((lo >> 3) << 7) | ((lo & 7) << 1) | (hi >> 3) | ((hi & 7) << 4)
    return out.astype(np.uint8)


def expected_packed(gate, up, down):
    """numpy: (data, scales) pairs of the canonical banks -> (units, dscales)
    bytes of the sliced layout moe_gemv.h documents for moe_packed_bank."""
    (gd, gs), (ud, us), (dd, ds) = gate, up, down
    E, I, Hh = gd.shape
    H = 2 * Hh
    nb = H // 32
    units, dsc = [], []
    for e in range(E):
        for j in range(I // 16):
            # A: the 128-row operand, row 32s + R = gate/up row R (gate 16j ..
            # 16j+15, then up) over K segment s of Ks = 64 T elements (T =
            # ceil(H / 256)); [K tile][half][operand row][16 bytes], standard
            # nibble order, zero past H
            T = (H + 255) // 256
            rows = np.zeros((32, 128 * T), np.uint8)
            rows[:16, :Hh] = gd[e, 16 * j:16 * j + 16]
            rows[16:, :Hh] = ud[e, 16 * j:16 * j + 16]
            units.append(rows.reshape(32, 4, T, 2, 16).transpose(2, 3, 1, 0, 4).reshape(-1))
            # B: [K tile][row R][segment][half] E8M0, zero past H
            sc = np.zeros((32, 8 * T), np.uint8)
            sc[:16, :nb] = gs[e, 16 * j:16 * j + 16]
            sc[16:, :nb] = us[e, 16 * j:16 * j + 16]
            units.append(sc.reshape(32, 4, T, 2).transpose(2, 0, 1, 3).reshape(-1))
            # C: [group][g][t][r][2 bytes] = columns 16j + 4t .. +3 of down row 32G + 8r + g
            cols = dd[e][:, 8 * j:8 * j + 8].reshape(H // 32, 4, 8, 4, 2)  # [G][r][g][t][2]
            c = cols.transpose(0, 2, 3, 1, 4)  # [G][g][t][r][2]
            units.append(relayout(c.reshape(-1)))
        for p in range(I // 32):
            # byte 32G + 4g + t = scale of down row 32G + 8t + g
            dsc.append(ds[e][:, p].reshape(H // 32, 4, 8).transpose(0, 2, 1).reshape(-1))
    return np.concatenate(units), np.concatenate(dsc)


@pytest.mark.parametrize("E,H,Inter", [(3, 256, 64), (2, 192, 192), (2, 96, 32), (2, 2560, 768)])
def test_pack_matches_documented_layout(B, E, H, Inter):
    g = torch.Generator().manual_seed(E * 1000 + H + Inter)
    banks = []
    for rows, cols in ((Inter, H), (Inter, H), (H, Inter)):
        w = (torch.randn((E, rows, cols), generator=g) * 0.02).to(torch.bfloat16)
        banks.append(B.moe_quantize_mxfp4(w.cuda()))
    packed = B.moe_pack_experts(tuple(banks))
    torch.cuda.synchronize()
    assert packed.fmt == B.Format.MXFP4_MOE_PACKED
    canon = [(b.data.cpu().numpy(), b.scales.cpu().numpy()) for b in banks]
    want_u, want_d = expected_packed(*canon)
    assert np.array_equal(packed.units.cpu().numpy(), want_u)
    assert np.array_equal(packed.dscales.cpu().numpy(), want_d)
    assert packed.nbytes() == want_u.size + want_d.size
    if H % 256 == 0:  # no K-tile padding: the same bytes, regrouped
        assert packed.nbytes() == sum(b.nbytes() for b in banks)


def test_pack_of_ling_shared_expert(B):
    s = I.LING_MOE
    banks = tuple(B.moe_quantize_mxfp4(I.expert_matrix(0, s, "shared", k).cuda()) for k in ("gate", "up", "down"))
    packed = B.moe_pack_experts(banks)
    canon = [(b.data.cpu().numpy(), b.scales.cpu().numpy()) for b in banks]
    want_u, want_d = expected_packed(*canon)
    assert np.array_equal(packed.units.cpu().numpy(), want_u)
    assert np.array_equal(packed.dscales.cpu().numpy(), want_d)


def expected_tiled_head(q):
    """numpy: the [V][H] E4M3 head -> the tiled bytes moe_gemv.h documents for
    MOE_FMT_FP8_E4M3_TILED (whole 16-row tiles, zero rows past V; per 64-byte
    K slice, [half][lane][16 bytes] = row (lane >> 2) + 8 half, bytes
    64 s + 16 (lane & 3) ...)."""
    V, H = q.shape
    T = (V + 15) // 16
    padded = np.zeros((T * 16, H), dtype=np.uint8)
    padded[:V] = q
    t = padded.reshape(T, 2, 8, H // 64, 4, 16)          # [tile][half][g][slice][tq][16]
    return t.transpose(0, 3, 1, 2, 4, 5).reshape(-1)     # [tile][slice][half][g][tq][16]


@pytest.mark.parametrize("V,H", [(4100, 320), (157184 // 16, 2560)])
def test_fp8_head_tiles_match_documented_layout(B, V, H):
    g = torch.Generator().manual_seed(V + H)
    w = (torch.randn((V, H), generator=g) * 0.02).to(torch.bfloat16)
    canon = B.lmhead_quantize_fp8(w.cuda(), tiled=False)
    tiled = B.lmhead_tile_fp8(canon)
    torch.cuda.synchronize()
    assert tiled.fmt == B.Format.FP8_E4M3_TILED and (tiled.vocab, tiled.hidden) == (V, H)
    assert tiled.row_scale.data_ptr() == canon.row_scale.data_ptr()
    assert np.array_equal(tiled.q.cpu().numpy(), expected_tiled_head(canon.q.cpu().numpy()))
