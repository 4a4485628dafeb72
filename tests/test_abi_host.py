"""The C-ABI library on a machine without a GPU: it loads, exports every
function include/*.h declares, and rejects bad arguments with the documented
status codes before any CUDA call (no compute happens here)."""
import ctypes
import glob
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    from moe_decode_gemv_b200 import build
    build.build()
    from moe_decode_gemv_b200 import binding
    return binding


def declared_functions():
    names = []
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        text = open(h).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        for m in re.finditer(r"^\s*(?:const\s+)?[A-Za-z_][\w\s\*]*?\b([a-z_][a-z0-9_]*)\s*\(", text, flags=re.M):
            if m.group(1) not in ("if", "for", "while", "return", "sizeof"):
                names.append(m.group(1))
    return sorted(set(names))


def test_header_declares_the_abi():
    names = declared_functions()
    for n in ("moe_quantize_mxfp4", "moe_decode", "lmhead_quantize_fp8", "lmhead_decode"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    missing = [n for n in declared_functions() if not hasattr(lib.library, n)]
    assert not missing, missing


def test_status_strings_and_path(lib):
    L = lib.library
    for s in lib.Status:
        assert L.moe_status_string(int(s)).decode() == "MOE_" + ("OK" if s == 0 else "ERR_" + s.name)
    path = lib.moe_query_path()
    assert "sm_100a" in path and "MXFP4" in path and "FP8" in path


def test_workspace_sizes(lib):
    assert lib.moe_workspace_bytes(1, 8, 512, 2560, 768) > 0
    assert lib.moe_workspace_bytes(4, 8, 512, 2560, 768) > 0
    assert lib.moe_workspace_bytes(5, 8, 512, 2560, 768) == 0          # M > 4
    assert lib.moe_workspace_bytes(1, 9, 512, 2560, 768) == 0          # top_k > 8
    assert lib.moe_workspace_bytes(1, 8, 512, 2561, 768) == 0          # H not a multiple of 32
    assert lib.moe_workspace_bytes(1, 8, 512, 2560, 80) == 0           # I not a multiple of 32
    assert lib.moe_workspace_bytes(1, 8, 512, 3872, 768) == 0          # H above 3840 (shared memory)
    assert lib.moe_workspace_bytes(1, 8, 512, 3840, 768) > 0
    assert lib.moe_workspace_bytes(1, 8, 1025, 2560, 768) == 0         # more than 1024 experts
    assert lib.moe_workspace_bytes(1, 8, 512, 96, 32) > 0              # the smallest odd sizes
    assert lib.lmhead_workspace_bytes(1, 29, 157184, 2560) > 0
    assert lib.lmhead_workspace_bytes(1, 65, 157184, 2560) == 0
    assert lib.lmhead_workspace_bytes(1, 8, 4, 256) == 0                # top_k > vocab


# fake device addresses: aligned and unaligned, never dereferenced because
# every call below fails validation first
A = 0x7F0000000000
U = A + 4


def _mx(lib, fmt, count, rows, K, data=A, scales=A):
    return lib._Mxfp4(fmt, count, rows, K, data, scales)


def _bank(lib, fmt=2, E=16, H=256, I=64):
    return lib._Bank(_mx(lib, fmt, E, I, H), _mx(lib, fmt, E, I, H), _mx(lib, fmt, E, H, I))


def _packed(lib, fmt=4, E=16, H=256, I=64, units=A, dscales=A):
    return lib._Packed(fmt, E, H, I, units, dscales)


def _decode(lib, experts, shared, M=1, top_k=2, x=A, ws=A, ws_bytes=1 << 24):
    L = lib.library
    return L.moe_decode(x, A, None, ctypes.byref(experts), ctypes.byref(shared), M, top_k, A, None, None,
                        ws, ws_bytes, None)


def test_moe_decode_rejects_bad_arguments(lib):
    S = lib.Status
    ok_bank, ok_shared = _packed(lib), _packed(lib, E=1)
    # the integration trap: a bank tagged as something other than the packed MXFP4 layout
    assert _decode(lib, _packed(lib, fmt=2), ok_shared) == S.FORMAT_MISMATCH     # canonical MXFP4, not packed
    assert _decode(lib, ok_bank, _packed(lib, fmt=3, E=1)) == S.FORMAT_MISMATCH
    assert _decode(lib, ok_bank, ok_shared, M=0) == S.INVALID_ARG
    assert _decode(lib, ok_bank, ok_shared, M=5) == S.INVALID_ARG
    assert _decode(lib, ok_bank, ok_shared, top_k=9) == S.INVALID_ARG
    assert _decode(lib, ok_bank, ok_shared, x=0) == S.INVALID_ARG
    assert _decode(lib, ok_bank, ok_shared, x=U) == S.MISALIGNED
    assert _decode(lib, ok_bank, ok_shared, ws_bytes=100) == S.WORKSPACE
    assert _decode(lib, _packed(lib, H=250), _packed(lib, E=1, H=250)) == S.UNSUPPORTED_SHAPE
    assert _decode(lib, ok_bank, _packed(lib, E=2)) == S.UNSUPPORTED_SHAPE          # shared count != 1
    assert _decode(lib, ok_bank, _packed(lib, E=1, I=128)) == S.UNSUPPORTED_SHAPE   # shared width differs
    assert _decode(lib, _packed(lib, units=U), ok_shared) == S.MISALIGNED
    assert _decode(lib, _packed(lib, dscales=0), ok_shared) == S.INVALID_ARG


def test_pack_rejects_bad_arguments_and_sizes(lib):
    S, L = lib.Status, lib.library
    # sizes: one 16-row item is 32 gate/up rows of H/2 + H/32 bytes and 16 down
    # columns of H rows (8 bytes each); the down scales are H bytes per 32 columns
    assert L.moe_packed_units_bytes(512, 2560, 768) == 512 * 48 * (32 * (1280 + 80) + 2560 * 8)
    assert L.moe_packed_dscales_bytes(512, 2560, 768) == 512 * 24 * 2560
    assert L.moe_packed_units_bytes(512, 2560, 768) + L.moe_packed_dscales_bytes(512, 2560, 768) == 512 * 3133440
    assert L.moe_packed_units_bytes(1, 250, 64) == 0 and L.moe_packed_dscales_bytes(1, 256, 80) == 0

    def pack(src, dst):
        return L.moe_pack_experts(ctypes.byref(src), ctypes.byref(dst), None)

    assert pack(_bank(lib, fmt=1), _packed(lib, fmt=0)) == S.FORMAT_MISMATCH
    assert pack(_bank(lib), _packed(lib, fmt=0, E=8)) == S.UNSUPPORTED_SHAPE        # dst count differs
    assert pack(_bank(lib), _packed(lib, fmt=0, units=U)) == S.MISALIGNED
    assert pack(_bank(lib), _packed(lib, fmt=0, dscales=0)) == S.INVALID_ARG
    bad_down = lib._Bank(_mx(lib, 2, 16, 64, 256), _mx(lib, 2, 16, 64, 256), _mx(lib, 2, 16, 64, 256))
    assert pack(bad_down, _packed(lib, fmt=0)) == S.UNSUPPORTED_SHAPE               # down not [H][I]


def test_lmhead_rejects_bad_arguments(lib):
    S, L = lib.Status, lib.library

    def call(head, M=1, k=1, ids=A, ws_bytes=1 << 22, fn=L.lmhead_decode):
        return fn(A, ctypes.byref(head), M, k, ids, A, None, A, ws_bytes, None)

    fp8 = lib._Fp8Head(5, 4096, 256, A, A)
    # an FP8 head handed to the BF16 path, and a BF16-tagged head handed to the
    # FP8 path, are both refused instead of being read with the wrong format;
    # so is an FP8 head that was quantised but not tiled
    assert call(lib._Fp8Head(1, 4096, 256, A, A)) == S.FORMAT_MISMATCH
    assert call(lib._Bf16Head(3, 4096, 256, A), fn=L.lmhead_decode_bf16) == S.FORMAT_MISMATCH
    assert call(lib._Fp8Head(0, 4096, 256, A, A)) == S.FORMAT_MISMATCH
    assert call(lib._Fp8Head(3, 4096, 256, A, A)) == S.FORMAT_MISMATCH
    assert L.lmhead_decode_noalloc(A, ctypes.byref(lib._Fp8Head(3, 4096, 256, A, A)), 1, 1, A, A, None,
                                   None) == S.FORMAT_MISMATCH
    assert L.lmhead_noalloc_status(None, None) == S.INVALID_ARG  # checked before any CUDA call
    assert call(fp8, M=0) == S.INVALID_ARG
    assert call(fp8, k=65) == S.INVALID_ARG
    assert call(fp8, ids=0) == S.INVALID_ARG
    assert call(fp8, ids=U) == S.MISALIGNED
    assert call(fp8, ws_bytes=10) == S.WORKSPACE
    assert call(lib._Fp8Head(5, 4096, 100, A, A)) == S.UNSUPPORTED_SHAPE
    assert call(lib._Fp8Head(5, 4096, 8192, A, A)) == S.UNSUPPORTED_SHAPE
    assert call(lib._Fp8Head(5, 0, 256, A, A)) in (S.UNSUPPORTED_SHAPE, S.INVALID_ARG)


def test_head_tiling_sizes_and_arguments(lib):
    S, L = lib.Status, lib.library
    # whole 16-row tiles: 157,184 rows are 9,824 tiles; 4,100 rows round up to 4,112
    assert L.lmhead_tiled_bytes(157184, 2560) == 157184 * 2560
    assert L.lmhead_tiled_bytes(4100, 256) == 4112 * 256
    assert L.lmhead_tiled_bytes(4096, 100) == 0 and L.lmhead_tiled_bytes(0, 256) == 0
    src, dst = lib._Fp8Head(3, 4096, 256, A, A), lib._Fp8Head(0, 4096, 256, A, A)
    tile = lambda a, b: L.lmhead_tile_fp8(ctypes.byref(a), ctypes.byref(b), None)
    assert tile(lib._Fp8Head(5, 4096, 256, A, A), dst) == S.FORMAT_MISMATCH      # already tiled
    assert tile(src, lib._Fp8Head(0, 4095, 256, A, A)) == S.INVALID_ARG         # sizes differ
    assert tile(src, lib._Fp8Head(0, 4096, 256, U, A)) == S.MISALIGNED
    assert tile(src, lib._Fp8Head(0, 4096, 256, 0, A)) == S.INVALID_ARG


def test_quantizers_reject_bad_arguments(lib):
    S, L = lib.Status, lib.library
    t = _mx(lib, 0, 1, 8, 48)
    assert L.moe_quantize_mxfp4(A, ctypes.byref(t), None) == S.UNSUPPORTED_SHAPE   # K not a multiple of 32
    t = _mx(lib, 0, 1, 8, 64, data=U)
    assert L.moe_quantize_mxfp4(A, ctypes.byref(t), None) == S.MISALIGNED
    assert L.moe_quantize_mxfp4(None, ctypes.byref(_mx(lib, 0, 1, 8, 64)), None) == S.INVALID_ARG
    h = lib._Fp8Head(0, 16, 100, A, A)
    assert L.lmhead_quantize_fp8(A, ctypes.byref(h), None) == S.UNSUPPORTED_SHAPE
    h = lib._Fp8Head(0, 16, 256, U, A)
    assert L.lmhead_quantize_fp8(A, ctypes.byref(h), None) == S.MISALIGNED


def test_sampling_and_accept_reject_bad_arguments(lib):
    S, L = lib.Status, lib.library
    f = ctypes.c_float
    assert L.lmhead_sample(A, A, 1, 29, f(0.0), f(0.95), A, A, None) == S.INVALID_ARG   # temperature 0
    assert L.lmhead_sample(A, A, 1, 29, f(0.6), f(1.5), A, A, None) == S.INVALID_ARG    # top_p > 1
    assert L.lmhead_sample(A, A, 1, 65, f(0.6), f(0.95), A, A, None) == S.INVALID_ARG   # top_k > 64
    assert L.lmhead_sample(A, A, 0, 29, f(0.6), f(0.95), A, A, None) == S.INVALID_ARG   # M = 0
    assert L.lmhead_sample(None, A, 1, 29, f(0.6), f(0.95), A, A, None) == S.INVALID_ARG
    assert L.lmhead_sample(A + 2, A, 1, 29, f(0.6), f(0.95), A, A, None) == S.MISALIGNED
    assert L.moe_mtp_accept(A, A, 0, A, A, None) == S.INVALID_ARG
    assert L.moe_mtp_accept(A, A, 65, A, A, None) == S.INVALID_ARG
    assert L.moe_mtp_accept(A, None, 3, A, A, None) == S.INVALID_ARG
    assert L.moe_mtp_accept(A, A + 1, 3, A, A, None) == S.MISALIGNED


def test_moe_decode_rejects_out_of_range_shapes_and_pointers(lib):
    S, L = lib.Status, lib.library
    ok_bank, ok_shared = _packed(lib), _packed(lib, E=1)
    assert _decode(lib, _packed(lib, E=4), ok_shared, top_k=8) == S.UNSUPPORTED_SHAPE           # top_k > E
    assert _decode(lib, _packed(lib, E=1025), ok_shared) == S.UNSUPPORTED_SHAPE                 # E > 1024
    assert _decode(lib, _packed(lib, H=3872), _packed(lib, E=1, H=3872)) == S.UNSUPPORTED_SHAPE  # H > 3840
    assert _decode(lib, _packed(lib, I=65568), _packed(lib, E=1, I=65568)) == S.UNSUPPORTED_SHAPE
    assert _decode(lib, ok_bank, ok_shared, ws=0) == S.INVALID_ARG
    assert _decode(lib, ok_bank, ok_shared, ws=U) == S.MISALIGNED

    def call(router_w=A, bias=None, out=A, ids=None, w=None):
        return L.moe_decode(A, router_w, bias, ctypes.byref(ok_bank), ctypes.byref(ok_shared), 1, 2, out, ids, w,
                            A, 1 << 24, None)

    assert call(router_w=None) == S.INVALID_ARG
    assert call(out=None) == S.INVALID_ARG
    assert call(router_w=U) == S.MISALIGNED
    assert call(bias=U) == S.MISALIGNED
    assert call(out=U) == S.MISALIGNED
    assert call(ids=U) == S.MISALIGNED
    assert call(w=U) == S.MISALIGNED
    # a NULL experts or shared bank is an argument error, not a crash
    assert L.moe_decode(A, A, None, None, ctypes.byref(ok_shared), 1, 2, A, None, None, A, 1 << 24,
                        None) == S.INVALID_ARG
    assert L.moe_decode(A, A, None, ctypes.byref(ok_bank), None, 1, 2, A, None, None, A, 1 << 24,
                        None) == S.INVALID_ARG


def test_stream_glue_and_housekeeping_reject_bad_arguments(lib):
    S, L = lib.Status, lib.library
    # RMSNorm between layers: y [M][H] fp32 -> bf16, H a multiple of 8, eps >= 0
    assert L.moe_rmsnorm_bf16(None, 1, 256, 1e-6, A, None) == S.INVALID_ARG
    assert L.moe_rmsnorm_bf16(A, 0, 256, 1e-6, A, None) == S.INVALID_ARG
    assert L.moe_rmsnorm_bf16(A, 1, 100, 1e-6, A, None) == S.INVALID_ARG
    assert L.moe_rmsnorm_bf16(A, 1, 256, -1.0, A, None) == S.INVALID_ARG
    assert L.moe_rmsnorm_bf16(A, 1, 256, float("nan"), A, None) == S.INVALID_ARG
    assert L.moe_rmsnorm_bf16(U, 1, 256, 1e-6, A, None) == S.MISALIGNED
    assert L.moe_rmsnorm_bf16(A, 1, 256, 1e-6, U, None) == S.MISALIGNED
    # embedding gather for the next step's input
    assert L.moe_embed_gather(A, 0, 256, A, 1, 1, A, None) == S.INVALID_ARG
    assert L.moe_embed_gather(A, 1000, 12, A, 1, 1, A, None) == S.INVALID_ARG
    assert L.moe_embed_gather(A, 1000, 256, None, 1, 1, A, None) == S.INVALID_ARG
    assert L.moe_embed_gather(A, 1000, 256, A, 0, 1, A, None) == S.INVALID_ARG
    assert L.moe_embed_gather(A, 1000, 256, A, 1, 0, A, None) == S.INVALID_ARG
    assert L.moe_embed_gather(U, 1000, 256, A, 1, 1, A, None) == S.MISALIGNED
    assert L.moe_embed_gather(A, 1000, 256, A + 2, 1, 1, A, None) == S.MISALIGNED
    # the read-ceiling probe: whole 16-byte words from an aligned source
    assert L.moe_stream_read(A, 8, A, None) == S.INVALID_ARG
    assert L.moe_stream_read(A, 24, A, None) == S.INVALID_ARG
    assert L.moe_stream_read(None, 1 << 20, A, None) == S.INVALID_ARG
    assert L.moe_stream_read(U, 1 << 20, A, None) == S.MISALIGNED
    assert L.moe_stream_read(A, 1 << 20, A + 2, None) == S.MISALIGNED
    # workspaces and the bounded-wait self-test
    assert L.moe_workspace_reset(None, 1 << 20, None) == S.INVALID_ARG
    assert L.moe_workspace_reset(A, 8, None) == S.INVALID_ARG
    assert L.moe_workspace_status(None, None) == S.INVALID_ARG
    assert L.moe_selftest_wait_timeout(None, 64, 100, None) == S.WORKSPACE
    assert L.moe_selftest_wait_timeout(A, 8, 100, None) == S.WORKSPACE
    assert L.moe_selftest_wait_timeout(U, 64, 100, None) == S.MISALIGNED
    assert L.moe_selftest_wait_timeout(A, 64, 0, None) == S.INVALID_ARG
    assert L.moe_selftest_wait_timeout(A, 64, 1000001, None) == S.INVALID_ARG
    buf = ctypes.create_string_buffer(8)
    assert L.moe_query_path(None, 8) == S.INVALID_ARG
    assert L.moe_query_path(buf, 0) == S.INVALID_ARG
    # too small: the text's beginning, NUL-terminated, and an argument error
    assert L.moe_query_path(buf, 8) == S.INVALID_ARG and buf.value == b"sm_100a"
    big = ctypes.create_string_buffer(1024)
    assert L.moe_query_path(big, 1024) == S.OK and big.value.startswith(b"sm_100a;")
