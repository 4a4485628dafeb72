"""Thin Python binding of the C ABI in include/moe_gemv.h.

Argument marshalling only: every step of the hot path runs in the CUDA
kernels of libmoe_gemv.so.  Tensors are torch CUDA tensors (torch provides
device memory and streams); the calls pass their data pointers and the
current CUDA stream through ctypes.  Importing this module loads the
library and raises if it is missing -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import enum
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
library_path = os.path.join(_PKG, "libmoe_gemv.so")


class Status(enum.IntEnum):
    OK = 0
    INVALID_ARG = -1
    UNSUPPORTED_SHAPE = -2
    MISALIGNED = -3
    FORMAT_MISMATCH = -4
    WORKSPACE = -5
    CUDA = -6
    TIMEOUT = -7
    DEVICE_CHECK = -8


class Format(enum.IntEnum):
    NONE = 0
    BF16 = 1
    MXFP4_E2M1_E8M0_32 = 2
    FP8_E4M3_ROWSCALE_F32 = 3
    MXFP4_MOE_PACKED = 4
    FP8_E4M3_TILED = 5


class MoEError(RuntimeError):
    def __init__(self, status: int, call: str):
        self.status = Status(status)
        super().__init__(f"{call} returned {self.status.name}")


class _Mxfp4(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("count", ctypes.c_int32), ("rows", ctypes.c_int64),
                ("K", ctypes.c_int64), ("data", ctypes.c_void_p), ("scales", ctypes.c_void_p)]


class _Bank(ctypes.Structure):
    _fields_ = [("gate", _Mxfp4), ("up", _Mxfp4), ("down", _Mxfp4)]


class _Packed(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("count", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("units", ctypes.c_void_p), ("dscales", ctypes.c_void_p)]


class _Fp8Head(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("vocab", ctypes.c_int64), ("hidden", ctypes.c_int64),
                ("q", ctypes.c_void_p), ("row_scale", ctypes.c_void_p)]


class _Bf16Head(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("vocab", ctypes.c_int64), ("hidden", ctypes.c_int64),
                ("w", ctypes.c_void_p)]


def _load() -> ctypes.CDLL:
    if not os.path.exists(library_path):
        raise ImportError(f"{library_path} is missing: build it with `python -m moe_decode_gemv_b200.build` "
                          "(the CUDA path has no fallback)")
    L = ctypes.CDLL(library_path)
    P, I32, I64, SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
    sig = {
        "moe_quantize_mxfp4": ([P, ctypes.POINTER(_Mxfp4), P], I32),
        "lmhead_quantize_fp8": ([P, ctypes.POINTER(_Fp8Head), P], I32),
        "lmhead_tiled_bytes": ([I64, I64], SZ),
        "lmhead_tile_fp8": ([ctypes.POINTER(_Fp8Head), ctypes.POINTER(_Fp8Head), P], I32),
        "moe_workspace_bytes": ([I32, I32, I32, I32, I32], SZ),
        "moe_packed_units_bytes": ([I32, I32, I32], SZ),
        "moe_packed_dscales_bytes": ([I32, I32, I32], SZ),
        "moe_pack_experts": ([ctypes.POINTER(_Bank), ctypes.POINTER(_Packed), P], I32),
        "moe_decode": ([P, P, P, ctypes.POINTER(_Packed), ctypes.POINTER(_Packed), I32, I32, P, P, P, P, SZ, P], I32),
        "lmhead_workspace_bytes": ([I32, I32, I64, I64], SZ),
        "lmhead_decode": ([P, ctypes.POINTER(_Fp8Head), I32, I32, P, P, P, P, SZ, P], I32),
        "lmhead_decode_bf16": ([P, ctypes.POINTER(_Bf16Head), I32, I32, P, P, P, P, SZ, P], I32),
        "lmhead_decode_noalloc": ([P, ctypes.POINTER(_Fp8Head), I32, I32, P, P, P, P], I32),
        "lmhead_noalloc_status": ([ctypes.POINTER(I32), P], I32),
        "moe_rmsnorm_bf16": ([P, I32, I32, ctypes.c_float, P, P], I32),
        "moe_embed_gather": ([P, I64, I64, P, I32, I32, P, P], I32),
        "moe_workspace_reset": ([P, SZ, P], I32),
        "moe_workspace_status": ([P, P], I32),
        "moe_query_path": ([ctypes.c_char_p, SZ], I32),
        "moe_status_string": ([I32], ctypes.c_char_p),
        "moe_selftest_wait_timeout": ([P, SZ, ctypes.c_uint32, P], I32),
        "lmhead_sample": ([P, P, I32, I32, ctypes.c_float, ctypes.c_float, P, P, P], I32),
        "moe_stream_read": ([P, SZ, P, P], I32),
        "moe_mtp_accept": ([P, P, I32, P, P, P], I32),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    return L


library = _load()


def _check(status: int, call: str) -> None:
    if status != 0:
        raise MoEError(status, call)


def _ptr(t: torch.Tensor | None):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


# ---------------------------------------------------------------------------
# quantised containers
# ---------------------------------------------------------------------------

@dataclass
class MXFP4Bank:
    """A stack of `count` MXFP4 matrices [rows][K]: data [count, rows, K/2]
    uint8 (element 2j in the low nibble of byte j) and scales [count, rows,
    K/32] uint8 (E8M0)."""
    data: torch.Tensor
    scales: torch.Tensor
    fmt: int = Format.NONE

    @property
    def count(self) -> int:
        return self.data.shape[0]

    @property
    def rows(self) -> int:
        return self.data.shape[1]

    @property
    def K(self) -> int:
        return self.data.shape[2] * 2

    def _c(self) -> _Mxfp4:
        return _Mxfp4(int(self.fmt), self.count, self.rows, self.K, self.data.data_ptr(), self.scales.data_ptr())

    def nbytes(self) -> int:
        return self.data.numel() + self.scales.numel()


def alloc_mxfp4_bank(count: int, rows: int, K: int, device="cuda") -> MXFP4Bank:
    return MXFP4Bank(torch.empty((count, rows, K // 2), dtype=torch.uint8, device=device),
                     torch.empty((count, rows, K // 32), dtype=torch.uint8, device=device))


@dataclass
class PackedBank:
    """An expert bank laid out for moe_decode (moe_pack_experts): units
    [count * I/16 * 25 H] uint8 (one contiguous run per 16-row work item) and
    dscales [count * I/32 * H] uint8 (the down scales of each 32-column pair)."""
    units: torch.Tensor
    dscales: torch.Tensor
    count: int
    hidden: int
    inter: int
    fmt: int = Format.NONE

    def _c(self) -> _Packed:
        return _Packed(int(self.fmt), self.count, self.hidden, self.inter, self.units.data_ptr(),
                       self.dscales.data_ptr())

    def nbytes(self) -> int:
        return self.units.numel() + self.dscales.numel()


@dataclass
class FP8Head:
    """The online-FP8 LM head: q uint8 (E4M3) -- [V, H] as quantised, or the
    flat tiled bytes lmhead_decode reads -- and row_scale [V] fp32."""
    q: torch.Tensor
    row_scale: torch.Tensor
    fmt: int = Format.NONE
    vocab: int = 0
    hidden: int = 0

    def __post_init__(self):
        if self.q.dim() == 2 and not self.vocab:
            self.vocab, self.hidden = self.q.shape

    def _c(self) -> _Fp8Head:
        return _Fp8Head(int(self.fmt), self.vocab, self.hidden, self.q.data_ptr(), self.row_scale.data_ptr())


def alloc_fp8_head(vocab: int, hidden: int, device="cuda") -> FP8Head:
    return FP8Head(torch.empty((vocab, hidden), dtype=torch.uint8, device=device),
                   torch.empty((vocab,), dtype=torch.float32, device=device))


def _bank_c(gate: MXFP4Bank, up: MXFP4Bank, down: MXFP4Bank) -> _Bank:
    return _Bank(gate._c(), up._c(), down._c())


# ---------------------------------------------------------------------------
# entry points
# ---------------------------------------------------------------------------

def moe_quantize_mxfp4(w_bf16: torch.Tensor, out: MXFP4Bank | None = None, stream=None) -> MXFP4Bank:
    """bf16 [count, rows, K] (or [rows, K]) -> MXFP4 bank."""
    w = w_bf16 if w_bf16.dim() == 3 else w_bf16.unsqueeze(0)
    assert w.dtype == torch.bfloat16 and w.is_cuda and w.is_contiguous()
    if out is None:
        out = alloc_mxfp4_bank(w.shape[0], w.shape[1], w.shape[2], device=w.device)
    c = out._c()
    _check(library.moe_quantize_mxfp4(_ptr(w), ctypes.byref(c), _stream(stream)), "moe_quantize_mxfp4")
    out.fmt = c.fmt
    return out


def moe_pack_experts(bank: tuple[MXFP4Bank, MXFP4Bank, MXFP4Bank], stream=None) -> PackedBank:
    """(gate, up, down) quantised banks -> the packed bank moe_decode reads."""
    gate, up, down = bank
    E, H, I = gate.count, gate.K, gate.rows
    gb = int(library.moe_packed_units_bytes(E, H, I))
    db = int(library.moe_packed_dscales_bytes(E, H, I))
    if gb == 0 or db == 0:
        raise MoEError(Status.UNSUPPORTED_SHAPE, "moe_pack_experts")
    dev = gate.data.device
    out = PackedBank(torch.empty((gb,), dtype=torch.uint8, device=dev), torch.empty((db,), dtype=torch.uint8, device=dev),
                     E, H, I)
    src, c = _bank_c(gate, up, down), out._c()
    _check(library.moe_pack_experts(ctypes.byref(src), ctypes.byref(c), _stream(stream)), "moe_pack_experts")
    out.fmt = c.fmt
    return out


def lmhead_quantize_fp8(w_bf16: torch.Tensor, out: FP8Head | None = None, stream=None,
                        tiled: bool = True) -> FP8Head:
    """bf16 [V, H] -> the FP8 head; tiled (the default) re-lays it for
    lmhead_decode by lmhead_tile_fp8, else it stays [V, H]."""
    assert w_bf16.dtype == torch.bfloat16 and w_bf16.is_cuda and w_bf16.is_contiguous()
    if out is None:
        out = alloc_fp8_head(w_bf16.shape[0], w_bf16.shape[1], device=w_bf16.device)
    c = out._c()
    _check(library.lmhead_quantize_fp8(_ptr(w_bf16), ctypes.byref(c), _stream(stream)), "lmhead_quantize_fp8")
    out.fmt = c.fmt
    return lmhead_tile_fp8(out, stream=stream) if tiled else out


def lmhead_tile_fp8(head: FP8Head, stream=None) -> FP8Head:
    """A quantised [V, H] head -> the tiled head lmhead_decode reads (its row
    scales are shared with `head`)."""
    nbytes = int(library.lmhead_tiled_bytes(head.vocab, head.hidden))
    if nbytes == 0:
        raise MoEError(Status.UNSUPPORTED_SHAPE, "lmhead_tile_fp8")
    out = FP8Head(torch.empty((nbytes,), dtype=torch.uint8, device=head.q.device), head.row_scale,
                  vocab=head.vocab, hidden=head.hidden)
    src, c = head._c(), out._c()
    _check(library.lmhead_tile_fp8(ctypes.byref(src), ctypes.byref(c), _stream(stream)), "lmhead_tile_fp8")
    out.fmt = c.fmt
    return out


def moe_workspace_bytes(M: int, top_k: int, num_experts: int, hidden: int, inter: int) -> int:
    return int(library.moe_workspace_bytes(M, top_k, num_experts, hidden, inter))


def lmhead_workspace_bytes(M: int, top_k: int, vocab: int, hidden: int) -> int:
    return int(library.lmhead_workspace_bytes(M, top_k, vocab, hidden))


def new_workspace(nbytes: int, device="cuda", stream=None) -> torch.Tensor:
    """A zeroed workspace buffer (16-byte aligned torch allocation)."""
    ws = torch.empty((max(nbytes, 64),), dtype=torch.uint8, device=device)
    _check(library.moe_workspace_reset(_ptr(ws), ws.numel(), _stream(stream)), "moe_workspace_reset")
    return ws


def moe_decode(hidden: torch.Tensor, router_w: torch.Tensor, router_bias: torch.Tensor | None,
               experts: PackedBank, shared: PackedBank, top_k: int, out: torch.Tensor,
               topk_ids: torch.Tensor | None = None, topk_w: torch.Tensor | None = None,
               workspace: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One MoE layer: out[M, H] fp32 = sum_i w_i expert_i(x) + shared(x)."""
    M = hidden.shape[0]
    if workspace is None:
        workspace = new_workspace(moe_workspace_bytes(M, top_k, experts.count, experts.hidden, experts.inter),
                                  hidden.device, stream)
    eb, sb = experts._c(), shared._c()
    st = library.moe_decode(_ptr(hidden), _ptr(router_w), _ptr(router_bias), ctypes.byref(eb), ctypes.byref(sb),
                            M, top_k, _ptr(out), _ptr(topk_ids), _ptr(topk_w), _ptr(workspace), workspace.numel(),
                            _stream(stream))
    _check(st, "moe_decode")
    return out


def lmhead_decode(hidden: torch.Tensor, head: FP8Head, top_k: int, topk_ids: torch.Tensor, topk_vals: torch.Tensor,
                  logits: torch.Tensor | None = None, workspace: torch.Tensor | None = None, stream=None):
    M = hidden.shape[0]
    if workspace is None:
        workspace = new_workspace(lmhead_workspace_bytes(M, top_k, head.vocab, head.hidden),
                                  hidden.device, stream)
    c = head._c()
    st = library.lmhead_decode(_ptr(hidden), ctypes.byref(c), M, top_k, _ptr(topk_ids), _ptr(topk_vals), _ptr(logits),
                               _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "lmhead_decode")
    return topk_ids, topk_vals


def lmhead_decode_bf16(hidden: torch.Tensor, w_bf16: torch.Tensor, top_k: int, topk_ids: torch.Tensor,
                       topk_vals: torch.Tensor, logits: torch.Tensor | None = None,
                       workspace: torch.Tensor | None = None, stream=None):
    M = hidden.shape[0]
    if workspace is None:
        workspace = new_workspace(lmhead_workspace_bytes(M, top_k, w_bf16.shape[0], w_bf16.shape[1]),
                                  hidden.device, stream)
    c = _Bf16Head(int(Format.BF16), w_bf16.shape[0], w_bf16.shape[1], w_bf16.data_ptr())
    st = library.lmhead_decode_bf16(_ptr(hidden), ctypes.byref(c), M, top_k, _ptr(topk_ids), _ptr(topk_vals),
                                    _ptr(logits), _ptr(workspace), workspace.numel(), _stream(stream))
    _check(st, "lmhead_decode_bf16")
    return topk_ids, topk_vals


def lmhead_decode_noalloc(hidden: torch.Tensor, head: FP8Head, top_k: int, topk_ids: torch.Tensor,
                          topk_vals: torch.Tensor, logits: torch.Tensor | None = None, stream=None):
    """lmhead_decode without a workspace: for callers that cannot allocate
    device memory; the library's fixed scratch array is used instead (calls
    that overlap on the GPU race on it)."""
    c = head._c()
    st = library.lmhead_decode_noalloc(_ptr(hidden), ctypes.byref(c), hidden.shape[0], top_k, _ptr(topk_ids),
                                       _ptr(topk_vals), _ptr(logits), _stream(stream))
    _check(st, "lmhead_decode_noalloc")
    return topk_ids, topk_vals


def lmhead_noalloc_status(stream=None) -> int:
    """The first device status a lmhead_decode_noalloc launch reported since
    the last read (Status.OK if none), cleared by the read; waits for
    `stream`."""
    out = ctypes.c_int32(0)
    st = library.lmhead_noalloc_status(ctypes.byref(out), _stream(stream))
    _check(st, "lmhead_noalloc_status")
    return int(out.value)


def lmhead_sample(topk_ids: torch.Tensor, topk_vals: torch.Tensor, temperature: float, top_p: float,
                  uniforms: torch.Tensor, out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    """One draw per token from the head's sorted top-k (temperature, top-p);
    uniforms [M] fp32 in [0, 1) are the caller's random numbers."""
    M, k = topk_ids.shape
    if out is None:
        out = torch.empty((M,), dtype=torch.int32, device=topk_ids.device)
    _check(library.lmhead_sample(_ptr(topk_ids), _ptr(topk_vals), M, k, float(temperature), float(top_p),
                                 _ptr(uniforms), _ptr(out), _stream(stream)), "lmhead_sample")
    return out


def moe_mtp_accept(draft_ids: torch.Tensor, verify_ids: torch.Tensor, stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """Greedy acceptance of D drafts against D + 1 verify argmaxes; returns
    (emitted [D + 1] int32, n_emitted [1] int32), device tensors."""
    D = draft_ids.numel()
    emitted = torch.empty((D + 1,), dtype=torch.int32, device=draft_ids.device)
    n = torch.empty((1,), dtype=torch.int32, device=draft_ids.device)
    _check(library.moe_mtp_accept(_ptr(draft_ids), _ptr(verify_ids), D, _ptr(emitted), _ptr(n), _stream(stream)),
           "moe_mtp_accept")
    return emitted, n


def moe_stream_read(src: torch.Tensor, sink: torch.Tensor, stream=None) -> None:
    """Read all of `src` (measurement aid for the HBM read ceiling)."""
    nbytes = src.numel() * src.element_size() // 16 * 16
    _check(library.moe_stream_read(_ptr(src), nbytes, _ptr(sink), _stream(stream)), "moe_stream_read")


def moe_rmsnorm_bf16(y: torch.Tensor, out: torch.Tensor, eps: float = 1e-6, stream=None) -> torch.Tensor:
    """bf16 [M, H] = RMSNorm (gain 1) of fp32 [M, H]: the next layer's input."""
    M, H = y.shape
    _check(library.moe_rmsnorm_bf16(_ptr(y), M, H, float(eps), _ptr(out), _stream(stream)), "moe_rmsnorm_bf16")
    return out


def moe_embed_gather(table: torch.Tensor, ids: torch.Tensor, out: torch.Tensor, ids_stride: int = 1,
                     stream=None) -> torch.Tensor:
    """out[m] = table[ids[m * ids_stride]] (bf16 rows)."""
    V, H = table.shape
    st = library.moe_embed_gather(_ptr(table), V, H, _ptr(ids), ids_stride, out.shape[0], _ptr(out), _stream(stream))
    _check(st, "moe_embed_gather")
    return out


def moe_workspace_status(workspace: torch.Tensor, stream=None) -> Status:
    return Status(library.moe_workspace_status(_ptr(workspace), _stream(stream)))


def moe_selftest_wait_timeout(workspace: torch.Tensor, limit_us: int, stream=None) -> None:
    """Enqueue a bounded wait on a flag that nothing sets (limit in
    microseconds); the kernel records TIMEOUT in the workspace status word."""
    _check(library.moe_selftest_wait_timeout(_ptr(workspace), workspace.numel(), int(limit_us), _stream(stream)),
           "moe_selftest_wait_timeout")


def moe_query_path() -> str:
    buf = ctypes.create_string_buffer(1024)
    _check(library.moe_query_path(buf, len(buf)), "moe_query_path")
    return buf.value.decode()
