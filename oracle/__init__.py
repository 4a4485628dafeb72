"""CPU oracle for MXFP4 MoE decode and the online-FP8 LM head (fp64, plain C).

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the
benchmark's CPU-baseline leg are the only callers.  The CUDA library never
imports, links or calls anything here, and nothing here is shared with it.

This module compiles ``oracle.c`` with gcc when the shared object is missing
or older than its source, and wraps each C function for numpy arrays.  bf16
data travels as ``numpy.uint16`` bit patterns; packed MXFP4 and E4M3 data as
``numpy.uint8``.  The C header ``oracle.h`` states what each function computes
and which passage of the pages or the format specification it follows.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "oracle.c")
HEADER = os.path.join(_HERE, "oracle.h")
LIBRARY = os.path.join(_HERE, "liboracle.so")
CFLAGS = ["-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fPIC", "-shared"]


def build(source: str = SOURCE, out: str = LIBRARY, force: bool = False) -> str:
    """Compile the oracle into a shared object (gcc, no CUDA)."""
    stale = (not os.path.exists(out)
             or os.path.getmtime(out) < max(os.path.getmtime(source), os.path.getmtime(HEADER)))
    if force or stale:
        cmd = ["gcc", *CFLAGS, "-I", _HERE, source, "-o", out + ".tmp", "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(out + ".tmp", out)
    return out


_P = ctypes.c_void_p
_I64 = ctypes.c_int64
_INT = ctypes.c_int
_DBL = ctypes.c_double


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _u16(a) -> np.ndarray:
    """Accept a numpy uint16 array or a torch bfloat16 tensor; return uint16 bits."""
    if hasattr(a, "dtype") and str(a.dtype) == "torch.bfloat16":
        import torch
        return a.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)
    a = np.ascontiguousarray(a)
    assert a.dtype == np.uint16, a.dtype
    return a


class Oracle:
    """ctypes view of one compiled oracle library."""

    def __init__(self, path: str):
        self.path = path
        L = ctypes.CDLL(path)
        self._L = L
        L.orc_bf16_to_double.restype = _DBL
        L.orc_bf16_to_double.argtypes = [ctypes.c_uint16]
        for n in ("orc_e2m1_to_double", "orc_e8m0_to_double", "orc_e4m3_to_double"):
            getattr(L, n).restype = _DBL
            getattr(L, n).argtypes = [ctypes.c_uint]
        L.orc_e2m1_encode.restype = ctypes.c_uint
        L.orc_e2m1_encode.argtypes = [_DBL]
        L.orc_e4m3_encode_satfinite.restype = ctypes.c_uint
        L.orc_e4m3_encode_satfinite.argtypes = [_DBL]
        L.orc_double_to_bf16.restype = ctypes.c_uint16
        L.orc_double_to_bf16.argtypes = [_DBL]
        L.orc_mxfp4_quantize.argtypes = [_I64, _I64, _P, _P, _P]
        L.orc_mxfp4_element.restype = _DBL
        L.orc_mxfp4_element.argtypes = [_I64, _P, _P, _I64, _I64]
        L.orc_fp8_rowquant.argtypes = [_I64, _I64, _P, _P, _P]
        L.orc_router.argtypes = [_INT, _INT, _INT, _INT, _P, _P, _P, _P, _P, _P]
        L.orc_expert_mlp.argtypes = [_INT, _INT, _P] + [_P] * 6 + [_P, _P]
        L.orc_moe_layer.argtypes = [_INT, _INT, _INT, _INT, _P, _P, _P] + [_P] * 12 + [_P]
        L.orc_lmhead_fp8.argtypes = [_I64, _I64, _INT, _P, _P, _P, _P, _P]
        L.orc_lmhead_bf16.argtypes = [_I64, _I64, _INT, _P, _P, _P]
        L.orc_topk.argtypes = [_I64, _P, _INT, _P, _P]
        L.orc_sample_topk.restype = _INT
        L.orc_sample_topk.argtypes = [_INT, _P, _DBL, _DBL, _DBL]
        L.orc_mtp_accept.restype = _INT
        L.orc_mtp_accept.argtypes = [_INT, _P, _P, _P]
        L.orc_rmsnorm_bf16.argtypes = [_INT, _P, _DBL, _P]

    # ---- scalar formats -------------------------------------------------
    def bf16_to_double(self, bits: int) -> float:
        return self._L.orc_bf16_to_double(int(bits))

    def e2m1(self, code: int) -> float:
        return self._L.orc_e2m1_to_double(int(code))

    def e8m0(self, code: int) -> float:
        return self._L.orc_e8m0_to_double(int(code))

    def e4m3(self, code: int) -> float:
        return self._L.orc_e4m3_to_double(int(code))

    def e2m1_encode(self, v: float) -> int:
        return int(self._L.orc_e2m1_encode(float(v)))

    def e4m3_encode(self, v: float) -> int:
        return int(self._L.orc_e4m3_encode_satfinite(float(v)))

    def double_to_bf16(self, v: float) -> int:
        return int(self._L.orc_double_to_bf16(float(v)))

    # ---- quantisers ------------------------------------------------------
    def mxfp4_quantize(self, w_bf16) -> tuple[np.ndarray, np.ndarray]:
        """[..., K] bf16 -> (data [..., K/2] u8, scales [..., K/32] u8)."""
        w = _u16(w_bf16)
        K = w.shape[-1]
        assert K % 32 == 0
        rows = w.size // K
        data = np.empty(w.shape[:-1] + (K // 2,), np.uint8)
        scales = np.empty(w.shape[:-1] + (K // 32,), np.uint8)
        self._L.orc_mxfp4_quantize(rows, K, _ptr(w), _ptr(data), _ptr(scales))
        return data, scales

    def mxfp4_dequantize(self, data: np.ndarray, scales: np.ndarray) -> np.ndarray:
        """Element-by-element dequantisation of a [rows, K] MXFP4 matrix (slow)."""
        rows, K = data.shape[0], data.shape[1] * 2
        d = np.ascontiguousarray(data)
        s = np.ascontiguousarray(scales)
        out = np.empty((rows, K), np.float64)
        f = self._L.orc_mxfp4_element
        for r in range(rows):
            for j in range(K):
                out[r, j] = f(K, _ptr(d), _ptr(s), r, j)
        return out

    def fp8_rowquant(self, w_bf16) -> tuple[np.ndarray, np.ndarray]:
        """[V, H] bf16 -> (q [V, H] u8 E4M3, s [V] f32)."""
        w = _u16(w_bf16)
        V, H = w.shape
        q = np.empty((V, H), np.uint8)
        s = np.empty((V,), np.float32)
        self._L.orc_fp8_rowquant(V, H, _ptr(w), _ptr(q), _ptr(s))
        return q, s

    # ---- router / experts -----------------------------------------------
    def router(self, x_bf16, Wr: np.ndarray, bias: np.ndarray | None, k: int):
        """-> (logits [M,E] f64, ids [M,k] i32, w [M,k] f64)."""
        x = _u16(x_bf16)
        M, H = x.shape
        Wr = np.ascontiguousarray(Wr, np.float32)
        E = Wr.shape[0]
        b = None if bias is None else np.ascontiguousarray(bias, np.float32)
        logits = np.empty((M, E), np.float64)
        ids = np.empty((M, k), np.int32)
        w = np.empty((M, k), np.float64)
        self._L.orc_router(M, E, H, k, _ptr(x), _ptr(Wr), _ptr(b), _ptr(logits), _ptr(ids), _ptr(w))
        return logits, ids, w

    def expert_mlp(self, x_bf16, gate, up, down):
        """One token through one expert; gate/up/down are (data, scales) pairs.
        -> (out [H] f64, h [I] f64)."""
        x = _u16(x_bf16).reshape(-1)
        H = x.shape[0]
        I = gate[0].shape[-2]
        out = np.empty((H,), np.float64)
        h = np.empty((I,), np.float64)
        args = [np.ascontiguousarray(a) for a in (*gate, *up, *down)]
        self._L.orc_expert_mlp(H, I, _ptr(x), *[_ptr(a) for a in args], _ptr(out), _ptr(h))
        return out, h

    def moe_layer(self, x_bf16, ids: np.ndarray, w: np.ndarray, bank: dict, shared: dict):
        """y [M,H] f64.  bank/shared map 'gate'/'up'/'down' to (data, scales),
        stacked over experts ([E, rows, K/2], [E, rows, K/32]); only the experts
        in ids are read, so unused experts may hold anything."""
        x = _u16(x_bf16)
        M, H = x.shape
        k = ids.shape[1]
        I = bank["gate"][0].shape[-2]
        ids = np.ascontiguousarray(ids, np.int32)
        w = np.ascontiguousarray(w, np.float64)
        y = np.empty((M, H), np.float64)
        parts = []
        for src in (bank, shared):
            for name in ("gate", "up", "down"):
                parts += [np.ascontiguousarray(a) for a in src[name]]
        self._L.orc_moe_layer(M, H, I, k, _ptr(x), _ptr(ids), _ptr(w),
                              *[_ptr(a) for a in parts], _ptr(y))
        return y

    # ---- LM head ----------------------------------------------------------
    def lmhead_fp8(self, x_bf16, q: np.ndarray, s: np.ndarray, want_abssum: bool = False):
        """-> logits [M,V] f64 (and abssum [M,V] f64 when asked)."""
        x = _u16(x_bf16)
        M, H = x.shape
        V = q.shape[0]
        q = np.ascontiguousarray(q, np.uint8)
        s = np.ascontiguousarray(s, np.float32)
        logits = np.empty((M, V), np.float64)
        abss = np.empty((M, V), np.float64) if want_abssum else None
        self._L.orc_lmhead_fp8(V, H, M, _ptr(x), _ptr(q), _ptr(s), _ptr(logits), _ptr(abss))
        return (logits, abss) if want_abssum else logits

    def lmhead_bf16(self, x_bf16, w_bf16) -> np.ndarray:
        x = _u16(x_bf16)
        w = _u16(w_bf16)
        M, H = x.shape
        V = w.shape[0]
        logits = np.empty((M, V), np.float64)
        self._L.orc_lmhead_bf16(V, H, M, _ptr(x), _ptr(w), _ptr(logits))
        return logits

    def topk(self, v: np.ndarray, k: int):
        """-> (ids [k] i32, vals [k] f64), descending, ties to the lower index."""
        v = np.ascontiguousarray(v, np.float64)
        ids = np.empty((k,), np.int32)
        vals = np.empty((k,), np.float64)
        self._L.orc_topk(v.shape[0], _ptr(v), k, _ptr(ids), _ptr(vals))
        return ids, vals

    def sample_topk(self, vals, temperature: float, top_p: float, u: float) -> int:
        v = np.ascontiguousarray(np.asarray(vals, dtype=np.float64))
        return int(self._L.orc_sample_topk(len(v), _ptr(v), float(temperature), float(top_p), float(u)))

    def mtp_accept(self, draft, verify) -> np.ndarray:
        d = np.ascontiguousarray(np.asarray(draft, dtype=np.int32))
        v = np.ascontiguousarray(np.asarray(verify, dtype=np.int32))
        assert len(v) == len(d) + 1
        out = np.zeros(len(v), np.int32)
        n = self._L.orc_mtp_accept(len(d), _ptr(d), _ptr(v), _ptr(out))
        return out[:n]

    def rmsnorm_bf16(self, y: np.ndarray, eps: float = 1e-6) -> np.ndarray:
        y = np.ascontiguousarray(y, np.float64)
        out = np.empty(y.shape, np.uint16)
        self._L.orc_rmsnorm_bf16(y.shape[0], _ptr(y), float(eps), _ptr(out))
        return out


_DEFAULT: Oracle | None = None


def load(path: str | None = None) -> Oracle:
    """The oracle compiled from this directory (built on first use), or the
    library at ``path``."""
    global _DEFAULT
    if path is not None:
        return Oracle(path)
    if _DEFAULT is None:
        _DEFAULT = Oracle(build())
    return _DEFAULT
