"""B200-native (sm_100a) weight-streaming hot path of batch-1 MoE decode.

Two operations, each a hand-written CUDA kernel chain behind a C ABI
(``include/moe_gemv.h``):

- the routed-expert MoE layer over MXFP4 weights (router GEMV, top-k softmax
  routing, gate/up GEMV, SiLU gate, down GEMV, shared expert, weighted
  combine) at M = 1 token and at the M = 4 verify step;
- the online-FP8 LM head (load-time per-row E4M3 quantisation, then a GEMV
  fused with the per-row scale and a top-k / argmax reduction).

``moe_decode_gemv_b200.inputs`` draws seeded synthetic inputs and needs no
GPU.  The ABI wrappers (``moe_decode``, ``lmhead_decode``...) live in
``moe_decode_gemv_b200.binding``; they load the compiled library on first
access and raise if it is missing -- there is no CPU fallback.
"""
from __future__ import annotations

_BINDING_NAMES = {
    "Status", "MoEError", "Format", "library", "library_path",
    "moe_quantize_mxfp4", "moe_pack_experts", "lmhead_quantize_fp8", "lmhead_tile_fp8",
    "moe_decode", "lmhead_decode", "lmhead_decode_bf16", "lmhead_decode_noalloc", "lmhead_noalloc_status",
    "lmhead_sample", "moe_mtp_accept", "moe_rmsnorm_bf16", "moe_embed_gather", "moe_stream_read",
    "moe_workspace_bytes", "lmhead_workspace_bytes", "new_workspace", "moe_workspace_status",
    "moe_query_path", "MXFP4Bank", "PackedBank", "FP8Head",
    "alloc_mxfp4_bank", "alloc_fp8_head",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
