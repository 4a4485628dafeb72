"""The workspace-free LM-head entry point, for callers that cannot allocate
device memory (a host that owns every allocation and hands a plugin only its
inputs and outputs, or a loop where cudaMalloc is not allowed).

It must agree with lmhead_decode, which takes a caller workspace, on two calls
in a row (the second reuses the scratch the first left behind), and refuse a
request too large for its fixed scratch.  Collected last on purpose."""
import ctypes

import numpy as np
import pytest
import torch

from gpu_support import MAX_ABS_TOL, REL_L2_TOL, rel_l2
from moe_decode_gemv_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from moe_decode_gemv_b200 import build
    build.build()
    from moe_decode_gemv_b200 import binding
    return binding


def _outputs(M, k, V, dev="cuda"):
    return (torch.empty((M, k), dtype=torch.int32, device=dev), torch.empty((M, k), dtype=torch.float32, device=dev),
            torch.empty((M, V), dtype=torch.float32, device=dev))


@pytest.mark.parametrize("shape,M,k", [(I.TINY_HEAD, 1, 1), (I.TINY_HEAD, 4, 29), (I.LING_HEAD, 1, 29),
                                       (I.LING_HEAD, 4, 29)])
def test_matches_workspace_entry_point_twice(B, shape, M, k):
    head = B.lmhead_quantize_fp8(I.lmhead_weight(0, shape).cuda())
    ref_ids, ref_vals, ref_logits = _outputs(M, k, shape.vocab)
    for call in range(2):
        x = I.hidden_states(call, M, shape.hidden, tag="noalloc").cuda()
        B.lmhead_decode(x, head, k, ref_ids, ref_vals, ref_logits)
        ids, vals, logits = _outputs(M, k, shape.vocab)
        B.lmhead_decode_noalloc(x, head, k, ids, vals, logits)
        torch.cuda.synchronize()
        assert torch.equal(ids, ref_ids), f"call {call}: ids differ"
        v, rv = vals.cpu().numpy(), ref_vals.cpu().numpy()
        assert np.abs(v - rv).max() <= MAX_ABS_TOL
        lg, rlg = logits.cpu().numpy(), ref_logits.cpu().numpy()
        assert rel_l2(lg, rlg) <= REL_L2_TOL and np.abs(lg - rlg).max() <= MAX_ABS_TOL
    assert B.lmhead_noalloc_status() == B.Status.OK  # no device error since the last read


def _need(G, M, k):
    """Scratch bytes of one call: the 64-byte header, then M lists of G x k
    candidates of 8 bytes, each list rounded up to an even entry count."""
    return 64 + M * ((G * k + 1) & ~1) * 8


def _raw(B, x, head, M, k, ids, vals, logits=None):
    c = head._c()
    return B.library.lmhead_decode_noalloc(ctypes.c_void_p(x.data_ptr()), ctypes.byref(c), M, k,
                                           ctypes.c_void_p(ids.data_ptr()), ctypes.c_void_p(vals.data_ptr()),
                                           None if logits is None else ctypes.c_void_p(logits.data_ptr()), None)


def test_refuses_requests_beyond_its_scratch(B):
    """M x top_k candidate lists for every SM must fit the fixed scratch."""
    head = B.lmhead_quantize_fp8(I.lmhead_weight(0, I.TINY_HEAD).cuda())
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    M, k = 4, 64
    need = _need(min(sms, I.TINY_HEAD.vocab // 16), M, k)
    x = I.hidden_states(0, M, I.TINY_HEAD.hidden).cuda()
    ids, vals, _ = _outputs(M, k, I.TINY_HEAD.vocab)
    st = _raw(B, x, head, M, k, ids, vals)  # raw C call: expect a status, not an exception
    expected = B.Status.WORKSPACE if need > 256 * 1024 else B.Status.OK
    assert st == expected, (st, need)
    torch.cuda.synchronize()
    assert B.lmhead_noalloc_status() == B.Status.OK


def test_largest_request_that_fits_and_the_next(B):
    """On the Ling head at M = 4: the largest top_k whose lists fit the scratch
    runs and matches lmhead_decode; one more is refused with WORKSPACE."""
    shape, M = I.LING_HEAD, 4
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    G = min(sms, shape.vocab // 16)
    fits = [k for k in range(1, 65) if _need(G, M, k) <= 256 * 1024]
    k = max(fits)
    head = B.lmhead_quantize_fp8(I.lmhead_weight(0, shape).cuda())
    x = I.hidden_states(5, M, shape.hidden, tag="noalloc-limit").cuda()
    ref_ids, ref_vals, _ = _outputs(M, k, shape.vocab)
    B.lmhead_decode(x, head, k, ref_ids, ref_vals)
    ids, vals, _ = _outputs(M, k, shape.vocab)
    assert _raw(B, x, head, M, k, ids, vals) == B.Status.OK
    torch.cuda.synchronize()
    assert torch.equal(ids, ref_ids)
    assert np.abs(vals.cpu().numpy() - ref_vals.cpu().numpy()).max() <= MAX_ABS_TOL
    assert B.lmhead_noalloc_status() == B.Status.OK
    if k < 64:
        ids2, vals2, _ = _outputs(M, k + 1, shape.vocab)
        assert _raw(B, x, head, M, k + 1, ids2, vals2) == B.Status.WORKSPACE
    print(f"no-alloc limit on {sms} SMs at M={M}: top_k {k} runs, {k + 1} is refused")
