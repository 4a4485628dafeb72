"""Failure detection without a GPU fault: a device wait that can never
complete ends, after its time limit, with MOE_ERR_TIMEOUT in the workspace
status word, and the context stays usable for the next calls."""
import time

import pytest
import torch

import oracle
from gpu_support import Layer, check_moe
from moe_decode_gemv_b200 import inputs as I

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from moe_decode_gemv_b200 import build
    build.build()
    from moe_decode_gemv_b200 import binding
    return binding


def test_wait_on_unset_flag_times_out_and_reports(B):
    ws = B.new_workspace(4096, "cuda")
    assert B.moe_workspace_status(ws) == B.Status.OK
    t0 = time.perf_counter()
    B.moe_selftest_wait_timeout(ws, 20_000)  # 20 ms
    st = B.moe_workspace_status(ws)  # synchronises the stream
    elapsed = time.perf_counter() - t0
    assert st == B.Status.TIMEOUT
    assert 0.015 < elapsed < 5.0  # the wait ran out near its limit, not at once and not never
    assert B.moe_workspace_status(ws) == B.Status.OK  # reading the status clears it


def test_context_usable_after_timeout(B):
    ws = B.new_workspace(4096, "cuda")
    B.moe_selftest_wait_timeout(ws, 5_000)
    assert B.moe_workspace_status(ws) == B.Status.TIMEOUT
    O = oracle.load()
    layer = Layer(B, 0, I.TINY_MOE)
    x = I.hidden_states(5, 1, I.TINY_MOE.hidden)
    y, ids, w = layer.run_gpu(x.cuda())
    check_moe(layer, O, x, y, ids, w)
    t = B.new_workspace(4096, "cuda")
    assert B.moe_workspace_status(t) == B.Status.OK


def test_selftest_rejects_bad_arguments(B):
    ws = B.new_workspace(4096, "cuda")
    for limit in (0, 1_000_001):
        with pytest.raises(B.MoEError):
            B.moe_selftest_wait_timeout(ws, limit)
    with pytest.raises(B.MoEError):
        B.moe_selftest_wait_timeout(ws[:32], 1000)
