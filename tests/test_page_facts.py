"""Facts the pages print, checked against the shapes and byte accounting this
library uses.  No GPU."""
import math

import pins
from moe_decode_gemv_b200 import accounting
from moe_decode_gemv_b200.inputs import LING_HEAD, LING_MOE, TINY_HEAD, TINY_MOE


def facts():
    return {row[0]: float(row[1]) for row in pins.read_golden("page_facts.txt")}


def test_ling_shapes_match_pages():
    f = facts()
    assert LING_MOE.experts == f["routed_experts"]
    assert LING_MOE.top_k == f["experts_per_token"]
    assert LING_MOE.inter == f["expert_intermediate"]
    assert LING_HEAD.vocab == f["lmhead_vocab"] and LING_HEAD.hidden == f["lmhead_hidden"]
    # the MoE layer's input is the model hidden size, the LM head's input width
    assert LING_MOE.hidden == LING_HEAD.hidden


def test_sparsity_arithmetic():
    f = facts()
    # about 4.1 percent of parameters active: 5.1B / 124B
    assert round(100 * f["active_params"] / f["total_params"], 1) == f["active_fraction_percent"]
    # the router's own sparsity is 8 of 512, i.e. 1 in 64 -- a different figure
    assert f["routed_experts"] / f["experts_per_token"] == f["router_sparsity_inverse"]
    assert not math.isclose(1 / f["router_sparsity_inverse"], f["active_fraction_percent"] / 100, rel_tol=0.1)
    # four verify positions wake at most 4 x 8 = 32 routed experts
    assert f["verify_positions"] * f["experts_per_token"] == f["verify_max_experts"]


def test_fp8_head_halves_the_reads():
    f = facts()
    bf16 = accounting.lmhead_bf16_bytes(LING_HEAD)
    assert bf16 == 804_782_080
    fp8_weights = LING_HEAD.vocab * LING_HEAD.hidden
    assert fp8_weights == 402_391_040 and fp8_weights / bf16 == f["fp8_head_read_ratio"]
    assert accounting.lmhead_fp8_bytes(LING_HEAD) == 402_391_040 + 628_736  # + fp32 row scales


def test_layer_bytes():
    assert accounting.mxfp4_row_bytes(2560) == 1280 + 80
    assert accounting.mxfp4_row_bytes(768) == 384 + 24
    assert accounting.expert_bytes(LING_MOE) == 3_133_440
    assert accounting.router_bytes(LING_MOE) == 5_242_880
    assert accounting.moe_layer_bytes(LING_MOE, 8) == 33_443_840
    assert accounting.moe_layer_bytes(LING_MOE, 32) == 108_646_400
    assert accounting.moe_layer_bytes(TINY_MOE, 2) == 16_384 + 3 * 26_112
    assert accounting.lmhead_fp8_bytes(TINY_HEAD) == 1_048_576 + 16_384
