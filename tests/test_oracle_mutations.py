"""Planted mistakes in the CPU oracle must be caught by its pins.

Each case copies oracle.c, applies one plausible mistake (a dropped term, a
wrong sign, bias or index, a transposed operand, a wrong tie rule), compiles
the copy with gcc into a temporary directory, and runs the pins against it:
at least one pin must fail.  This shows that the pins in tests/pins.py
constrain every step of the oracle.  No GPU; nothing here touches the CUDA
library.
"""
import os
import shutil
import subprocess

import pytest

import oracle
import pins

MUTATIONS = {
    "nibble_order_decode": ("unsigned code = (j & 1) ? (unsigned)(byte >> 4) : (unsigned)(byte & 15u);",
                            "unsigned code = (j & 1) ? (unsigned)(byte & 15u) : (unsigned)(byte >> 4);"),
    "nibble_order_pack": ("d[i / 2] = (uint8_t)(lo | (hi << 4));", "d[i / 2] = (uint8_t)(hi | (lo << 4));"),
    "mx_scale_exponent": ("xexp = (e - 1) - 2;", "xexp = (e - 1) - 1;"),
    "mx_amax_signed": ("else if (fabs(v) > amax)", "else if (v > amax)"),
    "e2m1_subnormal": ("0.5 * (double)m : ldexp", "1.0 * (double)m : ldexp"),
    "e2m1_tie_odd": ("(err == best_err && (c & 1u) == 0u)", "(err == best_err && (c & 1u) == 1u)"),
    "e8m0_bias": ("return ldexp(1.0, (int)code - 127);", "return ldexp(1.0, (int)code - 126);"),
    "e4m3_bias": ("ldexp(1.0 + (double)m / 8.0, (int)e - 7)", "ldexp(1.0 + (double)m / 8.0, (int)e - 8)"),
    "e4m3_no_satfinite": ("mag = 0x7Eu;", "mag = 0x7Fu;"),
    "e4m3_truncate": ("double t = nearbyint(f * 16.0);", "double t = floor(f * 16.0);"),
    "fp8_scale_447": ("amax / 448.0f", "amax / 447.0f"),
    "fp8_multiply_scale": ("float t = (float)orc_bf16_to_double(row[j]) / sv;",
                           "float t = (float)orc_bf16_to_double(row[j]) * sv;"),
    "topk_tie_upper": ("if (best < 0 || v[j] > v[best])", "if (best < 0 || v[j] >= v[best])"),
    "router_weight_sign": ("w[(int64_t)m * k + i] = exp(sel[i] - sel[0]) / z;",
                           "w[(int64_t)m * k + i] = exp(sel[0] - sel[i]) / z;"),
    "router_bias_dropped": ("acc += (double)bias[e];", "acc += 0.0;"),
    "silu_on_up": ("h[r] = g / (1.0 + exp(-g)) * u;", "h[r] = u / (1.0 + exp(-u)) * g;"),
    "sigmoid_sign": ("h[r] = g / (1.0 + exp(-g)) * u;", "h[r] = g / (1.0 + exp(g)) * u;"),
    "down_transposed": ("orc_mxfp4_element(I, down_d, down_s, i, r)", "orc_mxfp4_element(I, down_d, down_s, r, i)"),
    "shared_dropped": ("        for (int j = 0; j < H; ++j)\n            ym[j] += out[j];",
                       "        for (int j = 0; j < H; ++j)\n            ym[j] += 0.0 * out[j];"),
    "combine_weight_dropped": ("ym[j] += w[(int64_t)m * k + i] * out[j];", "ym[j] += out[j];"),
    "lmhead_scale_dropped": ("logits[(int64_t)m * V + v] = (double)s[v] * acc;", "logits[(int64_t)m * V + v] = acc;"),
    "bf16_truncate": ("double t = nearbyint(ldexp(f, 8));", "double t = floor(ldexp(f, 8));"),
    "rmsnorm_mean": ("sqrt(ss / (double)H + eps)", "sqrt(ss / (double)(H - 1) + eps)"),
    "sample_temperature_multiplies": ("p[i] = exp((vals[i] - vals[0]) / temperature);",
                                      "p[i] = exp((vals[i] - vals[0]) * temperature);"),
    "sample_nucleus_inclusive": ("while (n < k && before < top_p * total) {", "while (n < k && before <= top_p * total) {"),
    "sample_draw_unnormalised": ("const double r = u * kept;", "const double r = u * total;"),
    "mtp_accept_skips_mismatch": ("while (a < D && draft[a] == verify[a]) {", "while (a < D && draft[a] != verify[a] + 1) {"),
    # a second batch: indexing, sign and special-value slips
    "e2m1_sign_bit": ("unsigned s = (code >> 3) & 1u, e = (code >> 1) & 3u", "unsigned s = (code >> 2) & 1u, e = (code >> 1) & 3u"),
    "e8m0_nan_as_inf": ("        return NAN;\n    return ldexp(1.0, (int)code - 127);",
                        "        return INFINITY;\n    return ldexp(1.0, (int)code - 127);"),
    "e4m3_subnormal_scale": ("ldexp((double)m, -9) : ldexp", "ldexp((double)m, -10) : ldexp"),
    "e4m3_binade_carry": ("            t = 8.0;\n            E += 1;", "            t = 8.0;"),
    "bf16_sign_dropped": ("return signbit(v) ? (uint16_t)(b | 0x8000u) : b;", "return b;"),
    "mx_block_scale_index": ("g_e8m0[scales[r * (K / 32) + j / 32]]", "g_e8m0[scales[r * (K / 32)]]"),
    "mx_nonfinite_block_scale": ("scales[r * nb + b] = 0xFFu;", "scales[r * nb + b] = 0x00u;"),
    "mx_zero_block_scale": ("                xexp = -127;\n            } else {", "                xexp = 0;\n            } else {"),
    "fp8_amax_signed": ("float a = fabsf((float)orc_bf16_to_double(row[j]));", "float a = (float)orc_bf16_to_double(row[j]);"),
    "fp8_zero_row_scale": ("(amax == 0.0f) ? 1.0f : amax / 448.0f", "(amax == 0.0f) ? 0.0f : amax / 448.0f"),
    "topk_ascending": ("if (best < 0 || v[j] > v[best])", "if (best < 0 || v[j] < v[best])"),
    "router_token0": ("acc += orc_bf16_to_double(x_bf16[(int64_t)m * H + j]) * (double)Wr[(int64_t)e * H + j];",
                      "acc += orc_bf16_to_double(x_bf16[j]) * (double)Wr[(int64_t)e * H + j];"),
    "router_not_renormalised": ("        for (int i = 0; i < k; ++i)\n            z += exp(sel[i] - sel[0]);",
                                "        for (int i = 0; i < E; ++i)\n            z += exp(lg[i] - sel[0]);"),
    "down_uses_gate_scales": ("orc_mxfp4_element(I, down_d, down_s, i, r)", "orc_mxfp4_element(I, down_d, gate_s, i, r)"),
    "layer_token0": ("const uint16_t* xm = x_bf16 + (int64_t)m * H;", "const uint16_t* xm = x_bf16;"),
    "shared_weighted": ("        for (int j = 0; j < H; ++j)\n            ym[j] += out[j];",
                        "        for (int j = 0; j < H; ++j)\n            ym[j] += w[(int64_t)m * k] * out[j];"),
    "lmhead_token0": ("            xd[j] = orc_bf16_to_double(x_bf16[(int64_t)m * H + j]);\n        for (int64_t v = 0; v < V; ++v) {\n            const uint8_t* row",
                      "            xd[j] = orc_bf16_to_double(x_bf16[j]);\n        for (int64_t v = 0; v < V; ++v) {\n            const uint8_t* row"),
    "lmhead_bf16_token0": ("            xd[j] = orc_bf16_to_double(x_bf16[(int64_t)m * H + j]);\n        for (int64_t v = 0; v < V; ++v) {\n            double acc",
                           "            xd[j] = orc_bf16_to_double(x_bf16[j]);\n        for (int64_t v = 0; v < V; ++v) {\n            double acc"),
    "rmsnorm_eps_outside": ("sqrt(ss / (double)H + eps)", "sqrt(ss / (double)H) + eps"),
    "mtp_emits_draft_after_accept": ("        emitted[a] = draft[a];\n        ++a;", "        emitted[a] = verify[a + 1 < D ? a + 1 : a];\n        ++a;"),
}


@pytest.fixture(scope="module")
def workdir(tmp_path_factory):
    d = tmp_path_factory.mktemp("mutants")
    shutil.copy(oracle.HEADER, d / "oracle.h")
    return d


def test_unmutated_source_matches(workdir):
    src = open(oracle.SOURCE).read()
    for name, (old, _) in MUTATIONS.items():
        assert src.count(old) == 1, f"{name}: anchor occurs {src.count(old)} times"


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutant_is_caught(workdir, name):
    old, new = MUTATIONS[name]
    src = open(oracle.SOURCE).read()
    assert src.count(old) == 1
    c = workdir / f"{name}.c"
    so = workdir / f"lib{name}.so"
    c.write_text(src.replace(old, new))
    subprocess.run(["gcc", *oracle.CFLAGS, "-I", str(workdir), str(c), "-o", str(so), "-lm"], check=True)
    O = oracle.load(str(so))
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(O)
        except AssertionError:
            failed.append(pin.__name__)
            break
    assert failed, f"no pin caught the planted mistake {name!r}"
