"""Plant plausible mistakes in copies of the oracle and check that the pins
catch every one: a flipped tie-break, a dropped term, a wrong sign or index,
a transposed operand, a wrong rounding.  Runs on the CPU only."""
import pytest

import oracle
import oracle_pins

MUTANTS = {
    "tie_to_higher_id": ("(double)row[e] > (double)row[best]",
                         "(double)row[e] >= (double)row[best]"),
    "softmax_sign": ("(float)(exp(sel[j] - sel[0]) / denom)",
                     "(float)(exp(sel[0] - sel[j]) / denom)"),
    "softmax_dropped_term": ("for (int32_t j = 0; j < top_k; ++j) denom +=",
                             "for (int32_t j = 1; j < top_k; ++j) denom +="),
    "inclusive_prefix": ("e2 < e; ++e2", "e2 <= e; ++e2"),
    "capacity_n_times_k": ("(top_k < per_rank ? top_k : per_rank)", "top_k"),
    "round_robin_rank_map": ("int32_t r = e / per_rank;", "int32_t r = e % n_ranks;"),
    "src_of_encoding": ("src_of[s] = (int32_t)(t * top_k + j);",
                        "src_of[s] = (int32_t)(j * n + t);"),
    "scatter_wrong_row": ("src + t * row_bytes", "src + (n - 1 - t) * row_bytes"),
    "dequant_block_index": ("scale[s * n_blocks + c / block]",
                            "scale[s * n_blocks + c % n_blocks]"),
    "swiglu_gate_up_swapped": ("double silu = g / (1.0 + exp(-g));\n"
                               "            uint16_t hb = bf16_from_double(silu * u);",
                               "double silu = u / (1.0 + exp(-u));\n"
                               "            uint16_t hb = bf16_from_double(silu * g);"),
    "silu_sign": ("double silu = g / (1.0 + exp(-g));", "double silu = g / (1.0 + exp(g));"),
    "fp8_silu_sign": ("bf16_from_double(g / (1.0 + exp(-g)) * u)",
                      "bf16_from_double(g / (1.0 + exp(g)) * u)"),
    "w_down_transposed": ("wd[(int64_t)c * inter + d]", "wd[(int64_t)d * hidden + c]"),
    "combine_weight_index": ("acc += (double)topk_w[t * top_k + j] * load_elem",
                             "acc += (double)topk_w[t * top_k] * load_elem"),
    "combine_float_accumulator": ("            double acc = 0.0;\n"
                                  "            for (int32_t j = 0; j < top_k; ++j) {\n"
                                  "                int64_t s = slot_of[t * top_k + j];\n"
                                  "                if (s < 0 || s >= total_slots) return ORACLE_BAD_INDEX;\n"
                                  "                acc += (double)topk_w",
                                  "            float acc = 0.0f;\n"
                                  "            for (int32_t j = 0; j < top_k; ++j) {\n"
                                  "                int64_t s = slot_of[t * top_k + j];\n"
                                  "                if (s < 0 || s >= total_slots) return ORACLE_BAD_INDEX;\n"
                                  "                acc += (float)topk_w"),
    "bf16_truncate": ("nearbyint(ldexp(a, -q_exp))", "floor(ldexp(a, -q_exp))"),
    "bf16_nine_bits": ("int q_exp = e - 8;", "int q_exp = e - 9;"),
    "e4m3_bias": ("ldexp(1.0 + (double)m / 8.0, ex - 7)", "ldexp(1.0 + (double)m / 8.0, ex - 8)"),
    "e4m3_subnormal": ("ldexp((double)m / 8.0, -6)", "ldexp((double)m / 8.0, -7)"),
    "bf16_decode_shift": ("(uint32_t)b << 16", "(uint32_t)b << 15"),
    "e4m3_encode_ties_odd": ("(c & 1) == 0 && (best & 1) == 1", "(c & 1) == 1 && (best & 1) == 0"),
    "e4m3_encode_no_saturation": ("if (a >= 448.0) return sign | 0x7E;", ""),
    "quant_divisor": ("(float)(amax / 448.0)", "(float)(amax / 240.0)"),
    "quant_signed_amax": ("double a = fabs(bf16_to_double(hb[c]));",
                          "double a = bf16_to_double(hb[c]);"),
    "fp8_x_scale_dropped": ("double xv = dec[xr[d]] * (double)xsr[d / block];",
                            "double xv = dec[xr[d]];"),
    "fp8_gate_scale_transposed": ("(double)wsc[(int64_t)(c / block) * kb + d / block]);\n"
                                  "                u +=",
                                  "(double)wsc[(int64_t)(d / block) * kb + c / block]);\n"
                                  "                u +="),
    "fp8_up_uses_gate_scale": ("(double)wsc[(cu / block) * kb + d / block]",
                               "(double)wsc[(int64_t)(c / block) * kb + d / block]"),
    "fp8_down_h_scale_block": ("(double)hsr[d / block]", "(double)hsr[0]"),
    "fp8_down_expert_scales": ("const float* wsc = w_down_s + e * (int64_t)rb * kb;",
                               "const float* wsc = w_down_s;"),
    "router_first_expert_row": ("const uint16_t* wr = w_router + (int64_t)e * hidden;",
                                "const uint16_t* wr = w_router;"),
    "router_dropped_last_term": ("for (int32_t d = 0; d < hidden; ++d) acc += bf16_to_double(xr[d])",
                                 "for (int32_t d = 0; d < hidden - 1; ++d) acc += bf16_to_double(xr[d])"),
    "router_float_accumulator": ("            double acc = 0.0;\n"
                                 "            for (int32_t d = 0; d < hidden; ++d) acc +=",
                                 "            float acc = 0.0f;\n"
                                 "            for (int32_t d = 0; d < hidden; ++d) acc += (float)"),
    "router_token_row": ("const uint16_t* xr = x + t * hidden;", "const uint16_t* xr = x;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.source_text()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    lib = oracle.build_variant(src.replace(old, new), str(tmp_path / f"mut_{name}.so"))
    o = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(o)
        except (AssertionError, ValueError) as exc:  # a pin failed
            caught.append((pin.__name__, type(exc).__name__))
    assert caught, f"no pin caught the planted mistake {name}"
