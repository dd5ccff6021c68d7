"""Plant plausible mistakes in a copy of the oracle and check the pins catch them.

Each mutant is a textual edit of ``oracle/moe_oracle.c`` compiled into a
temporary library on the CPU.  The pins of ``test_oracle.py`` run against it,
and at least one must fail: a pin set that lets a mutant through would not
pin the oracle.
"""
import importlib.util
import inspect
import os

import pytest

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))

MUTANTS = {
    "bias_added_to_logit": [
        ("s[e] = oracle_sigmoid_f32(lg[e]);",
         "s[e] = oracle_sigmoid_f32(lg[e] + (bias ? bias[e] : 0.0f));")],
    "bias_kept_in_weights": [
        ("for (int32_t j = 0; j < top_k; ++j) wsum += (double)s[order[j].idx];",
         "for (int32_t j = 0; j < top_k; ++j) wsum += (double)order[j].key;"),
        ("weights[(size_t)t * top_k + j] = (float)((double)s[order[j].idx] / wsum);",
         "weights[(size_t)t * top_k + j] = (float)((double)order[j].key / wsum);")],
    "higher_index_wins_ties": [
        ("return (a->idx < b->idx) ? -1 : (a->idx > b->idx);",
         "return (a->idx > b->idx) ? -1 : (a->idx < b->idx);")],
    "sigmoid_sign_flipped": [
        ("return (float)(1.0 / (1.0 + exp(-(double)logit)));",
         "return (float)(1.0 / (1.0 + exp((double)logit)));")],
    "weights_not_normalised": [
        ("weights[(size_t)t * top_k + j] = (float)((double)s[order[j].idx] / wsum);",
         "weights[(size_t)t * top_k + j] = (float)((double)s[order[j].idx]);")],
    "map_not_stable": [
        ("for (int64_t r = 0; r < rows; ++r) {\n        int32_t p = fill",
         "for (int64_t r = rows - 1; r >= 0; --r) {\n        int32_t p = fill")],
    "matmul_weight_transposed": [
        ("acc += bf16_to_f64(We[(size_t)c * k + i]) * bf16_to_f64(xr[i]);",
         "acc += bf16_to_f64(We[(size_t)i * n + c]) * bf16_to_f64(xr[i]);")],
    "matmul_slotted_reads_token_row": [
        ("const uint16_t *xr = x + (size_t)(layout == 0 ? t : r) * k;",
         "const uint16_t *xr = x + (size_t)t * k;")],
    "ffn_missing_up_factor": [
        ("a[i] = g / (1.0 + exp(-g)) * u;", "a[i] = g / (1.0 + exp(-g));")],
    "ffn_gate_up_swapped": [
        ("a[i] = g / (1.0 + exp(-g)) * u;", "a[i] = u / (1.0 + exp(-u)) * g;")],
    "ffn_sigmoid_not_silu": [
        ("a[i] = g / (1.0 + exp(-g)) * u;", "a[i] = 1.0 / (1.0 + exp(-g)) * u;")],
    "ffn_combine_unweighted": [("yt[h] += w * d;", "yt[h] += d;")],
    "ffn_down_transposed": [
        ("d += bf16_to_f64(Wd[(size_t)h * inter + i]) * a[i];",
         "d += bf16_to_f64(Wd[(size_t)i * hidden + h]) * a[i];")],
    "ffn_slotted_reads_token_row": [
        ("const uint16_t *xr = x + (size_t)(layout == 0 ? t : r) * hidden;",
         "const uint16_t *xr = x + (size_t)t * hidden;")],
    "router_weight_transposed": [
        ("for (int32_t c = 0; c < hidden; ++c) acc += bf16_to_f64(we[c]) * bf16_to_f64(xt[c]);",
         "for (int32_t c = 0; c < hidden; ++c) acc += bf16_to_f64(W_router[(size_t)c * n_experts + e]) * bf16_to_f64(xt[c]);")],
    "shared_gate_sign_flipped": [
        ("const double gate = 1.0 / (1.0 + exp(-logit));",
         "const double gate = 1.0 / (1.0 + exp(logit));")],
    "shared_gate_not_applied": [("yt[h] += gate * d_s;", "yt[h] += d_s;")],
    "shared_missing_silu": [
        ("h_s[i] = a_s / (1.0 + exp(-a_s)) * b_s;", "h_s[i] = a_s * b_s;")],
    "shared_down_transposed": [
        ("d_s += bf16_to_f64(W_sh_down[(size_t)h * inter_sh + i]) * h_s[i];",
         "d_s += bf16_to_f64(W_sh_down[(size_t)i * hidden + h]) * h_s[i];")],
    "shared_logit_from_gate_row": [
        ("logit += bf16_to_f64(w_sh[c]) * bf16_to_f64(xt[c]);",
         "logit += bf16_to_f64(W_sh_gate[c]) * bf16_to_f64(xt[c]);")],
    "shared_drops_routed_part": [
        ("oracle_ffn(x, ids, weights, W_gate, W_up, W_down, y, m, hidden, inter, top_k, n_experts, 0,\n"
         "               act_mode, tokens, n_tokens);",
         "memset(y, 0, sizeof(double) * (size_t)n_tokens * hidden);")],
    "nan_key_not_demoted": [
        ("    if (isnan(k)) return -INFINITY;\n", "")],
    "map_inverse_not_inverted": [("        inv_perm[r] = p;\n", "        inv_perm[p] = (int32_t)r;\n")],
    "map_stores_token_not_row": [
        ("        perm[p] = (int32_t)r;\n", "        perm[p] = (int32_t)(r / top_k);\n")],
    "matmul_expert_from_wrong_slot": [
        ("const uint16_t *We = W + (size_t)ids[r] * n * k;",
         "const uint16_t *We = W + (size_t)ids[t * top_k + (top_k - 1 - r % top_k)] * n * k;")],
    "ffn_weight_from_wrong_slot": [
        ("const double w = (double)weights[r];",
         "const double w = (double)weights[t * top_k + (top_k - 1 - j)];")],
    "fp16_activation_unscaled": [
        ("    const float f = (float)v * 0.0625f;", "    const float f = (float)v;"),
        ("    return (double)h * 16.0;", "    return (double)h;")],
    "fp16_activation_scale_inverted": [
        ("    const float f = (float)v * 0.0625f;", "    const float f = (float)v * 16.0f;"),
        ("    return (double)h * 16.0;", "    return (double)h * 0.0625;")],
    "fp16_activation_scale_not_undone": [("    return (double)h * 16.0;", "    return (double)h;")],
    "fp16_activation_is_bf16": [
        ("    const _Float16 h = (_Float16)f;\n    return (double)h * 16.0;",
         "    return round_to_bf16((double)f) * 16.0;")],
    "forced_weights_unnormalised": [
        ("weights[(size_t)t * top_k + j] = (float)(s / wsum);",
         "weights[(size_t)t * top_k + j] = (float)s;")],
}


def _pins():
    spec = importlib.util.spec_from_file_location("_pins", os.path.join(HERE, "test_oracle.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    calls = []
    for name, fn in inspect.getmembers(mod, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        params = inspect.signature(fn).parameters
        if "oracle_mod" not in params:
            continue
        if "case" in params:
            for case in mod.ROUTE_CASES:
                calls.append((f"{name}[{case['name']}]", fn, {"case": case}))
        else:
            calls.append((name, fn, {}))
    return calls


@pytest.mark.parametrize("mutant", sorted(MUTANTS))
def test_pins_catch_mutant(mutant, tmp_path):
    src = open(oracle.SOURCE).read()
    for old, new in MUTANTS[mutant]:
        assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
        src = src.replace(old, new)
    c_path = tmp_path / "mutant.c"
    c_path.write_text(src)
    lib = oracle.compile_source(str(c_path), str(tmp_path / "libmutant.so"))
    mutated = oracle.Oracle(lib)
    caught = []
    for name, fn, kw in _pins():
        try:
            fn(oracle_mod=mutated, **kw)
        except (AssertionError, ValueError):
            caught.append(name)
            break
    assert caught, f"no pin caught mutant {mutant}"
