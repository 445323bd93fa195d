"""Plant one mistake at a time in a copy of the oracle (on the CPU) and check
that the pins catch it: each mutant must fail at least one pin.  This shows the
pins are strong enough that a dropped term, a wrong sign, a wrong index or a
transposed operand anywhere in the oracle would not go unnoticed."""
import pytest

import oracle_pins

# (name, text in lightning_oracle.c, replacement, which occurrence)
MUTANTS = [
    ("recurrent_state_transposed", "S[(size_t)a * d + b] += kt[a] * vt[b];",
     "S[(size_t)a * d + b] += kt[b] * vt[a];", 0),
    ("recurrent_output_transposed", "o[b] += qt[a] * S[(size_t)a * d + b];",
     "o[b] += qt[a] * S[(size_t)b * d + a];", 0),
    ("recurrent_ignores_state_in", "if (state_in)\n            memcpy(S,", "if (0)\n            memcpy(S,", 0),
    ("recurrent_wrong_head", "const int h = heads ? heads[j] : j;", "const int h = j;", 0),
    ("quadratic_strict_mask", "for (int s = t0; s <= t; ++s) {", "for (int s = t0; s < t; ++s) {", 0),
    ("quadratic_key_index", "score += widen_bf16(ROW(q, t, h)[a]) * widen_bf16(ROW(k, s, h)[a]);",
     "score += widen_bf16(ROW(q, t, h)[a]) * widen_bf16(ROW(k, t, h)[a]);", 0),
    ("quadratic_drops_state_in", "o[b] += qa * Sin[(size_t)a * d + b];",
     "o[b] += 0.0 * qa * Sin[(size_t)a * d + b];", 0),
    ("quadratic_state_transposed", "S[(size_t)a * d + b] += ka * widen_bf16(ROW(v, s, h)[b]);",
     "S[(size_t)b * d + a] += ka * widen_bf16(ROW(v, s, h)[b]);", 0),
    ("blocked_strict_mask", "for (int s = b0; s <= t; ++s) {", "for (int s = b0; s < t; ++s) {", 0),
    ("blocked_inter_sign", "for (int b = 0; b < d; ++b) o[b] += qa * S[(size_t)a * d + b];",
     "for (int b = 0; b < d; ++b) o[b] -= qa * S[(size_t)a * d + b];", 0),
    ("blocked_update_before_output", "/* S_{<=b} = S_{<b} + K_b^T V_b */",
     "/* mutated */ for (int s = b0; s < b1; ++s) for (int a = 0; a < d; ++a) "
     "S[(size_t)a * d + a] += 0.5;", 0),
    ("blocked_short_block", "const int b1 = (b0 + block < t1) ? b0 + block : t1;",
     "const int b1 = (b0 + block < t1) ? b0 + block - (block > 1) : t1;", 0),
    ("segmented_inclusive_prefix", "for (int r2 = 0; r2 < r; ++r2)", "for (int r2 = 0; r2 <= r; ++r2)", 0),
    ("segmented_final_state_drops_last", "for (int r = 0; r < nseg; ++r)\n                for (size_t e = 0; e < dd; ++e) So[e]",
     "for (int r = 0; r < nseg - 1; ++r)\n                for (size_t e = 0; e < dd; ++e) So[e]", 0),
    ("decode_output_transposed", "for (int b = 0; b < d; ++b) o[b] += qa * S[(size_t)a * d + b];",
     "for (int b = 0; b < d; ++b) o[b] += qa * S[(size_t)b * d + a];", 1),
    ("decode_update_index", "S[(size_t)a * d + b] += ka * widen_bf16(vp[b]);",
     "S[(size_t)a * d + b] += ka * widen_bf16(vp[a]);", 0),
    ("widen_wrong_shift", "((uint32_t)bits) << 16", "((uint32_t)bits) << 15", 0),
    ("backward_dq_strict_mask", "for (int s2 = 0; s2 <= t; ++s2) {", "for (int s2 = 0; s2 < t; ++s2) {", 0),
    ("backward_dq_state_transposed", "o[a] += Sin[(size_t)a * d + b] * G[(size_t)t * d + b];",
     "o[a] += Sin[(size_t)b * d + a] * G[(size_t)t * d + b];", 0),
    ("backward_dkdv_strict_mask", "for (int t = s2; t < n; ++t) {", "for (int t = s2 + 1; t < n; ++t) {", 0),
    ("backward_dk_wrong_factor", "ok[a] += wk * Q[(size_t)t * d + a];", "ok[a] += wk * K[(size_t)t * d + a];", 0),
    ("backward_dv_wrong_score", "wv += Q[(size_t)t * d + b] * K[(size_t)s2 * d + b];",
     "wv += Q[(size_t)t * d + b] * Q[(size_t)s2 * d + b];", 0),
    ("backward_dk_drops_state_grad", "ok[a] += GS[(size_t)a * d + b] * V[(size_t)s2 * d + b];",
     "ok[a] += 0.0 * GS[(size_t)a * d + b] * V[(size_t)s2 * d + b];", 0),
    ("backward_dk_state_grad_transposed", "ok[a] += GS[(size_t)a * d + b] * V[(size_t)s2 * d + b];",
     "ok[a] += GS[(size_t)b * d + a] * V[(size_t)s2 * d + b];", 0),
    ("backward_dv_state_grad_transposed", "ov[b] += K[(size_t)s2 * d + a] * GS[(size_t)a * d + b];",
     "ov[b] += K[(size_t)s2 * d + a] * GS[(size_t)b * d + a];", 0),
    ("backward_dsin_drops_state_grad", "D[e] = GS ? GS[e] : 0.0;", "D[e] = 0.0;", 0),
    ("backward_dsin_transposed", "D[(size_t)a * d + b] += Q[(size_t)t * d + a] * G[(size_t)t * d + b];",
     "D[(size_t)b * d + a] += Q[(size_t)t * d + a] * G[(size_t)t * d + b];", 0),
    # per-head decay
    ("decay_recurrent_decays_new_token", "S[(size_t)a * d + b] = lam * S[(size_t)a * d + b] + kt[a] * vt[b];",
     "S[(size_t)a * d + b] = lam * (S[(size_t)a * d + b] + kt[a] * vt[b]);", 0),
    ("decay_recurrent_position_not_head", "const double lam = decay[h];", "const double lam = decay[j];", 0),
    ("decay_quadratic_exponent_plus_one", "const double w = score * pow(lam, (double)(t - s));",
     "const double w = score * pow(lam, (double)(t - s + 1));", 0),
    ("decay_quadratic_state_in_factor", "const double f = pow(lam, (double)(t - t0 + 1));",
     "const double f = pow(lam, (double)(t - t0));", 0),
    ("decay_quadratic_final_state_exponent", "const double w = pow(lam, (double)(t1 - 1 - s));",
     "const double w = pow(lam, (double)(t1 - s));", 0),
    ("decay_blocked_intra_exponent", "const double w = score * pow(lam, (double)(t - s));",
     "const double w = score * pow(lam, (double)(s - t));", 1),
    ("decay_blocked_inter_factor", "const double f = pow(lam, (double)(t - b0 + 1));",
     "const double f = pow(lam, (double)(t - b0));", 0),
    ("decay_blocked_state_factor", "const double f = pow(lam, (double)(b1 - b0));",
     "const double f = pow(lam, (double)(b1 - b0 - 1));", 0),
    ("decay_segmented_local_exponent", "const double w = pow(lam, (double)(s1 - 1 - s));",
     "const double w = pow(lam, (double)(s1 - s));", 0),
    ("decay_segmented_prefix_factor", "const double f = pow(lam, (double)(s0 - e2));",
     "const double f = pow(lam, (double)(s0 - e2 + 1));", 0),
    ("decay_decode_decays_new_token",
     "S[(size_t)a * d + b] = lam * S[(size_t)a * d + b] + ka * widen_bf16(vp[b]);",
     "S[(size_t)a * d + b] = lam * (S[(size_t)a * d + b] + ka * widen_bf16(vp[b]));", 0),
]


def _replace_nth(text, old, new, n):
    idx = -1
    for _ in range(n + 1):
        idx = text.find(old, idx + 1)
        if idx < 0:
            raise AssertionError(f"mutation site not found: {old!r} (occurrence {n})")
    return text[:idx] + new + text[idx + len(old):]


@pytest.mark.parametrize("name,old,new,occ", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(oracle_mod, tmp_path, name, old, new, occ):
    src = _replace_nth(oracle_mod.oracle.source_text(), old, new, occ)
    lib = oracle_mod.oracle.build_variant(src, str(tmp_path / f"mut_{name}.so"))
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(oracle_mod, lib)
        except (AssertionError, ValueError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
