"""Pin strength: plant one plausible mistake at a time into a copy of the
oracle source (CPU only), rebuild it, and require that at least one pin
catches it.  The real oracle source is never modified."""
import os

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "lizard_oracle.cpp")

# (name, exact text in the oracle, replacement).  Each text is replaced once
# (its first occurrence).
MUTANTS = [
    ("add_before_decay", "decay * S[(size_t)i * dv + j] + kt[i] * vt[j];",
     "decay * (S[(size_t)i * dv + j] + kt[i] * vt[j]);"),
    ("decay_uses_minus_g", "double decay = std::exp(gt[i]);", "double decay = std::exp(-gt[i]);"),
    ("output_transposed_index", "acc += qt[i] * S[(size_t)i * dv + j];",
     "acc += qt[i] * S[(size_t)j * dv + i];"),
    ("chunk_exclusive_cumsum", "run += g[(size_t)(c0 + r) * dk + i];\n        b[(size_t)r * dk + i] = run;",
     "b[(size_t)r * dk + i] = run;\n        run += g[(size_t)(c0 + r) * dk + i];"),
    ("window_one_too_wide", "int lo = std::max(0, t - w + 1);", "int lo = std::max(0, t - w);"),
    ("sink_not_in_denominator", "l += p;  // a sink always enters the denominator", ";"),
    ("meta_logit_unscaled", "      a *= scale;\n      logit[nwin + m] = a;", "      logit[nwin + m] = a;"),
    ("alpha_on_wrong_branch", "o[tv + x] = og[x] + alpha * os[x];", "o[tv + x] = alpha * og[x] + os[x];"),
    ("dq_reads_v", "a += St[(size_t)i * dv + j] * dot[j];", "a += St[(size_t)i * dv + j] * vt[j];"),
    ("dk_reads_state", "bsum += dS[(size_t)i * dv + j] * vt[j];", "bsum += St[(size_t)i * dv + j] * vt[j];"),
    ("dg_missing_gate", "dg[(size_t)t * dk + i] = std::exp(gt[i]) * gsum;", "dg[(size_t)t * dk + i] = gsum;"),
    ("dg_uses_current_state", "gsum += dS[(size_t)i * dv + j] * Sp[(size_t)i * dv + j];",
     "gsum += dS[(size_t)i * dv + j] * St[(size_t)i * dv + j];"),
    ("softmax_grad_drops_D", "double ds = p[x] * (dp[x] - D);", "double ds = p[x] * dp[x];"),
    ("dv_drops_prob", "dval[c] += p[x] * dot[c];", "dval[c] += dot[c];"),
    ("dalpha_sign", "for (size_t x = 0; x < (size_t)T * dv; ++x) s += dO[tv + x] * os[x];",
     "for (size_t x = 0; x < (size_t)T * dv; ++x) s -= dO[tv + x] * os[x];"),
    ("decode_wrong_slot", "int slot = (int)(p % w);", "int slot = (int)((p + 1) % w);"),
    ("decode_window_short", "int nwin = (int)std::min<int64_t>(p + 1, w);",
     "int nwin = (int)std::min<int64_t>(p, w);"),
    ("mse_gradient_drops_two", "if (dO) dO[x] = 2.0 * diff / (double)n;", "if (dO) dO[x] = diff / (double)n;"),
    ("mse_sum_not_mean", "*loss = n > 0 ? s / (double)n : 0.0;", "*loss = n > 0 ? s : 0.0;"),
    ("mse_gradient_sign", "const double diff = o[x] - target[x];", "const double diff = target[x] - o[x];"),
    ("gate_logit_unscaled", "g_out[x] = scale * ls;", "g_out[x] = ls;"),
    ("dlogits_sigmoid_of_z", "dz[x] = dg[x] * scale * sneg;", "dz[x] = dg[x] * scale * (1.0 - sneg);"),
    ("proj_layout_token_major", "double* dst = out[which] + (((size_t)b * H + h) * T + t) * dk;",
     "double* dst = out[which] + (((size_t)b * T + t) * H + h) * dk;"),
    ("proj_gate_map_on_keys", "if (which == 2) {", "if (which == 1) {"),
    ("proj_weight_rows_of_head0", "const double* wr = W[which] + ((size_t)h * dk + i) * Dm;",
     "const double* wr = W[which] + ((size_t)i) * Dm;"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(SRC).read()
    assert old in src, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    path = tmp_path / f"mut_{name}.cpp"
    path.write_text(mutated)
    so = str(tmp_path / f"libmut_{name}.so")
    oracle.build(str(path), so)
    lib = oracle.load(so)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError, FloatingPointError) as exc:
            caught.append((pin.__name__, str(exc)[:80]))
            break
    assert caught, f"mutant {name} passed every pin"
