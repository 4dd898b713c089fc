"""Each plausible mistake planted in a copy of the oracle (on the CPU) must make
at least one pin of tests/test_oracle_pins.py fail.  This shows the pins are
strong enough to catch a dropped term, a wrong sign or index, or a transposed
operand anywhere in the recurrence or the chunkwise steps."""
import pytest

import oracle
import tests.test_oracle_pins as pins

# (name, original text, mutated text) -- each replacement hits one place only
MUTATIONS = [
    ("gdn: decay dropped from the erase term",
     "- a * b * r[i] * k[j] + b * v[i] * k[j]", "- b * r[i] * k[j] + b * v[i] * k[j]"),
    ("gdn: write term sign flipped",
     "- a * b * r[i] * k[j] + b * v[i] * k[j]", "- a * b * r[i] * k[j] - b * v[i] * k[j]"),
    ("read-out before the update (old state)",
     [("        if (!p->channel_decay) {\n            /* S <- alpha",
       "        { double *o0 = p->o + (t * H + h) * dv;\n"
       "          for (int i = 0; i < dv; ++i) { double acc = 0.0;\n"
       "            for (int j = 0; j < dk; ++j) acc += S[i * dk + j] * q[j]; o0[i] = acc; } }\n"
       "        if (!p->channel_decay) {\n            /* S <- alpha"),
      ("            o[i] = acc;\n", "            (void)o; (void)acc;\n")], None),
    ("read-out with the key instead of the query",
     "acc += S[i * dk + j] * q[j];", "acc += S[i * dk + j] * k[j];"),
    ("kda: one channel's decay used for all channels",
     "const double a = exp(log_decay(p, t, h, j));", "const double a = exp(log_decay(p, t, h, 0));"),
    ("kda: erase reads the undecayed state",
     "for (int i = 0; i < dv; ++i) S[i * dk + j] *= a;", "for (int i = 0; i < dv; ++i) r[i] += 0.0 * a;"),
    ("chunk A: decay of the wrong token",
     "* exp(G[r * dk + c] - G[s * dk + c]);\n            A[r * L + s]",
     "* exp(G[s * dk + c] - G[s * dk + c]);\n            A[r * L + s]"),
    ("chunk A: beta of the wrong token",
     "A[r * L + s] = beta[r] * acc;", "A[r * L + s] = beta[s] * acc;"),
    ("UT solve: a term skipped",
     "for (int m = j; m < i; ++m) acc += A[i * L + m] * T[m * L + j];",
     "for (int m = j + 1; m < i; ++m) acc += A[i * L + m] * T[m * L + j];"),
    ("W without the decay", "* k[s * dk + c] * exp(G[s * dk + c]);", "* k[s * dk + c];"),
    ("V' sign", "Vp[r * dv + i] = U[r * dv + i] - acc;", "Vp[r * dv + i] = U[r * dv + i] + acc;"),
    ("intra-chunk product not causal (strict)",
     "for (int s = 0; s <= r; ++s) {\n                double qk",
     "for (int s = 0; s < r; ++s) {\n                double qk"),
    ("chunk end state: key decay dropped",
     "acc += Vp[s * dv + i] * k[s * dk + c] * exp(gL - G[s * dk + c]);",
     "acc += Vp[s * dv + i] * k[s * dk + c];"),
    ("chunk end state: state transposed",
     "double acc = S[i * dk + c] * exp(gL);", "double acc = S[c * dk + i] * exp(gL);"),
    ("fg2: key rate not rooted",
     "kt[c] = sqrt(p->beta_k[(t * H + h) * dk + c]) * k[c];",
     "kt[c] = p->beta_k[(t * H + h) * dk + c] * k[c];"),
    ("fg2: value gate ignored",
     "vt[i] = p->beta_v ? sqrt(p->beta_v[(t * H + h) * dv + i]) * v[i] : v[i];",
     "vt[i] = v[i];"),
    ("fg2: erase along the unscaled key",
     "for (int c = 0; c < dk; ++c) e += kt[c] * S[i * dk + c];",
     "for (int c = 0; c < dk; ++c) e += k[c] * S[i * dk + c];"),
    ("fg2: decay dropped",
     "const double ac = exp(log_decay(p, t, h, c));   /* column c decays */",
     "const double ac = 1.0;"),
    ("fg2: write along the unscaled key",
     "S[i * dk + c] += (vt[i] - r[i]) * kt[c];",
     "S[i * dk + c] += vt[i] * k[c] - r[i] * kt[c];"),
    ("prologue: norm not rooted", "double nrm = sqrt(ss);", "double nrm = ss;"),
    ("prologue: sigmoid of the negated logit",
     "static double sigmoid(double x) { return 1.0 / (1.0 + exp(-x)); }",
     "static double sigmoid(double x) { return 1.0 / (1.0 + exp(x)); }"),
    ("prologue: softplus tail loses x",
     "return x > 0 ? x + log1p(exp(-x)) : log1p(exp(x));",
     "return x > 0 ? log1p(exp(-x)) : log1p(exp(x));"),
    ("prologue: decay bias dropped",
     "log_alpha[i] = -softplus(a_logit[i] + bias);", "log_alpha[i] = -softplus(a_logit[i]);"),
    ("prologue: decay sign", "log_alpha[i] = -softplus(a_logit[i] + bias);",
     "log_alpha[i] = softplus(a_logit[i] + bias);"),
]

PIN_TESTS = [
    (pins.test_hand_worked_example, [("gdn",), ("kda",)]),
    (pins.test_delta_rule_is_one_sgd_step, [(False,), (True,)]),
    (pins.test_retrieval_with_orthonormal_keys, [()]),
    (pins.test_orthogonal_keys_reduce_to_decayed_linear_attention, [()]),
    (pins.test_channel_decay_with_disjoint_keys, [()]),
    (pins.test_brute_force_transition_products, [(False,), (True,)]),
    (pins.test_chunkwise_equals_recurrent, [(False, 16), (True, 16)]),
    (pins.test_chunk_stage_ut_factor, [(False,), (True,)]),
    (pins.test_prologue_gate_closed_forms, [()]),
    (pins.test_fg2_uniform_rates_equal_kda, [()]),
    (pins.test_fg2_is_kda_on_scaled_keys_and_values_chunkwise_too, [()]),
    (pins.test_fg2_erase_is_exact_along_a_unit_scaled_key, [()]),
    (pins.test_prologue_decay_bias_per_head_and_channel, [()]),
    (pins.test_prologue_unit_norm_scale_invariance_and_direction, [()]),
]


@pytest.mark.parametrize("name,orig,mut", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_mutation_is_caught(name, orig, mut, tmp_path, monkeypatch):
    src = oracle.source()
    for a, b in (orig if isinstance(orig, list) else [(orig, mut)]):
        assert src.count(a) == 1, f"mutation anchor not unique/found: {name}"
        src = src.replace(a, b)
    lib = oracle._bind(oracle.build_variant(src, str(tmp_path / "mut.so")))
    monkeypatch.setattr(oracle, "_lib", lib)
    caught = []
    for fn, arglists in PIN_TESTS:
        for args in arglists:
            try:
                fn(*args)
            except AssertionError:
                caught.append(fn.__name__)
    assert caught, f"no pin caught the planted mistake: {name}"
