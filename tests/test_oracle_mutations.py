"""The oracle's pins catch plausible mistakes: each case plants one mistake in a copy
of la_oracle.c (on the CPU), compiles it, and requires at least one pin to fail."""
import os

import pytest

import oracle
from tests import pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "la_oracle.c")

# (name, text to find, replacement, which occurrence (0-based))
MUTATIONS = [
    ("phi_drops_plus_one", "x > 0.0 ? x + 1.0 : exp(x); }", "x > 0.0 ? x : exp(x); }", 0),
    ("phi_prime_constant", "x > 0.0 ? 1.0 : exp(x); }", "x > 0.0 ? 1.0 : 1.0; }", 0),
    ("fwd_drops_eps", "double n = jb->eps;", "double n = 0.0;", 0),
    ("bwd_drops_eps", "double n = jb->eps;", "double n = 0.0;", 1),
    ("fwd_state_transposed", "u += fq[i] * S[i * D + j];", "u += fq[i] * S[j * D + i];", 0),
    ("fwd_z_dropped", "z[i] += fk;", "z[i] += 1.0;", 0),
    ("bwd_dz_sign", "dz[i] -= fq[i] * go / n;", "dz[i] += fq[i] * go / n;", 0),
    ("bwd_dq_drops_norm_term", "(gs - go * z[i]) / n", "gs / n", 0),
    ("bwd_dq_wrong_state_index", "gs += g[t * D + j] * S[i * D + j];", "gs += g[t * D + j] * S[j * D + i];", 0),
    ("bwd_dv_transposed", "a += fk * dS[i * D + j];", "a += fk * dS[j * D + i];", 0),
    ("bwd_dk_drops_dz", "double a = dz[i];", "double a = 0.0;", 0),
    ("bwd_dk_uses_phi_not_dphi", "double fp = jb->use_phi ? dphi(k[s * D + i]) : 1.0;",
     "double fp = jb->use_phi ? phi(k[s * D + i]) : 1.0;", 0),
    ("bwd_dq_no_dphi", "double fp = jb->use_phi ? dphi(q[t * D + i]) : 1.0;", "double fp = 1.0;", 0),
    ("ret_fwd_no_decay", "S[i * D + j] = gamma * S[i * D + j] + k[t * D + i] * v[t * D + j];",
     "S[i * D + j] = S[i * D + j] + k[t * D + i] * v[t * D + j];", 0),
    ("ret_fwd_output_before_update_index", "a += q[t * D + i] * S[i * D + j];", "a += q[t * D + i] * S[j * D + i];", 0),
    ("ret_bwd_reverse_no_decay", "R[i * D + j] = gamma * R[i * D + j] + q[s * D + i] * g[s * D + j];",
     "R[i * D + j] = R[i * D + j] + q[s * D + i] * g[s * D + j];", 0),
    ("ret_bwd_dq_transposed", "a += S[i * D + j] * g[t * D + j];", "a += S[j * D + i] * g[t * D + j];", 0),
    ("ret_bwd_dv_transposed", "a += k[s * D + i] * R[i * D + j];", "a += k[s * D + i] * R[j * D + i];", 0),
    ("ret_fwd_gamma_head_index", "const double gamma = jb->gamma[bh % jb->H];", "const double gamma = jb->gamma[0];", 0),
    ("ret_bwd_gamma_head_index", "const double gamma = jb->gamma[bh % jb->H];", "const double gamma = jb->gamma[0];", 1),
    ("head_offset_dropped", "const long off = bh * T * D;", "const long off = 0;", 0),
    ("step_no_decay", "Sh[i * D + j] = g * Sh[i * D + j] + kh[i] * vh[j];",
     "Sh[i * D + j] = Sh[i * D + j] + kh[i] * vh[j];", 0),
    ("step_output_transposed", "a += qh[i] * Sh[i * D + j];", "a += qh[i] * Sh[j * D + i];", 0),
    ("step_outer_product_transposed", "+ kh[i] * vh[j];", "+ kh[j] * vh[i];", 0),
    ("step_gamma_head_index", "const double g = gamma[bh % H];", "const double g = gamma[0];", 0),
    ("fwd_state_in_ignored", "    if (jb->state_in)\n", "    if (0)\n", 0),
    ("bwd_state_in_ignored", "    if (jb->state_in) memcpy(S,", "    if (0) memcpy(S,", 0),
    ("bwd_dstate_in_ignored", "    if (jb->dstate_in) memcpy(R,", "    if (0) memcpy(R,", 0),
    ("bwd_dstate_out_is_state", "memcpy(jb->dstate_out + bh * D * D, R,", "memcpy(jb->dstate_out + bh * D * D, S,", 0),
    ("causal_drops_eps", "double n = jb->eps;\n        for (long i = 0; i < D; ++i) n += fq[i] * z[i];\n        for (long j",
     "double n = 0.0;\n        for (long i = 0; i < D; ++i) n += fq[i] * z[i];\n        for (long j", 0),
    ("causal_z_not_decayed", "z[i] = gamma * z[i] + fk[i];", "z[i] = z[i] + fk[i];", 0),
    ("causal_bwd_dn_sign", "const double dn = -go / n;", "const double dn = go / n;", 0),
    ("causal_bwd_drops_r", "double a = r[i];", "double a = 0.0;", 0),
    ("causal_bwd_dk_uses_f", "dk[s * D + i] = a * dfeat(jb, k[s * D + i]);", "dk[s * D + i] = a * feat(jb, k[s * D + i]);", 0),
    ("causal_bwd_dq_drops_z", "double a = z[i] * dn;", "double a = 0.0;", 0),
    ("focus_drops_norm_ratio", "y[i] = b > 0.0 ? (a / b) * pow(r, p) : 0.0;", "y[i] = b > 0.0 ? pow(r, p) : 0.0;", 0),
    ("focus_bwd_s_term_sign", "+ s * r / (a * b) - s * a * p", "- s * r / (a * b) - s * a * p", 0),
    ("polarity_halves_swapped", "y[i] = kind == 1 ? pos : neg;", "y[i] = kind == 1 ? neg : pos;", 0),
    ("polarity_bwd_neg_sign", "const double dneg = x[i] < 0.0 ? -p * pow(-x[i], p - 1.0) : 0.0;",
     "const double dneg = x[i] < 0.0 ? p * pow(-x[i], p - 1.0) : 0.0;", 0),
    ("normed_uses_phi", "jb.eps = eps; jb.use_phi = 0; jb.use_norm = 1;\n    return for_each_head(&jb, state_fwd_head",
     "jb.eps = eps; jb.use_phi = 1; jb.use_norm = 1;\n    return for_each_head(&jb, state_fwd_head", 0),
    ("gated_reverse_gate_of_t", "const double a = t + 1 < T ? exp(lg[(t + 1) * D + i]) : 0.0;",
     "const double a = t + 1 < T ? exp(lg[t * D + i]) : 0.0;", 0),
    ("gated_dg_forward_cumsum", "    for (long t = T - 1; t >= 0; --t)\n        for (long i = 0; i < D; ++i) {\n            acc[i] +=",
     "    for (long t = 0; t < T; ++t)\n        for (long i = 0; i < D; ++i) {\n            acc[i] +=", 0),
    ("gated_dg_k_sign", "acc[i] += q[t * D + i] * dq[t * D + i] - k[t * D + i] * dk[t * D + i];",
     "acc[i] += q[t * D + i] * dq[t * D + i] + k[t * D + i] * dk[t * D + i];", 0),
    ("gated_fwd_gate_not_exp", "            const double a = exp(lg[t * D + i]);\n            for (long j = 0; j < D; ++j) S[i * D + j] = a * S[i * D + j] + k[t * D + i] * v[t * D + j];\n        }\n        for (long j = 0; j < D; ++j) {\n            double u",
     "            const double a = 1.0 + lg[t * D + i];\n            for (long j = 0; j < D; ++j) S[i * D + j] = a * S[i * D + j] + k[t * D + i] * v[t * D + j];\n        }\n        for (long j = 0; j < D; ++j) {\n            double u", 0),
    ("fwd_state_out_before_last_token", "    if (jb->state_out) memcpy(jb->state_out + bh * D * D, S,",
     "    if (jb->state_out) memcpy(jb->state_out + bh * D * D, jb->state_in ? jb->state_in + bh * D * D : S,", 0),
]


def _mutate(text, find, repl, occurrence):
    pos = -1
    for _ in range(occurrence + 1):
        pos = text.find(find, pos + 1)
        if pos < 0:
            raise ValueError("mutation target not found: %r (occurrence %d)" % (find, occurrence))
    return text[:pos] + repl + text[pos + len(find):]


@pytest.mark.parametrize("name,find,repl,occ", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutation(tmp_path, name, find, repl, occ):
    text = open(SRC).read()
    mutated = _mutate(text, find, repl, occ)
    assert mutated != text
    src = tmp_path / "mut.c"
    src.write_text(mutated)
    lib = oracle.build(force=True, src=str(src), out=str(tmp_path / "libmut.so"))
    orc = oracle.load_variant(lib)
    failures = []
    for check in pins.ALL_CHECKS:
        try:
            check(orc)
        except (AssertionError, FloatingPointError) as e:
            failures.append((check.__name__, str(e)[:80]))
    assert failures, "mutation %s was not caught by any pin" % name
