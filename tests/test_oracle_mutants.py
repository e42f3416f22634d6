"""Plant one plausible mistake at a time in a copy of the oracle's C source,
compile the copy, and check that the pin battery rejects it.  This shows the
pins can tell a wrong oracle from a right one; the real oracle is untouched."""
import os

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "attn_jvp_oracle.c")

# (name, text in the oracle source, replacement)
MUTANTS = [
    ("drop_q_dot_term", "Sd[j] = scale * (dot(qdi, kj, d) + dot(qi, kdj, d));",
     "Sd[j] = scale * (dot(qi, kdj, d));"),
    ("drop_k_dot_term", "Sd[j] = scale * (dot(qdi, kj, d) + dot(qi, kdj, d));",
     "Sd[j] = scale * (dot(qdi, kj, d));"),
    ("swapped_tangent_operands", "Sd[j] = scale * (dot(qdi, kj, d) + dot(qi, kdj, d));",
     "Sd[j] = scale * (dot(qdi, kdj, d) + dot(qi, kj, d));"),
    ("tangent_logits_unscaled", "Sd[j] = scale * (dot(qdi, kj, d) + dot(qi, kdj, d));",
     "Sd[j] = (dot(qdi, kj, d) + dot(qi, kdj, d));"),
    ("drop_v_dot_term", "tvd[c] += P[j] * vdj[c];", "tvd[c] += 0.0 * vdj[c];"),
    ("mu_sign_flipped", "double w = P[j] * (Sd[j] - mu);", "double w = P[j] * (Sd[j] + mu);"),
    ("mu_dropped", "double w = P[j] * (Sd[j] - mu);", "double w = P[j] * Sd[j];"),
    ("mu_from_logits", "mu += P[j] * Sd[j];", "mu += P[j] * S[j];"),
    ("softmax_not_normalised", "for (int j = 0; j < n; ++j) P[j] = P[j] / l;", ""),
    ("logits_scaled_twice", "S[j] = scale * dot(qi, kj, d);", "S[j] = scale * scale * dot(qi, kj, d);"),
    ("no_max_subtraction", "P[j] = exp(S[j] - m);", "P[j] = exp(S[j]);"),
    ("lse_log2", "*lse = m + log(l);", "*lse = m + log2(l);"),
    ("lse_without_max", "*lse = m + log(l);", "*lse = log(l);"),
    ("mask_off_by_one", "n = kv_len[b];", "n = kv_len[b] + 1;"),
    ("value_row_index", "for (int c = 0; c < d; ++c) o[c] += P[j] * vj[c];",
     "for (int c = 0; c < d; ++c) o[c] += P[j] * vj[(c + 1) % d];"),
    ("lse_dot_sign", "if (lse_dot) *lse_dot = mu;", "if (lse_dot) *lse_dot = -mu;"),
    ("lse_dot_unnormalised", "if (lse_dot) *lse_dot = mu;", "if (lse_dot) *lse_dot = mu * l;"),
    ("query_tangent_row", "widen_row(qd, dtype, qoff, d, qdi);",
     "widen_row(qd, dtype, qoff - (i > 0 ? d : 0), d, qdi);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    msrc = tmp_path / f"mutant_{name}.c"
    msrc.write_text(src.replace(old, new))
    lib = oracle.load_library(oracle.compile_oracle(str(msrc), str(tmp_path / f"{name}.so")))
    failed = []
    for pin in oracle_pins.PINS:
        try:
            pin(lib)
        except Exception as e:  # noqa: BLE001 - any failure counts as caught
            failed.append((pin.__name__, type(e).__name__))
    assert failed, f"no pin caught the planted mistake {name}"
