"""The oracle's pins must catch plausible mistakes.

Each case copies the oracle's C source to a temporary directory, plants one
mistake there (the committed source is never touched), builds it, and runs a pin
from the oracle test files against the mutated build, which must fail.
"""
import importlib.util
import os

import pytest

import tests.test_oracle_attention as pa
import tests.test_oracle_backward as pb
import tests.test_oracle_gate_gather as pg
import tests.test_oracle_topk as pt

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = [
    # (name, original text, planted mistake, pin that must fail)
    ("bias_sign", "(double)gain[h] * (double)logsig[j]", "-(double)gain[h] * (double)logsig[j]",
     lambda o: pa.test_zero_query_closed_form(o)),
    ("temperature_dropped", "double scale = 1.0 / (sqrt((double)dh) * (double)temp[h]);",
     "double scale = 1.0 / sqrt((double)dh);",
     lambda o: pa.test_temperature_equals_query_scaling(o)),
    ("temperature_on_bias",
     "double lg = dot * scale + (logsig ? (double)gain[h] * (double)logsig[j] : 0.0);",
     "double lg = dot * scale + (logsig ? (double)gain[h] * (double)logsig[j] : 0.0) / (double)temp[h];",
     lambda o: pa.test_equal_keys_make_temperature_irrelevant_to_bias(o)),
    ("gqa_mapping", "int32_t hk = h / group;", "int32_t hk = h % Hkv;",
     lambda o: pa.test_reduces_to_causal_attention(o, [37], 4, 2, 16)),
    ("tie_break_reversed", "    return a->idx < b->idx;\n}", "    return a->idx > b->idx;\n}",
     lambda o: pt.test_all_equal_scores_keep_lowest_indices(o)),
    ("question_dropped", "for (int32_t p = e; p < n; ++p) kept[m++] = p;", "",
     lambda o: pt.test_brute_force_small(o, 3)),
    ("gelu_tanh", "erf(a / sqrt(2.0))", "tanh(0.7978845608 * (a + 0.044715 * a * a * a))",
     lambda o: pg.test_gate_closed_form_identity_slice(o)),
    ("rope_sign", "out[i] = x0 * c - x1 * s;", "out[i] = x0 * c + x1 * s;",
     lambda o: pg.test_rope_matches_complex_rotation(o, 64, 1e6)),
    ("rope_pairing", "double x0 = x[i], x1 = x[i + half];", "double x0 = x[2 * i], x1 = x[2 * i + 1];",
     lambda o: pg.test_rope_matches_complex_rotation(o, 64, 1e6)),
    ("logsig_on_question", "out[i] = is_doc ? log_sigmoid((double)z[row]) : 0.0;",
     "out[i] = log_sigmoid((double)z[row]);",
     lambda o: pg.test_logsig_matches_torch_and_protects_question(o)),
    # the attention row behind the backward's loss (tgo_attention_loss)
    ("loss_bias_sign", "double lg = dot * scale + gain[h] * logsig[j];",
     "double lg = dot * scale - gain[h] * logsig[j];",
     lambda o: pb.test_loss_is_the_forward_inner_product(o)),
    ("loss_temperature_on_bias", "double lg = dot * scale + gain[h] * logsig[j];",
     "double lg = dot * scale + gain[h] * logsig[j] / temp[h];",
     lambda o: pb.test_loss_is_the_forward_inner_product(o)),
    ("loss_gqa_mapping", "const float* kj = k + (j * Hkv + hk) * (int64_t)dh;\n        double dot = 0.0;\n"
     "        for (int32_t c = 0; c < dh; ++c) dot += (double)qi[c] * (double)kj[c];\n"
     "        s[j - j0] = dot;",
     "const float* kj = k + (j * Hkv + h % Hkv) * (int64_t)dh;\n        double dot = 0.0;\n"
     "        for (int32_t c = 0; c < dh; ++c) dot += (double)qi[c] * (double)kj[c];\n"
     "        s[j - j0] = dot;",
     lambda o: pb.test_loss_is_the_forward_inner_product(o)),
]


def _mutant(tmp_path, name, old, new):
    src = open(os.path.join(ROOT, "oracle", "tg_oracle.c")).read()
    assert src.count(old) >= 1, f"mutation {name}: text not found in oracle source"
    d = tmp_path / name
    d.mkdir()
    (d / "tg_oracle.c").write_text(src.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"oracle_mut_{name}",
                                                  os.path.join(ROOT, "oracle", "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    mod._SRC = str(d / "tg_oracle.c")
    mod._LIB = str(d / "libtg_oracle.so")
    mod._lib = None
    return mod


@pytest.mark.parametrize("name,old,new,pin", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pin_catches_planted_mistake(tmp_path, name, old, new, pin):
    mod = _mutant(tmp_path, name, old, new)
    with pytest.raises((AssertionError, ValueError)):
        pin(mod)
