"""The oracle pins must catch plausible mistakes.

Each case copies the oracle's C source, plants one mistake of the kind a
reader could make when writing the formulas of "Kwai Keye-VL-2.0 Technical
Report" review (xllm-io), 核心公式, and report translation sections 2.3.1 /
2.3.2 (a dropped ReLU or scale, a wrong sign or index, a reversed tie rule, a
wrong GQA group map, a missing normalisation, a wrong FP8 exponent bias) and
2.3.3 (the indexer's distillation losses),
compiles it with gcc, and runs the pin suite against that copy in a fresh
process.  The pin suite must fail for every one of them.  Everything runs on
the CPU.
"""
import os
import subprocess
import sys

import pytest

from conftest import ROOT

SRC = os.path.join(ROOT, "oracle", "dsa_oracle.c")

MUTATIONS = {
    "relu_dropped": ("double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;"),
    "query_scale_dropped": ("q8_t[(size_t)j * dI + c]) * sq_t;", "q8_t[(size_t)j * dI + c]);"),
    "key_scale_dropped": ("dsa_oracle_e4m3_to_double(k8_s[c]) * sk_s;", "dsa_oracle_e4m3_to_double(k8_s[c]);"),
    "weight_sign_lost": ("I += (double)w_t[j] * relu;", "I += fabs((double)w_t[j]) * relu;"),
    "self_excluded": ("if (s > t) { row[s] = -INFINITY; continue; }", "if (s >= t) { row[s] = -INFINITY; continue; }"),
    "tie_to_higher_index": ("return (x->s > y->s) - (x->s < y->s);", "return (x->s < y->s) - (x->s > y->s);"),
    "output_not_ascending": ("qsort(out, (size_t)k, sizeof(int32_t), cmp_int32);", ";"),
    "short_row_truncated": ("for (int i = 0; i < n; ++i) out[i] = i;", "for (int i = 0; i < n - 1; ++i) out[i] = i; if (n) out[n - 1] = -1;"),
    "gqa_group_interleaved": ("int g = h / G;\n            int n = 0;\n            for (int i = 0; i < k; ++i) {\n                int32_t s = idx[(size_t)r * k + i];",
                              "int g = h % Hkv;\n            int n = 0;\n            for (int i = 0; i < k; ++i) {\n                int32_t s = idx[(size_t)r * k + i];"),
    "softmax_not_normalised": ("for (int d = 0; d < D; ++d) o_h[d] /= denom;", ";"),
    "sm_scale_dropped": ("logit[i] = sm_scale * dot;", "logit[i] = dot;"),
    "e4m3_bias_off": ("mag = ldexp(1.0 + (double)m / 8.0, e - 7);", "mag = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "e4m3_subnormal_scale": ("mag = ldexp((double)m / 8.0, 1 - 7);", "mag = ldexp((double)m / 8.0, -7);"),
    "kl_sign_flipped": ("if (a > 0.0) kl += a * (log(a) - (Ir[S[i]] - logz));",
                        "if (a > 0.0) kl += a * ((Ir[S[i]] - logz) - log(a));"),
    "kl_target_not_renormalised": ("double a = pr[S[i]] / mass;", "double a = pr[S[i]];"),
    "kl_softmax_not_normalised": ("double logz = mx + log(z);", "double logz = mx;"),
    "kl_sparse_padding_counted": ("if (s >= 0 && s <= t) S[n++] = s;", "if (s <= t) S[n++] = s < 0 ? 0 : s;"),
    "page_slot_swapped": ("size_t slot = (size_t)p * page + (size_t)(s % page);\n            out[(size_t)b * ld + s]",
                          "size_t slot = (size_t)p * page + (size_t)((page - 1) - s % page);\n            out[(size_t)b * ld + s]"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new))
    lib = tmp_path / "libmutant.so"
    subprocess.check_call(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-fvisibility=hidden",
                           "-o", str(lib), str(mutated), "-lm"])
    env = dict(os.environ, DSA_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutation {name}:\n{r.stdout[-2000:]}"
