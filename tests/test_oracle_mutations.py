"""The oracle's pins (decode and prefill) catch plausible mistakes.

Each case plants one mistake in a copy of oracle.c (a dropped term, a wrong
sign, a wrong index, a transposed operand ...), builds it into a temporary
library and runs the pin suite against it in a child process; the suite must
fail.  Nothing here touches a GPU.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTATIONS = {
    "scale_dropped": ("x[t] = scale * dot;", "x[t] = dot;"),
    "softmax_sign": ("x[t] = exp(x[t] - m);", "x[t] = exp(m - x[t]);"),
    "sum_not_accumulated": ("Z += x[t];", "Z = x[t];"),
    "not_normalised": ("double p = x[t] / Z;", "double p = x[t];"),
    "key_value_swapped": ("dot += q[d] * K[t * D + d];", "dot += q[d] * V[t * D + d];"),
    "offset_from_block_index": ("int64_t o = t % B;", "int64_t o = (t / B) % B;"),
    "block_from_offset": ("int32_t p = table_row[t / B];", "int32_t p = table_row[(t % B) % 3];"),
    "head_group_interleaved": ("for (int h = g * G; h < (g + 1) * G && rc == OR_OK; ++h) {",
                               "for (int h = g; h < Hq && rc == OR_OK; h += Hkv) {"),
    "f16_exponent_bias": ("v = ldexp((double)(f | 0x400), e - 25);",
                          "v = ldexp((double)(f | 0x400), e - 24);"),
    "scatter_offset": ("int64_t frame = slot / B, off = slot % B;",
                       "int64_t frame = slot / B, off = (B - 1) - slot % B;"),
    "round_ties_away_from_zero": ("if (r > 0.5 || (r == 0.5 && fmod(f, 2.0) != 0.0)) f += 1.0;",
                                  "if (r >= 0.5) f += 1.0;"),
    "round_truncates": ("if (r > 0.5 || (r == 0.5 && fmod(f, 2.0) != 0.0)) f += 1.0;",
                        "(void)r;"),
    "round_no_carry": ("      f = ldexp(1.0, frac_bits);\n      e += 1;", "      f = ldexp(1.0, sig) - 1.0;"),
    "prefill_not_causal": ("attend(out + ((int64_t)i * Hq + h) * D, NULL, x, qd, K, V, (int64_t)p0 + i + 1, D, scale);",
                           "attend(out + ((int64_t)i * Hq + h) * D, NULL, x, qd, K, V, n, D, scale);"),
    "prefill_excludes_self": ("attend(out + ((int64_t)i * Hq + h) * D, NULL, x, qd, K, V, (int64_t)p0 + i + 1, D, scale);",
                              "attend(out + ((int64_t)i * Hq + h) * D, NULL, x, qd, K, V, (int64_t)p0 + i, D, scale);"),
    "prefill_head_group_interleaved": ("for (int32_t i = 0; i < T && rc == OR_OK; ++i) {\n      for (int h = g * G; h < (g + 1) * G; ++h) {",
                                       "for (int32_t i = 0; i < T && rc == OR_OK; ++i) {\n      for (int h = g; h < Hq; h += Hkv) {"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_fail_on_planted_mistake(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    mutated = tmp_path / "oracle_mut.c"
    mutated.write_text(src.replace(old, new))
    so = tmp_path / "liboracle_mut.so"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-fPIC", "-shared", "-o", str(so),
                           str(mutated), "-lm"])
    env = dict(os.environ, PKV_ORACLE_LIB=str(so))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py"),
                        os.path.join(ROOT, "tests", "test_oracle_prefill.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"pins did not catch mutation {name}:\n{r.stdout[-2000:]}"
    assert "failed" in r.stdout or "error" in r.stdout.lower()
