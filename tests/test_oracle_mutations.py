"""Mutation check of the oracle's pins (CPU, opt-in: SAGE_MUTATION=1, a few
minutes).  Each case is the oracle's C source with one plausible mistake
planted; the pin tests must fail on it.  The one equivalent mutant (E4M3
saturation moved from 448 to 480: the encoder's range check saturates the
same inputs) must leave every pin passing."""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.skipif(os.environ.get("SAGE_MUTATION") != "1",
                                reason="opt-in: set SAGE_MUTATION=1")

# name: (text in oracle/sage_oracle.c, replacement), first occurrence only
MUTANTS = {
    "mean_divisor_Lk_minus_1": ("/ (double)Lk;", "/ (double)(Lk > 1 ? Lk - 1 : 1);"),
    "smoothing_adds_the_mean": ("- m[ch];", "+ m[ch];"),
    "quant_range_128": ("float r = 127.0f / a;", "float r = 128.0f / a;"),
    "round_half_away_from_zero": ("float t = nearbyintf(y);", "float t = roundf(y);"),
    "scale_a_over_128": ("return a / 127.0f;", "return a / 128.0f;"),
    "amax_without_abs": ("float m = fabsf(x[i]);", "float m = x[i];"),
    "no_log2e_fold": ("sm_scale * 1.4426950408889634074", "sm_scale * 1.0"),
    "q_scale_without_fold": ("q_scale[(int64_t)bh * nqb + blk] = s * c;",
                             "q_scale[(int64_t)bh * nqb + blk] = s;"),
    "k_blocks_of_128": ("const int BK = 64;", "const int BK = 128;"),
    "causal_off_by_one": ("(int64_t)i + (Lk - Lq) + 1;", "(int64_t)i + (Lk - Lq);"),
    "causal_top_left": ("(int64_t)i + (Lk - Lq) + 1;", "(int64_t)i + 1;"),
    "noncausal_one_key_short": ("        return Lk;", "        return Lk - 1;"),
    "p_not_rounded_to_fp16": ("oracle_half_to_double(oracle_double_to_half(exp2(s[j] - mx)))",
                              "exp2(s[j] - mx)"),
    "natural_exp_in_sim": ("oracle_double_to_half(exp2(s[j] - mx))",
                           "oracle_double_to_half(exp(s[j] - mx))"),
    "k_scale_indexed_by_query": ("k_scale[bhk * nkb + j / 64]", "k_scale[bhk * nkb + i / 64]"),
    "gqa_modulo_mapping": ("(int64_t)b * Hkv + h / group;", "(int64_t)b * Hkv + h % Hkv;"),
    "q_scale_ignores_block_rows": ("q_scale[bh * nqb + i / BQ]", "q_scale[bh * nqb + i / 128]"),
    "v_read_transposed": ("o[c] += p * oracle_half_to_double(vj[c]);",
                          "o[c] += p * oracle_half_to_double(v[(bhk * d + c) * Lk + j]);"),
    "sim_without_normalization": ("for (int c = 0; c < d; ++c) o[c] /= l;", ""),
    "half_subnormal_scale": ("ldexp((double)m, -24);", "ldexp((double)m, -25);"),
    "half_ties_away": ("double n = nearbyint(ldexp(a, 10 - E));",
                       "double n = floor(ldexp(a, 10 - E) + 0.5);"),
    "fp64_uses_exp2": ("double p = exp(s[j] - mx);", "double p = exp2(s[j] - mx);"),
    "fp64_without_sm_scale": ("s[j] = acc * sm_scale;", "s[j] = acc;"),
    "e4m3_ties_away": ("double m = nearbyint((2.0 * f - 1.0) * 8.0);",
                       "double m = floor((2.0 * f - 1.0) * 8.0 + 0.5);"),
    "e4m3_subnormal_grid": ("double t = a * 512.0;", "double t = a * 256.0;"),
    "v8_scale_over_447": ("a / 448.0f : 0.0f;", "a / 447.0f : 0.0f;"),
    "v8_amax_without_abs": ("float x = (float)fabs(oracle_half_to_double(src[(int64_t)t * d]));",
                            "float x = (float)oracle_half_to_double(src[(int64_t)t * d]);"),
    "fp8_without_row_sum": ("o[c] = acc * (double)v_scale[bhk * d + c] / l;",
                            "o[c] = acc * (double)v_scale[bhk * d + c];"),
    "fp8_p_scale_240": ("float p448 = (float)p * 448.0f;", "float p448 = (float)p * 240.0f;"),
    "fp8_p_not_rounded": ("pq[j] = oracle_e4m3_decode(oracle_e4m3_encode(p448)) / 448.0;",
                          "pq[j] = p;"),
}
EQUIVALENT = {"e4m3_saturation_480": ("if (a >= 448.0)", "if (a >= 480.0)")}


def _run_pins(tmp_path, text, replacement):
    src = open(os.path.join(ROOT, "oracle", "sage_oracle.c")).read()
    assert text in src, text
    (tmp_path / "oracle").mkdir()
    shutil.copy(os.path.join(ROOT, "oracle", "__init__.py"), tmp_path / "oracle")
    (tmp_path / "oracle" / "sage_oracle.c").write_text(src.replace(text, replacement, 1))
    shutil.copytree(os.path.join(ROOT, "tests"), tmp_path / "tests",
                    ignore=shutil.ignore_patterns("__pycache__"))
    os.symlink(os.path.join(ROOT, "bit_quantized_attention_mean_b200"),
               tmp_path / "bit_quantized_attention_mean_b200")
    shutil.copy(os.path.join(ROOT, "pytest.ini"), tmp_path)
    env = dict(os.environ, SAGE_MUTATION="0")
    return subprocess.run([sys.executable, "-m", "pytest", "tests/test_oracle_pins.py", "-q", "-x",
                           "-p", "no:cacheprovider"], cwd=tmp_path, capture_output=True,
                          text=True, timeout=900, env=env)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_the_mutant(name, tmp_path):
    r = _run_pins(tmp_path, *MUTANTS[name])
    assert r.returncode != 0, f"{name} survived the pins"


@pytest.mark.parametrize("name", sorted(EQUIVALENT))
def test_equivalent_mutant_changes_nothing(name, tmp_path):
    r = _run_pins(tmp_path, *EQUIVALENT[name])
    assert r.returncode == 0, r.stdout[-2000:]
