"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a temporary copy of the oracle source (on the
CPU, never in the CUDA path), compiles it, and runs the pin suite against it
in a subprocess: the suite has to fail.
"""
import os
import subprocess
import sys
import tempfile

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "strata_oracle.c")

MUTATIONS = {
    "q2_offset_sign": ("w = d * ((float)c - 1.5f);", "w = d * ((float)c + 1.5f);"),
    "q2_bit_order": ("(codes[k / 4] >> (2 * (k % 4))) & 3", "(codes[k / 4] >> (6 - 2 * (k % 4))) & 3"),
    "q4_nibble_order": ("(k % 2 == 0) ? (byte & 15) : (byte >> 4)",
                        "(k % 2 == 0) ? (byte >> 4) : (byte & 15)"),
    "q4_codebook_entry": ("1,    13,   25,  38,", "1,    13,   26,  38,"),
    "tie_break": ("return (x->i < y->i) ? -1 : (x->i > y->i);",
                  "return (x->i > y->i) ? -1 : (x->i < y->i);"),
    "no_renormalise": ("w[(size_t)t * k + j] = (float)(p[s[j].i] / chosen);",
                       "w[(size_t)t * k + j] = (float)(p[s[j].i]);"),
    "bias_dropped": ("if (bias) l = l + bias[e];", "(void)bias;"),
    "silu_sign": ("double silu = g / (1.0 + exp(-g));", "double silu = g / (1.0 + exp(g));"),
    "gate_up_swapped": ("double silu = g / (1.0 + exp(-g));\n    hd[i] = silu * u;\n    hf[i] = (float)(silu * u);",
                        "double silu = u / (1.0 + exp(-u));\n    hd[i] = silu * g;\n    hf[i] = (float)(silu * g);"),
    "combine_reversed": ("float prod = w[j] * yj[j][h];", "float prod = w[k - 1 - j] * yj[k - 1 - j][h];"),
    "bucket_unstable": ("for (int p = 0; p < P; ++p) {\n    int e = ids[p];",
                        "for (int p = P - 1; p >= 0; --p) {\n    int e = ids[p];"),
    "gate_up_planes_swapped": ("if (m == which) {", "if (m == (which < 2 ? 1 - which : 2)) {"),
    "scale_block_size": ("uint16_t dbits = (uint16_t)(scales[2 * (k / 32)] | (scales[2 * (k / 32) + 1] << 8));",
                         "uint16_t dbits = (uint16_t)(scales[2 * (k / 64)] | (scales[2 * (k / 64) + 1] << 8));"),
    "mxfp4_nibble_order": (">> (4 * (k % 2))) & 15;", ">> (4 - 4 * (k % 2))) & 15;"),
    "mxfp4_e2m1_bias": ("ldexp(1.0 + 0.5 * man, ex - 1)", "ldexp(1.0 + 0.5 * man, ex)"),
    "mxfp4_e2m1_subnormal": ("ex == 0 ? 0.5 * man", "ex == 0 ? 1.0 * man"),
    "mxfp4_sign_bit": ("const int sign = (c >> 3) & 1,", "const int sign = (c >> 2) & 1,"),
    "mxfp4_e8m0_bias": ("ldexp(1.0, e - 127); }", "ldexp(1.0, e - 128); }"),
    "mxfp4_e8m0_nan": ("e == 255 ? NAN :", "e == 256 ? NAN :"),
    "mxfp4_scale_width": ("(fmt == 3 ? 1 : 2)", "2"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(name, tmp_path):
    before, after = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor not found once: {name}"
    mut = tmp_path / "mut.c"
    mut.write_text(src.replace(before, after))
    lib = tmp_path / "libmut.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC",
                    "-o", str(lib), str(mut), "-lm"], check=True)
    env = dict(os.environ, STRATA_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-q", "-x",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode != 0, f"pins did not catch mutation {name}:\n{r.stdout[-2000:]}"
