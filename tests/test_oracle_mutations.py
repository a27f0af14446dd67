"""Plant plausible mistakes in a copy of the oracle's C source (on the CPU, in a
temporary directory) and check that the pins in ``test_oracle_pins.py`` catch
every one of them.  The committed oracle is never modified."""
import inspect
import json
import os
import subprocess

import pytest

import oracle as O
from oracle import build_oracle
import tests.test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(build_oracle.__file__), "nf4_oracle.c")

# (name, text to find, replacement).  Every occurrence is replaced.
MUTANTS = [
    ("nibble order swapped", "(idx[2 * i] << 4) | idx[2 * i + 1]", "(idx[2 * i + 1] << 4) | idx[2 * i]"),
    ("ties to the upper index", "if (d < best_d)", "if (d <= best_d)"),
    ("reciprocal multiply instead of division", "float x = blk[j] / am;",
     "float x = blk[j] * (1.0f / am);"),
    ("left-to-right mean", "for (int i = 0; i < h; ++i) a[i] = a[i] + a[i + h];",
     "for (int i = 0; i < h; ++i) a[i] = a[i] + a[i + h];\n    a[0] = 0;\n"
     "    for (int i = 0; i < count; ++i) a[0] = a[0] + v[i];"),
    ("residual sign flipped", "float r = absmax[b] - mu;", "float r = mu - absmax[b];"),
    ("8-bit range 128", "127.0f", "128.0f"),
    ("outermost probability off", "1.0 / 32.0", "1.0 / 31.0"),
    ("zero block mapped to level 8", "idx[j] = 7;", "idx[j] = 8;"),
    ("bf16 truncation instead of rounding", "u += 0x7FFFu + lsb;", "u += 0u * lsb;"),
    ("mean dropped from absmax dequant", "return u + mu;", "return u;"),
    ("dequant scale index off by a block", "absmax_scale[b / 256]", "absmax_scale[b / 255]"),
    ("weight operand transposed", "(double)bf16_bits_to_f32(w[j * k + t])",
     "(double)bf16_bits_to_f32(w[t * n + j])"),
    ("absmax from the signed maximum", "float a = fabsf(blk[j]);", "float a = blk[j];"),
    ("negative levels one short", "for (int i = 0; i < 7; ++i) v[k++] = -orc_norm_ppf",
     "for (int i = 1; i < 8; ++i) v[k++] = -orc_norm_ppf"),
    ("FP4 exponent bias 0", "ldexp(1.0 + 0.5 * m, e - 1)", "ldexp(1.0 + 0.5 * m, e)"),
    ("FP4 subnormals flushed", "(e == 0) ? 0.5 * m :", "(e == 0) ? 0.0 * m :"),
    ("FP4 zero block mapped to -0", "if (qt == ORC_FP4) idx[j] = 0;", "if (qt == ORC_FP4) idx[j] = 8;"),
    ("FP4 quantized with the NF4 levels", "const float* c = table_of(qt);", "const float* c = codebook();"),
    # rounding-order readings (each result is still close; only the bits differ)
    ("absmax dequant as q * (s / 127)",
     "float t = (float)absmax_q[b] / 127.0f;\n    float u = t * absmax_scale[b / 256];",
     "float t = absmax_scale[b / 256] / 127.0f;\n    float u = (float)absmax_q[b] * t;"),
    ("absmax dequant with the rounded reciprocal of 127", "float t = (float)absmax_q[b] / 127.0f;",
     "float t = (float)absmax_q[b] * (1.0f / 127.0f);"),
    ("DQ code as r * (127 / s)", "float t = r / s;\n                float u = t * 127.0f;",
     "float t = 127.0f / s;\n                float u = r * t;"),
    ("DQ code rounds half away from zero", "q = (int)nearbyintf(u);", "q = (int)roundf(u);"),
    ("DQ mean divided in fp32", "return (float)(orc_dq_sum(absmax, nb) / (double)nb);",
     "return (float)orc_dq_sum(absmax, nb) / (float)nb;"),
    ("weight dequant product in fp64 with a tiny bias", "out_f32[e] = c[idx] * a;",
     "out_f32[e] = (float)((double)c[idx] * (double)a * (1.0 + 1e-9));"),
]


def _run_pins() -> list:
    """Run every pin; return the names of those that fail."""
    with open(os.path.join(os.path.dirname(__file__), "golden", "pages_figures.json")) as f:
        golden = json.load(f)
    failed = []
    for name, fn in inspect.getmembers(pins, inspect.isfunction):
        if not name.startswith("test_"):
            continue
        kwargs = {"golden": golden} if "golden" in inspect.signature(fn).parameters else {}
        try:
            fn(**kwargs)
        except Exception:  # noqa: BLE001 -- any failure counts as caught
            failed.append(name)
    return failed


def test_unmodified_oracle_passes_every_pin():
    assert _run_pins() == []


@pytest.mark.parametrize("name,find,repl", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_the_mutant(tmp_path, name, find, repl):
    src = open(SRC).read()
    assert find in src, "mutation site not found: %s" % name
    mutated = src.replace(find, repl)
    c_path = tmp_path / "nf4_oracle.c"
    c_path.write_text(mutated)
    (tmp_path / "nf4_oracle.h").write_text(open(SRC[:-2] + ".h").read())
    so = tmp_path / "liboracle_mut.so"
    subprocess.run(["gcc", *build_oracle.CFLAGS, str(c_path), "-o", str(so), "-lm"], check=True)
    try:
        O.use_library(str(so))
        failed = _run_pins()
    finally:
        O.use_library(None)
    assert failed, "no pin caught the mutant '%s'" % name
