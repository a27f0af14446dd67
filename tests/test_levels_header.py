"""The CUDA library's level / threshold header is what its generator produces,
and the thresholds are exactly the round-down midpoints of the oracle's
levels (checked in rational arithmetic)."""
import importlib.util
import os
import re
from fractions import Fraction

import numpy as np

import oracle as O

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "quantized_linear_layers_nf4_b200", "csrc")


def _gen():
    spec = importlib.util.spec_from_file_location("gen_levels", os.path.join(CSRC, "gen_levels.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _parse(name):
    text = open(os.path.join(CSRC, "nf4_levels.h")).read()
    body = re.search(r"#define %s \{(.*?)\}" % name, text, re.S).group(1)
    return [float.fromhex(h[:-1]) for h in re.findall(r"-?0x[0-9a-fA-Fp.+-]+f", body)]


def test_header_is_up_to_date():
    gen = _gen()
    assert open(os.path.join(CSRC, "nf4_levels.h")).read() == gen.render()


def test_header_levels_equal_oracle_levels():
    lv = np.array(_parse("NF4_LEVELS_INIT"), dtype=np.float32)
    assert lv.size == 16
    assert np.array_equal(lv.view(np.uint32), O.codebook().view(np.uint32))


def test_thresholds_are_round_down_midpoints():
    c = [Fraction(float(v)) for v in O.codebook()]
    t = _parse("NF4_THRESHOLDS_INIT")
    assert len(t) == 15
    for j in range(15):
        mid = (c[j] + c[j + 1]) / 2
        tj = Fraction(t[j])
        assert tj <= mid
        nxt = Fraction(float(np.nextafter(np.float32(t[j]), np.float32(2))))
        assert nxt > mid, "t_%d is not the largest fp32 <= midpoint" % j


def test_header_fp4_levels_equal_oracle_fp4_codebook():
    lv = np.array(_parse("FP4_LEVELS_INIT"), dtype=np.float32)
    assert lv.size == 16
    assert np.array_equal(lv.view(np.uint32), O.codebook("fp4").view(np.uint32))


def test_fp4_thresholds_are_round_down_midpoints_of_the_magnitudes():
    c = [Fraction(float(v)) for v in O.codebook("fp4")[:8]]
    t = _parse("FP4_THRESHOLDS_INIT")
    assert len(t) == 7
    for j in range(7):
        mid = (c[j] + c[j + 1]) / 2
        assert Fraction(t[j]) <= mid
        assert Fraction(float(np.nextafter(np.float32(t[j]), np.float32(2)))) > mid
