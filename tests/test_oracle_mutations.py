"""Plausible mistakes planted in a copy of the oracle must each fail at least one pin.

Each mutation is a textual edit of conv2d_oracle.c compiled to a temporary
library; the shipped oracle is never modified.  Every mutation keeps all memory
accesses inside the arrays (bounds checks are tightened, never loosened)."""
import os

import pytest

import oracle
import oracle_pins

MUTATIONS = {
    "bias dropped": ("double acc = bias ? bias[oc] : 0.0;", "double acc = 0.0;"),
    "bias indexed by group": ("bias ? bias[oc]", "bias ? bias[g]"),
    "padding added instead of subtracted": ("kh * dilation - pad;", "kh * dilation + pad;"),
    "padding forgotten on columns": ("kw * dilation - pad;", "kw * dilation;"),
    "stride forgotten on rows": ("long ih = oh * stride", "long ih = oh"),
    "dilation forgotten": ("kh * dilation - pad", "kh - pad"),
    "last row dropped by the bounds check": ("ih >= H)", "ih >= H - 1)"),
    "first column dropped by the bounds check": ("iw < 0 ||", "iw < 1 ||"),
    "column index built from the row tap": ("long iw = ow * stride + kw", "long iw = ow * stride + kh"),
    "row index built from the output column": ("long ih = oh * stride", "long ih = ow * stride"),
    "group offset dropped": ("long ic = g * cin_g + c;", "long ic = c;"),
    "weight channel index dropped": ("w[((oc * cin_g + c) * Kh", "w[((oc * cin_g) * Kh"),
    "weight taps transposed": ("* Kh + kh) * Kw + kw]", "* Kh + (kw % Kh)) * Kw + (kh % Kw)]"),
    "subtraction instead of accumulation": ("acc += xv * wv;", "acc -= xv * wv;"),
    "single-precision accumulator": ("double acc = bias", "float acc = bias"),
    "output size off by one": ("*out = numer / stride + 1;", "*out = numer / stride;"),
    "output size rounded up": ("*out = numer / stride + 1;", "*out = (numer + stride - 1) / stride + 1;"),
}


def _build_mutant(tmp_path, name, old, new):
    src = open(oracle.SOURCE, encoding="utf-8").read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    mutated = src.replace(old, new)
    tag = "".join(ch if ch.isalnum() else "_" for ch in name)
    c_path = os.path.join(tmp_path, f"{tag}.c")
    so_path = os.path.join(tmp_path, f"lib{tag}.so")
    with open(c_path, "w", encoding="utf-8") as f:
        f.write(mutated)
    oracle.build(c_path, so_path)
    return oracle.load(so_path)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    lib = _build_mutant(str(tmp_path), name, old, new)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake: {name}"
