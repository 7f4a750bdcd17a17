"""The conv3d oracle against its pins, and planted mistakes the pins must catch (CPU
only).  Each mutation is a textual edit of conv3d_oracle.c compiled to a temporary
library; the shipped oracle is never modified, and every mutation keeps all memory
accesses inside the arrays."""
import os

import pytest

import oracle
import oracle_pins_conv3d


@pytest.fixture(scope="module")
def lib():
    return oracle.load_conv3d()


@pytest.mark.parametrize("pin", oracle_pins_conv3d.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(lib, pin):
    pin(lib)


MUTATIONS = {
    "depth stride forgotten": ("long id = od * stride", "long id = od"),
    "depth dilation forgotten": ("long id = od * stride + kd * dilation - pad;", "long id = od * stride + kd - pad;"),
    "depth padding forgotten": ("long id = od * stride + kd * dilation - pad;", "long id = od * stride + kd * dilation;"),
    "last frame dropped": ("if (id < 0 || id >= D)", "if (id < 0 || id >= D - 1)"),
    "weight depth index dropped": ("w[(((oc * cin_g + c) * Kd + kd) * Kh + kh) * Kw + kw]",
                                   "w[(((oc * cin_g + c) * Kd) * Kh + kh) * Kw + kw]"),
    "input depth index from the row": ("x[(((n * C_in + ic) * D + id) * H + ih)", "x[(((n * C_in + ic) * D + (ih % D)) * H + ih)"),
    "group offset dropped": ("long ic = g * cin_g + c;", "long ic = c;"),
    "bias dropped": ("double acc = bias ? bias[oc] : 0.0;", "double acc = 0.0;"),
    "depth extent off by one": ("*Do = extent(D, Kd, stride, pad, dilation);",
                                "*Do = extent(D, Kd, stride, pad, dilation) - (D > 1 ? 1 : 0);"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(oracle.C3D_SOURCE, encoding="utf-8").read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    tag = "".join(ch if ch.isalnum() else "_" for ch in name)
    c_path = os.path.join(tmp_path, f"{tag}.c")
    so_path = os.path.join(tmp_path, f"lib{tag}.so")
    with open(c_path, "w", encoding="utf-8") as f:
        f.write(src.replace(old, new))
    oracle.build(c_path, so_path)
    mutant = oracle.load_conv3d(so_path)
    caught = []
    for pin in oracle_pins_conv3d.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake: {name}"
