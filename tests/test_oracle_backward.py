"""The backward oracle against its pins, and planted mistakes that the pins must catch
(CPU only).  Each mutation is a textual edit of conv2d_backward_oracle.c compiled to a
temporary library; the shipped oracle is never modified, and every mutation keeps all
memory accesses inside the arrays."""
import os

import numpy as np
import pytest

import oracle
import oracle_pins_backward


@pytest.fixture(scope="module")
def lib():
    return oracle.load_backward()


@pytest.mark.parametrize("pin", oracle_pins_backward.ALL_PINS, ids=lambda p: p.__name__)
def test_pin(lib, pin):
    pin(lib)


def test_rejects_bad_shapes(lib):
    x = np.zeros((1, 4, 5, 5))
    w = np.zeros((2, 4, 3, 3))
    with pytest.raises(ValueError):
        oracle.conv2d_backward(np.zeros((1, 2, 4, 4)), x, w, 1, 1, lib=lib)  # dy is 5x5 for pad 1
    with pytest.raises(ValueError):
        oracle.conv2d_backward(np.zeros((1, 3, 3, 3)), x, w, lib=lib)       # C_out mismatch


MUTATIONS = {
    "dx assigned instead of accumulated": (
        "dx[((n * C_in + ic) * H + ih) * W + iw] +=", "dx[((n * C_in + ic) * H + ih) * W + iw] ="),
    "dW assigned instead of accumulated": (
        "dW[((oc * cin_g + c) * Kh + kh) * Kw + kw] +=", "dW[((oc * cin_g + c) * Kh + kh) * Kw + kw] ="),
    "dW taps transposed": ("dW[((oc * cin_g + c) * Kh + kh) * Kw + kw] +=",
                           "dW[((oc * cin_g + c) * Kh + (kw % Kh)) * Kw + (kh % Kw)] +="),
    "dx scattered with the weight's taps transposed": (
        "w[((oc * cin_g + c) * Kh + kh) * Kw + kw] * grad_out;",
        "w[((oc * cin_g + c) * Kh + (kw % Kh)) * Kw + (kh % Kw)] * grad_out;"),
    "padding forgotten in the scatter": ("long ih = oh * stride + kh * dilation - pad;\n                                if (ih < 0 || ih >= H)\n                                    continue;\n                                for (long kw = 0; kw < Kw; ++kw) {\n                                    long iw = ow * stride + kw * dilation - pad;\n                                    if (iw < 0 || iw >= W)\n                                        continue;\n                                    dx",
                                         "long ih = oh * stride + kh * dilation;\n                                if (ih < 0 || ih >= H)\n                                    continue;\n                                for (long kw = 0; kw < Kw; ++kw) {\n                                    long iw = ow * stride + kw * dilation;\n                                    if (iw < 0 || iw >= W)\n                                        continue;\n                                    dx"),
    "stride forgotten in the weight gradient": ("long ih = oh * stride + kh * dilation - pad;\n                                if (ih < 0 || ih >= H)\n                                    continue;\n                                for (long kw = 0; kw < Kw; ++kw) {\n                                    long iw = ow * stride + kw * dilation - pad;\n                                    if (iw < 0 || iw >= W)\n                                        continue;\n                                    dW",
                                                "long ih = oh + kh * dilation - pad;\n                                if (ih < 0 || ih >= H)\n                                    continue;\n                                for (long kw = 0; kw < Kw; ++kw) {\n                                    long iw = ow + kw * dilation - pad;\n                                    if (iw < 0 || iw >= W)\n                                        continue;\n                                    dW"),
    "bias gradient over the first image only": ("for (long n = 0; n < N; ++n)\n                for (long oh = 0; oh < Ho; ++oh)\n                    for (long ow = 0; ow < Wo; ++ow)\n                        acc +=",
                                                "for (long n = 0; n < 1; ++n)\n                for (long oh = 0; oh < Ho; ++oh)\n                    for (long ow = 0; ow < Wo; ++ow)\n                        acc +="),
    "group offset dropped": ("long ic = g * cin_g + c;", "long ic = c;"),
    "last input row dropped": ("if (ih < 0 || ih >= H)", "if (ih < 0 || ih >= H - 1)"),
    "single-precision accumulation": ("double grad_out =", "float grad_out ="),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutation_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(oracle.BWD_SOURCE, encoding="utf-8").read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    tag = "".join(ch if ch.isalnum() else "_" for ch in name)
    c_path = os.path.join(tmp_path, f"{tag}.c")
    so_path = os.path.join(tmp_path, f"lib{tag}.so")
    with open(c_path, "w", encoding="utf-8") as f:
        f.write(src.replace(old, new))
    oracle.build(c_path, so_path)
    mutant = oracle.load_backward(so_path)
    caught = []
    for pin in oracle_pins_backward.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the planted mistake: {name}"
