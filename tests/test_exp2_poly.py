"""The cubic the attention kernel uses for part of its exp2 evaluations:
the kernel source carries the coefficients that csrc/fit_exp2.py fits, and
the float32 emulation of the kernel's bit manipulation stays within 2e-4
relative error of 2^x over the arguments it can receive."""

import os
import re

import numpy as np

from long_context_mean_b200.csrc import fit_exp2

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                   "long_context_mean_b200", "csrc", "attn_tc.cu")


def kernel_coefficients():
    text = open(SRC).read()
    vals = {}
    for name, val in re.findall(r"kExpC(\d)\s*=\s*([-+0-9.eE]+)f", text):
        vals[int(name)] = np.float32(float(val))
    return [vals[i] for i in range(4)]


def test_kernel_carries_fitted_coefficients():
    fitted = fit_exp2.fit()
    assert np.allclose(kernel_coefficients(), fitted, rtol=2e-6, atol=0)


def test_emulation_error_bound():
    c = kernel_coefficients()
    assert fit_exp2.max_rel_error(c, -125.0, 8.0, 400001) < 2e-4
    # the clamp keeps very negative arguments tiny and positive
    tiny = fit_exp2.emulate(np.array([-1000.0, -200.0, -125.0], np.float32), c)
    assert np.all(tiny > 0) and np.all(tiny < 1e-37)
