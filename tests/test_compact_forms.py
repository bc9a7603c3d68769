"""The accuracy claims of the compact step-preparation forms of the bf16
tensor-core kernel (selective_state_space_12_b200/csrc/common.cuh:
softplus_compact, expm1_compact), checked on the CPU in fp64:

* log1p(e) for e < 2^-6 by e - e^2/2 + e^3/3 - e^4/4: relative truncation
  below 2e-8 (the next term is below e^5/5);
* for e >= 2^-6 the hardware log's absolute error bound of 2^-21.41 on
  [0.5, 2] (CUDA's published bound for __logf) gives a relative error below
  3e-5 of log1p(e) >= log1p(2^-6);
* expm1(x) for |x| < 1/2 by x (1 + x/2 + ... + x^6/5040): relative truncation
  below 3e-7.
Both stay far inside bf16 I/O's 2^-8 rounding."""
import numpy as np

CUT = 2.0 ** -6


def test_log1p_series_below_the_cut():
    e = np.logspace(-30, np.log10(CUT), 20001)
    e = e[e < CUT]
    series = e * (1 + e * (-0.5 + e * (1 / 3 + e * (-0.25))))
    rel = np.abs(series - np.log1p(e)) / np.log1p(e)
    assert rel.max() < 2e-8


def test_hardware_log_branch_bound_above_the_cut():
    assert 2.0 ** -21.41 / np.log1p(CUT) < 3e-5


def test_expm1_series_inside_half():
    x = np.linspace(-0.5, 0.5, 40001)
    x = x[(x != 0) & (np.abs(x) < 0.5)]
    q = 1 / 5040
    for c in (1 / 720, 1 / 120, 1 / 24, 1 / 6, 0.5, 1.0):
        q = q * x + c
    rel = np.abs(x * q - np.expm1(x)) / np.abs(np.expm1(x))
    assert rel.max() < 3e-7
