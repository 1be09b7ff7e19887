"""The log1p polynomial of kernel (a)'s softplus: the generator reproduces the
coefficients written in the CUDA source, and their float32 error bound holds."""
import os

from mamba_ssd_sequence_b200 import gen_log1p_poly

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_coefficients_match_source_and_bound():
    c = gen_log1p_poly.coefficients(8)
    src = open(os.path.join(ROOT, "mamba_ssd_sequence_b200", "csrc", "ssd_math.cuh")).read()
    for v in c:
        assert f"{abs(float(v)):.9e}f" in src
    assert gen_log1p_poly.max_rel_error(c) < 3e-7
