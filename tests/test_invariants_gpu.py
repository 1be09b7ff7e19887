"""Invariants of the operator, checked on the CUDA path itself.

The oracle pins the same properties on the CPU; here they hold for the
kernels, exactly where the arithmetic allows it:
  * heads are independent problems (each head has its own q, k, v, dt, A, D),
    so permuting heads -- or batch rows -- permutes the output, bit for bit;
  * the scores are q.k raised to the order, so without the residual
    y(alpha q) = alpha^order y(q); with the normaliser the factor cancels,
    y(alpha q) = y(q).  For alpha = 2 the scaling commutes with every
    rounding step (bf16 inputs and products, fp32 sums), so the identity is
    exact; for alpha = 3 the bf16 rounding of 3q enters and the identity
    holds to the bf16 tolerance.
Sources: the 2Mamba2Furious summary, Algorithm 5 (the squared scores and the
normaliser) and Algorithm 2 (per-head A and dt); the Mamba-2 post's SSD
definition for order 1.
"""
import numpy as np
import pytest

import mamba_ssd_sequence_b200 as ssd
from mamba_ssd_sequence_b200 import inputs
from helpers import TOL, rel_err, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

# (B, H, N, d_h, order, normalize, chunk, dtype, path)
CASES = [
    (2, 4, 1024, 64, 1, False, 128, "bf16", "tc_order1"),
    (2, 3, 1024, 64, 1, False, 256, "bf16", "tc_order1"),
    (2, 3, 512, 32, 2, True, 64, "bf16", "tc_order2_quad"),
    (2, 3, 512, 32, 2, False, 64, "bf16", "tc_order2_quad"),
    (2, 3, 512, 64, 2, True, 64, "bf16", "tc_order2_quad"),
    (2, 3, 512, 64, 2, False, 64, "bf16", "tc_order2_quad"),
    (2, 3, 256, 16, 1, False, 64, "f32", "simt"),
    (2, 3, 256, 16, 2, True, 64, "f32", "simt"),
]
IDS = [f"{c[8]}-o{c[4]}-d{c[3]}-n{int(c[5])}-c{c[6]}" for c in CASES]


def _run(dev, order, normalize, chunk, D="dev"):
    Dt = dev["D"] if D == "dev" else D
    y = ssd.ssd_fwd(dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"], dev["dt_bias"], Dt,
                    order, normalize, chunk)
    torch.cuda.synchronize()
    return y


def _setup(case, seed):
    B, H, N, d, order, normalize, chunk, dtype, path = case
    code = ssd.SSD_BF16 if dtype == "bf16" else ssd.SSD_F32
    assert ssd.ssd_fwd_path(B, H, N, d, code, order, chunk)[0] == path
    x = inputs.make_inputs(B, H, N, d, dtype, seed=seed, residual=True)
    return to_device(x, dtype)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_head_permutation(case):
    B, H, N, d, order, normalize, chunk, dtype, path = case
    dev = _setup(case, seed=31)
    perm = torch.tensor(np.random.default_rng(3).permutation(H), device="cuda")
    y = _run(dev, order, normalize, chunk)
    pd = {
        "q": dev["q"][:, perm].contiguous(), "k": dev["k"][:, perm].contiguous(),
        "v": dev["v"][:, perm].contiguous(), "dt_p": dev["dt_p"][:, perm].contiguous(),
        "A_log": dev["A_log"][perm].contiguous(), "dt_bias": dev["dt_bias"][perm].contiguous(),
        "D": dev["D"].view(H, d)[perm].reshape(-1).contiguous(),
    }
    yp = _run(pd, order, normalize, chunk)
    assert torch.equal(yp, y[:, perm])


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_batch_permutation(case):
    B, H, N, d, order, normalize, chunk, dtype, path = case
    dev = _setup(case, seed=32)
    perm = torch.tensor([1, 0], device="cuda")
    y = _run(dev, order, normalize, chunk)
    pd = dict(dev)
    for name in ("q", "k", "v", "dt_p"):
        pd[name] = dev[name][perm].contiguous()
    yp = _run(pd, order, normalize, chunk)
    assert torch.equal(yp, y[perm])


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_homogeneity_in_q_power_of_two(case):
    """y(2q) = 2^order y(q) without the normaliser, y(2q) = y(q) with it:
    exact, since scaling by 2 commutes with every rounding."""
    B, H, N, d, order, normalize, chunk, dtype, path = case
    dev = _setup(case, seed=33)
    y = _run(dev, order, normalize, chunk, D=None)
    d2 = dict(dev)
    d2["q"] = dev["q"] * 2
    y2 = _run(d2, order, normalize, chunk, D=None)
    factor = 1.0 if normalize else float(2 ** order)
    assert torch.equal(y2, y * factor)


@pytest.mark.parametrize("case", CASES, ids=IDS)
def test_homogeneity_in_q_general(case):
    """y(3q) = 3^order y(q) (or y(q) with the normaliser) to the dtype's
    tolerance: 3q is rounded to the input dtype first."""
    B, H, N, d, order, normalize, chunk, dtype, path = case
    dev = _setup(case, seed=34)
    y = _run(dev, order, normalize, chunk, D=None).double().cpu().numpy()
    d3 = dict(dev)
    d3["q"] = (dev["q"].float() * 3).to(dev["q"].dtype)
    y3 = _run(d3, order, normalize, chunk, D=None).double().cpu().numpy()
    factor = 1.0 if normalize else float(3 ** order)
    assert rel_err(y3 / factor, y) <= TOL[dtype]
