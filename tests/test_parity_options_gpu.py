"""Parity of the Mamba-2S options of ssd_fwd_ex (a given per-token log-decay
and value discretisation V (.) dt, 2Mamba2Furious Algorithm 4) with the CPU
oracle, on every path: order-1 tensor cores (chunk 128 and 256), order-2
tensor cores (log-decay), the SIMT path (fp32, and order 2 with V (.) dt).
Tolerances as for ssd_fwd: 1e-4 (fp32) and 1.5e-2 (bf16) of max|y_ref|."""
import numpy as np
import pytest

import mamba_ssd_sequence_b200 as ssd
import oracle
from mamba_ssd_sequence_b200 import inputs
from helpers import TOL, rel_err, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

# (dtype, d_h, order, normalize, chunk, chunks)
SHAPES = [
    ("bf16", 64, 1, False, 128, 5),   # order-1 tensor-core path
    ("bf16", 64, 1, False, 128, 7),   # longer heads (more chunk states to carry)
    ("bf16", 64, 1, False, 128, 15),
    ("bf16", 64, 1, False, 256, 3),   # order-1 tensor-core path, two 128-row tiles per chunk
    ("f32", 16, 1, False, 64, 5),     # SIMT path
    ("f32", 16, 1, True, 64, 4),      # SIMT path with the normaliser
    ("bf16", 32, 2, True, 64, 5),     # order-2 tensor-core path (value dt scales V in place)
    ("bf16", 32, 2, False, 64, 4),    # order 2 without the normaliser
    ("bf16", 64, 2, True, 64, 3),     # order-2 cluster of 8 CTAs
]
OPTIONS = [("log_decay", True, False), ("value_dt", False, True), ("both", True, True)]


def _run(x, ld, dtype, order, normalize, chunk, use_ld, vdt):
    dev = to_device(x, dtype)
    ldd = torch.from_numpy(ld).cuda() if use_ld else None
    out = ssd.ssd_fwd(dev["q"], dev["k"], dev["v"], dev["dt_p"],
                      None if use_ld else dev["A_log"], dev["dt_bias"], dev["D"], order, normalize, chunk,
                      log_decay=ldd, value_dt=vdt)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("shape", SHAPES, ids=lambda s: f"{s[0]}-d{s[1]}-o{s[2]}-n{int(s[3])}-c{s[4]}x{s[5]}")
@pytest.mark.parametrize("opt", OPTIONS, ids=lambda o: o[0])
@pytest.mark.parametrize("residual", [True, False])
def test_options_match_oracle(shape, opt, residual):
    dtype, d, order, normalize, chunk, n_chunks = shape
    _, use_ld, vdt = opt
    B, H, N = 1, 3, n_chunks * chunk
    x = inputs.make_inputs(B, H, N, d, dtype, seed=31, residual=residual)
    if order == 1 and normalize:
        # order-1 row sums of SiLU features can cross zero, which makes y / N
        # ill-conditioned; positive features keep them away from zero
        for key in ("q", "k"):
            x[key] = np.abs(x[key])
            if dtype == "bf16":
                x[key + "_bits"] = inputs.bf16_round_bits(x[key])
    ld = inputs.make_log_decay(B, H, N, seed=31)
    y = _run(x, ld, dtype, order, normalize, chunk, use_ld, vdt)
    ref = oracle.ssd_quadratic(x["q"], x["k"], x["v"], x["dt_p"], None if use_ld else x["A_log"],
                               x["dt_bias"], x["D"], order, normalize,
                               log_decay=ld if use_ld else None, value_dt=vdt)
    assert np.isfinite(y).all()
    assert rel_err(y, ref) <= TOL[dtype], rel_err(y, ref)


def test_log_decay_equal_to_a_dt_gives_plain_result():
    """Feeding a_t = -exp(A_log) softplus(dt_p + dt_bias) as the log-decay
    reproduces ssd_fwd on the headline shape's tensor-core path."""
    x = inputs.make_inputs(1, 2, 512, 64, "bf16", seed=32, residual=True)
    z = x["dt_p"].astype(np.float64) + x["dt_bias"][None, :, None]
    dt = np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))
    ld = (-np.exp(x["A_log"].astype(np.float64))[None, :, None] * dt).astype(np.float32)
    y_ld = _run(x, ld, "bf16", 1, False, 128, True, False)
    dev = to_device(x, "bf16")
    y = ssd.ssd_fwd(dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"], dev["dt_bias"], dev["D"],
                    1, False, 128).float().cpu().numpy().astype(np.float64)
    assert rel_err(y_ld, y) <= 2e-3
