"""Parity of the conv1d + SiLU prologue (2Mamba2Furious Algorithm 3's
Q, K, V = SiLU(conv_1d(h W_QKV)), window 2 on the Algorithm 6 page) with the
CPU oracle, alone and followed by the operator."""
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


def _weights(H, d, width, seed):
    rng = np.random.default_rng(seed)
    w = (rng.standard_normal((H * d, width)) / np.sqrt(width)).astype(np.float32)
    b = (0.1 * rng.standard_normal(H * d)).astype(np.float32)
    return w, b


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("width", [1, 2, 3, 4])
@pytest.mark.parametrize("silu,use_bias", [(True, True), (False, False), (True, False)])
def test_conv1d_matches_oracle(dtype, width, silu, use_bias):
    B, H, N, d = 2, 3, 77, 32
    x = inputs.make_inputs(B, H, N, d, dtype, seed=51)
    w, b = _weights(H, d, width, 51)
    dev = to_device(x, dtype)
    wd = torch.from_numpy(w).cuda()
    bd = torch.from_numpy(b).cuda() if use_bias else None
    y = ssd.ssd_conv1d(dev["q"], wd, bd, silu=silu)
    torch.cuda.synchronize()
    ref = oracle.conv1d(x["q"], w, b if use_bias else None, silu=silu)
    got = y.float().cpu().numpy().astype(np.float64)
    # the operator's measure, max|d| / max|ref|: an elementwise relative error
    # is meaningless where the window's terms cancel; fp32 accumulation of a
    # few terms, and bf16 output rounding (2^-9 relative) bound it
    tol = 1e-5 if dtype == "f32" else 2 ** -8
    assert rel_err(got, ref) <= tol


@pytest.mark.parametrize("dtype,B,H,N,d,width", [
    ("f32", 2, 40, 1000, 16, 3),   # 640 tiles of 128 tokens, ragged last tile of each sequence
    ("bf16", 1, 16, 4096, 64, 2),  # the bench's sequence length
    ("bf16", 3, 20, 700, 32, 4),
])
def test_conv1d_many_tiles_per_cta(dtype, B, H, N, d, width):
    """More tiles than two per SM: each CTA walks a range of tiles through its
    two tile buffers, crossing from one head's sequence to the next."""
    x = inputs.make_inputs(B, H, N, d, dtype, seed=53)
    w, b = _weights(H, d, width, 53)
    dev = to_device(x, dtype)
    y = ssd.ssd_conv1d(dev["q"], torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda(), silu=True)
    torch.cuda.synchronize()
    ref = oracle.conv1d(x["q"], w, b, silu=True)
    got = y.float().cpu().numpy().astype(np.float64)
    tol = 1e-5 if dtype == "f32" else 2 ** -8
    assert rel_err(got, ref) <= tol


def test_prologue_then_operator():
    """conv1d + SiLU on q, k, v, then the order-1 tensor-core operator, agrees
    with the oracle's prologue followed by the oracle's operator."""
    B, H, N, d, chunk = 1, 2, 384, 64, 128
    x = inputs.make_inputs(B, H, N, d, "bf16", seed=52, residual=True)
    dev = to_device(x, "bf16")
    conv = {}
    ref_in = {}
    for i, name in enumerate(("q", "k", "v")):
        w, b = _weights(H, d, 2, 60 + i)
        conv[name] = ssd.ssd_conv1d(dev[name], torch.from_numpy(w).cuda(), torch.from_numpy(b).cuda())
        r = oracle.conv1d(x[name], w, b).astype(np.float32)
        ref_in[name] = inputs.bf16_bits_to_f32(inputs.bf16_round_bits(r))  # the operator reads bf16
    y = ssd.ssd_fwd(conv["q"], conv["k"], conv["v"], dev["dt_p"], dev["A_log"], dev["dt_bias"], dev["D"],
                    1, False, chunk)
    torch.cuda.synchronize()
    ref = oracle.ssd_quadratic(ref_in["q"], ref_in["k"], ref_in["v"], x["dt_p"], x["A_log"], x["dt_bias"],
                               x["D"], 1, False)
    assert rel_err(y.float().cpu().numpy().astype(np.float64), ref) <= TOL["bf16"]


def test_silu_accuracy():
    """The convolutions' SiLU (one exponential, a Newton-Raphson reciprocal)
    against u / (1 + e^-u) in double precision: an identity convolution
    (width 1, tap 1, no bias) of float32 values spanning [-60, 60] keeps its
    relative error within a few float32 ulps plus the error of forming the
    exponent y = |u| log2(e) in float32 (the constant and the product each
    round by 2^-24 relative, so y is off by up to |y| 2^-23 and 2^y by a
    relative |y| ln(2) 2^-23 = |u| 2^-23, which any float32 exp of -u
    carries); far negative inputs give (near) zero."""
    d = 64
    u = np.linspace(-60.0, 60.0, 4 * 4096 * d // 4 * 4).astype(np.float32)
    u = np.concatenate([u, np.array([0.0, 1e-30, -1e-30, 1e-3, -1e-3, 0.5, -0.5], np.float32)])
    n_tok = -(-u.size // d)
    x = np.zeros(n_tok * d, np.float32)
    x[:u.size] = u
    x = x.reshape(1, 1, n_tok, d)
    w = np.ones((d, 1), np.float32)
    y = ssd.ssd_conv1d(torch.from_numpy(x).cuda(), torch.from_numpy(w).cuda(), None, silu=True)
    torch.cuda.synchronize()
    got = y.cpu().numpy().reshape(-1)[:u.size].astype(np.float64)
    ud = u.astype(np.float64)
    ref = ud / (1.0 + np.exp(-ud))
    rel = np.abs(got - ref) / np.maximum(np.abs(ref), 1e-30)
    bound = 4.0 * 2.0 ** -24 + np.abs(ud) * 2.0 ** -23
    assert np.all(rel <= bound), (rel.max(), ud[np.argmax(rel / bound)])
    far = np.array([-80.0, -100.0, -1e4], np.float32)
    xf = np.zeros((1, 1, 1, d), np.float32)
    xf[0, 0, 0, :3] = far
    yf = ssd.ssd_conv1d(torch.from_numpy(xf).cuda(), torch.from_numpy(w).cuda(), None, silu=True)
    torch.cuda.synchronize()
    assert np.all(np.abs(yf.cpu().numpy()[0, 0, 0, :3]) <= 1e-20)
