"""The operator with its convolution prologue fused (ssd_fwd_conv: q, k, v =
SiLU(conv_1d(x)) of 2Mamba2Furious Algorithm 3, window 2 on its Algorithm 6
page) against the CPU oracle's convolution followed by the oracle's
operator, and bit for bit against the unfused sequence ssd_conv1d x 3 then
ssd_fwd_ex."""
import numpy as np
import pytest

import mamba_ssd_sequence_b200 as ssd
import oracle
from mamba_ssd_sequence_b200 import inputs
from helpers import TOL, rel_err, sample_rows, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _taps(H, d, width, seed, use_bias=True):
    rng = np.random.default_rng(seed)
    w = [(rng.standard_normal((H * d, width)) / np.sqrt(width)).astype(np.float32) for _ in range(3)]
    b = [(0.1 * rng.standard_normal(H * d)).astype(np.float32) if use_bias else None for _ in range(3)]
    return w, b


def _dev(a):
    return None if a is None else torch.from_numpy(a).cuda()


def _oracle_inputs(x, w, b, silu, dtype):
    """The oracle's prologue, rounded to the operator's input type."""
    out = {}
    for i, name in enumerate(("q", "k", "v")):
        r = oracle.conv1d(x[name], w[i], b[i], silu=silu).astype(np.float32)
        out[name] = inputs.bf16_bits_to_f32(inputs.bf16_round_bits(r)) if dtype == "bf16" else r
    return out


def _run_fused(dev, w, b, order, normalize, chunk, silu, log_decay=None, value_dt=False):
    y = ssd.ssd_fwd_conv(dev["q"], dev["k"], dev["v"], [_dev(t) for t in w], [_dev(t) for t in b],
                         dev["dt_p"], dev["A_log"], dev["dt_bias"], dev["D"], order, normalize, chunk,
                         silu=silu, log_decay=log_decay, value_dt=value_dt)
    torch.cuda.synchronize()
    return y


def _run_unfused(dev, w, b, order, normalize, chunk, silu, log_decay=None, value_dt=False):
    c = [ssd.ssd_conv1d(dev[n], _dev(w[i]), _dev(b[i]), silu=silu) for i, n in enumerate(("q", "k", "v"))]
    y = ssd.ssd_fwd(c[0], c[1], c[2], dev["dt_p"], dev["A_log"], dev["dt_bias"], dev["D"], order, normalize,
                    chunk, log_decay=log_decay, value_dt=value_dt)
    torch.cuda.synchronize()
    return y


def _as64(y):
    return y.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("chunk", [128, 256])
@pytest.mark.parametrize("width,silu,use_bias", [(2, True, True), (1, True, False), (3, False, True),
                                                 (4, True, True)])
def test_fused_prologue_matches_oracle(chunk, width, silu, use_bias):
    """Order-1 tensor-core path (fused): several heads, several chunks per
    head (the halo crosses chunk boundaries and is zero at head starts)."""
    B, H, N, d = 2, 3, 5 * chunk, 64
    x = inputs.make_inputs(B, H, N, d, "bf16", seed=70 + width, residual=True)
    assert ssd.ssd_fwd_path(B, H, N, d, ssd.SSD_BF16, 1, chunk)[0] == "tc_order1"  # the fused path
    w, b = _taps(H, d, width, 80 + width, use_bias)
    y = _run_fused(to_device(x, "bf16"), w, b, 1, False, chunk, silu)
    ri = _oracle_inputs(x, w, b, silu, "bf16")
    ref = oracle.ssd_quadratic(ri["q"], ri["k"], ri["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"], 1, False)
    assert rel_err(_as64(y), ref) <= TOL["bf16"]


@pytest.mark.parametrize("chunk", [128, 256])
@pytest.mark.parametrize("opt", ["none", "log_decay", "value_dt"])
def test_fused_prologue_equals_unfused_bitwise(chunk, opt):
    """The fused path computes the same bits as the standalone convolution
    followed by the operator (same taps arithmetic, same kernels after it)."""
    B, H, N, d = 1, 4, 6 * chunk, 64
    x = inputs.make_inputs(B, H, N, d, "bf16", seed=90, residual=True)
    dev = to_device(x, "bf16")
    w, b = _taps(H, d, 2, 91)
    kw = {}
    if opt == "log_decay":
        rng = np.random.default_rng(92)
        kw["log_decay"] = torch.from_numpy(-rng.uniform(0.0, 0.3, size=(B, H, N)).astype(np.float32)).cuda()
    if opt == "value_dt":
        kw["value_dt"] = True
    yf = _run_fused(dev, w, b, 1, False, chunk, True, **kw)
    yu = _run_unfused(dev, w, b, 1, False, chunk, True, **kw)
    assert torch.equal(yf, yu)


@pytest.mark.parametrize("order,normalize,dtype,d,chunk", [(2, True, "bf16", 32, 64), (1, False, "f32", 32, 64),
                                                           (2, False, "bf16", 64, 64), (2, True, "bf16", 64, 64),
                                                           (1, False, "bf16", 64, 256)])
def test_other_paths_match_oracle(order, normalize, dtype, d, chunk):
    """Shapes off the fused path (order 2, fp32, order 1 at chunk 256) run the
    standalone convolution, then the operator."""
    B, H, N = 1, 2, 3 * chunk
    x = inputs.make_inputs(B, H, N, d, dtype, seed=95, residual=True)
    w, b = _taps(H, d, 2, 96)
    y = _run_fused(to_device(x, dtype), w, b, order, normalize, chunk, True)
    ri = _oracle_inputs(x, w, b, True, dtype)
    ref = oracle.ssd_quadratic(ri["q"], ri["k"], ri["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"], order,
                               normalize)
    assert rel_err(_as64(y), ref) <= TOL[dtype]


@pytest.mark.parametrize("d,normalize,opt", [(32, True, "none"), (64, True, "none"), (32, False, "value_dt"),
                                             (64, True, "log_decay")])
def test_order2_prologue_equals_unfused_bitwise(d, normalize, opt):
    """Order 2 through ssd_fwd_conv (the standalone convolution, then the
    order-2 tensor-core kernel) gives the same bits as ssd_conv1d x 3
    followed by the operator."""
    B, H, N = 1, 3, 5 * 64
    x = inputs.make_inputs(B, H, N, d, "bf16", seed=93, residual=True)
    dev = to_device(x, "bf16")
    w, b = _taps(H, d, 2, 94)
    kw = {}
    if opt == "log_decay":
        rng = np.random.default_rng(95)
        kw["log_decay"] = torch.from_numpy(-rng.uniform(0.0, 0.3, size=(B, H, N)).astype(np.float32)).cuda()
    if opt == "value_dt":
        kw["value_dt"] = True
    yf = _run_fused(dev, w, b, 2, normalize, 64, True, **kw)
    yu = _run_unfused(dev, w, b, 2, normalize, 64, True, **kw)
    assert torch.equal(yf, yu)


@pytest.mark.parametrize("name", ["order1-bf16-B4H16N2048d64-c128", "order1-bf16-B1H32N65536d64-c256",
                                  "order2-bf16-B4H16N4096d32-c64", "order2-bf16-B2H8N16384d64-c64"])
def test_fused_prologue_full_size(name):
    """The order-1 workloads at full size with the prologue: sampled rows
    against the oracle, and every output bit against the unfused sequence."""
    wl = inputs.WORKLOADS[name]
    x = inputs.make_workload_inputs(wl, seed=0)
    dev = to_device(x, "bf16")
    w, b = _taps(wl.H, wl.d, 2, 97)
    yf = _run_fused(dev, w, b, wl.order, wl.normalize, wl.chunk, True)
    yu = _run_unfused(dev, w, b, wl.order, wl.normalize, wl.chunk, True)
    assert torch.equal(yf, yu)
    rows = sample_rows(wl.N, wl.chunk, seed=3, n_random=8)
    ri = _oracle_inputs(x, w, b, True, "bf16")
    ref = oracle.ssd_quadratic(ri["q"], ri["k"], ri["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"], wl.order,
                               wl.normalize, rows=rows)
    assert rel_err(_as64(yf)[:, :, rows, :], ref) <= TOL["bf16"]
