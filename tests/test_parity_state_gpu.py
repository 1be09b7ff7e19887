"""Parity of the carried-state entry points with the CPU oracle: a prefill
from a given state that also returns the final state (ssd_fwd_state), and the
one-token recurrent step (ssd_decode_step) continuing it -- 2Mamba2Furious
Algorithm 6 run token by token.  Tolerances as for ssd_fwd, applied to the
outputs (of max|y_ref|) and to the states (of max|h_ref|)."""
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


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _state(B, H, d, order, seed, scale=0.5):
    """A carried state to start from.  Order 1: random entries (z0 > 0).
    Order 2: the state a 64-token prefix leaves (the oracle's recurrence over
    seeded inputs), since the normaliser phi(q) . z0 of an arbitrary z0 can
    come out near zero or negative, which no real prefix gives."""
    if order == 2:
        p = inputs.make_inputs(B, H, 64, d, "f32", seed=seed)
        _, _, h0, z0 = oracle.ssd_recurrent(p["q"], p["k"], p["v"], p["dt_p"], p["A_log"], p["dt_bias"],
                                           None, 2, False, return_norm=True, return_state=True)
        return h0.astype(np.float32), z0.astype(np.float32)
    rng = np.random.default_rng(seed)
    Dphi = d ** order
    h0 = (scale * rng.standard_normal((B, H, Dphi, d))).astype(np.float32)
    z0 = np.abs(scale * rng.standard_normal((B, H, Dphi))).astype(np.float32)
    return h0, z0


# (dtype, d_h, order, normalize, chunk, use z, chunks per head)
PREFILL = [
    ("bf16", 64, 1, False, 128, False, 3),   # order-1 tensor-core path (h only)
    ("bf16", 64, 1, False, 128, False, 7),   # longer heads: the state pass carries h0 over more chunks
    ("bf16", 64, 1, False, 128, False, 15),
    ("bf16", 64, 1, False, 256, False, 3),
    ("f32", 16, 1, False, 64, True, 3),      # SIMT path with the normaliser state
    ("bf16", 32, 2, True, 64, True, 3),      # order-2 tensor-core path with h and z
    ("bf16", 32, 2, False, 64, True, 4),     # order 2 without the normaliser, z still carried
    ("bf16", 64, 2, True, 64, True, 2),      # order 2, cluster of 8 CTAs per head
]


@pytest.mark.parametrize("case", PREFILL,
                         ids=lambda c: f"{c[0]}-d{c[1]}-o{c[2]}-c{c[4]}-z{int(c[5])}-n{c[6]}")
@pytest.mark.parametrize("in_place", [False, True])
def test_prefill_state_in_and_out(case, in_place):
    dtype, d, order, norm, chunk, use_z, n_chunks = case
    B, H, N = 1, 3, n_chunks * chunk
    x = inputs.make_inputs(B, H, N, d, dtype, seed=41, residual=True)
    h0, z0 = _state(B, H, d, order, 41)
    dev = to_device(x, dtype)
    h0d = torch.from_numpy(h0).cuda()
    z0d = torch.from_numpy(z0).cuda() if use_z else None
    ho = h0d if in_place else torch.empty_like(h0d)
    zo = (z0d if in_place else torch.empty_like(z0d)) if use_z else None
    y = ssd.ssd_fwd_state(dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"], dev["dt_bias"], dev["D"],
                          order, norm, chunk, h0=h0d, z0=z0d, h_out=ho, z_out=zo)
    torch.cuda.synchronize()
    y_ref, _, h_ref, z_ref = oracle.ssd_recurrent(
        x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"], order, norm,
        return_norm=True, return_state=True, h0=h0, z0=z0 if use_z else None)
    assert rel_err(_np(y), y_ref) <= TOL[dtype]
    assert rel_err(_np(ho), h_ref) <= TOL[dtype]
    if use_z:
        assert rel_err(_np(zo), z_ref) <= TOL[dtype]


# (dtype, d_h, order, normalize)
DECODE = [("f32", 16, 1, False), ("f32", 32, 1, True), ("bf16", 64, 1, False), ("f32", 16, 2, True),
          ("bf16", 32, 2, True), ("bf16", 64, 2, True), ("bf16", 64, 2, False)]


@pytest.mark.parametrize("case", DECODE, ids=lambda c: f"{c[0]}-d{c[1]}-o{c[2]}-n{int(c[3])}")
@pytest.mark.parametrize("opt", ["plain", "log_decay", "value_dt"])
def test_decode_steps_continue_the_recurrence(case, opt):
    """Four decode steps from a carried state agree with the oracle's
    recurrence over the same tokens, output by output, and in the final state."""
    dtype, d, order, norm = case
    B, H, T = 2, 3, 4
    x = inputs.make_inputs(B, H, T, d, dtype, seed=42, residual=True)
    ld = inputs.make_log_decay(B, H, T, seed=42) if opt == "log_decay" else None
    vdt = opt == "value_dt"
    h0, z0 = _state(B, H, d, order, 42)
    dev = to_device(x, dtype)
    h = torch.from_numpy(h0).cuda()
    z = torch.from_numpy(z0).cuda()
    ldd = torch.from_numpy(ld).cuda() if ld is not None else None
    ys = []
    for t in range(T):
        sl = lambda a: a[:, :, t].contiguous()
        y = ssd.ssd_decode_step(sl(dev["q"]), sl(dev["k"]), sl(dev["v"]), sl(dev["dt_p"]), dev["A_log"],
                                dev["dt_bias"], dev["D"], order, norm, h, z,
                                log_decay=None if ldd is None else sl(ldd), value_dt=vdt)
        ys.append(_np(y))
    torch.cuda.synchronize()
    y_ref, _, h_ref, z_ref = oracle.ssd_recurrent(
        x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"], order, norm,
        return_norm=True, return_state=True, log_decay=ld, value_dt=vdt, h0=h0, z0=z0)
    y = np.stack(ys, axis=2)
    assert rel_err(y, y_ref) <= TOL[dtype]
    assert rel_err(_np(h), h_ref) <= TOL[dtype]
    assert rel_err(_np(z), z_ref) <= TOL[dtype]


def test_prefill_then_decode_equals_one_pass():
    """A prefill of N tokens that returns its state, then decode steps, gives
    the outputs a single pass over all tokens gives (order 1, tensor cores)."""
    d, chunk, N, T = 64, 128, 256, 3
    x = inputs.make_inputs(1, 2, N + T, d, "bf16", seed=43, residual=True)
    dev = to_device(x, "bf16")
    pre = lambda a: a[:, :, :N].contiguous()
    h = torch.zeros((1, 2, d, d), dtype=torch.float32, device="cuda")
    y_pre = ssd.ssd_fwd_state(pre(dev["q"]), pre(dev["k"]), pre(dev["v"]), pre(dev["dt_p"]), dev["A_log"],
                              dev["dt_bias"], dev["D"], 1, False, chunk, h_out=h)
    ys = [_np(y_pre)]
    for t in range(N, N + T):
        sl = lambda a: a[:, :, t].contiguous()
        ys.append(_np(ssd.ssd_decode_step(sl(dev["q"]), sl(dev["k"]), sl(dev["v"]), sl(dev["dt_p"]),
                                          dev["A_log"], dev["dt_bias"], dev["D"], 1, False, h))[:, :, None])
    torch.cuda.synchronize()
    y = np.concatenate(ys, axis=2)
    ref = oracle.ssd_recurrent(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"], 1, False)
    assert rel_err(y, ref) <= TOL["bf16"]


# (dtype, d_h, order, normalize, chunk, chunks per head): every path that takes a state
MAMBA2S_PREFILL = [
    ("bf16", 64, 1, False, 128, 5),   # order-1 tensor-core path
    ("bf16", 64, 1, False, 256, 2),
    ("bf16", 32, 2, True, 64, 4),     # order-2 tensor-core path
    ("bf16", 64, 2, True, 64, 2),
    ("f32", 16, 1, False, 64, 3),     # SIMT path
]


@pytest.mark.parametrize("case", MAMBA2S_PREFILL, ids=lambda c: f"{c[0]}-d{c[1]}-o{c[2]}-c{c[4]}-n{c[5]}")
def test_prefill_state_with_mamba2s_options(case):
    """A given per-token log-decay and value discretisation (Algorithm 4)
    together with a carried state in and out, against the oracle's
    recurrence with the same options."""
    dtype, d, order, norm, chunk, n_chunks = case
    B, H, N = 1, 3, n_chunks * chunk
    x = inputs.make_inputs(B, H, N, d, dtype, seed=44, residual=True)
    ld = inputs.make_log_decay(B, H, N, seed=44)
    h0, z0 = _state(B, H, d, order, 44)
    use_z = norm
    dev = to_device(x, dtype)
    h0d = torch.from_numpy(h0).cuda()
    z0d = torch.from_numpy(z0).cuda() if use_z else None
    ho = torch.empty_like(h0d)
    zo = torch.empty_like(z0d) if use_z else None
    y = ssd.ssd_fwd_state(dev["q"], dev["k"], dev["v"], dev["dt_p"], None, dev["dt_bias"], dev["D"],
                          order, norm, chunk, h0=h0d, z0=z0d, h_out=ho, z_out=zo,
                          log_decay=torch.from_numpy(ld).cuda(), value_dt=True)
    torch.cuda.synchronize()
    y_ref, _, h_ref, z_ref = oracle.ssd_recurrent(
        x["q"], x["k"], x["v"], x["dt_p"], None, x["dt_bias"], x["D"], order, norm,
        return_norm=True, return_state=True, log_decay=ld, value_dt=True, h0=h0,
        z0=z0 if use_z else None)
    assert rel_err(_np(y), y_ref) <= TOL[dtype]
    assert rel_err(_np(ho), h_ref) <= TOL[dtype]
    if use_z:
        assert rel_err(_np(zo), z_ref) <= TOL[dtype]


@pytest.mark.parametrize("n_chunks", [17, 20, 64])
def test_prefill_state_heads_longer_than_sixteen_chunks(n_chunks):
    """The order-1 state pass keeps sixteen chunks' inputs in flight for heads
    of up to 16 chunks and eight for longer ones; a carried state in and out on
    heads of 17, 20 and 64 chunks runs the second variant."""
    d, chunk = 64, 128
    B, H, N = 1, 2, n_chunks * chunk
    x = inputs.make_inputs(B, H, N, d, "bf16", seed=45 + n_chunks, residual=True)
    h0, _ = _state(B, H, d, 1, 45)
    dev = to_device(x, "bf16")
    h0d = torch.from_numpy(h0).cuda()
    ho = torch.empty_like(h0d)
    y = ssd.ssd_fwd_state(dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"], dev["dt_bias"], dev["D"],
                          1, False, chunk, h0=h0d, h_out=ho)
    torch.cuda.synchronize()
    y_ref, _, h_ref, _ = oracle.ssd_recurrent(
        x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"], 1, False,
        return_norm=True, return_state=True, h0=h0)
    assert rel_err(_np(y), y_ref) <= TOL["bf16"]
    assert rel_err(_np(ho), h_ref) <= TOL["bf16"]
