"""Parity of the Mamba-2S options and of the carried state at the full
workload sizes, launched as the benchmark launches the plain operator, so
that every persistent CTA takes several tiles (or a cluster walks every chunk
of a long head) with the options on.

Outputs are checked on rows the oracle's quadratic form evaluates one by one
(2Mamba2Furious, Algorithms 1, 4 and 5, with the carried state of Algorithm
6 entering before token 0).  The final states are checked on a slice of
heads against the oracle's token recurrence over the same heads (Algorithm
6); heads are independent, so a slice of them is an exact sub-problem."""
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


def _np(t):
    return t.float().cpu().numpy().astype(np.float64)


def _carried_state(w, seed):
    """A state to start from.  Order 1: 0.5 N(0,1) entries and |0.5 N(0,1)| for
    z.  Order 2: the state the oracle's recurrence leaves after a seeded
    64-token prefix (an arbitrary z can make the normaliser cross zero)."""
    if w.order == 2:
        p = inputs.make_inputs(w.B, w.H, 64, w.d, "f32", seed=seed)
        _, _, h0, z0 = oracle.ssd_recurrent(p["q"], p["k"], p["v"], p["dt_p"], p["A_log"], p["dt_bias"],
                                           None, 2, False, return_norm=True, return_state=True)
        return h0.astype(np.float32), z0.astype(np.float32)
    rng = np.random.default_rng(seed)
    h0 = (0.5 * rng.standard_normal((w.B, w.H, w.d, w.d))).astype(np.float32)
    z0 = np.abs(0.5 * rng.standard_normal((w.B, w.H, w.d))).astype(np.float32)
    return h0, z0


def _head_slice(x, ld, h0, z0, b, hs):
    """The oracle's arguments restricted to batch b and heads hs (a slice)."""
    sl = lambda a: None if a is None else np.ascontiguousarray(a[b:b + 1, hs])
    d = x["q"].shape[-1]
    D = None if x["D"] is None else np.ascontiguousarray(x["D"].reshape(-1, d)[hs].reshape(-1))
    return (sl(x["q"]), sl(x["k"]), sl(x["v"]), sl(x["dt_p"]), x["A_log"][hs], x["dt_bias"][hs], D,
            sl(ld), sl(h0), sl(z0))


# (workload, per-token log-decay, value discretisation, carried state)
CASES = [
    ("order1-bf16-B1H32N65536d64-c256", True, True, False),
    ("order1-bf16-B1H32N65536d64-c256", False, False, True),
    ("order1-bf16-B1H32N65536d64-c256", True, True, True),
    ("order1-bf16-B4H16N2048d64-c128", True, True, True),
    ("order2-bf16-B4H16N4096d32-c64", True, True, True),
    ("order2-bf16-B2H8N16384d64-c64", False, False, True),
    ("order2-bf16-B2H8N16384d64-c64", True, True, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[0]}-ld{int(c[1])}-vdt{int(c[2])}-state{int(c[3])}")
def test_full_size_options_and_state_sampled(case):
    name, use_ld, vdt, use_state = case
    w = inputs.WORKLOADS[name]
    x = inputs.make_workload_inputs(w, seed=3)
    ld = inputs.make_log_decay(w.B, w.H, w.N, seed=3) if use_ld else None
    dev = to_device(x, w.dtype)
    h0 = z0 = None
    h0d = z0d = ho = zo = None
    if use_state:
        h0, z0 = _carried_state(w, 3)
        h0d = torch.from_numpy(h0).cuda()
        ho = torch.empty_like(h0d)
        if w.order == 2:  # the order-1 tensor-core path carries h only
            z0d = torch.from_numpy(z0).cuda()
            zo = torch.empty_like(z0d)
        else:
            z0 = None
    path, _ = ssd.ssd_fwd_path(w.B, w.H, w.N, w.d, ssd.SSD_BF16, w.order, w.chunk)
    # without a carried state order 2 takes the quadratic form; with one, the chunked kernel
    assert path == ("tc_order1" if w.order == 1 else "tc_order2_quad"), "the workload runs on its tensor-core path"
    y = ssd.ssd_fwd_state(dev["q"], dev["k"], dev["v"], dev["dt_p"], None if use_ld else dev["A_log"],
                          dev["dt_bias"], dev["D"], w.order, w.normalize, w.chunk,
                          h0=h0d, z0=z0d, h_out=ho, z_out=zo,
                          log_decay=None if ld is None else torch.from_numpy(ld).cuda(), value_dt=vdt)
    torch.cuda.synchronize()
    yn = _np(y)
    assert np.all(np.isfinite(yn))
    rows = sample_rows(w.N, w.chunk, seed=2)
    ref = oracle.ssd_quadratic(x["q"], x["k"], x["v"], x["dt_p"], None if use_ld else x["A_log"],
                               x["dt_bias"], x["D"], w.order, w.normalize, rows=rows,
                               log_decay=ld, value_dt=vdt, h0=h0, z0=z0)
    assert rel_err(yn[:, :, rows, :], ref) <= TOL[w.dtype]
    if use_state:
        # final state of two heads of the last batch, against the recurrence
        b, hs = w.B - 1, slice(0, 2)
        q, k, v, dt, Al, db, D, lds, h0s, z0s = _head_slice(x, ld, h0, z0, b, hs)
        _, _, h_ref, z_ref = oracle.ssd_recurrent(q, k, v, dt, None if use_ld else Al, db, D, w.order,
                                                  w.normalize, return_norm=True, return_state=True,
                                                  log_decay=lds, value_dt=vdt, h0=h0s, z0=z0s)
        assert rel_err(_np(ho)[b:b + 1, hs], h_ref) <= TOL[w.dtype]
        if zo is not None:
            assert rel_err(_np(zo)[b:b + 1, hs], z_ref) <= TOL[w.dtype]
