"""Parity of the CUDA path (called through the C ABI) with the CPU oracle.

Tolerances are the operator's stated ones: max|y - y_ref| / max|y_ref| <=
1e-4 for fp32 inputs and <= 1.5e-2 for bf16 inputs with fp32 accumulation.
The full-size workloads are run in exactly the launch configuration the
benchmark times and checked on rows the oracle evaluates one by one.
"""
import numpy as np
import pytest

import mamba_ssd_sequence_b200 as ssd
import oracle
from mamba_ssd_sequence_b200 import inputs
from helpers import TOL, rel_err, run_gpu, sample_rows, to_device

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def _oracle_full(x, order, normalize, D="inputs"):
    Dv = x["D"] if D == "inputs" else D
    return oracle.ssd_recurrent(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"],
                                Dv, order, normalize)


# ------------------------------------------------------------ kernel (a)
@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_chunk_cumsum_matches_oracle(chunk):
    x = inputs.make_inputs(2, 3, 4 * chunk, 16, "f32", seed=21)
    dev = to_device(x, "f32")
    acs, lam = ssd.ssd_chunk_cumsum(dev["dt_p"], dev["A_log"], dev["dt_bias"], chunk)
    torch.cuda.synchronize()
    ref = oracle.log_decay(x["dt_p"], x["A_log"], x["dt_bias"])  # global, inclusive
    B, H, N = ref.shape
    g = ref.reshape(B, H, N // chunk, chunk)
    start = np.concatenate([np.zeros((B, H, 1)), g[:, :, :-1, -1]], axis=2)[..., None]
    local = (g - start).reshape(B, H, N)
    got = acs.cpu().numpy()
    scale = np.maximum(1.0, np.abs(local))
    assert np.max(np.abs(got - local) / scale) < 2e-5
    np.testing.assert_allclose(lam.cpu().numpy(), local.reshape(B, H, -1, chunk)[..., -1],
                               rtol=2e-5, atol=2e-5)


# -------------------------------------------------- small cases, every row
@pytest.mark.parametrize("residual", [True, False])
def test_small_fp32_workload_all_rows(residual):
    w = inputs.WORKLOADS[inputs.SMALL]
    x = inputs.make_workload_inputs(w, seed=0, residual=residual)
    y = run_gpu(x, w.dtype, w.order, w.normalize, w.chunk)
    ref = _oracle_full(x, w.order, w.normalize)
    assert rel_err(y, ref) <= TOL["f32"]
    ref_q = oracle.ssd_quadratic(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"],
                                 x["D"], w.order, w.normalize)
    assert rel_err(y, ref_q) <= TOL["f32"]


def _reduced(w, B, H, n_chunks):
    return dict(B=B, H=H, N=n_chunks * w.chunk, d=w.d, dtype=w.dtype, order=w.order,
                normalize=w.normalize, chunk=w.chunk)


@pytest.mark.parametrize("name", inputs.WORKLOAD_ORDER[1:])
@pytest.mark.parametrize("residual", [True, False])
def test_reduced_workloads_all_rows(name, residual):
    """Each workload's d_h, chunk, order, normaliser and dtype on fewer heads
    and tokens (still several chunks, so the carried state is exercised)."""
    w = inputs.WORKLOADS[name]
    r = _reduced(w, 2, 3, 5)
    x = inputs.make_inputs(r["B"], r["H"], r["N"], r["d"], r["dtype"], seed=1, residual=residual)
    y = run_gpu(x, r["dtype"], r["order"], r["normalize"], r["chunk"])
    ref = _oracle_full(x, r["order"], r["normalize"])
    assert rel_err(y, ref) <= TOL[r["dtype"]]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("d", [16, 32, 64])
@pytest.mark.parametrize("order", [1, 2])
@pytest.mark.parametrize("chunk", [64, 128, 256])
def test_shape_grid(dtype, d, order, chunk):
    normalize = order == 2
    x = inputs.make_inputs(1, 2, 3 * chunk, d, dtype, seed=d + chunk + order)
    y = run_gpu(x, dtype, order, normalize, chunk)
    ref = _oracle_full(x, order, normalize)
    assert rel_err(y, ref) <= TOL[dtype]


def test_single_chunk_and_one_head():
    for dtype, order in [("f32", 1), ("bf16", 1), ("bf16", 2)]:
        x = inputs.make_inputs(1, 1, 64, 64, dtype, seed=3)
        y = run_gpu(x, dtype, order, order == 2, 64)
        assert rel_err(y, _oracle_full(x, order, order == 2)) <= TOL[dtype]


@pytest.mark.parametrize("n_chunks", [1, 2, 3, 4, 7, 15])
def test_chunk_counts_and_segment_boundaries(n_chunks):
    """Heads split into segments at chunk boundaries (odd and even split
    points, one-chunk heads) give the same result as the oracle."""
    x = inputs.make_inputs(1, 3, n_chunks * 128, 64, "bf16", seed=40 + n_chunks)
    for residual in (True, False):
        y = run_gpu(x, "bf16", 1, False, 128, D="inputs" if residual else None)
        ref = _oracle_full(x, 1, False, D="inputs" if residual else None)
        assert rel_err(y, ref) <= TOL["bf16"]


def test_order1_normalised_with_positive_features():
    x = inputs.make_inputs(2, 2, 512, 64, "bf16", seed=4)
    for key in ("q", "k"):
        x[key] = np.abs(x[key])
        x[key + "_bits"] = inputs.bf16_round_bits(x[key])
    y = run_gpu(x, "bf16", 1, True, 128)
    assert rel_err(y, _oracle_full(x, 1, True)) <= TOL["bf16"]


@pytest.mark.parametrize("A_log", [-1000.0, 0.0, 80.0])
def test_decay_extremes(A_log):
    """No decay (plain causal linear attention), slow decay, and decay so
    fast that only the diagonal survives."""
    x = inputs.make_inputs(1, 2, 256, 64, "bf16", seed=5)
    x["A_log"] = np.full(2, A_log, dtype=np.float32)
    for order in (1, 2):
        y = run_gpu(x, "bf16", order, order == 2, 64)
        assert rel_err(y, _oracle_full(x, order, order == 2)) <= TOL["bf16"]


def test_chunk_size_invariance():
    """The chunk length only changes the blocking: 64, 128 and 256 agree."""
    x = inputs.make_inputs(1, 4, 1024, 64, "bf16", seed=6)
    for order in (1, 2):
        ys = [run_gpu(x, "bf16", order, order == 2, c) for c in (64, 128, 256)]
        ref = _oracle_full(x, order, order == 2)
        for y in ys:
            assert rel_err(y, ref) <= TOL["bf16"]
        assert rel_err(ys[0], ys[2]) <= TOL["bf16"]


def test_repeatable_and_status_clean():
    x = inputs.make_inputs(2, 4, 512, 64, "bf16", seed=7)
    dev = to_device(x, "bf16")
    ws = ssd.alloc_workspace(2, 4, 512, 64, ssd.SSD_BF16, 1, 128)
    outs = []
    for _ in range(2):
        outs.append(ssd.ssd_fwd(dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"],
                                dev["dt_bias"], dev["D"], 1, False, 128, workspace=ws))
    assert ssd.ssd_status_from_workspace(ws) == 0
    assert torch.equal(outs[0], outs[1])


def test_output_guard_bands_untouched():
    """Nothing is written outside out[]: canaries before and after it."""
    for dtype, order, chunk in [("f32", 1, 64), ("bf16", 1, 64), ("bf16", 1, 128),
                                ("bf16", 2, 64)]:
        x = inputs.make_inputs(1, 2, 256, 64, dtype, seed=8)
        dev = to_device(x, dtype)
        n = dev["q"].numel()
        pad = 4096
        buf = torch.full((n + 2 * pad,), 7.0, dtype=dev["q"].dtype, device="cuda")
        out = buf[pad:pad + n].view_as(dev["q"])
        ssd.ssd_fwd(dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"], dev["dt_bias"],
                    dev["D"], order, order == 2, chunk, out=out)
        torch.cuda.synchronize()
        assert torch.all(buf[:pad] == 7.0) and torch.all(buf[pad + n:] == 7.0)


def test_host_entry_point_matches_device_entry_point():
    x = inputs.make_inputs(1, 4, 512, 64, "bf16", seed=9)
    dev = to_device(x, "bf16")
    ref = ssd.ssd_fwd(dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"],
                      dev["dt_bias"], dev["D"], 1, False, 128)
    host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in dev.items()}
    out_h = torch.empty_like(host["q"]).pin_memory()
    scratch = {k: (torch.empty_like(v) if v is not None else None) for k, v in dev.items()}
    scratch["out"] = torch.empty_like(dev["q"])
    ws = ssd.alloc_workspace(1, 4, 512, 64, ssd.SSD_BF16, 1, 128)
    ssd.ssd_fwd_host(host["q"], host["k"], host["v"], host["dt_p"], host["A_log"],
                     host["dt_bias"], host["D"], 1, False, 128, out_h, scratch, ws)
    torch.cuda.synchronize()
    assert torch.equal(out_h, ref.cpu())


@pytest.mark.parametrize("B,H,N,d,dtype,order,chunk", [
    (3, 4, 4096, 64, "bf16", 1, 128),   # three slices of whole batches
    (1, 10, 4096, 64, "bf16", 1, 256),  # one batch: heads [0, 4) and [4, 10)
    (2, 8, 4096, 32, "bf16", 2, 64),    # order 2 (clusters of two), two slices
    (2, 8, 2048, 64, "bf16", 2, 64),    # order 2 with the reduction through L2
    (4, 2, 4096, 64, "f32", 1, 64),     # the SIMT path, four slices
])
def test_host_entry_point_in_slices(B, H, N, d, dtype, order, chunk):
    """Inputs of 4 MiB and more go in by slices of heads, each slice's copies
    overlapping the previous slice's pass: the same bytes as the device entry
    point on the whole problem, twice in a row, with a clean status word."""
    import torch
    assert B * H * N * d * (2 if dtype == "bf16" else 4) >= 4 << 20
    x = inputs.make_inputs(B, H, N, d, dtype, seed=11)
    dev = to_device(x, dtype)
    norm = order == 2
    ref = ssd.ssd_fwd(dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"],
                      dev["dt_bias"], dev["D"], order, norm, chunk).cpu()
    host = {k: (v.cpu().pin_memory() if v is not None else None) for k, v in dev.items()}
    scratch = {k: (torch.empty_like(v) if v is not None else None) for k, v in dev.items()}
    scratch["out"] = torch.empty_like(dev["q"])
    ws = ssd.alloc_workspace(B, H, N, d, ssd.SSD_BF16 if dtype == "bf16" else ssd.SSD_F32, order, chunk)
    for _ in range(2):
        out_h = torch.empty_like(host["q"]).pin_memory()
        ssd.ssd_fwd_host(host["q"], host["k"], host["v"], host["dt_p"], host["A_log"],
                         host["dt_bias"], host["D"], order, norm, chunk, out_h, scratch, ws)
        torch.cuda.synchronize()
        assert torch.equal(out_h, ref)
    assert ssd.ssd_status_from_workspace(ws) == 0


# --------------------------------------------- full-size workloads, sampled
@pytest.mark.parametrize("name", inputs.WORKLOAD_ORDER[1:])
def test_full_size_workload_sampled_rows(name):
    """The workload at its full size, launched exactly as the benchmark does,
    checked on the rows the oracle evaluates one by one."""
    w = inputs.WORKLOADS[name]
    x = inputs.make_workload_inputs(w, seed=0)
    y = run_gpu(x, w.dtype, w.order, w.normalize, w.chunk)
    rows = sample_rows(w.N, w.chunk, seed=1)
    ref = oracle.ssd_quadratic(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"],
                               x["D"], w.order, w.normalize, rows=rows)
    assert rel_err(y[:, :, rows, :], ref) <= TOL[w.dtype]
    assert np.all(np.isfinite(y))


def test_headline_workload_every_row():
    w = inputs.WORKLOADS[inputs.HEADLINE]
    x = inputs.make_workload_inputs(w, seed=0)
    y = run_gpu(x, w.dtype, w.order, w.normalize, w.chunk)
    assert rel_err(y, _oracle_full(x, w.order, w.normalize)) <= TOL[w.dtype]
