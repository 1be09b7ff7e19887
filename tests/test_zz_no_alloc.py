"""ssd_fwd_noalloc: the forward pass for callers that cannot allocate device
memory (their host application owns the device memory pool, or they must
not trigger the synchronisation cudaMalloc can cause).  It runs on a fixed
scratch buffer inside the library; this test calls it through the C ABI and
checks it against ssd_fwd and against the CPU oracle's token recurrence on
two calls in a row, so a second call that wrongly relied on the first call's
leftovers would show.

The file is named so that pytest collects it last."""
import ctypes

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


def _noalloc_fn():
    lib = ssd.load_library()
    fn = lib.ssd_fwd_noalloc
    vp, ci = ctypes.c_void_p, ctypes.c_int
    fn.argtypes = [vp] * 7 + [ci] * 8 + [vp, vp]
    fn.restype = ci
    return fn


def _call(fn, dev, shape, dtype, order, normalize, chunk, out):
    B, H, N, d = shape
    code = ssd.SSD_BF16 if dtype == "bf16" else ssd.SSD_F32
    D = dev["D"].data_ptr() if dev["D"] is not None else None
    return fn(dev["q"].data_ptr(), dev["k"].data_ptr(), dev["v"].data_ptr(),
              dev["dt_p"].data_ptr(), dev["A_log"].data_ptr(), dev["dt_bias"].data_ptr(), D,
              B, H, N, d, code, order, int(normalize), chunk, out.data_ptr(),
              torch.cuda.current_stream().cuda_stream)


CASES = [  # (shape, dtype, order, normalize, chunk)
    ((1, 2, 256, 16), "f32", 1, False, 64),
    ((2, 4, 512, 64), "bf16", 1, False, 128),
    ((1, 3, 256, 32), "bf16", 2, True, 64),
]


@pytest.mark.parametrize("shape,dtype,order,normalize,chunk", CASES)
def test_noalloc_matches_ssd_fwd_on_two_calls(shape, dtype, order, normalize, chunk):
    fn = _noalloc_fn()
    B, H, N, d = shape
    outs = []
    for seed in (31, 32):  # two calls in a row, different inputs
        x = inputs.make_inputs(B, H, N, d, dtype, seed=seed)
        dev = to_device(x, dtype)
        ref = ssd.ssd_fwd(dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"],
                          dev["dt_bias"], dev["D"], order, normalize, chunk)
        out = torch.full_like(dev["q"], float("nan"))
        rc = _call(fn, dev, shape, dtype, order, normalize, chunk, out)
        assert rc == 0, ssd.status_str(rc)
        torch.cuda.synchronize()
        got = out.float().cpu().numpy().astype(np.float64)
        want = ref.float().cpu().numpy().astype(np.float64)
        assert np.all(np.isfinite(got))
        assert rel_err(got, want) <= TOL[dtype]
        ref = oracle.ssd_recurrent(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"],
                                   order, normalize)
        assert rel_err(got, ref) <= TOL[dtype]
        outs.append(got)
    assert not np.array_equal(outs[0], outs[1])


def test_noalloc_rejects_problems_beyond_its_scratch():
    fn = _noalloc_fn()
    x = inputs.make_inputs(1, 1, 64, 16, "bf16", seed=1)
    dev = to_device(x, "bf16")
    out = torch.empty_like(dev["q"])
    B, H, N, d = 4, 16, 2048, 64  # order 2 needs ~1 GiB of scratch: refused up front
    code = fn(dev["q"].data_ptr(), dev["k"].data_ptr(), dev["v"].data_ptr(),
              dev["dt_p"].data_ptr(), dev["A_log"].data_ptr(), dev["dt_bias"].data_ptr(), None,
              B, H, N, d, ssd.SSD_BF16, 2, 1, 64, out.data_ptr(),
              torch.cuda.current_stream().cuda_stream)
    assert code == 7  # SSD_ERR_WORKSPACE, nothing enqueued
