"""Device-side failure detection on the tensor-core paths.

The kernels' waits are bounded: a wait that runs out records SSD_ERR_TIMEOUT
in the workspace status, raises the kernel's abort flag so that every other
role stops too, lets the copies and matrix products already in flight land,
frees the tensor memory and returns.  Nothing traps.  The test hook
ssd_debug_fwd makes one producer skip one publication (a TMA stage in the
order-1 kernels, a state slab in the order-2 kernel) with a 2 ms wait limit;
the host then reads the timeout back, and the same workspace serves a clean
call whose output matches the oracle.  The pages have no counterpart: this is
the library's own failure contract.
"""
import time

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

SSD_ERR_TIMEOUT = 9

# (B, H, N, d_h, order, normalize, chunk, step skipped, path)
CASES = [
    (1, 2, 1024, 64, 1, False, 128, 0, "tc_order1"),
    (1, 2, 2048, 64, 1, False, 256, 0, "tc_order1"),
    (1, 2, 256, 32, 2, True, 64, 1, "tc_order2"),       # the chunked kernel (a slab's state)
    (1, 2, 256, 64, 2, True, 64, 5, "tc_order2"),
    (1, 2, 256, 32, 2, True, 64, 1, "tc_order2_quad"),  # the quadratic form (a K, V stage)
    (1, 2, 512, 64, 2, True, 64, 2, "tc_order2_quad"),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"{c[8]}-d{c[3]}-c{c[6]}")
def test_skipped_publication_times_out_then_clean_call(case):
    B, H, N, d, order, normalize, chunk, skip, path = case
    force = 2 if path == "tc_order2" else -1  # the chunked kernel: as a call with a carried state
    if force < 0:
        assert ssd.ssd_fwd_path(B, H, N, d, ssd.SSD_BF16, order, chunk)[0] == path
    x = inputs.make_inputs(B, H, N, d, "bf16", seed=5, residual=True)
    dev = to_device(x, "bf16")
    ws = ssd.alloc_workspace(B, H, N, d, ssd.SSD_BF16, order, chunk, state=ssd.SSD_STATE_H if force == 2 else 0)
    out = torch.empty_like(dev["q"])
    args = (dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"], dev["dt_bias"], dev["D"])

    t0 = time.monotonic()
    ssd.ssd_debug_fwd(*args, order, normalize, chunk, skip_publish=skip, wait_ns=2_000_000,
                      out=out, workspace=ws, path=force)
    torch.cuda.synchronize()  # the kernels returned: no trap, the context is usable
    elapsed = time.monotonic() - t0
    assert ssd.ssd_status_from_workspace(ws) == SSD_ERR_TIMEOUT
    assert elapsed < 5.0

    # the same workspace and context serve the next call (on the same path)
    out.zero_()
    ssd.ssd_debug_fwd(*args, order, normalize, chunk, skip_publish=-1, wait_ns=0, out=out, workspace=ws,
                      path=force)
    torch.cuda.synchronize()
    assert ssd.ssd_status_from_workspace(ws) == 0
    ref = oracle.ssd_recurrent(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"],
                               order, normalize)
    y = out.float().cpu().numpy().astype(np.float64)
    assert rel_err(y, ref) <= TOL["bf16"]


def test_no_skip_is_a_plain_call():
    """skip_publish = -1 runs the kernels unchanged (status OK, oracle parity)."""
    B, H, N, d = 1, 2, 512, 64
    x = inputs.make_inputs(B, H, N, d, "bf16", seed=6, residual=True)
    dev = to_device(x, "bf16")
    ws = ssd.alloc_workspace(B, H, N, d, ssd.SSD_BF16, 1, 128)
    y = ssd.ssd_debug_fwd(dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"], dev["dt_bias"],
                          dev["D"], 1, False, 128, skip_publish=-1, wait_ns=0, workspace=ws)
    torch.cuda.synchronize()
    assert ssd.ssd_status_from_workspace(ws) == 0
    ref = oracle.ssd_recurrent(x["q"], x["k"], x["v"], x["dt_p"], x["A_log"], x["dt_bias"], x["D"], 1, False)
    assert rel_err(y.float().cpu().numpy().astype(np.float64), ref) <= TOL["bf16"]
