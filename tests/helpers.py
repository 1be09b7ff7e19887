"""Shared helpers for the GPU tests: upload the generator's arrays, run the
CUDA path through the binding, and compare with the oracle."""
import numpy as np

import mamba_ssd_sequence_b200 as ssd

TOL = {"f32": 1e-4, "bf16": 1.5e-2}


def to_device(x, dtype):
    """Upload one input set from inputs.make_inputs to cuda tensors."""
    import torch
    dev = {}
    for name in ("q", "k", "v"):
        if dtype == "bf16":
            bits = np.ascontiguousarray(x[name + "_bits"]).view(np.int16)
            dev[name] = torch.from_numpy(bits).cuda().view(torch.bfloat16)
        else:
            dev[name] = torch.from_numpy(np.ascontiguousarray(x[name])).cuda()
    for name in ("dt_p", "A_log", "dt_bias"):
        dev[name] = torch.from_numpy(np.ascontiguousarray(x[name])).cuda()
    dev["D"] = None if x["D"] is None else torch.from_numpy(x["D"]).cuda()
    return dev


def run_gpu(x, dtype, order, normalize, chunk, D="inputs"):
    """Run ssd_fwd on the inputs; returns the output as float64 numpy."""
    import torch
    dev = to_device(x, dtype)
    Dt = dev["D"] if D == "inputs" else D
    out = ssd.ssd_fwd(dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"], dev["dt_bias"],
                      Dt, order, normalize, chunk)
    torch.cuda.synchronize()
    return out.float().cpu().numpy().astype(np.float64)


def rel_err(y, ref):
    """max |y - ref| / max |ref| (the operator's stated error measure)."""
    return float(np.max(np.abs(y - ref)) / np.max(np.abs(ref)))


def sample_rows(N, chunk, seed=0, n_random=16):
    """Rows the oracle evaluates one by one at full size: the first rows,
    both sides of the first chunk boundaries, the middle, the last rows and
    a seeded random set."""
    fixed = [0, 1, chunk - 1, chunk, chunk + 1, 2 * chunk - 1, 2 * chunk, N // 2 - 1, N // 2,
             N - chunk - 1, N - chunk, N - 2, N - 1]
    rng = np.random.default_rng(seed)
    rnd = rng.integers(0, N, size=n_random).tolist()
    return sorted(set(r for r in fixed + rnd if 0 <= r < N))
