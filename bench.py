"""Benchmark of the SSD forward operator on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--impl ours|reference] [--no-cpu-baseline]

One step is one ssd_fwd() call -- the whole hot path (decay, intra-chunk
quadratic form, carried state, normaliser / residual epilogue) -- over one
batch of seeded synthetic input of the workload's shape, with the inputs
resident in HBM.  Before every step the L2 is flushed: a 256 MiB buffer is
written (evicting the inputs) and then read back (so the flush's own dirty
lines are written back before, not during, the timed kernels).  Each step is
timed by its own CUDA-event pair on the launching stream.  With N > 1 (torchrun) every rank runs an
independent replica of the workload on its own GPU (the operator has no
cross-GPU step); the time is the max over ranks and `value` counts the tokens
of all ranks ("weak" scaling).

Rank 0 prints one JSON line.  `--impl reference` times the CPU oracle (the
only other implementation of the method) on the host cores instead, on a
bounded sample of the same workload.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mamba_ssd_sequence_b200 import inputs  # noqa: E402

METRIC = "SSD fwd tokens/s and TFLOP/s (frac. of bf16 TC peak) at H=16,d_h=64,N=2K–64K"
L2_FLUSH_BYTES = 256 << 20
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def max_over_ranks(value: float, device="cpu") -> float:
    """The largest `value` over all ranks (identity without a process group)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank: float, steps: int, world: int, total_ms: float) -> float:
    """Whole-job throughput: every rank processes `units_per_rank` per step;
    the job's time is the slowest rank's."""
    return world * units_per_rank * steps / (total_ms / 1e3)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return p, "measured"
    except (OSError, ValueError):
        return dict(FALLBACK_PEAKS), "fallback"


# DRAM bytes of one call, dram__bytes_read.sum + dram__bytes_write.sum summed
# over the path's kernels, each captured by ncu with caches flushed before it
# (the captures summarised under profiles/, taken on the kernels in this tree;
# a workload without a capture of the current kernels reports null).
DRAM_TRAFFIC = {
    # chunk states 34.11 MB + state pass 8.40 MB + chunk outputs 59.47 MB
    "order1-bf16-B4H16N2048d64-c128": 101_977_344,
    # chunk states 607.3 MB + state pass 87.1 MB + chunk outputs 1127.6 MB
    "order1-bf16-B1H32N65536d64-c256": 1_821_930_752,
    # quadratic form: decay factors 1.05 MB + the loop over key tiles 53.2 MB
    "order2-bf16-B4H16N4096d32-c64": 54_286_336,
    # quadratic form: decay factors 1.05 MB + the loop over key tiles 117.5 MB
    "order2-bf16-B2H8N16384d64-c64": 118_563_328,
}


def algorithmic_work(w: inputs.Workload):
    """Per-launch algorithmic bytes and FLOPs of one call.

    bytes per token-head: q, k, v and out (d_h elements each) plus dt_p (fp32);
    the carried state never leaves the chip and is not counted.
    FLOPs per token-head: the causal half of the intra-chunk score and value
    products 2(C+1)d, the state build and state readout 4*D_phi*d, and the
    normaliser 4*D_phi + C + 1 when it is on."""
    e = 2 if w.dtype == "bf16" else 4
    d, C = w.d, w.chunk
    dphi = d if w.order == 1 else d * d
    per_tok_bytes = 4 * d * e + 4
    per_tok_flops = 2 * (C + 1) * d + 4 * dphi * d + ((4 * dphi + C + 1) if w.normalize else 0)
    T = w.token_heads
    return T * per_tok_bytes, T * per_tok_flops, per_tok_bytes, per_tok_flops


def quad_tile_pairs(w: inputs.Workload, x) -> int:
    """(query tile, key tile) pairs of 128 tokens that the order-2 quadratic
    form multiplies on these inputs: per query tile I its own tile, tile
    I - 1, and earlier tiles while the decay over the tiles between stays at
    or above 2^-200 (the kernel's rule, evaluated here in float64 from the
    same inputs, so a pair at the boundary may count differently)."""
    T = 128
    NT = w.N // T
    dt_p = x["dt_p"].reshape(w.B, w.H, w.N).astype(np.float64)
    dt = np.logaddexp(0.0, dt_p + x["dt_bias"].astype(np.float64)[None, :, None])
    a = -np.exp(x["A_log"].astype(np.float64))[None, :, None] * dt / np.log(2.0)
    lam = a.reshape(w.B, w.H, NT, T).sum(-1)
    pairs = 0
    for b in range(w.B):
        for h in range(w.H):
            negc = -np.concatenate([[0.0], np.cumsum(lam[b, h])])  # -sum of lam over tiles < k, increasing
            for I in range(NT):
                n = 1 + (1 if I >= 1 else 0)
                if I >= 2:  # tiles J <= I - 2: decay over tiles J + 1 .. I - 1 = negc[J + 1] - negc[I] <= 200
                    m0 = int(np.searchsorted(negc, negc[I] - 200.0, side="left"))
                    lo = max(m0, 1)
                    n += max(0, (I - 1) - lo + 1)
                pairs += n
    return pairs


def roofline_of(w: inputs.Workload, mean_ms: float, peaks, peak_src: str):
    """The roofline object of one call of workload `w` that took `mean_ms`:
    order 1 is bound by HBM (algorithmic bytes / time against hbm_gbs), order
    2 by the tensor cores (algorithmic FLOPs / time against bf16_tflops)."""
    alg_bytes, alg_flops, _, _ = algorithmic_work(w)
    tflops = alg_flops / (mean_ms / 1e3) / 1e12
    gbs = alg_bytes / (mean_ms / 1e3) / 1e9
    if w.order == 1:
        bound, achieved, peak, unit = "hbm", gbs, float(peaks["hbm_gbs"]), "GB/s"
    else:
        bound, achieved, peak, unit = "tensor", tflops, float(peaks["bf16_tflops"]), "TFLOP/s"
    traffic = DRAM_TRAFFIC.get(w.name)
    return {"bound": bound, "achieved": achieved, "peak": peak, "unit": unit,
            "frac": achieved / peak, "traffic": traffic,
            "traffic_over_algorithmic": None if traffic is None else traffic / alg_bytes,
            "peak_source": f"{peak_src} ({'hbm_gbs' if bound == 'hbm' else 'bf16_tflops'})",
            "algorithmic_bytes_per_launch": alg_bytes,
            "algorithmic_flops_per_launch": alg_flops}, tflops, gbs


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled every 200 ms while running."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = os.path.join("/tmp", f"ssd_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.fh = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=self.fh, stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.fh.close()

    def summary(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        with open(self.path) as f:
            rows = [parts for parts in ([p.strip() for p in line.split(",")] for line in f) if len(parts) >= 9]
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        sm = [float(r[1]) for r in rows if r[1].replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i] == "Active"})
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


def make_device_inputs(w, seed, torch):
    x = inputs.make_workload_inputs(w, seed=seed)
    dev = {}
    for name in ("q", "k", "v"):
        if w.dtype == "bf16":
            t = torch.from_numpy(x[name + "_bits"].view(np.int16)).view(torch.bfloat16)
        else:
            t = torch.from_numpy(x[name])
        dev[name] = t
    for name in ("dt_p", "A_log", "dt_bias"):
        dev[name] = torch.from_numpy(x[name])
    dev["D"] = None if x["D"] is None else torch.from_numpy(x["D"])
    return x, dev


def _oracle_sample(w, x, heads):
    """Arguments of the oracle for the first `heads` (b, h) rows of the
    workload (batch-major), every token."""
    bsel = (heads + w.H - 1) // w.H
    q = x["q"][:bsel].reshape(-1, w.N, w.d)[:heads][None]
    k = x["k"][:bsel].reshape(-1, w.N, w.d)[:heads][None]
    v = x["v"][:bsel].reshape(-1, w.N, w.d)[:heads][None]
    dt = x["dt_p"][:bsel].reshape(-1, w.N)[:heads][None]
    hidx = np.arange(heads) % w.H
    D = None if x["D"] is None else x["D"].reshape(w.H, w.d)[hidx].reshape(-1)
    return q, k, v, dt, x["A_log"][hidx], x["dt_bias"][hidx], D


def _time_oracle(w, x, target_s):
    """Times the oracle's quadratic form on a sample of (b, h) rows sized to
    take about `target_s` seconds; returns (tokens/s, threads, description)."""
    import oracle
    bh_all = w.B * w.H
    t0 = time.perf_counter()
    oracle.ssd_quadratic(*_oracle_sample(w, x, 1), w.order, w.normalize)
    t1 = max(time.perf_counter() - t0, 1e-6)
    heads = max(1, min(bh_all, int(target_s / t1)))
    reps = 1
    if heads == bh_all:
        reps = max(1, int(target_s / (t1 * bh_all)))
    args = _oracle_sample(w, x, heads)
    t0 = time.perf_counter()
    for _ in range(reps):
        oracle.ssd_quadratic(*args, w.order, w.normalize)
    t = time.perf_counter() - t0
    tokens = reps * w.N * heads / w.H  # equivalent full (all-heads) tokens
    desc = (f"quadratic form (float64, OpenMP) over {heads} of the {bh_all} (b, h) rows, "
            f"all {w.N} tokens, {reps} pass(es): {t:.2f} s")
    return tokens / t, oracle.num_threads(), desc


def cpu_baseline(w, x, target_s=12.0):
    """The CPU oracle as it stands, timed on the host cores on a bounded
    sample of the same workload (the JSON object of the bench line)."""
    value, threads, desc = _time_oracle(w, x, target_s)
    return {"value": value, "unit": "tokens/s", "cores": threads, "kind": "oracle",
            "sample": desc}


def run_reference(args, w):
    """The reference arm: the CPU oracle, timed on the host cores."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    x = inputs.make_workload_inputs(w, seed=0)
    per_step = min(10.0, 120.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        _time_oracle(w, x, per_step / 4)
    vals, descs = [], []
    for _ in range(args.steps):
        v_, threads, d_ = _time_oracle(w, x, per_step)
        vals.append(v_)
        descs.append(d_)
    value = len(vals) / sum(1.0 / v_ for v_ in vals)
    times = [w.tokens / v_ for v_ in vals]
    line = {"metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * sum(times) / len(times), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "impl": "reference",
            "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d_h": w.d,
                       "chunk": w.chunk, "order": w.order, "normalize": w.normalize,
                       "residual": w.residual},
            "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": threads,
                             "kind": "oracle",
                             "sample": "each step: " + descs[-1]},
            "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=30)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=inputs.HEADLINE, choices=inputs.WORKLOAD_ORDER)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="time only the selected workload (skip the other bf16 workloads)")
    args = ap.parse_args()
    w = inputs.WORKLOADS[args.workload]
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist
    import mamba_ssd_sequence_b200 as ssd

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev_name = f"cuda:{local}"
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device(dev_name))

    x, host = make_device_inputs(w, seed=rank, torch=torch)
    dev = {k: (v.to(dev_name) if v is not None else None) for k, v in host.items()}
    out = torch.empty_like(dev["q"])
    dcode = ssd.SSD_BF16 if w.dtype == "bf16" else ssd.SSD_F32
    ws = ssd.alloc_workspace(w.B, w.H, w.N, w.d, dcode, w.order, w.chunk, dev_name)
    path, n_launch = ssd.ssd_fwd_path(w.B, w.H, w.N, w.d, dcode, w.order, w.chunk)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev_name)
    stream = torch.cuda.current_stream()

    def step():
        ssd.ssd_fwd(dev["q"], dev["k"], dev["v"], dev["dt_p"], dev["A_log"], dev["dt_bias"],
                    dev["D"], w.order, w.normalize, w.chunk, out=out, workspace=ws,
                    stream=stream)

    def flush_l2(v):
        flush.fill_(v)
        flush_sink.add_(flush.sum())  # read back: leaves the L2 clean

    flush_sink = torch.zeros((), dtype=torch.float32, device=dev_name)
    for _ in range(max(3, args.warmup)):
        flush_l2(1.0)
        step()
    torch.cuda.synchronize()
    if ssd.ssd_status_from_workspace(ws) != 0:
        raise RuntimeError("device status not clean after warm-up")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local) as clk:
        for i in range(args.steps):
            flush_l2(float(i))
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
        # keep the sampler alive for at least a few samples on short runs
        time.sleep(0.5)
    if world > 1:
        dist.barrier()
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = max_over_ranks(sum(step_ms), dev_name)
    status = ssd.ssd_status_from_workspace(ws)

    # the other bf16 workloads (order 2 at 4K tokens, order 1 at 64K tokens,
    # order 2 at 16K tokens with d_h = 64), each timed the same way: inputs
    # resident, L2 flushed before every step, one CUDA-event pair per step
    others = {}
    if not args.no_workloads:
        for name in inputs.WORKLOAD_ORDER[1:]:
            if name == w.name:
                continue
            ow = inputs.WORKLOADS[name]
            ox, oh = make_device_inputs(ow, seed=rank, torch=torch)
            od = {k: (v.to(dev_name) if v is not None else None) for k, v in oh.items()}
            del oh
            oout = torch.empty_like(od["q"])
            ows = ssd.alloc_workspace(ow.B, ow.H, ow.N, ow.d, ssd.SSD_BF16, ow.order, ow.chunk, dev_name)
            opath, olaunch = ssd.ssd_fwd_path(ow.B, ow.H, ow.N, ow.d, ssd.SSD_BF16, ow.order, ow.chunk)

            def ostep(od=od, oout=oout, ows=ows, ow=ow):
                ssd.ssd_fwd(od["q"], od["k"], od["v"], od["dt_p"], od["A_log"], od["dt_bias"], od["D"],
                            ow.order, ow.normalize, ow.chunk, out=oout, workspace=ows, stream=stream)

            osteps = max(5, min(args.steps, 20))
            for _ in range(max(3, args.warmup)):
                flush_l2(1.0)
                ostep()
            oev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(osteps)]
            for i in range(osteps):
                flush_l2(float(i))
                oev[i][0].record(stream)
                ostep()
                oev[i][1].record(stream)
            torch.cuda.synchronize()
            oms = max_over_ranks(sum(a_.elapsed_time(b_) for a_, b_ in oev), dev_name) / osteps
            others[name] = {"ms": oms, "steps": osteps, "path": opath, "launches_per_step": olaunch,
                            "status": ssd.ssd_status_from_workspace(ows),
                            "value": weak_scaling_rate(ow.tokens, osteps, world, oms * osteps)}
            if opath == "tc_order2_quad":
                # the tensor work the quadratic form actually does, next to the
                # algorithmic FLOPs of the chunked form that the roofline counts
                others[name]["quad_pairs"] = quad_tile_pairs(ow, ox)
            del od, oout, ows, ox
            torch.cuda.empty_cache()

    # kernel (a) on its own: the chunk-local cumsum of A dt and the chunk
    # totals, which the tensor-core paths fuse into their first kernel.  It
    # reads dt_p and writes acs and the chunk totals: HBM-bound.
    acs_a = torch.empty_like(dev["dt_p"])
    csum_a = torch.empty((w.B, w.H, w.N // w.chunk), dtype=torch.float32, device=dev_name)

    def step_a():
        ssd.ssd_chunk_cumsum(dev["dt_p"], dev["A_log"], dev["dt_bias"], w.chunk, acs=acs_a,
                             chunk_sum=csum_a, stream=stream)

    for _ in range(max(3, args.warmup)):
        flush_l2(1.0)
        step_a()
    a_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in range(args.steps)]
    for i in range(args.steps):
        flush_l2(float(i))
        a_ev[i][0].record(stream)
        step_a()
        a_ev[i][1].record(stream)
    torch.cuda.synchronize()
    a_ms = max_over_ranks(sum(s.elapsed_time(e) for s, e in a_ev), dev_name) / args.steps
    a_bytes = 4 * (dev["dt_p"].numel() + acs_a.numel() + csum_a.numel())

    # the memory-bound entry points beside the operator, each timed alone with
    # the L2 flushed before every call: one order-2 decode step at d_h = 64
    # (it reads and writes the whole state, 1 MiB per head) and the conv1d +
    # SiLU prologue over this workload's q
    def time_calls(fn):
        for _ in range(max(3, args.warmup)):
            flush_l2(1.0)
            fn()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(args.steps)]
        for i in range(args.steps):
            flush_l2(float(i))
            ev[i][0].record(stream)
            fn()
            ev[i][1].record(stream)
        torch.cuda.synchronize()
        return max_over_ranks(sum(s_.elapsed_time(e_) for s_, e_ in ev), dev_name) / args.steps

    dB, dH, dd = 2, 8, 64
    xd = inputs.make_inputs(dB, dH, 1, dd, "bf16", seed=rank)
    dq, dk, dv = (torch.from_numpy(xd[n + "_bits"].view(np.int16)).view(torch.bfloat16)
                  .reshape(dB, dH, dd).to(dev_name) for n in ("q", "k", "v"))
    ddt = torch.from_numpy(xd["dt_p"]).reshape(dB, dH).to(dev_name)
    dpar = {n: torch.from_numpy(xd[n]).to(dev_name) for n in ("A_log", "dt_bias", "D")}
    hst = torch.zeros((dB, dH, dd * dd, dd), dtype=torch.float32, device=dev_name)
    zst = torch.zeros((dB, dH, dd * dd), dtype=torch.float32, device=dev_name)
    dout = torch.empty_like(dq)
    dws = torch.empty(ssd.ssd_decode_workspace_bytes(dB, dH, dd, 2), dtype=torch.uint8, device=dev_name)
    dec_ms = time_calls(lambda: ssd.ssd_decode_step(dq, dk, dv, ddt, dpar["A_log"], dpar["dt_bias"], dpar["D"],
                                                    2, True, hst, zst, out=dout, workspace=dws, stream=stream))
    dec_bytes = 2 * 4 * (hst.numel() + zst.numel()) + 2 * (4 * dq.numel()) + 4 * ddt.numel()

    cw = torch.from_numpy(np.random.default_rng(rank).standard_normal((w.H * w.d, 4)).astype(np.float32) / 2.0)
    cw = cw.to(dev_name)
    cout = torch.empty_like(dev["q"])
    conv_ms = time_calls(lambda: ssd.ssd_conv1d(dev["q"], cw, None, True, out=cout, stream=stream))
    conv_bytes = 2 * dev["q"].numel() * dev["q"].element_size() + 4 * cw.numel()

    # the operator with its convolution prologue (window 2 + SiLU on q, k,
    # v), through ssd_fwd_conv (fused into the chunk-state kernel on the
    # order-1 tensor-core path at chunk 128) against ssd_conv1d x 3 followed by
    # the operator, on this workload
    prologue = None
    if w.order == 1 and w.dtype == "bf16":
        prng = np.random.default_rng(100 + rank)
        ptaps = [torch.from_numpy((prng.standard_normal((w.H * w.d, 2)) / 1.5).astype(np.float32)).to(dev_name)
                 for _ in range(3)]
        pbias = [torch.from_numpy((0.1 * prng.standard_normal(w.H * w.d)).astype(np.float32)).to(dev_name)
                 for _ in range(3)]
        pws = torch.empty(ssd.ssd_fwd_conv_workspace_bytes(w.B, w.H, w.N, w.d, ssd.SSD_BF16, 1, w.chunk),
                          dtype=torch.uint8, device=dev_name)
        pc = [torch.empty_like(dev["q"]) for _ in range(3)]
        pout = torch.empty_like(dev["q"])

        def fused_call():
            ssd.ssd_fwd_conv(dev["q"], dev["k"], dev["v"], ptaps, pbias, dev["dt_p"], dev["A_log"], dev["dt_bias"],
                             dev["D"], 1, False, w.chunk, out=pout, workspace=pws, stream=stream)

        def unfused_call():
            for i, n in enumerate(("q", "k", "v")):
                ssd.ssd_conv1d(dev[n], ptaps[i], pbias[i], True, out=pc[i], stream=stream)
            ssd.ssd_fwd(pc[0], pc[1], pc[2], dev["dt_p"], dev["A_log"], dev["dt_bias"], dev["D"], 1, False,
                        w.chunk, out=pout, workspace=ws, stream=stream)

        fused_ms = time_calls(fused_call)
        unfused_ms = time_calls(unfused_call)
        prologue = {"what": "conv1d (width 2, bias) + SiLU on q, k, v, then the operator, on this workload, "
                            "L2 flushed before each call",
                    "fused": path == "tc_order1" and w.chunk == 128,
                    "ms_fused": fused_ms, "ms_conv1d_x3_then_operator": unfused_ms,
                    "ms_operator_alone": total_ms / args.steps}

    # end to end: pinned host inputs -> device -> ssd_fwd -> host, per step
    e2e = None
    if not args.no_e2e:
        host_p = {k: (v.pin_memory() if v is not None else None) for k, v in host.items()}
        out_h = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        scratch = dict(dev)
        scratch["out"] = out
        h2d = sum(v.numel() * v.element_size() for v in host_p.values() if v is not None)
        d2h = out_h.numel() * out_h.element_size()

        def e2e_step():
            ssd.ssd_fwd_host(host_p["q"], host_p["k"], host_p["v"], host_p["dt_p"],
                             host_p["A_log"], host_p["dt_bias"], host_p["D"], w.order,
                             w.normalize, w.chunk, out_h, scratch, ws, stream=stream)

        for _ in range(max(3, args.warmup)):
            e2e_step()
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            e2e_step()
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(e0.elapsed_time(e1), dev_name)
        e2e = {"value": weak_scaling_rate(w.tokens, args.steps, world, e2e_ms), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h)}

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    mean_ms = total_ms / args.steps
    peaks, peak_src = load_peaks()
    roofline, tflops, gbs = roofline_of(w, mean_ms, peaks, peak_src)
    line = {
        "metric": METRIC,
        "value": weak_scaling_rate(w.tokens, args.steps, world, total_ms),
        "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": max(3, args.warmup),
        "ms_per_step": mean_ms,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.dtype == "bf16" else "f32",
        "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "H": w.H, "N": w.N, "d_h": w.d,
                   "chunk": w.chunk, "order": w.order, "normalize": w.normalize,
                   "residual": w.residual, "parallelism": f"replicas{world}",
                   "l2": "flushed before every step (256 MiB written, then read back so no "
                         "dirty lines remain); each step timed by its own CUDA-event pair",
                   "path": path},
        "tflops": tflops,
        "tc_frac": tflops / float(peaks["bf16_tflops"]),
        "hbm_gbs": gbs,
        "roofline": roofline,
        "gpu_launches": n_launch * args.steps,
        "kernel_a": {"what": "chunk cumsum of A dt and chunk totals, launched alone (L2 flushed before each)",
                     "ms_per_launch": a_ms, "bytes_per_launch": a_bytes,
                     "achieved_gbs": a_bytes / (a_ms / 1e3) / 1e9,
                     "frac_of_hbm": a_bytes / (a_ms / 1e3) / 1e9 / float(peaks["hbm_gbs"])},
        "decode_step": {"what": "one order-2 recurrent step with the normaliser, B=2 H=8 d_h=64 "
                                "(reads and writes h and z), L2 flushed before each",
                        "ms_per_call": dec_ms, "bytes_per_call": dec_bytes,
                        "achieved_gbs": dec_bytes / (dec_ms / 1e3) / 1e9,
                        "frac_of_hbm": dec_bytes / (dec_ms / 1e3) / 1e9 / float(peaks["hbm_gbs"])},
        "conv1d": {"what": "causal depthwise conv1d (width 4) + SiLU over this workload's q, "
                           "L2 flushed before each",
                   "ms_per_call": conv_ms, "bytes_per_call": conv_bytes,
                   "achieved_gbs": conv_bytes / (conv_ms / 1e3) / 1e9,
                   "frac_of_hbm": conv_bytes / (conv_ms / 1e3) / 1e9 / float(peaks["hbm_gbs"])},
        "conv_prologue": prologue,
        "device_status": status,
        "clocks": clk.summary(),
    }
    if others:
        wl = {}
        for name, o in others.items():
            ow = inputs.WORKLOADS[name]
            rl, otf, ogbs = roofline_of(ow, o["ms"], peaks, peak_src)
            wl[name] = {"ms_per_step": o["ms"], "steps": o["steps"], "tokens_per_s": o["value"],
                        "tflops": otf, "hbm_gbs": ogbs, "roofline": rl,
                        "path": {0: "simt", 1: "tc_order1", 2: "tc_order2", 3: "tc_order2_quad"}.get(o["path"], o["path"]),
                        "launches_per_step": o["launches_per_step"], "device_status": o["status"],
                        "config": {"B": ow.B, "H": ow.H, "N": ow.N, "d_h": ow.d, "chunk": ow.chunk,
                                   "order": ow.order, "normalize": ow.normalize,
                                   "residual": ow.residual}}
            if "quad_pairs" in o:
                # S = Q K^T and Y += P V per pair: 2 (128 x 128 x d) + 2 (128 x d x 128)
                ex = o["quad_pairs"] * 4 * 128 * 128 * ow.d
                extf = ex / (o["ms"] / 1e3) / 1e12
                wl[name]["executed"] = {
                    "what": "tensor FLOPs the quadratic form performs (tile pairs x 4 x 128^2 x d_h); the "
                            "roofline counts the chunked form's algorithmic FLOPs",
                    "tile_pairs": o["quad_pairs"], "tensor_flops": ex, "tflops": extf,
                    "frac_of_peak": extf / float(peaks["bf16_tflops"])}
        line["workloads"] = wl
    if e2e is not None:
        line["e2e"] = e2e
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w, x)
    print(json.dumps(line), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
