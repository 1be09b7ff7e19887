"""Host logic of bench.py: the algorithmic work per token-head of each
workload (the roofline's numerator), and the parsing of the clock samples
taken during the timed region."""
import bench
from mamba_ssd_sequence_b200 import inputs

# per token-head (bytes, FLOPs), worked by hand from the definitions:
# bytes = 4 d e + 4 (q, k, v, out of d elements of e bytes, dt_p in fp32);
# FLOPs = 2 (C + 1) d + 4 D_phi d [+ 4 D_phi + C + 1 with the normaliser]
EXPECTED = {
    "order1-fp32-B1H2N256d16-c64": (260, 2 * 65 * 16 + 4 * 16 * 16),              # 3,104
    "order1-bf16-B4H16N2048d64-c128": (516, 2 * 129 * 64 + 4 * 64 * 64),          # 32,896
    "order2-bf16-B4H16N4096d32-c64": (260, 2 * 65 * 32 + 4 * 1024 * 32 + 4 * 1024 + 65),  # 139,393
    "order1-bf16-B1H32N65536d64-c256": (516, 2 * 257 * 64 + 4 * 64 * 64),         # 49,280
    "order2-bf16-B2H8N16384d64-c64": (516, 2 * 65 * 64 + 4 * 4096 * 64 + 4 * 4096 + 65),  # 1,073,345
}


def test_algorithmic_work_per_token_head():
    assert set(EXPECTED) == set(inputs.WORKLOAD_ORDER)
    for name, (bpt, fpt) in EXPECTED.items():
        w = inputs.WORKLOADS[name]
        total_b, total_f, got_b, got_f = bench.algorithmic_work(w)
        assert (got_b, got_f) == (bpt, fpt), name
        assert total_b == w.token_heads * bpt and total_f == w.token_heads * fpt


def test_headline_totals():
    w = inputs.WORKLOADS[inputs.HEADLINE]
    total_b, total_f, _, _ = bench.algorithmic_work(w)
    assert total_b == 67_633_152 and total_f == 4_311_744_512


def test_clock_summary_parses_samples(tmp_path):
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "clocks.csv")
    s.proc = object()  # a sampler that ran
    with open(s.path, "w") as f:
        f.write("0, 1965, 1965, 700.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")
        f.write("0, 1900, 1965, 990.5, 0x4, Not Active, Not Active, Not Active, Active\n")
        f.write("0, 1950, 1965, 800.0, 0x0, Not Active, Not Active, Not Active, Not Active\n")
        f.write("garbage line\n")
    out = s.summary()
    assert out == {"sm_mhz": 1950.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 3}


def test_clock_summary_without_nvidia_smi():
    s = bench.ClockSampler(0)
    assert s.summary()["reasons"] == ["nvidia-smi unavailable"]


def test_quad_tile_pairs_matches_a_walk_over_the_tiles():
    """The bench's count of the quadratic form's (query, key) tile pairs
    equals a direct walk over each query tile's key tiles with the kernel's
    rule (its own tile, the tile before, then earlier tiles while the decay
    over the tiles between is at least 2^-200)."""
    import numpy as np
    w = inputs.Workload("t", 2, 3, 2048, 32, 64, 2, True, False, "bf16")
    x = inputs.make_inputs(w.B, w.H, w.N, w.d, "bf16", seed=4)
    # strong decays in some heads, so that walks stop early
    x["A_log"] = np.log(np.array([1.0, 8.0, 16.0], np.float32))
    x["dt_bias"] = np.array([-6.0, 0.0, 1.0], np.float32)
    T, NT = 128, w.N // 128
    dt = np.logaddexp(0.0, x["dt_p"].reshape(w.B, w.H, w.N).astype(np.float64) + x["dt_bias"][None, :, None])
    a = -np.exp(x["A_log"].astype(np.float64))[None, :, None] * dt / np.log(2.0)
    lam = a.reshape(w.B, w.H, NT, T).sum(-1)
    want = 0
    for b in range(w.B):
        for h in range(w.H):
            for I in range(NT):
                want += 1
                J, G = I, 0.0
                while J > 0:
                    J -= 1
                    if J <= I - 2:
                        G += lam[b, h, J + 1]
                        if G < -200.0:
                            break
                    want += 1
    got = bench.quad_tile_pairs(w, x)
    assert got == want
    assert got < w.B * w.H * NT * (NT + 1) // 2  # the strong decays skip tiles
