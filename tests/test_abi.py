"""The C ABI: libssd.so loads, exports every function include/ssd.h declares,
and rejects bad arguments before touching the device (no GPU needed)."""
import ctypes
import os
import re

import pytest

import mamba_ssd_sequence_b200 as ssd
from mamba_ssd_sequence_b200 import build as ssd_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    ssd_build.build()
    return ssd.load_library()


def _declared_functions():
    names = []
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            text = open(os.path.join(ROOT, "include", fn)).read()
            text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
            names += re.findall(r"\b(ssd_[a-z0-9_]+)\s*\(", text)
    return sorted(set(names))


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert "ssd_fwd" in names and "ssd_workspace_bytes" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in include/ but not exported"


def test_workspace_bytes_rejects_invalid(lib):
    ok = ssd.ssd_workspace_bytes(4, 16, 2048, 64, ssd.SSD_BF16, 1, 128)
    assert ok > 0 and ok % 256 == 0
    assert ssd.ssd_workspace_bytes(4, 16, 2000, 64, ssd.SSD_BF16, 1, 128) == 0  # N % chunk
    assert ssd.ssd_workspace_bytes(4, 16, 2048, 48, ssd.SSD_BF16, 1, 128) == 0  # d_h
    assert ssd.ssd_workspace_bytes(4, 16, 2048, 64, 7, 1, 128) == 0             # dtype
    assert ssd.ssd_workspace_bytes(4, 16, 2048, 64, ssd.SSD_BF16, 3, 128) == 0  # order
    assert ssd.ssd_workspace_bytes(4, 16, 2048, 64, ssd.SSD_BF16, 1, 96) == 0   # chunk
    assert ssd.ssd_workspace_bytes(0, 16, 2048, 64, ssd.SSD_BF16, 1, 128) == 0  # empty batch


def _call_fwd(lib, **over):
    a = dict(q=16, k=32, v=48, dt_p=64, A_log=80, dt_bias=96, D=None, B=1, H=2, N=256, d=16,
             dtype=ssd.SSD_F32, order=1, normalize=0, chunk=64, out=112, ws=256, ws_bytes=1 << 30)
    a.update(over)
    return lib.ssd_fwd(a["q"], a["k"], a["v"], a["dt_p"], a["A_log"], a["dt_bias"], a["D"],
                       a["B"], a["H"], a["N"], a["d"], a["dtype"], a["order"], a["normalize"],
                       a["chunk"], a["out"], a["ws"], a["ws_bytes"], None)


def test_fwd_validation_codes(lib):
    """Every rejection happens on the host, before any CUDA call (the fake
    pointers are never dereferenced)."""
    assert _call_fwd(lib, q=None) == 1          # SSD_ERR_NULL
    assert _call_fwd(lib, out=None) == 1
    assert _call_fwd(lib, N=250) == 2           # SSD_ERR_SHAPE (N % chunk)
    assert _call_fwd(lib, N=0) == 2
    assert _call_fwd(lib, d=24) == 2
    assert _call_fwd(lib, dtype=5) == 3         # SSD_ERR_DTYPE
    assert _call_fwd(lib, order=0) == 4         # SSD_ERR_ORDER
    assert _call_fwd(lib, chunk=32) == 5        # SSD_ERR_CHUNK
    assert _call_fwd(lib, k=33) == 6            # SSD_ERR_ALIGN
    assert _call_fwd(lib, D=8) == 6
    assert _call_fwd(lib, ws=128) == 6          # workspace needs 256-byte alignment
    assert _call_fwd(lib, ws=None) == 7         # SSD_ERR_WORKSPACE
    assert _call_fwd(lib, ws_bytes=100) == 7


def test_simt_path_chunk_count_bound(lib):
    """The SIMT path puts the chunk index in gridDim.y (at most 65535): a
    problem that would need more chunks there is rejected as a shape error
    before anything is enqueued, and has no workspace size."""
    N = 65536 * 64  # 65536 chunks of 64 tokens on the fp32 (SIMT) path
    assert ssd.ssd_workspace_bytes(1, 1, N, 16, ssd.SSD_F32, 1, 64) == 0
    assert _call_fwd(lib, B=1, H=1, N=N) == 2   # SSD_ERR_SHAPE
    assert ssd.ssd_workspace_bytes(1, 1, 65535 * 64, 16, ssd.SSD_F32, 1, 64) > 0


def test_status_strings(lib):
    for code in range(11):
        s = ssd.status_str(code)
        assert s.startswith("SSD_")
    assert ssd.status_str(99) == "unknown ssd status"


def test_path_selection(lib):
    path, n = ssd.ssd_fwd_path(1, 2, 256, 16, ssd.SSD_F32, 1, 64)
    assert path == "simt" and n == 4
    path, n = ssd.ssd_fwd_path(4, 16, 2048, 64, ssd.SSD_BF16, 1, 128)
    assert path == "tc_order1" and n == 3
    path, n = ssd.ssd_fwd_path(1, 32, 65536, 64, ssd.SSD_BF16, 1, 256)
    assert path == "tc_order1" and n == 3
    path, n = ssd.ssd_fwd_path(1, 4, 1024, 64, ssd.SSD_BF16, 1, 64)
    assert path == "simt" and n == 4
    # order 2 without a carried state: the quadratic form when N is a multiple
    # of 128, else the chunked kernel
    path, n = ssd.ssd_fwd_path(4, 16, 4096, 32, ssd.SSD_BF16, 2, 64)
    assert path == "tc_order2_quad" and n == 2
    path, n = ssd.ssd_fwd_path(2, 8, 16384, 64, ssd.SSD_BF16, 2, 64)
    assert path == "tc_order2_quad" and n == 2
    path, n = ssd.ssd_fwd_path(2, 8, 16320, 64, ssd.SSD_BF16, 2, 64)
    assert path == "tc_order2" and n == 1
    path, n = ssd.ssd_fwd_path(2, 8, 1024, 16, ssd.SSD_BF16, 2, 64)
    assert path == "simt" and n == 4
    with pytest.raises(ValueError):
        ssd.ssd_fwd_path(1, 2, 250, 16, ssd.SSD_F32, 1, 64)


def test_cumsum_validation(lib):
    assert lib.ssd_chunk_cumsum(16, 32, 48, 1, 1, 100, 64, 64, 80, None) == 2
    assert lib.ssd_chunk_cumsum(16, 32, 48, 1, 1, 128, 48, 64, 80, None) == 5
    assert lib.ssd_chunk_cumsum(None, 32, 48, 1, 1, 128, 64, 64, 80, None) == 1
    # 16-byte vector loads and stores: dt_p and acs must be aligned
    assert lib.ssd_chunk_cumsum(20, 32, 48, 1, 1, 128, 64, 64, 80, None) == 6
    assert lib.ssd_chunk_cumsum(16, 32, 48, 1, 1, 128, 64, 68, 80, None) == 6


def _call_fwd_ex(lib, **over):
    a = dict(q=16, k=32, v=48, dt_p=64, A_log=80, dt_bias=96, D=None, ld=None, B=1, H=2, N=256, d=16,
             dtype=ssd.SSD_F32, order=1, normalize=0, chunk=64, flags=0, out=112, ws=256, ws_bytes=1 << 30)
    a.update(over)
    return lib.ssd_fwd_ex(a["q"], a["k"], a["v"], a["dt_p"], a["A_log"], a["dt_bias"], a["D"], a["ld"],
                          a["B"], a["H"], a["N"], a["d"], a["dtype"], a["order"], a["normalize"],
                          a["chunk"], a["flags"], a["out"], a["ws"], a["ws_bytes"], None)


def test_fwd_ex_validation_codes(lib):
    """ssd_fwd_ex rejects unknown flags and missing inputs of the chosen
    decay / value form on the host (fake pointers, never dereferenced)."""
    assert _call_fwd_ex(lib, flags=2) == 11                              # SSD_ERR_FLAGS
    assert _call_fwd_ex(lib, flags=-1) == 11
    assert _call_fwd_ex(lib, A_log=None) == 1                            # A*dt needs A_log
    assert _call_fwd_ex(lib, dt_p=None) == 1                             # ... and dt_p
    assert _call_fwd_ex(lib, ld=128, A_log=None, flags=1, dt_p=None) == 1  # V (.) dt needs dt_p
    assert _call_fwd_ex(lib, ld=128, A_log=None, flags=1, dt_bias=None) == 1
    assert _call_fwd_ex(lib, ld=136) == 6                                # SSD_ERR_ALIGN
    assert _call_fwd_ex(lib, ld=128, N=250) == 2
    assert ssd.status_str(11).startswith("SSD_ERR_FLAGS")


def test_state_and_decode_validation_codes(lib):
    """ssd_fwd_state / ssd_decode_step reject bad arguments on the host."""
    vp = ctypes.c_void_p
    assert ssd.ssd_workspace_bytes_ex(1, 2, 256, 16, ssd.SSD_F32, 1, 64, 2, 0) == 0   # unknown flag
    assert ssd.ssd_workspace_bytes_ex(1, 2, 256, 16, ssd.SSD_F32, 1, 64, 0, 4) == 0   # unknown state bit
    assert ssd.ssd_workspace_bytes_ex(1, 2, 256, 16, ssd.SSD_F32, 1, 64, 0, 3) > 0
    assert ssd.ssd_decode_workspace_bytes(2, 8, 64, 2) >= 2 * 8 * 64 * 65 * 4
    assert ssd.ssd_decode_workspace_bytes(2, 8, 48, 2) == 0
    assert ssd.ssd_decode_workspace_bytes(2, 8, 64, 3) == 0

    def st(**o):
        a = dict(q=16, k=32, v=48, dt_p=64, A_log=80, dt_bias=96, D=None, ld=None, B=1, H=2, N=256, d=16,
                 dtype=ssd.SSD_F32, order=1, normalize=0, chunk=64, flags=0, h0=None, z0=None, ho=None,
                 zo=None, out=112, ws=256, wsb=1 << 30)
        a.update(o)
        return lib.ssd_fwd_state(a["q"], a["k"], a["v"], a["dt_p"], a["A_log"], a["dt_bias"], a["D"], a["ld"],
                                 a["B"], a["H"], a["N"], a["d"], a["dtype"], a["order"], a["normalize"],
                                 a["chunk"], a["flags"], a["h0"], a["z0"], a["ho"], a["zo"], a["out"], a["ws"],
                                 a["wsb"], None)
    assert st(h0=136) == 6 and st(zo=8) == 6      # SSD_ERR_ALIGN
    assert st(flags=4, h0=128) == 11              # SSD_ERR_FLAGS
    assert st(q=None, h0=128) == 1

    def dec(**o):
        a = dict(q=16, k=32, v=48, dt_p=64, A_log=80, dt_bias=96, D=None, ld=None, B=1, H=2, d=16,
                 dtype=ssd.SSD_F32, order=1, normalize=0, flags=0, h=128, z=None, out=112, ws=256, wsb=1 << 30)
        a.update(o)
        return lib.ssd_decode_step(a["q"], a["k"], a["v"], a["dt_p"], a["A_log"], a["dt_bias"], a["D"], a["ld"],
                                   a["B"], a["H"], a["d"], a["dtype"], a["order"], a["normalize"], a["flags"],
                                   a["h"], a["z"], a["out"], a["ws"], a["wsb"], None)
    assert dec(h=None) == 1                       # the state is required
    assert dec(normalize=1) == 1                  # ... and z when normalising
    assert dec(A_log=None) == 1
    assert dec(flags=2) == 11
    assert dec(d=48) == 2
    assert dec(order=3) == 4
    assert dec(dtype=9) == 3
    assert dec(h=136) == 6
    assert dec(dt_p=66) == 6                      # per-token scalars need 4-byte alignment
    assert dec(wsb=100) == 7


def test_conv1d_validation_codes(lib):
    def cv(**o):
        a = dict(x=1024, w=64, b=None, B=1, H=2, N=8, d=16, width=2, silu=1, dtype=ssd.SSD_BF16, out=4096)
        a.update(o)
        return lib.ssd_conv1d(a["x"], a["w"], a["b"], a["B"], a["H"], a["N"], a["d"], a["width"], a["silu"],
                              a["dtype"], a["out"], None)
    assert cv(x=None) == 1 and cv(w=None) == 1 and cv(out=None) == 1
    assert cv(dtype=4) == 3
    assert cv(width=0) == 2 and cv(width=5) == 2 and cv(d=24) == 2 and cv(N=0) == 2
    assert cv(x=1032) == 6 and cv(w=66) == 6
    assert cv(out=1024 + 256) == 2       # out overlaps x


def test_fwd_conv_validation_codes(lib):
    """ssd_fwd_conv rejects bad taps and arguments on the host; its workspace
    is the operator's plus three activation blocks."""
    base = ssd.ssd_workspace_bytes_ex(1, 2, 256, 64, ssd.SSD_BF16, 1, 128, 0, 0)
    need = ssd.ssd_fwd_conv_workspace_bytes(1, 2, 256, 64, ssd.SSD_BF16, 1, 128)
    assert base > 0 and need == base + 3 * 2 * 256 * 64 * 2
    assert ssd.ssd_fwd_conv_workspace_bytes(1, 2, 250, 64, ssd.SSD_BF16, 1, 128) == 0

    def fc(**o):
        a = dict(xq=16, xk=32, xv=48, w=(64, 80, 96), b=(None, None, None), width=2, silu=1, dt_p=112,
                 A_log=128, dt_bias=144, B=1, H=2, N=256, d=64, dtype=ssd.SSD_BF16, flags=0, out=160, ws=256,
                 ws_bytes=need, params=True)
        a.update(o)
        cp = ssd.ConvParams()
        for i in range(3):
            cp.w[i] = a["w"][i]
            cp.bias[i] = a["b"][i]
        cp.width, cp.silu = a["width"], a["silu"]
        return lib.ssd_fwd_conv(a["xq"], a["xk"], a["xv"], ctypes.byref(cp) if a["params"] else None,
                                a["dt_p"], a["A_log"], a["dt_bias"], None, None, a["B"], a["H"], a["N"], a["d"],
                                a["dtype"], 1, 0, 128, a["flags"], a["out"], a["ws"], a["ws_bytes"], None)
    assert fc(xq=None) == 1 and fc(params=False) == 1 and fc(w=(64, None, 96)) == 1   # SSD_ERR_NULL
    assert fc(width=0) == 2 and fc(width=5) == 2 and fc(N=250) == 2                    # SSD_ERR_SHAPE
    assert fc(flags=4) == 11                                                           # SSD_ERR_FLAGS
    assert fc(xk=40) == 6 and fc(w=(64, 82, 96)) == 6 and fc(b=(None, None, 98)) == 6  # SSD_ERR_ALIGN
    assert fc(ws=None) == 7 and fc(ws_bytes=need - 1) == 7                             # SSD_ERR_WORKSPACE


def test_debug_hook_and_order2_paths(lib):
    """The failure hook validates its path argument and wait limit on the
    host; the order-2 paths and workspaces follow the carried state."""
    def dbg(**o):
        a = dict(q=16, k=32, v=48, dt_p=64, A_log=80, dt_bias=96, D=None, B=1, H=2, N=256, d=32,
                 dtype=ssd.SSD_BF16, order=2, normalize=1, chunk=64, out=112, ws=256, wsb=1 << 30,
                 skip=-1, wait=0, path=-1)
        a.update(o)
        return lib.ssd_debug_fwd(a["q"], a["k"], a["v"], a["dt_p"], a["A_log"], a["dt_bias"], a["D"],
                                 a["B"], a["H"], a["N"], a["d"], a["dtype"], a["order"], a["normalize"],
                                 a["chunk"], a["out"], a["ws"], a["wsb"], None, a["skip"], a["wait"], a["path"])
    assert dbg(path=3) == 10 and dbg(path=0) == 10   # only -1 and the chunked order-2 path
    assert dbg(wait=-1) == 2                         # a negative wait limit
    assert dbg(path=2, dt_p=None) == 1
    # without a carried state order 2 takes the quadratic form, whose scratch
    # (per-token decay factors) differs from the chunked kernel's (partials)
    quad = ssd.ssd_workspace_bytes_ex(2, 8, 16384, 64, ssd.SSD_BF16, 2, 64, 0, 0)
    chunked = ssd.ssd_workspace_bytes_ex(2, 8, 16384, 64, ssd.SSD_BF16, 2, 64, 0, ssd.SSD_STATE_H)
    assert quad >= 256 + 3 * 2 * 8 * 16384 * 4 and chunked > 0 and quad != chunked
    assert ssd.ssd_fwd_path(1, 2, 256, 32, ssd.SSD_BF16, 2, 64)[0] == "tc_order2_quad"
    assert ssd.ssd_fwd_path(1, 2, 192, 32, ssd.SSD_BF16, 2, 64)[0] == "tc_order2"   # N % 128 != 0
    assert ssd.ssd_fwd_path(1, 2, 256, 16, ssd.SSD_BF16, 2, 64)[0] == "simt"        # d_h 16
