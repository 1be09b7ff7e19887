"""B200 (sm_100a) implementation of the decay-masked linear-attention (SSD)
forward operator of Mamba-2 / Mamba-2S / 2Mamba.

This module is a thin ctypes binding over libssd.so (C ABI in
include/ssd.h).  It only marshals arguments: every step of the operator runs
in the library's CUDA kernels.  Tensors are torch tensors; device tensors must
be contiguous and live on the current CUDA device.  If libssd.so has not been
built, every call raises -- there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssd.so")

SSD_F32 = 0
SSD_BF16 = 1
SSD_VALUE_DT = 1  # ssd_fwd_ex flag: contract with v * dt (Algorithm 4, V_dt)
SSD_STATE_H = 1   # state-mask bits for ssd_workspace_bytes_ex
SSD_STATE_Z = 2
PATH_NAMES = {0: "simt", 1: "tc_order1", 2: "tc_order2", 3: "tc_order2_quad"}

_lib = None


class SSDError(RuntimeError):
    """A libssd.so entry point returned a non-zero ssd_status."""

    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {status_str(code)} (code {code})")


class ConvParams(ctypes.Structure):
    """include/ssd.h ssd_conv_params: the taps of the convolution prologue."""
    _fields_ = [("w", ctypes.c_void_p * 3), ("bias", ctypes.c_void_p * 3), ("width", ctypes.c_int),
                ("silu", ctypes.c_int)]


def load_library():
    """Load libssd.so (ctypes) and declare the C signatures.  Raises if the
    library has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m mamba_ssd_sequence_b200.build` "
            "(there is no CPU or Python fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, sz, ci = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int
    lib.ssd_workspace_bytes.argtypes = [ci] * 7
    lib.ssd_workspace_bytes.restype = sz
    lib.ssd_fwd.argtypes = [vp] * 7 + [ci] * 8 + [vp, vp, sz, vp]
    lib.ssd_fwd.restype = ci
    lib.ssd_fwd_ex.argtypes = [vp] * 8 + [ci] * 9 + [vp, vp, sz, vp]
    lib.ssd_fwd_ex.restype = ci
    lib.ssd_fwd_state.argtypes = [vp] * 8 + [ci] * 9 + [vp] * 4 + [vp, vp, sz, vp]
    lib.ssd_fwd_state.restype = ci
    lib.ssd_workspace_bytes_ex.argtypes = [ci] * 9
    lib.ssd_workspace_bytes_ex.restype = sz
    lib.ssd_decode_workspace_bytes.argtypes = [ci] * 4
    lib.ssd_decode_workspace_bytes.restype = sz
    lib.ssd_decode_step.argtypes = [vp] * 8 + [ci] * 7 + [vp, vp, vp, vp, sz, vp]
    lib.ssd_decode_step.restype = ci
    lib.ssd_conv1d.argtypes = [vp] * 3 + [ci] * 7 + [vp, vp]
    lib.ssd_conv1d.restype = ci
    lib.ssd_fwd_conv_workspace_bytes.argtypes = [ci] * 8
    lib.ssd_fwd_conv_workspace_bytes.restype = sz
    lib.ssd_fwd_conv.argtypes = [vp, vp, vp, ctypes.POINTER(ConvParams)] + [vp] * 5 + [ci] * 9 + [vp, vp, sz, vp]
    lib.ssd_fwd_conv.restype = ci
    lib.ssd_fwd_host.argtypes = [vp] * 7 + [ci] * 8 + [vp] + [vp] * 8 + [vp, sz, vp]
    lib.ssd_fwd_host.restype = ci
    lib.ssd_chunk_cumsum.argtypes = [vp] * 3 + [ci] * 4 + [vp, vp, vp]
    lib.ssd_chunk_cumsum.restype = ci
    lib.ssd_status_from_workspace.argtypes = [vp, vp]
    lib.ssd_status_from_workspace.restype = ci
    lib.ssd_status_str.argtypes = [ci]
    lib.ssd_status_str.restype = ctypes.c_char_p
    lib.ssd_fwd_path.argtypes = [ci] * 7 + [ctypes.POINTER(ci)]
    lib.ssd_fwd_path.restype = ci
    lib.ssd_debug_fwd.argtypes = [vp] * 7 + [ci] * 8 + [vp, vp, sz, vp, ci, ctypes.c_longlong, ci]
    lib.ssd_debug_fwd.restype = ci
    _lib = lib
    return lib


def status_str(code: int) -> str:
    return load_library().ssd_status_str(int(code)).decode()


def _check(code: int, where: str):
    if code != 0:
        raise SSDError(code, where)


def _dtype_code(t) -> int:
    import torch
    if t.dtype == torch.float32:
        return SSD_F32
    if t.dtype == torch.bfloat16:
        return SSD_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {t.dtype}")


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors passed to libssd must be contiguous")
    return t.data_ptr()


def _stream_handle(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def ssd_workspace_bytes(B: int, H: int, N: int, d_h: int, dtype: int, order: int,
                        chunk: int) -> int:
    """Device workspace (bytes) ssd_fwd needs; 0 for invalid arguments."""
    return int(load_library().ssd_workspace_bytes(B, H, N, d_h, dtype, order, chunk))


def ssd_fwd_path(B: int, H: int, N: int, d_h: int, dtype: int, order: int, chunk: int):
    """(path name, kernels launched per call) for these arguments."""
    n = ctypes.c_int(0)
    p = load_library().ssd_fwd_path(B, H, N, d_h, dtype, order, chunk, ctypes.byref(n))
    if p < 0:
        raise ValueError("invalid ssd arguments")
    return PATH_NAMES[p], n.value


def ssd_workspace_bytes_ex(B: int, H: int, N: int, d_h: int, dtype: int, order: int, chunk: int,
                           flags: int = 0, state: int = 0) -> int:
    """Device workspace (bytes) ssd_fwd_ex / ssd_fwd_state need for these
    options (state: SSD_STATE_H | SSD_STATE_Z bits in use); 0 when invalid."""
    return int(load_library().ssd_workspace_bytes_ex(B, H, N, d_h, dtype, order, chunk, flags, state))


def alloc_workspace(B, H, N, d_h, dtype, order, chunk, device=None, flags: int = 0, state: int = 0):
    """A torch uint8 device buffer of ssd_workspace_bytes_ex() bytes."""
    import torch
    nbytes = ssd_workspace_bytes_ex(B, H, N, d_h, dtype, order, chunk, flags, state)
    if nbytes == 0:
        raise ValueError("invalid ssd arguments")
    return torch.empty(nbytes, dtype=torch.uint8, device=device or "cuda")


def ssd_fwd(q, k, v, dt_p, A_log, dt_bias, D, order: int, normalize: bool, chunk: int,
            out=None, workspace=None, stream=None, log_decay=None, value_dt: bool = False):
    """y = SSD forward (include/ssd.h: ssd_fwd, or ssd_fwd_ex when a Mamba-2S
    option is used) on CUDA tensors.

    q, k, v: [B, H, N, d_h] float32 or bfloat16; dt_p: [B, H, N] float32;
    A_log, dt_bias: [H] float32; D: [H*d_h] float32 or None.  log_decay:
    [B, H, N] float32 per-token log-decay replacing A*dt (A_log may then be
    None); value_dt: contract with v * dt.  Returns `out` ([B, H, N, d_h], the
    input dtype), allocating it and the workspace with torch when not given.
    Asynchronous on `stream` (default: the current torch stream)."""
    import torch
    B, H, N, d = q.shape
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    flags = SSD_VALUE_DT if value_dt else 0
    if workspace is None:
        workspace = alloc_workspace(B, H, N, d, dt, order, chunk, q.device, flags)
    lib = load_library()
    if log_decay is None and not value_dt:
        rc = lib.ssd_fwd(
            _ptr(q), _ptr(k), _ptr(v), _ptr(dt_p), _ptr(A_log), _ptr(dt_bias), _ptr(D),
            B, H, N, d, dt, int(order), int(bool(normalize)), int(chunk),
            _ptr(out), _ptr(workspace), workspace.numel(), _stream_handle(stream))
        _check(rc, "ssd_fwd")
    else:
        rc = lib.ssd_fwd_ex(
            _ptr(q), _ptr(k), _ptr(v), _ptr(dt_p), _ptr(A_log), _ptr(dt_bias), _ptr(D),
            _ptr(log_decay), B, H, N, d, dt, int(order), int(bool(normalize)), int(chunk),
            SSD_VALUE_DT if value_dt else 0, _ptr(out), _ptr(workspace), workspace.numel(),
            _stream_handle(stream))
        _check(rc, "ssd_fwd_ex")
    return out


def ssd_debug_fwd(q, k, v, dt_p, A_log, dt_bias, D, order: int, normalize: bool, chunk: int,
                  skip_publish: int, wait_ns: int, out=None, workspace=None, stream=None, path: int = -1):
    """Failure-detection test hook (include/ssd.h: ssd_debug_fwd): ssd_fwd in
    which one producer skips its publication at pipeline step `skip_publish`
    (-1: none) and every bounded device-side wait gives up after `wait_ns`
    nanoseconds; `path` 2 runs the chunked order-2 kernel that calls with a
    carried state take.  Returns `out`; read the device status with
    ssd_status_from_workspace(workspace)."""
    import torch
    B, H, N, d = q.shape
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        workspace = alloc_workspace(B, H, N, d, dt, order, chunk, q.device,
                                    state=SSD_STATE_H if path == 2 else 0)
    rc = load_library().ssd_debug_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dt_p), _ptr(A_log), _ptr(dt_bias), _ptr(D),
        B, H, N, d, dt, int(order), int(bool(normalize)), int(chunk),
        _ptr(out), _ptr(workspace), workspace.numel(), _stream_handle(stream),
        int(skip_publish), int(wait_ns), int(path))
    _check(rc, "ssd_debug_fwd")
    return out


def ssd_fwd_state(q, k, v, dt_p, A_log, dt_bias, D, order: int, normalize: bool, chunk: int,
                  h0=None, z0=None, h_out=None, z_out=None, out=None, workspace=None, stream=None,
                  log_decay=None, value_dt: bool = False):
    """ssd_fwd with the carried state in and out (include/ssd.h, ssd_fwd_state).

    h0 / h_out: [B, H, d_h^order, d_h] float32, z0 / z_out: [B, H, d_h^order]
    float32 CUDA tensors or None (h_out may be h0: updated in place).
    Returns `out`."""
    import torch
    B, H, N, d = q.shape
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    flags = SSD_VALUE_DT if value_dt else 0
    state = (SSD_STATE_H if (h0 is not None or h_out is not None) else 0) | \
        (SSD_STATE_Z if (z0 is not None or z_out is not None) else 0)
    if workspace is None:
        workspace = alloc_workspace(B, H, N, d, dt, order, chunk, q.device, flags, state)
    rc = load_library().ssd_fwd_state(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dt_p), _ptr(A_log), _ptr(dt_bias), _ptr(D), _ptr(log_decay),
        B, H, N, d, dt, int(order), int(bool(normalize)), int(chunk), flags,
        _ptr(h0), _ptr(z0), _ptr(h_out), _ptr(z_out),
        _ptr(out), _ptr(workspace), workspace.numel(), _stream_handle(stream))
    _check(rc, "ssd_fwd_state")
    return out


def ssd_decode_workspace_bytes(B: int, H: int, d_h: int, order: int) -> int:
    """Device workspace (bytes) ssd_decode_step needs; 0 when invalid."""
    return int(load_library().ssd_decode_workspace_bytes(B, H, d_h, order))


def ssd_decode_step(q, k, v, dt_p, A_log, dt_bias, D, order: int, normalize: bool, h, z=None,
                    out=None, workspace=None, stream=None, log_decay=None, value_dt: bool = False):
    """One recurrent step (include/ssd.h, ssd_decode_step): q, k, v [B, H, d_h];
    dt_p / log_decay [B, H]; h [B, H, d_h^order, d_h] and z [B, H, d_h^order]
    float32, updated in place.  Returns `out` [B, H, d_h]."""
    import torch
    B, H, d = q.shape
    dt = _dtype_code(q)
    if out is None:
        out = torch.empty_like(q)
    if workspace is None:
        n = ssd_decode_workspace_bytes(B, H, d, order)
        if n == 0:
            raise ValueError("invalid ssd_decode_step arguments")
        workspace = torch.empty(n, dtype=torch.uint8, device=q.device)
    rc = load_library().ssd_decode_step(
        _ptr(q), _ptr(k), _ptr(v), _ptr(dt_p), _ptr(A_log), _ptr(dt_bias), _ptr(D), _ptr(log_decay),
        B, H, d, dt, int(order), int(bool(normalize)), SSD_VALUE_DT if value_dt else 0,
        _ptr(h), _ptr(z), _ptr(out), _ptr(workspace), workspace.numel(), _stream_handle(stream))
    _check(rc, "ssd_decode_step")
    return out


def ssd_fwd_host(q_h, k_h, v_h, dt_p_h, A_log_h, dt_bias_h, D_h, order: int,
                 normalize: bool, chunk: int, out_h, dev: dict, workspace, stream=None):
    """ssd_fwd_host (include/ssd.h): host (pinned) tensors in and out, with the
    caller's device buffers `dev` (keys q, k, v, dt_p, A_log, dt_bias, D, out)
    receiving the copies.  Asynchronous on `stream`."""
    B, H, N, d = q_h.shape
    dt = _dtype_code(q_h)
    rc = load_library().ssd_fwd_host(
        _ptr(q_h), _ptr(k_h), _ptr(v_h), _ptr(dt_p_h), _ptr(A_log_h), _ptr(dt_bias_h),
        _ptr(D_h), B, H, N, d, dt, int(order), int(bool(normalize)), int(chunk), _ptr(out_h),
        _ptr(dev["q"]), _ptr(dev["k"]), _ptr(dev["v"]), _ptr(dev["dt_p"]),
        _ptr(dev["A_log"]), _ptr(dev["dt_bias"]), _ptr(dev.get("D")), _ptr(dev["out"]),
        _ptr(workspace), workspace.numel(), _stream_handle(stream))
    _check(rc, "ssd_fwd_host")
    return out_h


def ssd_chunk_cumsum(dt_p, A_log, dt_bias, chunk: int, acs=None, chunk_sum=None, stream=None):
    """Kernel (a): chunk-local inclusive cumsum of A*dt and chunk totals
    (include/ssd.h, ssd_chunk_cumsum).  Returns (acs [B,H,N], chunk_sum [B,H,N/chunk])."""
    import torch
    B, H, N = dt_p.shape
    if acs is None:
        acs = torch.empty_like(dt_p)
    if chunk_sum is None:
        chunk_sum = torch.empty((B, H, N // chunk), dtype=torch.float32, device=dt_p.device)
    rc = load_library().ssd_chunk_cumsum(_ptr(dt_p), _ptr(A_log), _ptr(dt_bias), B, H, N,
                                         int(chunk), _ptr(acs), _ptr(chunk_sum),
                                         _stream_handle(stream))
    _check(rc, "ssd_chunk_cumsum")
    return acs, chunk_sum


def ssd_status_from_workspace(workspace, stream=None) -> int:
    """Synchronise and read the device status left in the workspace."""
    return int(load_library().ssd_status_from_workspace(_ptr(workspace),
                                                        _stream_handle(stream)))


def ssd_fwd_conv_workspace_bytes(B: int, H: int, N: int, d_h: int, dtype: int, order: int, chunk: int,
                                 flags: int = 0) -> int:
    return int(load_library().ssd_fwd_conv_workspace_bytes(B, H, N, d_h, dtype, order, chunk, flags))


def ssd_fwd_conv(xq, xk, xv, w, bias, dt_p, A_log, dt_bias, D, order: int, normalize: bool, chunk: int,
                 silu: bool = True, out=None, workspace=None, stream=None, log_decay=None, value_dt: bool = False):
    """The operator with its convolution prologue (include/ssd.h, ssd_fwd_conv):
    q, k, v = SiLU(conv(xq)), SiLU(conv(xk)), SiLU(conv(xv)), then ssd_fwd.

    xq, xk, xv: [B, H, N, d_h] CUDA tensors (before the convolution); w: three
    [H*d_h, width] float32 tensors (for q, k, v); bias: three [H*d_h] float32
    tensors or None (the tuple or its entries).  Other arguments as ssd_fwd.
    Returns `out`."""
    import torch
    B, H, N, d = xq.shape
    dt = _dtype_code(xq)
    if out is None:
        out = torch.empty_like(xq)
    flags = SSD_VALUE_DT if value_dt else 0
    if workspace is None:
        nbytes = ssd_fwd_conv_workspace_bytes(B, H, N, d, dt, order, chunk, flags)
        if nbytes == 0:
            raise ValueError("invalid ssd arguments")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=xq.device)
    biases = bias if bias is not None else (None, None, None)
    cp = ConvParams()
    for i in range(3):
        cp.w[i] = _ptr(w[i])
        cp.bias[i] = _ptr(biases[i])
    cp.width = int(w[0].shape[1])
    if any(int(t.shape[1]) != cp.width for t in w):
        raise ValueError("the three tap tensors must have the same width")
    cp.silu = int(bool(silu))
    rc = load_library().ssd_fwd_conv(
        _ptr(xq), _ptr(xk), _ptr(xv), ctypes.byref(cp), _ptr(dt_p), _ptr(A_log), _ptr(dt_bias), _ptr(D),
        _ptr(log_decay), B, H, N, d, dt, int(order), int(bool(normalize)), int(chunk), flags,
        _ptr(out), _ptr(workspace), workspace.numel(), _stream_handle(stream))
    _check(rc, "ssd_fwd_conv")
    return out


def ssd_conv1d(x, w, bias=None, silu: bool = True, out=None, stream=None):
    """Causal depthwise conv over tokens (+ SiLU) on a CUDA tensor
    (include/ssd.h, ssd_conv1d): x [B, H, N, d_h]; w [H*d_h, width] float32
    (w[:, j] multiplies token t - j); bias [H*d_h] or None.  Returns `out`."""
    import torch
    B, H, N, d = x.shape
    if out is None:
        out = torch.empty_like(x)
    rc = load_library().ssd_conv1d(_ptr(x), _ptr(w), _ptr(bias), B, H, N, d, int(w.shape[1]),
                                   int(bool(silu)), _dtype_code(x), _ptr(out), _stream_handle(stream))
    _check(rc, "ssd_conv1d")
    return out
