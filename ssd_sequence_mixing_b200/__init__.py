"""B200-native chunked SSD (Mamba-2 sequence mixing) forward pass.

A thin ctypes binding over ``libssd.so`` (C ABI in ``include/ssd.h``).  This
module only marshals arguments: shapes are read off torch tensors, outputs are
allocated with torch when the caller does not pass them, and every step of the
computation runs in the library's CUDA kernels.  There is no CPU fallback:
without the built library, importing this package raises.

Entry points: ``ssd_forward`` (device buffers), ``ssd_forward_host`` (host
buffers, copies pipelined with the compute), ``ssd_forward_noalloc`` (no device
allocation), ``ssd_forward_dt`` (step size from the raw projection inside the
kernels), ``ssd_decode_step`` (one generation step), ``causal_conv1d_silu`` and
``gated_rmsnorm`` (the block's steps around the SSD), ``segment_logdecay`` and
``state_prefix`` (sequence parallelism, see ``sequence_parallel``).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssd.so")

SSD_F32, SSD_BF16 = 0, 1
PATH_AUTO, PATH_SIMT, PATH_TC = 0, 1, 2
STATUS = {
    0: "SSD_OK",
    1: "SSD_ERR_INVALID_ARG",
    2: "SSD_ERR_UNSUPPORTED",
    3: "SSD_ERR_MISALIGNED",
    4: "SSD_ERR_CUDA",
    5: "SSD_ERR_DEVICE_TIMEOUT",
    6: "SSD_ERR_BAD_SEQLENS",
    7: "SSD_ERR_SCRATCH_LIMIT",
}
# Size of the static scratch array behind ssd_forward_noalloc (SSD_NOALLOC_SCRATCH_BYTES).
NOALLOC_SCRATCH_BYTES = 32 << 20
# Every entry point include/ssd.h declares.
EXPORTS = (
    "ssd_forward",
    "ssd_forward_host",
    "ssd_workspace_bytes",
    "ssd_query_status",
    "ssd_status_string",
    "ssd_set_path",
    "ssd_select_path",
    "ssd_profile_dominant",
    "ssd_kernel_launch_count",
    "ssd_forward_noalloc",
    "ssd_decode_step",
    "ssd_forward_dt",
    "ssd_causal_conv1d_silu",
    "ssd_gated_rmsnorm",
    "ssd_segment_logdecay",
    "ssd_state_prefix",
    "ssd_set_test_hooks",
)


class SsdDtPrologue(ctypes.Structure):
    _fields_ = [
        ("dt_bias", ctypes.c_void_p),
        ("softplus", ctypes.c_int),
        ("dt_min", ctypes.c_float),
        ("dt_max", ctypes.c_float),
    ]


class SsdShape(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("seqlen", ctypes.c_int64),
        ("nheads", ctypes.c_int64),
        ("headdim", ctypes.c_int64),
        ("dstate", ctypes.c_int64),
        ("ngroups", ctypes.c_int64),
        ("nseq", ctypes.c_int64),
        ("io_dtype", ctypes.c_int),
        ("cu_seqlens_host", ctypes.c_void_p),
    ]


class SsdError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {STATUS.get(code, code)} ({_lib.ssd_status_string(code).decode()})")


def _open() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python ssd_sequence_mixing_b200/build.py`")
    lib = ctypes.CDLL(LIB_PATH)
    V, I, SP = ctypes.c_void_p, ctypes.c_int, ctypes.POINTER(SsdShape)
    fwd = [SP, V, V, V, V, V, V, V, V, I, V, V, V]
    for name in ("ssd_forward", "ssd_forward_host", "ssd_forward_noalloc"):
        getattr(lib, name).argtypes = fwd
        getattr(lib, name).restype = I
    lib.ssd_workspace_bytes.argtypes = [SP, I]
    lib.ssd_workspace_bytes.restype = ctypes.c_size_t
    lib.ssd_query_status.argtypes = [V]
    lib.ssd_query_status.restype = I
    lib.ssd_status_string.argtypes = [I]
    lib.ssd_status_string.restype = ctypes.c_char_p
    lib.ssd_set_path.argtypes = [I]
    lib.ssd_set_path.restype = I
    lib.ssd_select_path.argtypes = [SP, I]
    lib.ssd_select_path.restype = I
    lib.ssd_profile_dominant.argtypes = [V, V]
    lib.ssd_profile_dominant.restype = I
    lib.ssd_kernel_launch_count.argtypes = []
    lib.ssd_kernel_launch_count.restype = ctypes.c_uint64
    lib.ssd_decode_step.argtypes = [SP, V, V, V, V, V, V, V, V, V]
    lib.ssd_decode_step.restype = I
    lib.ssd_forward_dt.argtypes = [SP, ctypes.POINTER(SsdDtPrologue)] + fwd[1:]
    lib.ssd_forward_dt.restype = I
    L = ctypes.c_int64
    lib.ssd_causal_conv1d_silu.argtypes = [L, L, L, I, V, V, V, V, L, V, V]
    lib.ssd_causal_conv1d_silu.restype = I
    lib.ssd_gated_rmsnorm.argtypes = [L, L, I, V, V, V, ctypes.c_float, V, V]
    lib.ssd_gated_rmsnorm.restype = I
    lib.ssd_segment_logdecay.argtypes = [L, L, V, V, V, V]
    lib.ssd_segment_logdecay.restype = I
    lib.ssd_state_prefix.argtypes = [I, L, L, L, V, V, V, V, V]
    lib.ssd_state_prefix.restype = I
    lib.ssd_set_test_hooks.argtypes = [L, I]
    lib.ssd_set_test_hooks.restype = I
    return lib


_lib = _open()


def library() -> ctypes.CDLL:
    return _lib


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _io_code(dtype: torch.dtype) -> int:
    if dtype == torch.float32:
        return SSD_F32
    if dtype == torch.bfloat16:
        return SSD_BF16
    raise TypeError(f"x, B, C must be float32 or bfloat16, got {dtype}")


def make_shape(x: torch.Tensor, B: torch.Tensor, cu_seqlens=None, cu_seqlens_host=None) -> SsdShape:
    """ssd_shape from x (batch, T, H, P) and B (batch, T, G, N)."""
    if x.dim() != 4 or B.dim() != 4:
        raise ValueError("x must be (batch, seqlen, H, P) and B, C (batch, seqlen, G, N)")
    batch, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    nseq = 0
    if cu_seqlens is not None:
        nseq = cu_seqlens.numel() - 1
    s = SsdShape(batch, T, H, P, N, G, nseq, _io_code(x.dtype), None)
    if cu_seqlens_host is not None:
        s.cu_seqlens_host = ctypes.c_void_p(cu_seqlens_host.data_ptr())
    return s


def _check(name, t, device, dtype=None, shape=None):
    if t is None:
        return
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")


def _prepare(x, dt, A, B, C, D, init_state, cu_seqlens, y, final_state, return_final, device):
    batch, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    rows = cu_seqlens.numel() - 1 if cu_seqlens is not None else batch
    _check("x", x, device)
    _check("dt", dt, device, torch.float32, (batch, T, H))
    _check("A", A, device, torch.float32, (H,))
    _check("B", B, device, x.dtype, (batch, T, G, N))
    _check("C", C, device, x.dtype, (batch, T, G, N))
    _check("D", D, device, torch.float32, (H,))
    _check("init_state", init_state, device, torch.float32, (rows, H, P, N))
    _check("cu_seqlens", cu_seqlens, device, torch.int32)
    pin = device.type == "cpu" and x.is_pinned()
    if y is None:
        y = torch.empty(x.shape, dtype=x.dtype, device=device, pin_memory=pin)
    _check("y", y, device, x.dtype, tuple(x.shape))
    if final_state is None and return_final:
        final_state = torch.empty((rows, H, P, N), dtype=torch.float32, device=device, pin_memory=pin)
    _check("final_state", final_state, device, torch.float32, (rows, H, P, N))
    return y, final_state


def ssd_forward(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor, C: torch.Tensor,
                D: Optional[torch.Tensor] = None, init_state: Optional[torch.Tensor] = None,
                cu_seqlens: Optional[torch.Tensor] = None, chunk: int = 256, y: Optional[torch.Tensor] = None,
                final_state: Optional[torch.Tensor] = None, return_final: bool = True, stream=None,
                cu_seqlens_host: Optional[torch.Tensor] = None) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Chunked SSD forward on CUDA tensors (see ``ssd_forward`` in include/ssd.h).

    x (batch, T, H, P) fp32/bf16; dt (batch, T, H) fp32; A (H,) fp32; B, C (batch, T, G, N);
    D (H,) fp32 or None; init_state (rows, H, P, N) fp32 or None; cu_seqlens (nseq+1,) int32
    (packed batch, batch == 1) or None.  Returns (y, final_state).  Asynchronous on ``stream``
    (default: torch's current stream).
    """
    device = x.device
    if device.type != "cuda":
        raise ValueError("ssd_forward takes CUDA tensors; use ssd_forward_host for host buffers")
    y, final_state = _prepare(x, dt, A, B, C, D, init_state, cu_seqlens, y, final_state, return_final, device)
    shape = make_shape(x, B, cu_seqlens, cu_seqlens_host)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(device):
        rc = _lib.ssd_forward(ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                              _ptr(init_state), _ptr(cu_seqlens), int(chunk), _ptr(y), _ptr(final_state),
                              ctypes.c_void_p(handle))
    if rc:
        raise SsdError(rc, "ssd_forward")
    return y, final_state


def ssd_final_state(x: torch.Tensor, dt: torch.Tensor, A: torch.Tensor, B: torch.Tensor,
                    init_state: Optional[torch.Tensor] = None, cu_seqlens: Optional[torch.Tensor] = None,
                    chunk: int = 256, final_state: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
    """Only the state after each sequence: ssd_forward with y = NULL, which reads neither C
    nor D (the tensor-core kernel then loads x, dt and B alone).  Returns final_state
    (rows, H, P, N) fp32."""
    device = x.device
    if device.type != "cuda":
        raise ValueError("ssd_final_state takes CUDA tensors")
    batch, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    rows = cu_seqlens.numel() - 1 if cu_seqlens is not None else batch
    _check("x", x, device)
    _check("dt", dt, device, torch.float32, (batch, T, H))
    _check("A", A, device, torch.float32, (H,))
    _check("B", B, device, x.dtype, (batch, T, G, N))
    _check("init_state", init_state, device, torch.float32, (rows, H, P, N))
    _check("cu_seqlens", cu_seqlens, device, torch.int32)
    if final_state is None:
        final_state = torch.empty((rows, H, P, N), dtype=torch.float32, device=device)
    _check("final_state", final_state, device, torch.float32, (rows, H, P, N))
    shape = make_shape(x, B, cu_seqlens)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(device):
        rc = _lib.ssd_forward(ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), None, None,
                              _ptr(init_state), _ptr(cu_seqlens), int(chunk), None, _ptr(final_state),
                              ctypes.c_void_p(handle))
    if rc:
        raise SsdError(rc, "ssd_forward (final state only)")
    return final_state


def ssd_forward_noalloc(x, dt, A, B, C, D=None, init_state=None, cu_seqlens=None, chunk: int = 256,
                        y: Optional[torch.Tensor] = None, final_state: Optional[torch.Tensor] = None,
                        return_final: bool = True, stream=None):
    """ssd_forward for callers that cannot allocate device memory inside the call.

    A caller that owns the GPU's memory through its own pool (a server that gives HBM to
    weights and KV caches up front) cannot let the library call cudaMallocAsync.  The C entry
    point allocates nothing: its scratch is a static device array of NOALLOC_SCRATCH_BYTES
    shared by all calls (serialise calls; the first call on a device should precede any
    stream capture).  Pass ``y`` and ``final_state`` to keep this wrapper allocation-free too;
    otherwise it creates them with torch before the call.  Shapes needing more scratch raise
    SsdError with SSD_ERR_SCRATCH_LIMIT.
    """
    device = x.device
    if device.type != "cuda":
        raise ValueError("ssd_forward_noalloc takes CUDA tensors")
    y, final_state = _prepare(x, dt, A, B, C, D, init_state, cu_seqlens, y, final_state, return_final, device)
    shape = make_shape(x, B, cu_seqlens)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(device):
        rc = _lib.ssd_forward_noalloc(ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                      _ptr(init_state), _ptr(cu_seqlens), int(chunk), _ptr(y), _ptr(final_state),
                                      ctypes.c_void_p(handle))
    if rc:
        raise SsdError(rc, "ssd_forward_noalloc")
    return y, final_state


def ssd_forward_dt(x, dt_raw, A, B, C, D=None, init_state=None, cu_seqlens=None, chunk: int = 256,
                   dt_bias: Optional[torch.Tensor] = None, softplus: bool = True, dt_min: float = 0.0,
                   dt_max: float = float("inf"), y: Optional[torch.Tensor] = None,
                   final_state: Optional[torch.Tensor] = None, return_final: bool = True, stream=None):
    """ssd_forward with the step size made inside the kernels: dt = clamp(softplus(dt_raw +
    dt_bias), dt_min, dt_max) per token and head (softplus=False skips the softplus)."""
    device = x.device
    if device.type != "cuda":
        raise ValueError("ssd_forward_dt takes CUDA tensors")
    y, final_state = _prepare(x, dt_raw, A, B, C, D, init_state, cu_seqlens, y, final_state, return_final, device)
    _check("dt_bias", dt_bias, device, torch.float32, (x.shape[2],))
    pro = SsdDtPrologue(None if dt_bias is None else dt_bias.data_ptr(), int(bool(softplus)), float(dt_min),
                        float(dt_max))
    shape = make_shape(x, B, cu_seqlens)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(device):
        rc = _lib.ssd_forward_dt(ctypes.byref(shape), ctypes.byref(pro), _ptr(x), _ptr(dt_raw), _ptr(A), _ptr(B),
                                 _ptr(C), _ptr(D), _ptr(init_state), _ptr(cu_seqlens), int(chunk), _ptr(y),
                                 _ptr(final_state), ctypes.c_void_p(handle))
    if rc:
        raise SsdError(rc, "ssd_forward_dt")
    return y, final_state


def causal_conv1d_silu(xbc, weight, bias=None, cu_seqlens=None, out: Optional[torch.Tensor] = None, stream=None):
    """Depthwise causal conv1d (kernel 4) + SiLU over the channels of xbc (batch, seqlen,
    channels); weight (channels, 4) and bias (channels,) float32; the window restarts at
    every sequence (rows of a dense batch, or cu_seqlens ranges)."""
    device = xbc.device
    if device.type != "cuda":
        raise ValueError("causal_conv1d_silu takes CUDA tensors")
    if xbc.dim() != 3:
        raise ValueError("xbc must be (batch, seqlen, channels)")
    batch, T, ch = xbc.shape
    _check("xbc", xbc, device)
    _check("weight", weight, device, torch.float32, (ch, 4))
    _check("bias", bias, device, torch.float32, (ch,))
    _check("cu_seqlens", cu_seqlens, device, torch.int32)
    if out is None:
        out = torch.empty_like(xbc)
    _check("out", out, device, xbc.dtype, tuple(xbc.shape))
    nseq = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(device):
        rc = _lib.ssd_causal_conv1d_silu(batch, T, ch, _io_code(xbc.dtype), _ptr(xbc), _ptr(weight), _ptr(bias),
                                         _ptr(cu_seqlens), nseq, _ptr(out), ctypes.c_void_p(handle))
    if rc:
        raise SsdError(rc, "ssd_causal_conv1d_silu")
    return out


def gated_rmsnorm(y, z, weight, eps: float = 1e-5, out: Optional[torch.Tensor] = None, stream=None):
    """Gate first, then RMSNorm over the last dimension: g = y silu(z), out = g / rms(g) * weight."""
    device = y.device
    if device.type != "cuda":
        raise ValueError("gated_rmsnorm takes CUDA tensors")
    dim = y.shape[-1]
    tokens = y.numel() // dim if dim else 0
    _check("y", y, device)
    _check("z", z, device, y.dtype, tuple(y.shape))
    _check("weight", weight, device, torch.float32, (dim,))
    if out is None:
        out = torch.empty_like(y)
    _check("out", out, device, y.dtype, tuple(y.shape))
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(device):
        rc = _lib.ssd_gated_rmsnorm(tokens, dim, _io_code(y.dtype), _ptr(y), _ptr(z), _ptr(weight), float(eps),
                                    _ptr(out), ctypes.c_void_p(handle))
    if rc:
        raise SsdError(rc, "ssd_gated_rmsnorm")
    return out


def segment_logdecay(dt, A, stream=None):
    """lambda[h] = A[h] * sum_t dt[t, h] over a segment; dt (tokens, H) or (1, tokens, H)."""
    device = dt.device
    H = dt.shape[-1]
    tokens = dt.numel() // H
    _check("dt", dt, device, torch.float32)
    _check("A", A, device, torch.float32, (H,))
    out = torch.empty(H, dtype=torch.float32, device=device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(device):
        rc = _lib.ssd_segment_logdecay(tokens, H, _ptr(dt), _ptr(A), _ptr(out), ctypes.c_void_p(handle))
    if rc:
        raise SsdError(rc, "ssd_segment_logdecay")
    return out


def state_prefix(rank: int, states, logdecay, init_state=None, stream=None):
    """Start state of segment ``rank`` from the preceding segments' zero-start end states
    (>= rank, H, P, N) and log-decays (>= rank, H): h_{q+1} = exp(lambda_q) h_q + s_q."""
    device = states.device
    _, H, P, N = states.shape
    _check("states", states, device, torch.float32)
    _check("logdecay", logdecay, device, torch.float32)
    _check("init_state", init_state, device, torch.float32, (H, P, N))
    if states.shape[0] < rank or logdecay.shape[0] < rank or logdecay.shape[1] != H:
        raise ValueError("states and logdecay must cover the preceding segments")
    out = torch.empty((H, P, N), dtype=torch.float32, device=device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(device):
        rc = _lib.ssd_state_prefix(int(rank), H, P, N, _ptr(states), _ptr(logdecay), _ptr(init_state), _ptr(out),
                                   ctypes.c_void_p(handle))
    if rc:
        raise SsdError(rc, "ssd_state_prefix")
    return out


def ssd_decode_step(x, dt, A, B, C, D, state, y: Optional[torch.Tensor] = None, stream=None):
    """One recurrent generation step for a batch of sequences, state updated in place.

    x (batch, H, P) and B, C (batch, G, N) in float32 or bfloat16; dt (batch, H), A and D (H,)
    float32 (D may be None); state (batch, H, P, N) float32 on the same device.  Returns y
    (batch, H, P) in x's dtype.
    """
    device = x.device
    if device.type != "cuda":
        raise ValueError("ssd_decode_step takes CUDA tensors")
    if x.dim() != 3 or B.dim() != 3:
        raise ValueError("x must be (batch, H, P) and B, C (batch, G, N)")
    batch, H, P = x.shape
    G, N = B.shape[1], B.shape[2]
    _check("x", x, device)
    _check("dt", dt, device, torch.float32, (batch, H))
    _check("A", A, device, torch.float32, (H,))
    _check("B", B, device, x.dtype, (batch, G, N))
    _check("C", C, device, x.dtype, (batch, G, N))
    _check("D", D, device, torch.float32, (H,))
    _check("state", state, device, torch.float32, (batch, H, P, N))
    if y is None:
        y = torch.empty_like(x)
    _check("y", y, device, x.dtype, (batch, H, P))
    shape = SsdShape(batch, 1, H, P, N, G, 0, _io_code(x.dtype), None)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    with torch.cuda.device(device):
        rc = _lib.ssd_decode_step(ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                  _ptr(state), _ptr(y), ctypes.c_void_p(handle))
    if rc:
        raise SsdError(rc, "ssd_decode_step")
    return y


def ssd_forward_host(x, dt, A, B, C, D=None, init_state=None, cu_seqlens=None, chunk: int = 256, y=None,
                     final_state=None, return_final: bool = True, stream=None):
    """The same on host (CPU, ideally pinned) tensors: the library copies in, runs and copies out,
    and returns after synchronising.  Runs on the current CUDA device."""
    device = torch.device("cpu")
    if x.device.type != "cpu":
        raise ValueError("ssd_forward_host takes host tensors")
    y, final_state = _prepare(x, dt, A, B, C, D, init_state, cu_seqlens, y, final_state, return_final, device)
    shape = make_shape(x, B, cu_seqlens)
    if stream is None:
        stream = torch.cuda.current_stream()
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    rc = _lib.ssd_forward_host(ctypes.byref(shape), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                               _ptr(init_state), _ptr(cu_seqlens), int(chunk), _ptr(y), _ptr(final_state),
                               ctypes.c_void_p(handle))
    if rc:
        raise SsdError(rc, "ssd_forward_host")
    return y, final_state


def query_status(stream=None) -> int:
    """Synchronise ``stream`` and return (and clear) the device status word as an ssd_status."""
    if stream is None:
        stream = torch.cuda.current_stream()
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return _lib.ssd_query_status(ctypes.c_void_p(handle))


def set_path(path: int) -> int:
    """Force the kernel path (PATH_AUTO, PATH_SIMT or PATH_TC); returns the previous one."""
    rc = _lib.ssd_set_path(int(path))
    if rc < 0:
        raise SsdError(-rc, "ssd_set_path")
    return rc


def select_path(shape: SsdShape, chunk: int) -> int:
    return _lib.ssd_select_path(ctypes.byref(shape), int(chunk))


def workspace_bytes(shape: SsdShape, chunk: int) -> int:
    return int(_lib.ssd_workspace_bytes(ctypes.byref(shape), int(chunk)))


def profile_dominant(start=None, stop=None) -> None:
    """Have later ssd_forward calls record torch.cuda.Event ``start``/``stop`` around their
    dominant kernel (both None: off)."""
    h = lambda e: None if e is None else ctypes.c_void_p(e.cuda_event)
    _lib.ssd_profile_dominant(h(start), h(stop))


def kernel_launch_count() -> int:
    """Kernels launched by the library so far in this process."""
    return int(_lib.ssd_kernel_launch_count())


def set_test_hooks(wait_limit_cycles: int = 0, withhold_carry: bool = False, withhold_split: bool = False) -> None:
    """Test hooks of the tensor-core kernel's failure path: the cycle limit of every
    device-side wait (0 = the default, about 2 s), whether CTAs withhold the flag that
    hands their state on (so that the CTAs waiting for it time out) and whether CTA 0
    withholds its flag of the barrier after the work split's tile weights (so that every
    CTA's wait there times out).  Defaults restore normal operation."""
    bits = (1 if withhold_carry else 0) | (2 if withhold_split else 0)
    rc = _lib.ssd_set_test_hooks(int(wait_limit_cycles), bits)
    if rc:
        raise SsdError(rc, "ssd_set_test_hooks")
