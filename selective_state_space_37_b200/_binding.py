"""ctypes binding of libselscan (the C ABI declared in include/selscan.h).

Argument marshalling only: every step of the scan runs in the library's CUDA
kernels.  PyTorch supplies device memory (tensors, the cached workspace) and
the current stream.  There is no CPU fallback: if the library is missing or a
call fails, an exception is raised.
"""
import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# SELSCAN_LIB selects another build of the same library (e.g. one compiled
# with different tuning macros); default: the in-tree build.
LIB_PATH = os.environ.get("SELSCAN_LIB") or os.path.join(_HERE, "csrc", "libselscan.so")

SS_OK = 0
SS_ERR_INVALID_ARG = -1
SS_ERR_UNSUPPORTED = -2
SS_ERR_CUDA = -3
SS_ERR_TIMEOUT = -4
SS_ERR_WORKSPACE = -5

SS_BF16 = 1 << 0
SS_DELTA_SOFTPLUS = 1 << 1
SS_SYNC_CHECK = 1 << 2
SS_FORCE_GENERAL_A = 1 << 3
SS_TEST_DROP_CARRY = 1 << 30

D_STATE = 16

# Every symbol include/selscan.h declares.
EXPORTED = ("ss_fwd", "ss_step", "ss_fwd_workspace_bytes", "ss_fwd_chunk_len", "ss_check",
            "ss_status_string", "ss_version", "ss_fwd_noalloc", "ss_bwd", "ss_bwd_workspace_bytes",
            "ss_fwd_conv", "ss_step_conv", "ss_block_fwd", "ss_block_scratch_bytes", "ss_ssd_fwd",
            "ss_fwd_host", "ss_fwd_host_workspace_bytes", "ss_ssd_fwd_workspace_bytes", "ss_fwd_with_state")


class ss_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("d_inner", ctypes.c_int64), ("d_state", ctypes.c_int64)]


class ss_launch(ctypes.Structure):
    _fields_ = [("stream", ctypes.c_void_p), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t), ("timeout_iters", ctypes.c_uint32),
                ("chunk_len", ctypes.c_int32)]


class ss_block_weights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in ("in_proj_x", "in_proj_z", "conv_w", "conv_b", "x_proj_dt",
                                                "x_proj_B", "x_proj_C", "dt_proj", "dt_bias", "A", "D",
                                                "out_proj")] + \
               [("d_model", ctypes.c_int64), ("d_inner", ctypes.c_int64), ("dt_rank", ctypes.c_int64)]


BLOCK_WEIGHT_SHAPES = {   # name: (shape as a function of (d_model, d_inner, dt_rank), dtype tag)
    "in_proj_x": (lambda m, i, r: (i, m), "bf16"), "in_proj_z": (lambda m, i, r: (i, m), "bf16"),
    "conv_w": (lambda m, i, r: (i, 4), "f32"), "conv_b": (lambda m, i, r: (i,), "f32"),
    "x_proj_dt": (lambda m, i, r: (r, i), "bf16"), "x_proj_B": (lambda m, i, r: (D_STATE, i), "bf16"),
    "x_proj_C": (lambda m, i, r: (D_STATE, i), "bf16"), "dt_proj": (lambda m, i, r: (i, r), "bf16"),
    "dt_bias": (lambda m, i, r: (i,), "f32"), "A": (lambda m, i, r: (i, D_STATE), "f32"),
    "D": (lambda m, i, r: (i,), "f32"), "out_proj": (lambda m, i, r: (m, i), "bf16"),
}


class ss_ssd_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64), ("nheads", ctypes.c_int64),
                ("headdim", ctypes.c_int64), ("d_state", ctypes.c_int64)]


class SelscanError(RuntimeError):
    def __init__(self, status, what):
        self.status = status
        super().__init__(f"{what}: {status_string(status)} ({status})")


_lib = None
_lock = threading.Lock()


def lib():
    """The loaded library with argument types set (raises if not built)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(
                f"libselscan.so not found at {LIB_PATH}; build it with "
                "`python -m selective_state_space_37_b200.csrc.build`")
        L = ctypes.CDLL(LIB_PATH)
        vp, f32p = ctypes.c_void_p, ctypes.c_void_p
        L.ss_fwd.argtypes = [vp, vp, f32p, f32p, vp, vp, f32p, vp, vp, f32p, ctypes.c_uint32,
                             ctypes.POINTER(ss_dims), ctypes.POINTER(ss_launch)]
        L.ss_fwd.restype = ctypes.c_int
        L.ss_step.argtypes = [f32p, vp, vp, f32p, vp, vp, f32p, vp, vp, f32p, ctypes.c_uint32,
                              ctypes.POINTER(ss_dims), ctypes.POINTER(ss_launch)]
        L.ss_step.restype = ctypes.c_int
        L.ss_fwd_workspace_bytes.argtypes = [ctypes.POINTER(ss_dims), ctypes.c_uint32, ctypes.c_int32]
        L.ss_fwd_workspace_bytes.restype = ctypes.c_size_t
        L.ss_fwd_with_state.argtypes = [vp, vp, f32p, f32p, vp, vp, f32p, vp, f32p, vp, f32p, ctypes.c_uint32,
                                        ctypes.POINTER(ss_dims), ctypes.POINTER(ss_launch)]
        L.ss_fwd_with_state.restype = ctypes.c_int
        L.ss_fwd_host.argtypes = [vp, vp, f32p, f32p, vp, vp, f32p, vp, vp, f32p, ctypes.c_uint32,
                                  ctypes.POINTER(ss_dims), ctypes.POINTER(ss_launch), ctypes.c_int32]
        L.ss_fwd_host.restype = ctypes.c_int
        L.ss_fwd_host_workspace_bytes.argtypes = [ctypes.POINTER(ss_dims), ctypes.c_uint32, ctypes.c_int32]
        L.ss_fwd_host_workspace_bytes.restype = ctypes.c_size_t
        L.ss_fwd_chunk_len.argtypes = [ctypes.POINTER(ss_dims), ctypes.c_uint32]
        L.ss_fwd_chunk_len.restype = ctypes.c_int32
        L.ss_check.argtypes = [ctypes.POINTER(ss_launch)]
        L.ss_check.restype = ctypes.c_int
        L.ss_status_string.argtypes = [ctypes.c_int]
        L.ss_status_string.restype = ctypes.c_char_p
        L.ss_version.argtypes = []
        L.ss_version.restype = ctypes.c_int
        L.ss_fwd_noalloc.argtypes = [vp, vp, f32p, f32p, vp, vp, f32p, vp, vp, f32p, ctypes.c_uint32,
                                     ctypes.POINTER(ss_dims), vp]
        L.ss_fwd_noalloc.restype = ctypes.c_int
        L.ss_bwd.argtypes = [vp, vp, f32p, f32p, vp, vp, f32p, vp, vp, f32p, vp, vp, f32p, f32p, f32p,
                             f32p, vp, f32p, ctypes.c_uint32, ctypes.POINTER(ss_dims),
                             ctypes.POINTER(ss_launch)]
        L.ss_bwd.restype = ctypes.c_int
        L.ss_bwd_workspace_bytes.argtypes = [ctypes.POINTER(ss_dims), ctypes.c_uint32]
        L.ss_bwd_workspace_bytes.restype = ctypes.c_size_t
        L.ss_fwd_conv.argtypes = [vp, f32p, f32p, vp, f32p, f32p, vp, vp, f32p, vp, vp, f32p, f32p,
                                  ctypes.c_uint32, ctypes.POINTER(ss_dims), ctypes.POINTER(ss_launch)]
        L.ss_fwd_conv.restype = ctypes.c_int
        L.ss_step_conv.argtypes = [f32p, f32p, vp, f32p, f32p, vp, f32p, vp, vp, f32p, vp, vp, f32p,
                                   ctypes.c_uint32, ctypes.POINTER(ss_dims), ctypes.POINTER(ss_launch)]
        L.ss_step_conv.restype = ctypes.c_int
        L.ss_block_fwd.argtypes = [vp, vp, ctypes.POINTER(ss_block_weights), ctypes.c_int64, ctypes.c_int64,
                                   vp, ctypes.c_size_t, vp]
        L.ss_block_fwd.restype = ctypes.c_int
        L.ss_block_scratch_bytes.argtypes = [ctypes.POINTER(ss_block_weights), ctypes.c_int64, ctypes.c_int64]
        L.ss_block_scratch_bytes.restype = ctypes.c_size_t
        L.ss_ssd_fwd.argtypes = [vp, vp, f32p, f32p, vp, vp, f32p, vp, f32p, ctypes.c_uint32,
                                 ctypes.POINTER(ss_ssd_dims), ctypes.POINTER(ss_launch)]
        L.ss_ssd_fwd.restype = ctypes.c_int
        L.ss_ssd_fwd_workspace_bytes.argtypes = [ctypes.POINTER(ss_ssd_dims), ctypes.c_uint32]
        L.ss_ssd_fwd_workspace_bytes.restype = ctypes.c_size_t
        _lib = L
    return _lib


def status_string(status: int) -> str:
    return lib().ss_status_string(int(status)).decode()


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _io_flag(t):
    if t.dtype == torch.bfloat16:
        return SS_BF16
    if t.dtype == torch.float32:
        return 0
    raise TypeError(f"u/delta/z/B/C must be bfloat16 or float32, got {t.dtype}")


def _check(t, name, shape, dtype, device):
    if t is None:
        return
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_ws_cache = {}


def workspace_for(nbytes, device, stream_handle):
    """A cached device workspace of at least nbytes for (device, stream).

    One buffer per (device, stream), grown when a call needs more; calls on
    one stream run in order, so they can share it.  A replaced buffer is
    returned to torch's stream-ordered allocator.  clear_workspaces() drops
    them all."""
    key = (device.index, int(stream_handle))
    ws = _ws_cache.get(key)
    if ws is None or ws.numel() < nbytes:
        ws = torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)
        _ws_cache[key] = ws
    return ws


def clear_workspaces():
    """Releases the cached workspaces (call after synchronizing the streams
    that used them)."""
    _ws_cache.clear()


def _stream_handle(stream, device):
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return stream.cuda_stream


def fwd_workspace_bytes(batch, seqlen, d_inner, bf16=True, chunk_len=0, d_state=D_STATE):
    dims = ss_dims(batch, seqlen, d_inner, d_state)
    return int(lib().ss_fwd_workspace_bytes(ctypes.byref(dims), SS_BF16 if bf16 else 0, int(chunk_len)))


def fwd_chunk_len(batch, seqlen, d_inner, bf16=True, d_state=D_STATE):
    dims = ss_dims(batch, seqlen, d_inner, d_state)
    return int(lib().ss_fwd_chunk_len(ctypes.byref(dims), SS_BF16 if bf16 else 0))


def ss_fwd(u, delta, A, B, C, D=None, z=None, delta_bias=None, *, y=None, last_state=None,
           return_last_state=True, softplus=True, force_general_A=False, chunk_len=0,
           timeout_iters=0, workspace=None, stream=None, sync_check=False, extra_flags=0,
           initial_state=None):
    """Selective-scan forward pass through libselscan's ss_fwd (or
    ss_fwd_with_state when initial_state [batch, d_inner, 16] fp32 is given).

    u, delta, z: [batch, L, d_inner]; B, C: [batch, L, 16] (bf16 or fp32, all the
    same); A: [d_inner, 16] fp32; D, delta_bias: [d_inner] fp32 or None.
    Returns (y, last_state); last_state is None when return_last_state is False
    and none was passed in.
    """
    if u.dim() != 3:
        raise ValueError("u must be [batch, L, d_inner]")
    batch, L, d = u.shape
    dev = u.device
    if dev.type != "cuda":
        raise ValueError("ss_fwd runs on CUDA tensors only")
    io = u.dtype
    for t, nm, shp in ((u, "u", (batch, L, d)), (delta, "delta", (batch, L, d)),
                       (z, "z", (batch, L, d)), (B, "B", (batch, L, D_STATE)),
                       (C, "C", (batch, L, D_STATE))):
        _check(t, nm, shp, io, dev)
    _check(A, "A", (d, D_STATE), torch.float32, dev)
    _check(D, "D", (d,), torch.float32, dev)
    _check(delta_bias, "delta_bias", (d,), torch.float32, dev)
    if y is None:
        y = torch.empty((batch, L, d), dtype=io, device=dev)
    _check(y, "y", (batch, L, d), io, dev)
    if last_state is None and return_last_state:
        last_state = torch.empty((batch, d, D_STATE), dtype=torch.float32, device=dev)
    _check(last_state, "last_state", (batch, d, D_STATE), torch.float32, dev)
    flags = _io_flag(u) | (SS_DELTA_SOFTPLUS if softplus else 0) | int(extra_flags)
    if force_general_A:
        flags |= SS_FORCE_GENERAL_A
    if sync_check:
        flags |= SS_SYNC_CHECK
    sh = _stream_handle(stream, dev)
    dims = ss_dims(batch, L, d, D_STATE)
    need = int(lib().ss_fwd_workspace_bytes(ctypes.byref(dims), flags, int(chunk_len)))
    if workspace is None:
        workspace = workspace_for(need, dev, sh)
    launch = ss_launch(sh, workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                       int(timeout_iters), int(chunk_len))
    if initial_state is not None:
        _check(initial_state, "initial_state", (batch, d, D_STATE), torch.float32, dev)
        rc = lib().ss_fwd_with_state(_ptr(u), _ptr(delta), _ptr(delta_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                     _ptr(z), _ptr(initial_state), _ptr(y), _ptr(last_state), flags,
                                     ctypes.byref(dims), ctypes.byref(launch))
    else:
        rc = lib().ss_fwd(_ptr(u), _ptr(delta), _ptr(delta_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                          _ptr(z), _ptr(y), _ptr(last_state), flags, ctypes.byref(dims),
                          ctypes.byref(launch))
    if rc != SS_OK:
        raise SelscanError(rc, "ss_fwd")
    return y, last_state


def ss_fwd_host(u, delta, A, B, C, D=None, z=None, delta_bias=None, *, y=None, last_state=None,
                return_last_state=True, softplus=True, rows_per_slice=1, workspace=None, stream=None,
                sync_check=False):
    """ss_fwd on activations in host memory through libselscan's ss_fwd_host.

    u, delta, z, B, C (and y, last_state if given) are CPU tensors -- pinned
    for overlapped copies -- with ss_fwd's shapes; A, D, delta_bias are CUDA
    tensors on the device that runs the scan.  Batch slices of rows_per_slice
    rows are uploaded, scanned and downloaded with the three overlapped.
    Returns (y, last_state) as CPU tensors, complete once the stream is
    synchronized (sync_check=True does it).
    """
    if u.dim() != 3:
        raise ValueError("u must be [batch, L, d_inner]")
    batch, L, d = u.shape
    host = torch.device("cpu")
    dev = A.device
    if dev.type != "cuda":
        raise ValueError("A, D and delta_bias must be CUDA tensors")
    io = u.dtype
    for t, nm, shp in ((u, "u", (batch, L, d)), (delta, "delta", (batch, L, d)),
                       (z, "z", (batch, L, d)), (B, "B", (batch, L, D_STATE)),
                       (C, "C", (batch, L, D_STATE))):
        _check(t, nm, shp, io, host)
    _check(A, "A", (d, D_STATE), torch.float32, dev)
    _check(D, "D", (d,), torch.float32, dev)
    _check(delta_bias, "delta_bias", (d,), torch.float32, dev)
    pin = u.is_pinned()
    if y is None:
        y = torch.empty((batch, L, d), dtype=io, pin_memory=pin)
    _check(y, "y", (batch, L, d), io, host)
    if last_state is None and return_last_state:
        last_state = torch.empty((batch, d, D_STATE), dtype=torch.float32, pin_memory=pin)
    _check(last_state, "last_state", (batch, d, D_STATE), torch.float32, host)
    flags = _io_flag(u) | (SS_DELTA_SOFTPLUS if softplus else 0) | (SS_SYNC_CHECK if sync_check else 0)
    sh = _stream_handle(stream, dev)
    dims = ss_dims(batch, L, d, D_STATE)
    need = int(lib().ss_fwd_host_workspace_bytes(ctypes.byref(dims), flags, int(rows_per_slice)))
    if workspace is None:
        workspace = workspace_for(need, dev, sh)
    launch = ss_launch(sh, workspace.data_ptr(), workspace.numel() * workspace.element_size(), 0, 0)
    rc = lib().ss_fwd_host(_ptr(u), _ptr(delta), _ptr(delta_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                           _ptr(z), _ptr(y), _ptr(last_state), flags, ctypes.byref(dims),
                           ctypes.byref(launch), int(rows_per_slice))
    if rc != SS_OK:
        raise SelscanError(rc, "ss_fwd_host")
    return y, last_state


def fwd_host_workspace_bytes(batch, seqlen, d_inner, bf16=True, rows_per_slice=1, d_state=D_STATE):
    dims = ss_dims(batch, seqlen, d_inner, d_state)
    return int(lib().ss_fwd_host_workspace_bytes(ctypes.byref(dims), SS_BF16 if bf16 else 0, int(rows_per_slice)))


def bwd_workspace_bytes(batch, seqlen, d_inner, bf16=True, d_state=D_STATE):
    dims = ss_dims(batch, seqlen, d_inner, d_state)
    return int(lib().ss_bwd_workspace_bytes(ctypes.byref(dims), SS_BF16 if bf16 else 0))


def ss_bwd(u, delta, A, B, C, dy, D=None, z=None, delta_bias=None, dlast_state=None, *,
           softplus=True, grads=None, chunk_len=0, workspace=None, stream=None, sync_check=False):
    """Backward of ss_fwd through libselscan's ss_bwd.

    Same inputs as ss_fwd plus dy [batch, L, d_inner] (the element type of u)
    and dlast_state [batch, d_inner, 16] fp32 or None.  Returns a dict with
    du, ddelta, dz (element type of u; dz only with z), dA [d_inner, 16],
    dB, dC [batch, L, 16], dD and ddelta_bias [d_inner] (fp32; only with D /
    delta_bias).  `grads` may supply preallocated output tensors by name;
    chunk_len > 0 fixes the time-chunk length (0: the library's choice).
    """
    if u.dim() != 3:
        raise ValueError("u must be [batch, L, d_inner]")
    batch, L, d = u.shape
    dev = u.device
    if dev.type != "cuda":
        raise ValueError("ss_bwd runs on CUDA tensors only")
    io = u.dtype
    for t, nm, shp in ((u, "u", (batch, L, d)), (delta, "delta", (batch, L, d)),
                       (z, "z", (batch, L, d)), (dy, "dy", (batch, L, d)),
                       (B, "B", (batch, L, D_STATE)), (C, "C", (batch, L, D_STATE))):
        _check(t, nm, shp, io, dev)
    _check(A, "A", (d, D_STATE), torch.float32, dev)
    _check(D, "D", (d,), torch.float32, dev)
    _check(delta_bias, "delta_bias", (d,), torch.float32, dev)
    _check(dlast_state, "dlast_state", (batch, d, D_STATE), torch.float32, dev)
    g = dict(grads or {})
    shapes = {"du": ((batch, L, d), io), "ddelta": ((batch, L, d), io), "dA": ((d, D_STATE), torch.float32),
              "dB": ((batch, L, D_STATE), torch.float32), "dC": ((batch, L, D_STATE), torch.float32)}
    if z is not None:
        shapes["dz"] = ((batch, L, d), io)
    if D is not None:
        shapes["dD"] = ((d,), torch.float32)
    if delta_bias is not None:
        shapes["ddelta_bias"] = ((d,), torch.float32)
    for k, (shp, dt) in shapes.items():
        if k not in g:
            g[k] = torch.empty(shp, dtype=dt, device=dev)
        _check(g[k], k, shp, dt, dev)
    flags = _io_flag(u) | (SS_DELTA_SOFTPLUS if softplus else 0) | (SS_SYNC_CHECK if sync_check else 0)
    sh = _stream_handle(stream, dev)
    dims = ss_dims(batch, L, d, D_STATE)
    need = int(lib().ss_bwd_workspace_bytes(ctypes.byref(dims), flags))
    if workspace is None:
        workspace = workspace_for(need, dev, sh)
    launch = ss_launch(sh, workspace.data_ptr(), workspace.numel() * workspace.element_size(), 0, int(chunk_len))
    rc = lib().ss_bwd(_ptr(u), _ptr(delta), _ptr(delta_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z),
                      _ptr(dy), _ptr(dlast_state), _ptr(g["du"]), _ptr(g["ddelta"]), _ptr(g["dA"]),
                      _ptr(g["dB"]), _ptr(g["dC"]), _ptr(g.get("dD")), _ptr(g.get("dz")),
                      _ptr(g.get("ddelta_bias")), flags, ctypes.byref(dims), ctypes.byref(launch))
    if rc != SS_OK:
        raise SelscanError(rc, "ss_bwd")
    return {k: g[k] for k in shapes}


def ss_fwd_conv(x, conv_w, delta, A, B, C, D=None, z=None, delta_bias=None, conv_b=None, *, y=None,
                last_state=None, return_last_state=True, conv_state=None, softplus=True, chunk_len=0,
                timeout_iters=0, workspace=None, stream=None, sync_check=False):
    """ss_fwd with the causal conv1d (width 4) + SiLU prologue: x takes u's
    place, conv_w [d_inner, 4] fp32, conv_b [d_inner] fp32 or None.  Returns
    (y, last_state); pass conv_state [batch, d_inner, 3] fp32 to receive the
    last three x of each channel (for ss_step_conv)."""
    if x.dim() != 3:
        raise ValueError("x must be [batch, L, d_inner]")
    batch, L, d = x.shape
    dev = x.device
    io = x.dtype
    for t, nm, shp in ((x, "x", (batch, L, d)), (delta, "delta", (batch, L, d)),
                       (z, "z", (batch, L, d)), (B, "B", (batch, L, D_STATE)),
                       (C, "C", (batch, L, D_STATE))):
        _check(t, nm, shp, io, dev)
    _check(conv_w, "conv_w", (d, 4), torch.float32, dev)
    _check(conv_b, "conv_b", (d,), torch.float32, dev)
    _check(A, "A", (d, D_STATE), torch.float32, dev)
    _check(D, "D", (d,), torch.float32, dev)
    _check(delta_bias, "delta_bias", (d,), torch.float32, dev)
    _check(conv_state, "conv_state", (batch, d, 3), torch.float32, dev)
    if y is None:
        y = torch.empty((batch, L, d), dtype=io, device=dev)
    _check(y, "y", (batch, L, d), io, dev)
    if last_state is None and return_last_state:
        last_state = torch.empty((batch, d, D_STATE), dtype=torch.float32, device=dev)
    _check(last_state, "last_state", (batch, d, D_STATE), torch.float32, dev)
    flags = _io_flag(x) | (SS_DELTA_SOFTPLUS if softplus else 0) | (SS_SYNC_CHECK if sync_check else 0)
    sh = _stream_handle(stream, dev)
    dims = ss_dims(batch, L, d, D_STATE)
    need = int(lib().ss_fwd_workspace_bytes(ctypes.byref(dims), flags, int(chunk_len)))
    if workspace is None:
        workspace = workspace_for(need, dev, sh)
    launch = ss_launch(sh, workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                       int(timeout_iters), int(chunk_len))
    rc = lib().ss_fwd_conv(_ptr(x), _ptr(conv_w), _ptr(conv_b), _ptr(delta), _ptr(delta_bias), _ptr(A),
                           _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(y), _ptr(last_state), _ptr(conv_state),
                           flags, ctypes.byref(dims), ctypes.byref(launch))
    if rc != SS_OK:
        raise SelscanError(rc, "ss_fwd_conv")
    return y, last_state


def ss_step_conv(state, conv_state, x, conv_w, delta, A, B, C, D=None, z=None, delta_bias=None, conv_b=None,
                 *, y=None, softplus=True, stream=None, sync_check=False):
    """One decode step with the conv prologue; state [batch, d_inner, 16] and
    conv_state [batch, d_inner, 3] (fp32) are updated in place.  Returns y."""
    batch, d = x.shape
    dev = x.device
    io = x.dtype
    _check(state, "state", (batch, d, D_STATE), torch.float32, dev)
    _check(conv_state, "conv_state", (batch, d, 3), torch.float32, dev)
    for t, nm, shp in ((x, "x", (batch, d)), (delta, "delta", (batch, d)), (z, "z", (batch, d)),
                       (B, "B", (batch, D_STATE)), (C, "C", (batch, D_STATE))):
        _check(t, nm, shp, io, dev)
    _check(conv_w, "conv_w", (d, 4), torch.float32, dev)
    _check(conv_b, "conv_b", (d,), torch.float32, dev)
    _check(A, "A", (d, D_STATE), torch.float32, dev)
    _check(D, "D", (d,), torch.float32, dev)
    _check(delta_bias, "delta_bias", (d,), torch.float32, dev)
    if y is None:
        y = torch.empty((batch, d), dtype=io, device=dev)
    flags = _io_flag(x) | (SS_DELTA_SOFTPLUS if softplus else 0) | (SS_SYNC_CHECK if sync_check else 0)
    sh = _stream_handle(stream, dev)
    dims = ss_dims(batch, 1, d, D_STATE)
    launch = ss_launch(sh, None, 0, 0, 0)
    rc = lib().ss_step_conv(_ptr(state), _ptr(conv_state), _ptr(x), _ptr(conv_w), _ptr(conv_b), _ptr(delta),
                            _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(z), _ptr(y), _ptr(delta_bias), flags,
                            ctypes.byref(dims), ctypes.byref(launch))
    if rc != SS_OK:
        raise SelscanError(rc, "ss_step_conv")
    return y


def _block_struct(weights, device):
    d_inner, d_model = weights["in_proj_x"].shape
    dt_rank = weights["x_proj_dt"].shape[0]
    st = ss_block_weights()
    for name, (shape_fn, tag) in BLOCK_WEIGHT_SHAPES.items():
        t = weights.get(name)
        if t is None and name in ("conv_b", "D"):
            continue
        _check(t, name, shape_fn(d_model, d_inner, dt_rank), torch.bfloat16 if tag == "bf16" else torch.float32,
               device)
        setattr(st, name, t.data_ptr())
    st.d_model, st.d_inner, st.dt_rank = d_model, d_inner, dt_rank
    return st


def block_scratch_bytes(weights, batch, seqlen):
    st = _block_struct(weights, weights["in_proj_x"].device)
    return int(lib().ss_block_scratch_bytes(ctypes.byref(st), batch, seqlen))


def ss_block_fwd(hidden, weights, *, out=None, scratch=None, stream=None):
    """Forward of one Mamba block's inner path through libselscan's
    ss_block_fwd.  hidden [batch, L, d_model] bf16; weights: a dict of
    tensors named as the fields of ss_block_weights (bf16 matrices, fp32
    vectors).  Returns out [batch, L, d_model] bf16."""
    batch, L, d_model = hidden.shape
    dev = hidden.device
    st = _block_struct(weights, dev)
    if st.d_model != d_model:
        raise ValueError("hidden's last dimension must equal d_model")
    _check(hidden, "hidden", (batch, L, d_model), torch.bfloat16, dev)
    if out is None:
        out = torch.empty_like(hidden)
    _check(out, "out", (batch, L, d_model), torch.bfloat16, dev)
    sh = _stream_handle(stream, dev)
    need = int(lib().ss_block_scratch_bytes(ctypes.byref(st), batch, L))
    if need == 0:
        raise SelscanError(SS_ERR_INVALID_ARG, "ss_block_fwd")
    if scratch is None:
        scratch = workspace_for(need, dev, sh)
    rc = lib().ss_block_fwd(_ptr(hidden), _ptr(out), ctypes.byref(st), batch, L, scratch.data_ptr(),
                            scratch.numel() * scratch.element_size(), sh)
    if rc != SS_OK:
        raise SelscanError(rc, "ss_block_fwd")
    return out


def ss_ssd_fwd(x, dt, A, B, C, D=None, dt_bias=None, *, softplus=True, y=None, final_state=None,
               return_final_state=True, chunk_len=0, split=True, workspace=None, stream=None, sync_check=False,
               timeout_iters=0, extra_flags=0):
    """Multi-head scan with a scalar decay per head (Mamba-2's SSD model).
    x [batch, L, nheads, 64] bf16; dt [batch, L, nheads] bf16; A [nheads] fp32;
    B, C [batch, L, d_state] bf16 (d_state 64 or 128); D, dt_bias [nheads] fp32
    or None.  Returns (y [batch, L, nheads, 64] bf16, final_state
    [batch, nheads, 64, d_state] fp32 or None).  split=False runs every
    sequence whole (no workspace); chunk_len > 0 fixes the segment length;
    timeout_iters bounds one wait in microseconds (0: two
    seconds); extra_flags adds raw SS_* flags (SS_TEST_DROP_CARRY in tests)."""
    batch, L, H, P = x.shape
    N = B.shape[-1]
    dev = x.device
    bf = torch.bfloat16
    _check(x, "x", (batch, L, H, P), bf, dev)
    _check(dt, "dt", (batch, L, H), bf, dev)
    _check(B, "B", (batch, L, N), bf, dev)
    _check(C, "C", (batch, L, N), bf, dev)
    _check(A, "A", (H,), torch.float32, dev)
    _check(D, "D", (H,), torch.float32, dev)
    _check(dt_bias, "dt_bias", (H,), torch.float32, dev)
    if y is None:
        y = torch.empty_like(x)
    _check(y, "y", (batch, L, H, P), bf, dev)
    if final_state is None and return_final_state:
        final_state = torch.empty((batch, H, P, N), dtype=torch.float32, device=dev)
    _check(final_state, "final_state", (batch, H, P, N), torch.float32, dev)
    flags = (SS_DELTA_SOFTPLUS if softplus else 0) | (SS_SYNC_CHECK if sync_check else 0) | int(extra_flags)
    dims = ss_ssd_dims(batch, L, H, P, N)
    sh = _stream_handle(stream, dev)
    if split:
        if workspace is None:
            workspace = workspace_for(int(lib().ss_ssd_fwd_workspace_bytes(ctypes.byref(dims), flags)), dev, sh)
        launch = ss_launch(sh, workspace.data_ptr(), workspace.numel() * workspace.element_size(),
                           int(timeout_iters), int(chunk_len))
    else:
        launch = ss_launch(sh, None, 0, int(timeout_iters), int(chunk_len))
    rc = lib().ss_ssd_fwd(_ptr(x), _ptr(dt), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(y),
                          _ptr(final_state), flags, ctypes.byref(dims), ctypes.byref(launch))
    if rc != SS_OK:
        raise SelscanError(rc, "ss_ssd_fwd")
    return y, final_state


def ss_check(workspace, stream=None, device=None):
    """Synchronize and return the device status recorded in `workspace`."""
    dev = workspace.device if device is None else device
    sh = _stream_handle(stream, dev)
    launch = ss_launch(sh, workspace.data_ptr(), workspace.numel() * workspace.element_size(), 0, 0)
    return int(lib().ss_check(ctypes.byref(launch)))


def ss_step(state, u, delta, A, B, C, D=None, z=None, delta_bias=None, *, y=None, softplus=True,
            stream=None, sync_check=False):
    """One decode step through libselscan's ss_step; `state` is updated in place.

    state: [batch, d_inner, 16] fp32; u, delta, z: [batch, d_inner]; B, C: [batch, 16]
    (bf16 or fp32); A: [d_inner, 16] fp32; D, delta_bias: [d_inner] fp32 or None.
    Returns y [batch, d_inner].
    """
    if state.dim() != 3:
        raise ValueError("state must be [batch, d_inner, 16]")
    batch, d, _ = state.shape
    dev = state.device
    if dev.type != "cuda":
        raise ValueError("ss_step runs on CUDA tensors only")
    io = u.dtype
    _check(state, "state", (batch, d, D_STATE), torch.float32, dev)
    for t, nm, shp in ((u, "u", (batch, d)), (delta, "delta", (batch, d)), (z, "z", (batch, d)),
                       (B, "B", (batch, D_STATE)), (C, "C", (batch, D_STATE))):
        _check(t, nm, shp, io, dev)
    _check(A, "A", (d, D_STATE), torch.float32, dev)
    _check(D, "D", (d,), torch.float32, dev)
    _check(delta_bias, "delta_bias", (d,), torch.float32, dev)
    if y is None:
        y = torch.empty((batch, d), dtype=io, device=dev)
    _check(y, "y", (batch, d), io, dev)
    flags = _io_flag(u) | (SS_DELTA_SOFTPLUS if softplus else 0) | (SS_SYNC_CHECK if sync_check else 0)
    sh = _stream_handle(stream, dev)
    dims = ss_dims(batch, 1, d, D_STATE)
    launch = ss_launch(sh, None, 0, 0, 0)
    rc = lib().ss_step(_ptr(state), _ptr(u), _ptr(delta), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                       _ptr(z), _ptr(y), _ptr(delta_bias), flags, ctypes.byref(dims),
                       ctypes.byref(launch))
    if rc != SS_OK:
        raise SelscanError(rc, "ss_step")
    return y
