"""Python binding of libssd (argument marshalling only).

Every step of the SSD path runs in the CUDA kernels of ``libssd.so``; this module
checks shapes and dtypes, passes ``data_ptr()`` values and the current CUDA stream
through the C ABI declared in ``include/ssd.h``, and turns non-OK statuses into
exceptions. There is no fallback: if the library is missing, importing this
module raises.

Functions mirror the C entry points:
  scan_fwd(x, dt_raw, dt_bias, A, B, C, D, init_state=None, cu_seqlens=None,
           chunk=128, y=None, final_state=None, workspace=None)
  state_update(state, x, dt_raw, dt_bias, A, B, C, D, y=None)
  ChunkCache.empty(...), strict_scan_fwd(...), strict_state_update(...)  (strict mode)
  device_status(), scan_variant(...), workspace_size(...), last_launch_count()
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libssd.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m mamba_ssd_state_02_b200.build` "
        "(nvcc, sm_100a). The SSD path has no fallback.")

_lib = ctypes.CDLL(LIB_PATH)

SSD_OK, SSD_ERR_INVALID_ARG, SSD_ERR_UNSUPPORTED, SSD_ERR_CUDA, SSD_ERR_TIMEOUT = range(5)
SSD_DTYPE_F32, SSD_DTYPE_BF16 = 0, 1
_STATUS = {1: "SSD_ERR_INVALID_ARG", 2: "SSD_ERR_UNSUPPORTED", 3: "SSD_ERR_CUDA", 4: "SSD_ERR_TIMEOUT"}


class SSDDims(ctypes.Structure):
    """Mirror of ``ssd_dims`` (include/ssd.h)."""
    _fields_ = [
        ("batch", ctypes.c_int64),
        ("seqlen", ctypes.c_int64),
        ("nseq", ctypes.c_int32),
        ("total_tokens", ctypes.c_int64),
        ("nheads", ctypes.c_int32),
        ("headdim", ctypes.c_int32),
        ("ngroups", ctypes.c_int32),
        ("dstate", ctypes.c_int32),
        ("dtype", ctypes.c_int32),
        ("workspace", ctypes.c_void_p),
        ("workspace_bytes", ctypes.c_size_t),
    ]


_p = ctypes.c_void_p
_lib.ssd_scan_fwd_workspace_size.argtypes = [ctypes.POINTER(SSDDims), ctypes.c_int,
                                             ctypes.POINTER(ctypes.c_size_t)]
_lib.ssd_scan_fwd_workspace_size.restype = ctypes.c_int
_lib.ssd_scan_fwd.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p,
                              ctypes.POINTER(SSDDims), ctypes.c_int, _p]
_lib.ssd_scan_fwd.restype = ctypes.c_int
_lib.ssd_scan_fwd_snapshots.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p, ctypes.c_int64,
                                        ctypes.POINTER(SSDDims), ctypes.c_int, _p]
_lib.ssd_scan_fwd_snapshots.restype = ctypes.c_int
_lib.ssd_scan_fwd_snapshots_workspace_size.argtypes = [ctypes.POINTER(SSDDims), ctypes.c_int, ctypes.c_int64,
                                                       ctypes.POINTER(ctypes.c_size_t)]
_lib.ssd_scan_fwd_snapshots_workspace_size.restype = ctypes.c_int
_lib.ssd_snapshot_count.argtypes = [ctypes.POINTER(SSDDims), _p, ctypes.c_int64, ctypes.POINTER(ctypes.c_int64)]
_lib.ssd_snapshot_count.restype = ctypes.c_int
_lib.ssd_conv1d_fwd.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _p, ctypes.POINTER(SSDDims), ctypes.c_int, _p]
_lib.ssd_conv1d_fwd.restype = ctypes.c_int
_lib.ssd_conv1d_update.argtypes = [_p, _p, _p, _p, _p, _p, _p, ctypes.POINTER(SSDDims), ctypes.c_int, _p]
_lib.ssd_conv1d_update.restype = ctypes.c_int
_lib.ssd_gated_rmsnorm.argtypes = [_p, _p, _p, _p, ctypes.c_int64, ctypes.c_int, ctypes.c_int, ctypes.c_float,
                                   ctypes.c_int, _p]
_lib.ssd_gated_rmsnorm.restype = ctypes.c_int
_lib.ssd_scan_fwd_noalloc.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, _p,
                                      ctypes.POINTER(SSDDims), ctypes.c_int, _p]
_lib.ssd_scan_fwd_noalloc.restype = ctypes.c_int
_lib.ssd_state_update.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _p, ctypes.POINTER(SSDDims), _p]
_lib.ssd_state_update.restype = ctypes.c_int
_lib.ssd_get_device_status.argtypes = [_p]
_lib.ssd_get_device_status.restype = ctypes.c_int
_lib.ssd_last_error.argtypes = []
_lib.ssd_last_error.restype = ctypes.c_char_p
_lib.ssd_scan_fwd_variant.argtypes = [ctypes.POINTER(SSDDims), ctypes.c_int]
_lib.ssd_scan_fwd_variant.restype = ctypes.c_char_p
_lib.ssd_set_segment_tokens.argtypes = [ctypes.c_int]
_lib.ssd_test_stall.argtypes = [ctypes.c_int]
_lib.ssd_test_stall.restype = None

_lib.ssd_set_segment_tokens.restype = None
_lib.ssd_scan_fwd_segment_tokens.argtypes = [ctypes.POINTER(SSDDims), ctypes.c_int]
_lib.ssd_scan_fwd_segment_tokens.restype = ctypes.c_int


class SSDChunkCache(ctypes.Structure):
    """Mirror of ``ssd_chunk_cache``."""
    _fields_ = [("state", ctypes.c_void_p), ("x", ctypes.c_void_p), ("B", ctypes.c_void_p),
                ("dt", ctypes.c_void_p), ("acum", ctypes.c_void_p), ("len", ctypes.c_void_p)]


_lib.ssd_strict_scan_fwd_workspace_size.argtypes = [ctypes.POINTER(SSDDims), ctypes.c_int,
                                                    ctypes.POINTER(ctypes.c_size_t)]
_lib.ssd_strict_scan_fwd_workspace_size.restype = ctypes.c_int
_lib.ssd_strict_scan_fwd.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _p, _p, ctypes.POINTER(SSDChunkCache),
                                     ctypes.c_int, ctypes.POINTER(SSDDims), ctypes.c_int, _p]
_lib.ssd_strict_scan_fwd.restype = ctypes.c_int
_lib.ssd_strict_state_update.argtypes = [ctypes.POINTER(SSDChunkCache), _p, _p, _p, _p, _p, _p, _p, _p,
                                         ctypes.POINTER(SSDDims), ctypes.c_int, _p]
_lib.ssd_strict_state_update.restype = ctypes.c_int
_lib.ssd_last_launch_count.argtypes = []
_lib.ssd_last_launch_count.restype = ctypes.c_int


class SSDKernelTime(ctypes.Structure):
    """Mirror of ``ssd_kernel_time``."""
    _fields_ = [("name", ctypes.c_char_p), ("launches", ctypes.c_int), ("total_ms", ctypes.c_double)]


_lib.ssd_selftest_umma.argtypes = [_p, _p, _p, _p]
_lib.ssd_selftest_umma.restype = ctypes.c_int
_lib.ssd_profile_enable.argtypes = [ctypes.c_int]
_lib.ssd_profile_enable.restype = None
_lib.ssd_profile_read.argtypes = [ctypes.POINTER(SSDKernelTime), ctypes.c_int, ctypes.POINTER(ctypes.c_int)]
_lib.ssd_profile_read.restype = ctypes.c_int


class SSDError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS.get(status, status)}: {msg}")
        self.status = status


def _check(status: int) -> None:
    if status != SSD_OK:
        raise SSDError(status, _lib.ssd_last_error().decode())


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return SSD_DTYPE_BF16
    if t.dtype == torch.float32:
        return SSD_DTYPE_F32
    raise TypeError(f"x/B/C must be float32 or bfloat16, got {t.dtype}")


def _need(t, name, shape, dtype, device):
    if t is None:
        raise ValueError(f"{name} is required")
    if not t.is_cuda or t.device != device:
        raise ValueError(f"{name} must be on {device}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    if t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def make_dims(T, H, P, G, N, dtype_code, batch=None, seqlen=None, nseq=None, workspace=None):
    d = SSDDims()
    if nseq is not None:          # packed varlen
        d.batch, d.seqlen, d.nseq, d.total_tokens = 0, 0, int(nseq), int(T)
    else:
        d.batch, d.seqlen, d.nseq, d.total_tokens = int(batch), int(seqlen), 0, 0
    d.nheads, d.headdim, d.ngroups, d.dstate, d.dtype = H, P, G, N, dtype_code
    if workspace is not None:
        d.workspace, d.workspace_bytes = workspace.data_ptr(), workspace.numel() * workspace.element_size()
    return d


def workspace_size(dims: SSDDims, chunk: int) -> int:
    b = ctypes.c_size_t(0)
    _check(_lib.ssd_scan_fwd_workspace_size(ctypes.byref(dims), int(chunk), ctypes.byref(b)))
    return int(b.value)


def snapshot_workspace_size(dims: SSDDims, chunk: int, snapshot_tokens: int) -> int:
    b = ctypes.c_size_t(0)
    _check(_lib.ssd_scan_fwd_snapshots_workspace_size(ctypes.byref(dims), int(chunk), int(snapshot_tokens),
                                                      ctypes.byref(b)))
    return int(b.value)


def snapshot_count(dims: SSDDims, snapshot_tokens: int, cu_seqlens_host=None) -> int:
    """Snapshots ssd_scan_fwd_snapshots writes (cu_seqlens_host: CPU int32 tensor for varlen)."""
    n = ctypes.c_int64(0)
    cu = None
    if cu_seqlens_host is not None:
        cu = cu_seqlens_host.to(torch.int32).contiguous()
        if cu.device.type != "cpu":
            raise ValueError("cu_seqlens_host must be a CPU tensor")
    _check(_lib.ssd_snapshot_count(ctypes.byref(dims), None if cu is None else ctypes.c_void_p(cu.data_ptr()),
                                   int(snapshot_tokens), ctypes.byref(n)))
    return int(n.value)


def scan_variant(dims: SSDDims, chunk: int) -> str:
    return _lib.ssd_scan_fwd_variant(ctypes.byref(dims), int(chunk)).decode()


def set_segment_tokens(tokens: int) -> None:
    """Force the tensor-core segment length for later calls (0 restores the planner)."""
    _lib.ssd_set_segment_tokens(int(tokens))


def test_stall(pass_: int) -> None:
    """Test hook: make the UMMA warp of tensor-core pass 1 (segment states) or 2 (chunk
    scan) wait on a barrier that nothing arrives at, so that the wait runs out (0: off)."""
    _lib.ssd_test_stall(int(pass_))


def segment_tokens(dims: SSDDims, chunk: int) -> int:
    return int(_lib.ssd_scan_fwd_segment_tokens(ctypes.byref(dims), int(chunk)))


def last_launch_count() -> int:
    return int(_lib.ssd_last_launch_count())


def profile_enable(on: bool = True) -> None:
    """Start (and reset) or stop per-kernel CUDA-event timing inside the library."""
    _lib.ssd_profile_enable(1 if on else 0)


def profile_read() -> dict:
    """{kernel name: (launches, total device ms)} since enable / the last read."""
    buf = (SSDKernelTime * 32)()
    dropped = ctypes.c_int(0)
    n = _lib.ssd_profile_read(buf, 32, ctypes.byref(dropped))
    if n < 0:
        raise SSDError(SSD_ERR_CUDA, _lib.ssd_last_error().decode())
    out = {buf[i].name.decode(): (int(buf[i].launches), float(buf[i].total_ms)) for i in range(min(n, 32))}
    if dropped.value:
        out["_dropped"] = (int(dropped.value), 0.0)
    return out


def selftest_umma(X1: torch.Tensor, X2: torch.Tensor) -> torch.Tensor:
    """Run the tensor-core operand-format diagnostic on two [128,128] bf16 matrices;
    returns out [5,128,128] float32 (see ssd_selftest_umma in include/ssd.h)."""
    dev = X1.device
    for name, t in (("X1", X1), ("X2", X2)):
        _need(t, name, (128, 128), torch.bfloat16, dev)
    out = torch.empty(5, 128, 128, dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(_lib.ssd_selftest_umma(_ptr(X1), _ptr(X2), _ptr(out), _stream(dev)))
    return out


def device_status(device=None) -> None:
    """Wait for the current stream and raise if a kernel latched an error."""
    _check(_lib.ssd_get_device_status(_stream(device)))


def scan_fwd(x, dt_raw, dt_bias, A, B, C, D, init_state=None, cu_seqlens=None, chunk=128,
             y=None, final_state=None, workspace=None, batch=None, snapshot_tokens=None, snapshots=None):
    """Chunked SSD prefill.

    Dense: x [batch, L, H, P], dt_raw [batch, L, H], B/C [batch, L, G, N].
    Packed varlen (cu_seqlens int32 [nseq+1] on the device): x [T, H, P],
    dt_raw [T, H], B/C [T, G, N].
    Returns (y, final_state); final_state [nseq, H, P, N] float32.
    With snapshot_tokens (ssd_scan_fwd_snapshots) returns (y, final_state, snapshots),
    snapshots [n_snap, H, P, N] float32: each sequence's state after every multiple of
    snapshot_tokens tokens (allocated here when not given; for varlen that reads
    cu_seqlens back to the host to count them).
    """
    dev = x.device
    varlen = cu_seqlens is not None
    if varlen:
        T, H, P = x.shape
        nseq = cu_seqlens.numel() - 1
        tok = (T,)
    else:
        if x.dim() != 4:
            raise ValueError("dense x must be [batch, L, H, P]")
        bsz, L, H, P = x.shape
        nseq = bsz
        tok = (bsz, L)
    G, N = B.shape[-2], B.shape[-1]
    dt = x.dtype
    _need(x, "x", tok + (H, P), dt, dev)
    _need(dt_raw, "dt_raw", tok + (H,), torch.float32, dev)
    _need(B, "B", tok + (G, N), dt, dev)
    _need(C, "C", tok + (G, N), dt, dev)
    for name, v in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _need(v, name, (H,), torch.float32, dev)
    if init_state is not None:
        _need(init_state, "init_state", (nseq, H, P, N), torch.float32, dev)
    if varlen:
        _need(cu_seqlens, "cu_seqlens", (nseq + 1,), torch.int32, dev)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", tok + (H, P), dt, dev)
    if final_state is None:
        final_state = torch.empty(nseq, H, P, N, dtype=torch.float32, device=dev)
    _need(final_state, "final_state", (nseq, H, P, N), torch.float32, dev)
    if varlen:
        dims = make_dims(x.shape[0], H, P, G, N, _dtype_code(x), nseq=nseq, workspace=workspace)
    else:
        dims = make_dims(bsz * L, H, P, G, N, _dtype_code(x), batch=bsz, seqlen=L, workspace=workspace)
    if snapshot_tokens is not None:
        if snapshots is None:
            n_snap = snapshot_count(dims, snapshot_tokens, cu_seqlens.cpu() if varlen else None)
            snapshots = torch.empty(n_snap, H, P, N, dtype=torch.float32, device=dev)
        if snapshots.dtype != torch.float32 or snapshots.device != dev or not snapshots.is_contiguous() or \
                tuple(snapshots.shape[1:]) != (H, P, N):
            raise ValueError("snapshots must be a contiguous float32 [n_snap, H, P, N] tensor on x's device")
        with torch.cuda.device(dev):
            _check(_lib.ssd_scan_fwd_snapshots(_ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C),
                                               _ptr(D), _ptr(init_state), _ptr(cu_seqlens), _ptr(y),
                                               _ptr(final_state), _ptr(snapshots), int(snapshot_tokens),
                                               ctypes.byref(dims), int(chunk), _stream(dev)))
        return y, final_state, snapshots
    with torch.cuda.device(dev):
        _check(_lib.ssd_scan_fwd(_ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C),
                                 _ptr(D), _ptr(init_state), _ptr(cu_seqlens), _ptr(y),
                                 _ptr(final_state), ctypes.byref(dims), int(chunk), _stream(dev)))
    return y, final_state


def scan_fwd_noalloc(x, dt_raw, dt_bias, A, B, C, D, init_state=None, cu_seqlens=None, chunk=128,
                     y=None, final_state=None):
    """scan_fwd through ssd_scan_fwd_noalloc: the library's own 32 MiB scratch array, no
    device allocation inside the call (y/final_state are allocated here only when the
    caller passes none). For callers whose memory budget is fixed up front; calls that
    overlap on the GPU share the scratch and must be serialised."""
    dev = x.device
    varlen = cu_seqlens is not None
    if varlen:
        T, H, P = x.shape
        nseq = cu_seqlens.numel() - 1
        tok = (T,)
    else:
        if x.dim() != 4:
            raise ValueError("dense x must be [batch, L, H, P]")
        bsz, L, H, P = x.shape
        nseq = bsz
        tok = (bsz, L)
    G, N = B.shape[-2], B.shape[-1]
    dt = x.dtype
    _need(x, "x", tok + (H, P), dt, dev)
    _need(dt_raw, "dt_raw", tok + (H,), torch.float32, dev)
    _need(B, "B", tok + (G, N), dt, dev)
    _need(C, "C", tok + (G, N), dt, dev)
    for name, v in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _need(v, name, (H,), torch.float32, dev)
    if init_state is not None:
        _need(init_state, "init_state", (nseq, H, P, N), torch.float32, dev)
    if varlen:
        _need(cu_seqlens, "cu_seqlens", (nseq + 1,), torch.int32, dev)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", tok + (H, P), dt, dev)
    if final_state is None:
        final_state = torch.empty(nseq, H, P, N, dtype=torch.float32, device=dev)
    _need(final_state, "final_state", (nseq, H, P, N), torch.float32, dev)
    if varlen:
        dims = make_dims(x.shape[0], H, P, G, N, _dtype_code(x), nseq=nseq)
    else:
        dims = make_dims(bsz * L, H, P, G, N, _dtype_code(x), batch=bsz, seqlen=L)
    with torch.cuda.device(dev):
        _check(_lib.ssd_scan_fwd_noalloc(_ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C),
                                         _ptr(D), _ptr(init_state), _ptr(cu_seqlens), _ptr(y),
                                         _ptr(final_state), ctypes.byref(dims), int(chunk), _stream(dev)))
    return y, final_state


def state_update(state, x, dt_raw, dt_bias, A, B, C, D, y=None):
    """One decode step in place on ``state`` [nseq,H,P,N] float32.
    x [nseq,H,P], dt_raw [nseq,H], B/C [nseq,G,N]. Returns y [nseq,H,P]."""
    dev = x.device
    nseq, H, P = x.shape
    G, N = B.shape[-2], B.shape[-1]
    _need(state, "state", (nseq, H, P, N), torch.float32, dev)
    _need(x, "x", (nseq, H, P), x.dtype, dev)
    _need(dt_raw, "dt_raw", (nseq, H), torch.float32, dev)
    _need(B, "B", (nseq, G, N), x.dtype, dev)
    _need(C, "C", (nseq, G, N), x.dtype, dev)
    for name, v in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _need(v, name, (H,), torch.float32, dev)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", (nseq, H, P), x.dtype, dev)
    dims = make_dims(nseq, H, P, G, N, _dtype_code(x), batch=nseq, seqlen=1)
    with torch.cuda.device(dev):
        _check(_lib.ssd_state_update(_ptr(state), _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A),
                                     _ptr(B), _ptr(C), _ptr(D), _ptr(y), ctypes.byref(dims),
                                     _stream(dev)))
    return y


def conv1d_fwd(xbc, weight, bias, nheads, headdim, ngroups, dstate, conv_state=None, cu_seqlens=None,
               x=None, B=None, C=None, conv_state_out=None, return_state=True):
    """Causal conv1d + bias + SiLU prologue (ssd_conv1d_fwd).

    Dense: xbc [batch, L, D]; packed varlen (cu_seqlens int32 [nseq+1]): xbc [T, D],
    D = nheads*headdim + 2*ngroups*dstate. weight [D, K] float32, bias [D] float32 or
    None, conv_state [nseq, D, K-1] (xbc's dtype) or None.
    Returns (x, B, C, conv_state_out): x [..., H, P], B/C [..., G, N] in the scan's
    layouts, conv_state_out [nseq, D, K-1] (None if return_state is False)."""
    dev = xbc.device
    varlen = cu_seqlens is not None
    H, P, G, N = int(nheads), int(headdim), int(ngroups), int(dstate)
    Dc = H * P + 2 * G * N
    if varlen:
        T = xbc.shape[0]
        nseq = cu_seqlens.numel() - 1
        tok = (T,)
    else:
        if xbc.dim() != 3:
            raise ValueError("dense xbc must be [batch, L, D]")
        bsz, L = xbc.shape[0], xbc.shape[1]
        nseq = bsz
        tok = (bsz, L)
    dt = xbc.dtype
    _need(xbc, "xbc", tok + (Dc,), dt, dev)
    if weight.dim() != 2 or weight.shape[0] != Dc:
        raise ValueError(f"weight must be [D={Dc}, K]")
    K = weight.shape[1]
    _need(weight, "weight", (Dc, K), torch.float32, dev)
    if bias is not None:
        _need(bias, "bias", (Dc,), torch.float32, dev)
    if conv_state is not None:
        _need(conv_state, "conv_state", (nseq, Dc, K - 1), dt, dev)
    if varlen:
        _need(cu_seqlens, "cu_seqlens", (nseq + 1,), torch.int32, dev)
    x = torch.empty(*tok, H, P, dtype=dt, device=dev) if x is None else x
    B = torch.empty(*tok, G, N, dtype=dt, device=dev) if B is None else B
    C = torch.empty(*tok, G, N, dtype=dt, device=dev) if C is None else C
    _need(x, "x", tok + (H, P), dt, dev)
    _need(B, "B", tok + (G, N), dt, dev)
    _need(C, "C", tok + (G, N), dt, dev)
    if return_state and conv_state_out is None:
        conv_state_out = torch.empty(nseq, Dc, K - 1, dtype=dt, device=dev)
    if conv_state_out is not None:
        _need(conv_state_out, "conv_state_out", (nseq, Dc, K - 1), dt, dev)
    if varlen:
        dims = make_dims(T, H, P, G, N, _dtype_code(xbc), nseq=nseq)
    else:
        dims = make_dims(bsz * L, H, P, G, N, _dtype_code(xbc), batch=bsz, seqlen=L)
    with torch.cuda.device(dev):
        _check(_lib.ssd_conv1d_fwd(_ptr(xbc), _ptr(weight), _ptr(bias), _ptr(conv_state), _ptr(cu_seqlens),
                                   _ptr(x), _ptr(B), _ptr(C), _ptr(conv_state_out), ctypes.byref(dims), int(K),
                                   _stream(dev)))
    return x, B, C, conv_state_out


def conv1d_update(conv_state, xbc, weight, bias, nheads, headdim, ngroups, dstate, x=None, B=None, C=None):
    """One decode step of the conv1d prologue (ssd_conv1d_update): conv_state [nseq, D, K-1]
    updated in place, xbc [nseq, D]. Returns (x [nseq,H,P], B [nseq,G,N], C [nseq,G,N])."""
    dev = xbc.device
    H, P, G, N = int(nheads), int(headdim), int(ngroups), int(dstate)
    Dc = H * P + 2 * G * N
    nseq = xbc.shape[0]
    dt = xbc.dtype
    _need(xbc, "xbc", (nseq, Dc), dt, dev)
    K = weight.shape[1]
    _need(weight, "weight", (Dc, K), torch.float32, dev)
    if bias is not None:
        _need(bias, "bias", (Dc,), torch.float32, dev)
    _need(conv_state, "conv_state", (nseq, Dc, K - 1), dt, dev)
    x = torch.empty(nseq, H, P, dtype=dt, device=dev) if x is None else x
    B = torch.empty(nseq, G, N, dtype=dt, device=dev) if B is None else B
    C = torch.empty(nseq, G, N, dtype=dt, device=dev) if C is None else C
    dims = make_dims(nseq, H, P, G, N, _dtype_code(xbc), batch=nseq, seqlen=1)
    with torch.cuda.device(dev):
        _check(_lib.ssd_conv1d_update(_ptr(conv_state), _ptr(xbc), _ptr(weight), _ptr(bias), _ptr(x), _ptr(B),
                                      _ptr(C), ctypes.byref(dims), int(K), _stream(dev)))
    return x, B, C


def gated_rmsnorm(y, z, weight, group_size=512, eps=1e-6, out=None):
    """Gated group RMSNorm (ssd_gated_rmsnorm): out = rmsnorm_group(y * silu(z)) * weight.
    y, z: [..., channels] (bf16 or float32, same shape); weight [channels] float32."""
    dev = y.device
    channels = y.shape[-1]
    ntok = y.numel() // channels if channels else 0
    _need(y, "y", tuple(y.shape), y.dtype, dev)
    _need(z, "z", tuple(y.shape), y.dtype, dev)
    _need(weight, "weight", (channels,), torch.float32, dev)
    if out is None:
        out = torch.empty_like(y)
    _need(out, "out", tuple(y.shape), y.dtype, dev)
    with torch.cuda.device(dev):
        _check(_lib.ssd_gated_rmsnorm(_ptr(y), _ptr(z), _ptr(weight), _ptr(out), int(ntok), int(channels),
                                      int(group_size), float(eps), _dtype_code(y), _stream(dev)))
    return out


# ---------------------------------------------------------------------------------
# Strict mode (ssd_strict_scan_fwd / ssd_strict_state_update): bitwise split invariance
# between a chunked prefill and the chunk-emulating decode.
class ChunkCache:
    """Per-sequence chunk cache of strict mode (``ssd_chunk_cache``): the state entering
    each sequence's open chunk ([nseq, H, P, N]) and that chunk's tokens (x [nseq, H, Q, P],
    B [nseq, G, Q, N], dt and Acum [nseq, H, Q], len [nseq, H]). Tensors are owned here;
    the library only reads and writes them."""

    def __init__(self, state, x, B, dt, acum, length, chunk):
        self.state, self.x, self.B, self.dt, self.acum, self.len = state, x, B, dt, acum, length
        self.chunk = int(chunk)

    @classmethod
    def empty(cls, nseq, H, P, G, N, chunk, dtype, device):
        f32 = dict(dtype=torch.float32, device=device)
        return cls(torch.zeros(nseq, H, P, N, **f32), torch.zeros(nseq, H, chunk, P, dtype=dtype, device=device),
                   torch.zeros(nseq, G, chunk, N, dtype=dtype, device=device), torch.zeros(nseq, H, chunk, **f32),
                   torch.zeros(nseq, H, chunk, **f32), torch.zeros(nseq, H, dtype=torch.int32, device=device),
                   chunk)

    def state_pn(self):
        """The cached states, [nseq, H, P, N]."""
        return self.state

    def set_state(self, states):
        """Set the cached states from [nseq, H, P, N] (the layout of init/final states);
        the open chunks are left as they are."""
        self.state.copy_(states)

    def clone(self):
        return ChunkCache(self.state.clone(), self.x.clone(), self.B.clone(), self.dt.clone(), self.acum.clone(),
                          self.len.clone(), self.chunk)

    def _check(self, nseq, H, P, G, N, dtype, device):
        Q = self.chunk
        _need(self.state, "cache.state", (nseq, H, P, N), torch.float32, device)
        _need(self.x, "cache.x", (nseq, H, Q, P), dtype, device)
        _need(self.B, "cache.B", (nseq, G, Q, N), dtype, device)
        _need(self.dt, "cache.dt", (nseq, H, Q), torch.float32, device)
        _need(self.acum, "cache.acum", (nseq, H, Q), torch.float32, device)
        _need(self.len, "cache.len", (nseq, H), torch.int32, device)

    def _c(self):
        return SSDChunkCache(_ptr(self.state), _ptr(self.x), _ptr(self.B), _ptr(self.dt), _ptr(self.acum),
                             _ptr(self.len))


def strict_workspace_size(dims: SSDDims, chunk: int) -> int:
    b = ctypes.c_size_t(0)
    _check(_lib.ssd_strict_scan_fwd_workspace_size(ctypes.byref(dims), int(chunk), ctypes.byref(b)))
    return int(b.value)


def strict_scan_fwd(x, dt_raw, dt_bias, A, B, C, D, cache: ChunkCache, resume=False, cu_seqlens=None,
                    y=None, final_state=None, workspace=None):
    """Strict chunked prefill (ssd_strict_scan_fwd). Shapes as scan_fwd; the chunk length
    is the cache's. resume=True starts from cache.state (its open chunks must be empty).
    Writes the cache in place; returns (y, final_state)."""
    dev = x.device
    varlen = cu_seqlens is not None
    if varlen:
        T, H, P = x.shape
        nseq = cu_seqlens.numel() - 1
        tok = (T,)
    else:
        if x.dim() != 4:
            raise ValueError("dense x must be [batch, L, H, P]")
        bsz, L, H, P = x.shape
        nseq = bsz
        tok = (bsz, L)
    G, N = B.shape[-2], B.shape[-1]
    dt = x.dtype
    _need(x, "x", tok + (H, P), dt, dev)
    _need(dt_raw, "dt_raw", tok + (H,), torch.float32, dev)
    _need(B, "B", tok + (G, N), dt, dev)
    _need(C, "C", tok + (G, N), dt, dev)
    for name, v in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _need(v, name, (H,), torch.float32, dev)
    if varlen:
        _need(cu_seqlens, "cu_seqlens", (nseq + 1,), torch.int32, dev)
    cache._check(nseq, H, P, G, N, dt, dev)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", tok + (H, P), dt, dev)
    if final_state is None:
        final_state = torch.empty(nseq, H, P, N, dtype=torch.float32, device=dev)
    _need(final_state, "final_state", (nseq, H, P, N), torch.float32, dev)
    if varlen:
        dims = make_dims(x.shape[0], H, P, G, N, _dtype_code(x), nseq=nseq, workspace=workspace)
    else:
        dims = make_dims(bsz * L, H, P, G, N, _dtype_code(x), batch=bsz, seqlen=L, workspace=workspace)
    cc = cache._c()
    with torch.cuda.device(dev):
        _check(_lib.ssd_strict_scan_fwd(_ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                        _ptr(cu_seqlens), _ptr(y), _ptr(final_state), ctypes.byref(cc),
                                        1 if resume else 0, ctypes.byref(dims), cache.chunk, _stream(dev)))
    return y, final_state


def strict_state_update(cache: ChunkCache, x, dt_raw, dt_bias, A, B, C, D, y=None):
    """Chunk-emulating decode step (ssd_strict_state_update). x [nseq,H,P], dt_raw
    [nseq,H], B/C [nseq,G,N]; updates the cache in place and returns y [nseq,H,P]."""
    dev = x.device
    nseq, H, P = x.shape
    G, N = B.shape[-2], B.shape[-1]
    dt = x.dtype
    _need(x, "x", (nseq, H, P), dt, dev)
    _need(dt_raw, "dt_raw", (nseq, H), torch.float32, dev)
    _need(B, "B", (nseq, G, N), dt, dev)
    _need(C, "C", (nseq, G, N), dt, dev)
    for name, v in (("dt_bias", dt_bias), ("A", A), ("D", D)):
        _need(v, name, (H,), torch.float32, dev)
    cache._check(nseq, H, P, G, N, dt, dev)
    if y is None:
        y = torch.empty_like(x)
    _need(y, "y", (nseq, H, P), dt, dev)
    dims = make_dims(nseq, H, P, G, N, _dtype_code(x), batch=nseq, seqlen=1)
    cc = cache._c()
    with torch.cuda.device(dev):
        _check(_lib.ssd_strict_state_update(ctypes.byref(cc), _ptr(x), _ptr(dt_raw), _ptr(dt_bias), _ptr(A), _ptr(B),
                                            _ptr(C), _ptr(D), _ptr(y), ctypes.byref(dims), cache.chunk,
                                            _stream(dev)))
    return y
