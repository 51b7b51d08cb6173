"""Python binding of libgnorm: the same entry points as include/gnorm.h.

Argument marshalling only.  Tensors are torch CUDA tensors (torch provides device memory
and streams); every step of the computation runs in the library's CUDA kernels.  Outputs
that are not passed in are allocated with ``torch.empty``; errors reported by the library
raise ``GnormError``.
"""
from __future__ import annotations

import ctypes
import threading

import torch

from ._lib import GNORM_OK, GnormBwdDesc, GnormFwdDesc, GnormPlan, GnormTuning, lib

__all__ = [
    "GnormError",
    "gnorm_fwd",
    "gnorm_bwd",
    "gnorm_ckpt_step",
    "gnorm_fwd_bwd",
    "gnorm_ckpt_step_host",
    "gnorm_ckpt_step_host_bytes",
    "gnorm_bwd_noalloc",
    "gnorm_dw_reduce",
    "gnorm_bwd_workspace_bytes",
    "gnorm_bwd_workspace_bytes_for",
    "gnorm_status_string",
    "gnorm_plan_query",
    "gnorm_device_error",
    "gnorm_selftest_wait_timeout",
    "gnorm_set_tuning",
    "gnorm_build_info",
    "workspace",
]


class GnormError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {gnorm_status_string(status)} (status {status})")


def gnorm_status_string(status: int) -> str:
    return lib.gnorm_status_string(int(status)).decode()


def gnorm_build_info() -> str:
    return lib.gnorm_build_info().decode()


def gnorm_bwd_workspace_bytes(M: int, N: int, deterministic: bool = True) -> int:
    return int(lib.gnorm_bwd_workspace_bytes(int(M), int(N), int(bool(deterministic))))


def gnorm_bwd_workspace_bytes_for(M: int, N: int, deterministic: bool, num_sms: int) -> int:
    return int(lib.gnorm_bwd_workspace_bytes_for(int(M), int(N), int(bool(deterministic)),
                                                 int(num_sms)))


def gnorm_plan_query(kind: int, M: int, N: int, deterministic: bool, num_sms: int,
                     smem_per_block: int = 0) -> dict:
    """The dispatch rule for `kind` (0 fwd, 1 bwd) on a device with `num_sms` SMs."""
    p = GnormPlan()
    st = lib.gnorm_plan_query(int(kind), int(M), int(N), int(bool(deterministic)), int(num_sms),
                              int(smem_per_block), ctypes.byref(p))
    if st != GNORM_OK:
        raise GnormError(st, "gnorm_plan_query")
    return p.as_dict()


def gnorm_device_error(reset: bool = False) -> int:
    """The device error word (nonzero: a bounded wait inside a kernel gave up).  A call that
    gave up may leave its workspace header nonzero, so the workspaces this module caches are
    zeroed again whenever the word is nonzero; workspaces passed in by the caller are the
    caller's to zero (include/gnorm.h, gnorm_bwd)."""
    word = int(lib.gnorm_device_error(int(bool(reset))))
    if word > 0:
        with _ws_lock:
            for buf in _ws_cache.values():
                buf[:256].zero_()
    return word


def gnorm_selftest_wait_timeout(timeout_us: int = 20000) -> int:
    """Make one bounded wait run out on purpose; returns how long it waited (ns)."""
    waited = ctypes.c_ulonglong(0)
    _check(lib.gnorm_selftest_wait_timeout(int(timeout_us), ctypes.byref(waited)),
           "gnorm_selftest_wait_timeout")
    return int(waited.value)


def gnorm_set_tuning(**knobs) -> None:
    """Process-wide experiment knobs (fields of gnorm_tuning; 0 = built-in).  No arguments
    restores every built-in choice.  Tri-state knobs (l2_prefetch, tail_reduce,
    chain_prefetch, fwd_direct, bwd_direct, fuse_fwd_bwd): 1 on, 2 off, 0 built-in."""
    t = GnormTuning()
    names = {f for f, _ in GnormTuning._fields_}
    for k, v in knobs.items():
        if k not in names:
            raise TypeError(f"unknown tuning knob {k!r}")
        setattr(t, k, int(v))
    lib.gnorm_set_tuning(ctypes.byref(t) if knobs else None)


# ----------------------------------------------------------------------------- helpers

def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr() if t.numel() else 0)


def _stream(stream, device) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _mat(t: torch.Tensor, name: str):
    """(M, N, row stride) of a BF16 CUDA tensor viewed as rows of its last dimension.

    Contiguous tensors of any rank are rows of the last dimension; a 2-D view with unit
    column stride may have any row stride (e.g. a column slice of a wider buffer)."""
    if t.dim() < 1:
        raise ValueError(f"{name} must have a last dimension N")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name} must be bfloat16, got {t.dtype}")
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    N = t.shape[-1]
    if t.is_contiguous():
        return (t.numel() // N if N else 0), N, N
    if t.dim() == 2 and t.stride(1) == 1:
        M = t.shape[0]
        return M, N, (t.stride(0) if M > 1 else N)
    raise ValueError(f"{name}: rows need unit column stride (2-D row-strided views or "
                     "contiguous tensors)")


def _same(a: torch.Tensor, b: torch.Tensor, an: str, bn: str):
    if a.shape != b.shape:
        raise ValueError(f"{an} {tuple(a.shape)} and {bn} {tuple(b.shape)} differ")
    if a.device != b.device:
        raise ValueError(f"{an} and {bn} are on different devices")


def _vec(t: torch.Tensor, N: int, dtypes, name: str, device):
    if t.dtype not in dtypes:
        raise TypeError(f"{name} must be one of {dtypes}, got {t.dtype}")
    if t.numel() != N or not t.is_contiguous() or t.device != device:
        raise ValueError(f"{name} must be a contiguous [{N}] tensor on {device}")


def _weight(w, N, device):
    _vec(w, N, (torch.bfloat16, torch.float32), "w", device)
    return 1 if w.dtype == torch.float32 else 0


def _device_buffer(t, name: str, device):
    """Scratch handed to the library: contiguous memory on the device that runs the call
    (a host buffer here would reach a kernel as a device pointer)."""
    if t.device != torch.device(device) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous tensor on {device}")


def _check(st: int, where: str):
    if st != GNORM_OK:
        raise GnormError(st, where)


_ws_lock = threading.Lock()
_ws_cache: dict = {}


def workspace(M: int, N: int, deterministic: bool, device) -> torch.Tensor:
    """A zero-initialised backward workspace for `device`, cached and grown as needed.

    The cache holds one buffer per device; calls that may run concurrently (other streams)
    must pass workspaces of their own.
    """
    device = torch.device(device)
    idx = device.index if device.index is not None else torch.cuda.current_device()
    with torch.cuda.device(idx):
        need = max(gnorm_bwd_workspace_bytes(M, N, deterministic), 256)
    with _ws_lock:
        buf = _ws_cache.get(idx)
        if buf is None or buf.numel() < need:
            buf = torch.zeros(need, dtype=torch.uint8, device=torch.device("cuda", idx))
            _ws_cache[idx] = buf
        return buf


_host_cache: dict = {}


def _host_step_buffer(M: int, N: int, deterministic: bool, device) -> torch.Tensor:
    """Device buffer for gnorm_ckpt_step_host, cached per device and grown as needed (calls
    that may overlap on the GPU must pass buffers of their own)."""
    idx = device.index if device.index is not None else torch.cuda.current_device()
    with torch.cuda.device(idx):
        need = max(gnorm_ckpt_step_host_bytes(M, N, deterministic), 256)
    with _ws_lock:
        buf = _host_cache.get(idx)
        if buf is None or buf.numel() < need:
            buf = torch.empty(need, dtype=torch.uint8, device=torch.device("cuda", idx))
            _host_cache[idx] = buf
        return buf


# ------------------------------------------------------------------------- entry points

def _fwd_desc(x, g, w, eps, y, rstd):
    M, N, ldx = _mat(x, "x")
    Mg, Ng, ldg = _mat(g, "g")
    _same(x, g, "x", "g")
    w_fp32 = _weight(w, N, x.device)
    if y is None:
        y = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    else:
        _same(x, y, "x", "y")
    _, _, ldy = _mat(y, "y")
    if rstd is None:
        rstd = torch.empty(M, dtype=torch.float32, device=x.device)
    else:
        _vec(rstd, M, (torch.float32,), "rstd", x.device)
    d = GnormFwdDesc(x=_ptr(x), ldx=ldx, g=_ptr(g), ldg=ldg, w=_ptr(w), w_fp32=w_fp32,
                     eps=float(eps), y=_ptr(y), ldy=ldy, rstd=_ptr(rstd), M=M, N=N)
    return d, y, rstd


def _bwd_desc(dy, x, g, w, rstd, dx, dg, dw, dw_fp32, deterministic, ws):
    M, N, ldx = _mat(x, "x")
    _, _, lddy = _mat(dy, "dy")
    _, _, ldg = _mat(g, "g")
    _same(x, dy, "x", "dy")
    _same(x, g, "x", "g")
    w_fp32 = _weight(w, N, x.device)
    if rstd is not None:
        _vec(rstd, M, (torch.float32,), "rstd", x.device)
    if dx is None:
        dx = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    if dg is None:
        dg = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    _same(x, dx, "x", "dx")
    _same(x, dg, "x", "dg")
    _, _, lddx = _mat(dx, "dx")
    _, _, lddg = _mat(dg, "dg")
    dw_dtype = torch.float32 if dw_fp32 else torch.bfloat16
    if dw is None:
        dw = torch.empty(N, dtype=dw_dtype, device=x.device)
    else:
        _vec(dw, N, (dw_dtype,), "dw", x.device)
    if ws is None:
        ws = workspace(M, N, deterministic, x.device)
    else:
        _device_buffer(ws, "workspace_buf", x.device)
    d = GnormBwdDesc(dy=_ptr(dy), lddy=lddy, x=_ptr(x), ldx=ldx, g=_ptr(g), ldg=ldg, w=_ptr(w),
                     w_fp32=w_fp32, rstd=_ptr(rstd), dx=_ptr(dx), lddx=lddx, dg=_ptr(dg),
                     lddg=lddg, dw=_ptr(dw), dw_fp32=int(bool(dw_fp32)),
                     deterministic=int(bool(deterministic)), M=M, N=N, workspace=_ptr(ws),
                     workspace_bytes=ws.numel() * ws.element_size())
    return d, dx, dg, dw


def gnorm_fwd(x, g, w, eps: float = 1e-6, *, y=None, rstd=None, stream=None):
    """Forward: returns (y, rstd).

    x, g: BF16 rows (contiguous, or 2-D views with any row stride); w: BF16 or FP32 [N];
    rstd: FP32 [M].  y is allocated packed unless given (it may be a strided view)."""
    d, y, rstd = _fwd_desc(x, g, w, eps, y, rstd)
    with torch.cuda.device(x.device):
        st = lib.gnorm_fwd_ex(ctypes.byref(d), _stream(stream, x.device))
    _check(st, "gnorm_fwd")
    return y, rstd


def gnorm_bwd(dy, x, g, w, rstd, *, dx=None, dg=None, dw=None, dw_fp32: bool = False,
              deterministic: bool = True, workspace_buf=None, stream=None):
    """Backward: returns (dx, dg, dw).  dw is FP32 if dw_fp32 else BF16.  Row-strided 2-D
    views are accepted for dy, x, g, dx, dg; w may be BF16 or FP32."""
    d, dx, dg, dw = _bwd_desc(dy, x, g, w, rstd, dx, dg, dw, dw_fp32, deterministic,
                              workspace_buf)
    if rstd is None:
        raise ValueError("rstd is required")
    with torch.cuda.device(x.device):
        st = lib.gnorm_bwd_ex(ctypes.byref(d), _stream(stream, x.device))
    _check(st, "gnorm_bwd")
    return dx, dg, dw


def gnorm_ckpt_step(x, g, w, eps: float, dy, *, y=None, rstd=None, dx=None, dg=None, dw=None,
                    dw_fp32: bool = False, deterministic: bool = True, workspace_buf=None,
                    stream=None):
    """Checkpointed step (forward, forward again, backward): returns (y, rstd, dx, dg, dw)."""
    fd, y, rstd = _fwd_desc(x, g, w, eps, y, rstd)
    bd, dx, dg, dw = _bwd_desc(dy, x, g, w, rstd, dx, dg, dw, dw_fp32, deterministic,
                               workspace_buf)
    with torch.cuda.device(x.device):
        st = lib.gnorm_ckpt_step_ex(ctypes.byref(fd), ctypes.byref(bd),
                                    _stream(stream, x.device))
    _check(st, "gnorm_ckpt_step")
    return y, rstd, dx, dg, dw


def gnorm_fwd_bwd(x, g, w, eps: float, dy, *, y=None, rstd=None, dx=None, dg=None, dw=None,
                  dw_fp32: bool = False, deterministic: bool = True, workspace_buf=None,
                  stream=None):
    """Forward and backward of the same rows in one pass (the recompute forward of a
    checkpointed layer and its backward): returns (y, rstd, dx, dg, dw)."""
    fd, y, rstd = _fwd_desc(x, g, w, eps, y, rstd)
    bd, dx, dg, dw = _bwd_desc(dy, x, g, w, rstd, dx, dg, dw, dw_fp32, deterministic,
                               workspace_buf)
    with torch.cuda.device(x.device):
        st = lib.gnorm_fwd_bwd_ex(ctypes.byref(fd), ctypes.byref(bd), _stream(stream, x.device))
    _check(st, "gnorm_fwd_bwd")
    return y, rstd, dx, dg, dw


def gnorm_ckpt_step_host_bytes(M: int, N: int, deterministic: bool = True) -> int:
    return int(lib.gnorm_ckpt_step_host_bytes(int(M), int(N), int(bool(deterministic))))


def _host_mat(t, M, N, name):
    if t.device.type != "cpu" or t.dtype != torch.bfloat16 or not t.is_contiguous() or \
            tuple(t.shape) != (M, N):
        raise ValueError(f"{name} must be a contiguous BF16 [{M}, {N}] CPU tensor")


def gnorm_ckpt_step_host(x, g, w, eps: float, dy, *, y=None, rstd=None, dx=None, dg=None,
                         dw=None, dw_fp32: bool = False, deterministic: bool = True,
                         dev_buf=None, device=None, stream=None):
    """Checkpointed step on HOST tensors (pinned for overlapped copies): the library copies
    the rows in, runs the step chunk by chunk and copies the outputs back, all ordered on
    `stream` of `device`.  Returns (y, rstd, dx, dg, dw) as CPU tensors; they are written
    once the stream has reached the end of the call."""
    if x.dim() != 2:
        raise ValueError("x must be a 2-D [M, N] CPU tensor")
    M, N = x.shape
    for t, n in ((x, "x"), (g, "g"), (dy, "dy")):
        _host_mat(t, M, N, n)
    if w.device.type != "cpu" or w.dtype != torch.bfloat16 or tuple(w.shape) != (N,):
        raise ValueError(f"w must be a BF16 [{N}] CPU tensor")
    pin = x.is_pinned()
    device = torch.device("cuda") if device is None else torch.device(device)
    if device.index is None:
        device = torch.device("cuda", torch.cuda.current_device())

    def new(shape, dtype):
        return torch.empty(shape, dtype=dtype, pin_memory=pin)

    y = new((M, N), torch.bfloat16) if y is None else y
    dx = new((M, N), torch.bfloat16) if dx is None else dx
    dg = new((M, N), torch.bfloat16) if dg is None else dg
    rstd = new((M,), torch.float32) if rstd is None else rstd
    dw_dtype = torch.float32 if dw_fp32 else torch.bfloat16
    dw = new((N,), dw_dtype) if dw is None else dw
    for t, n in ((y, "y"), (dx, "dx"), (dg, "dg")):
        _host_mat(t, M, N, n)
    for t, n, length, dt in ((rstd, "rstd", M, torch.float32), (dw, "dw", N, dw_dtype)):
        if t.device.type != "cpu" or t.dtype != dt or tuple(t.shape) != (length,):
            raise ValueError(f"{n} must be a {dt} [{length}] CPU tensor")
    with torch.cuda.device(device):
        if dev_buf is None:
            dev_buf = _host_step_buffer(M, N, deterministic, device)
        else:
            _device_buffer(dev_buf, "dev_buf", device)
        st = lib.gnorm_ckpt_step_host(_ptr(x), _ptr(g), _ptr(w), float(eps), _ptr(dy), _ptr(y),
                                      _ptr(rstd), _ptr(dx), _ptr(dg), _ptr(dw),
                                      int(bool(dw_fp32)), int(bool(deterministic)), M, N,
                                      _ptr(dev_buf), dev_buf.numel() * dev_buf.element_size(),
                                      _stream(stream, device))
    _check(st, "gnorm_ckpt_step_host")
    return y, rstd, dx, dg, dw


def gnorm_dw_reduce(partials, *, dw=None, dw_fp32: bool = True, stream=None):
    """Fixed-order sum of FP32 partial rows [P, N] into dw [N] (BF16 or FP32)."""
    if (partials.device.type != "cuda" or partials.dtype != torch.float32 or
            partials.dim() != 2 or not partials.is_contiguous()):
        raise ValueError("partials must be a contiguous FP32 [P, N] CUDA tensor")
    P, N = partials.shape
    dw_dtype = torch.float32 if dw_fp32 else torch.bfloat16
    if dw is None:
        dw = torch.empty(N, dtype=dw_dtype, device=partials.device)
    else:
        _vec(dw, N, (dw_dtype,), "dw", partials.device)
    with torch.cuda.device(partials.device):
        st = lib.gnorm_dw_reduce(_ptr(partials), P, N, _ptr(dw), int(bool(dw_fp32)),
                                 _stream(stream, partials.device))
    _check(st, "gnorm_dw_reduce")
    return dw


def gnorm_bwd_noalloc(dy, x, g, w, rstd, *, dx=None, dg=None, dw=None, dw_fp32: bool = False,
                      deterministic: bool = True, stream=None):
    """Backward with the library's static scratch instead of a workspace.

    For callers that cannot allocate device memory.  Calls that overlap on the GPU share
    the scratch and race; see include/gnorm.h.
    """
    M, N, _ = _mat(x, "x")
    for t, n in ((dy, "dy"), (g, "g")):
        _same(x, t, "x", n)
    if dx is None:
        dx = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    if dg is None:
        dg = torch.empty(x.shape, dtype=torch.bfloat16, device=x.device)
    for t, n in ((x, "x"), (dy, "dy"), (g, "g"), (dx, "dx"), (dg, "dg")):
        if _mat(t, n)[2] != N:
            raise ValueError(f"gnorm_bwd_noalloc takes packed rows only ({n} is strided)")
    _vec(w, N, (torch.bfloat16,), "w", x.device)
    _vec(rstd, M, (torch.float32,), "rstd", x.device)
    dw_dtype = torch.float32 if dw_fp32 else torch.bfloat16
    if dw is None:
        dw = torch.empty(N, dtype=dw_dtype, device=x.device)
    else:
        _vec(dw, N, (dw_dtype,), "dw", x.device)
    with torch.cuda.device(x.device):
        st = lib.gnorm_bwd_noalloc(_ptr(dy), _ptr(x), _ptr(g), _ptr(w), _ptr(rstd), _ptr(dx),
                                   _ptr(dg), _ptr(dw), int(bool(dw_fp32)),
                                   int(bool(deterministic)), M, N, _stream(stream, x.device))
    _check(st, "gnorm_bwd_noalloc")
    return dx, dg, dw
