"""B200 (sm_100a) speculative-sampling verification behind a C ABI.

The work runs in ``libspecverify.so`` (CUDA kernels for sm_100a, declared in
``include/spec_verify.h``).  This module is a thin ctypes binding: it checks
tensor shapes, dtypes and devices, passes raw pointers and the current CUDA
stream, and turns status codes into exceptions.  ``host`` binds the host-side
drafters and schedulers of ``include/sv_host.h``; ``graph`` replays a whole
step as one CUDA graph.  PyTorch is used only for device memory
and streams.  There is no CPU fallback: without the built library every call
raises.

Typical use::

    import speculative_decoding_verification_92_b200 as sv
    accept_len, tokens = sv.spec_verify(target, draft, draft_tokens, draft_lens,
                                        uniforms, temperature=1.0)
"""
from __future__ import annotations

import ctypes
import enum
import os
from pathlib import Path

__all__ = [
    "Status", "StatsKernel", "SpecVerifyError", "library", "workspace_bytes",
    "spec_verify", "spec_verify_stats", "spec_verify_accept_sim", "spec_verify_host", "host_staging_bytes",
    "abi_version", "auto_draw_path", "DrawPath", "F32", "BF16", "MAX_K", "MAX_V",
]

F32 = 0
BF16 = 1
MAX_K = 1024      # SV_MAX_K of the C header: largest supported k_max
MAX_V = 393216    # SV_MAX_V of the C header: largest supported vocabulary


class Status(enum.IntEnum):
    OK = 0
    EINVAL = 1
    ECUDA = 2
    EUNSUPPORTED = 3
    ESCRATCH = 4


class StatsKernel(enum.IntEnum):
    AUTO = 0
    TMA = 1
    VEC16 = 2
    SCALAR = 3


class DrawPath(enum.IntEnum):
    AUTO = 0
    QUEUE = 1     # scan kernel, draw kernel over a queue of pieces, selection kernel
    CLUSTER = 2   # one thread-block cluster per request: scan and draw in one kernel


class SpecVerifyError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = Status(status)
        super().__init__(f"{what}: {self.status.name}")


class _Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("k_max", ctypes.c_int32), ("V", ctypes.c_int32),
                ("dtype", ctypes.c_int32), ("row_stride", ctypes.c_int64)]


class _Options(ctypes.Structure):
    _fields_ = [("stats_kernel", ctypes.c_int32), ("wait_timeout_us", ctypes.c_int32),
                ("event_stats_begin", ctypes.c_void_p), ("event_stats_end", ctypes.c_void_p),
                ("lost_copy_request", ctypes.c_int32), ("lost_draw_request", ctypes.c_int32),
                ("draw_path", ctypes.c_int32), ("reserved", ctypes.c_int32 * 5)]


_LIB = None

# C signatures, in header order.
_VP, _I32, _F32, _SZ = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
_SIGNATURES = {
    "spec_verify_workspace_bytes": (_SZ, [ctypes.POINTER(_Shape)]),
    "spec_verify": (_I32, [ctypes.POINTER(_Shape), _VP, _VP, _VP, _VP, _VP, _F32, _I32, _VP, _VP, _VP, _SZ, _VP]),
    "spec_verify_ex": (_I32, [ctypes.POINTER(_Shape), _VP, _VP, _VP, _VP, _VP, _F32, _I32, _VP, _VP, _VP, _SZ,
                              _VP, ctypes.POINTER(_Options)]),
    "spec_verify_stats": (_I32, [ctypes.POINTER(_Shape), _VP, _VP, _VP, _VP, _F32, _VP, _VP, _VP, _VP, _VP, _SZ,
                                 _VP, ctypes.POINTER(_Options)]),
    "spec_verify_accept_sim": (_I32, [ctypes.POINTER(_Shape), _VP, _VP, _VP, _VP, _VP, _F32, _F32, _VP, _VP, _VP, _VP,
                                      _VP, _SZ, _VP]),
    "spec_verify_host_staging_bytes": (_SZ, [ctypes.POINTER(_Shape), _I32, _I32]),
    "spec_verify_host": (_I32, [ctypes.POINTER(_Shape), _VP, _VP, _VP, _VP, _VP, _F32, _I32, _VP, _VP, _VP, _SZ,
                                _VP, _SZ, _VP]),
    "spec_verify_status_string": (ctypes.c_char_p, [_I32]),
    "spec_verify_abi_version": (_I32, []),
    "spec_verify_auto_draw_path": (_I32, [ctypes.POINTER(_Shape)]),
    "spec_verify_static_scratch": (_I32, [ctypes.POINTER(_Shape), _VP, _VP, _VP, _VP, _VP, _F32, _I32, _VP, _VP,
                                          _VP]),
}


def library_path() -> Path:
    return Path(__file__).resolve().parent / "libspecverify.so"


def library() -> ctypes.CDLL:
    """Load libspecverify.so (building it with nvcc first if the sources
    changed).  The environment variable SPECVERIFY_LIBRARY names another
    build of the same library to load instead (no rebuild).  Raises if the
    library cannot be built or loaded."""
    global _LIB
    if _LIB is None:
        override = os.environ.get("SPECVERIFY_LIBRARY")
        if override:
            path = Path(override)
        else:
            from . import build as _build
            if _build.is_stale():
                _build.build()
            path = library_path()
        lib = ctypes.CDLL(str(path))
        for name, (res, args) in _SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _LIB = lib
    return _LIB


def abi_version() -> int:
    return int(library().spec_verify_abi_version())


def auto_draw_path(B: int, k_max: int, V: int, dtype: int, row_stride: int = 0) -> "DrawPath":
    """The draw path DrawPath.AUTO takes for a sampling call of this shape on
    the current device (needs a GPU)."""
    shape = _shape(B, k_max, V, dtype, row_stride or V)
    r = int(library().spec_verify_auto_draw_path(ctypes.byref(shape)))
    if r < 0:
        raise SpecVerifyError(int(Status.EINVAL), "spec_verify_auto_draw_path")
    return DrawPath(r)


def _check(status: int, what: str):
    if status != 0:
        raise SpecVerifyError(status, what)


def _shape(B, k_max, V, dtype, row_stride=0) -> _Shape:
    return _Shape(int(B), int(k_max), int(V), int(dtype), int(row_stride))


def workspace_bytes(B: int, k_max: int, V: int, dtype: int, row_stride: int = 0) -> int:
    return int(library().spec_verify_workspace_bytes(ctypes.byref(_shape(B, k_max, V, dtype, row_stride))))


def host_staging_bytes(B, k_max, V, dtype, row_stride=0, has_draft=True, has_lens=False) -> int:
    return int(library().spec_verify_host_staging_bytes(ctypes.byref(_shape(B, k_max, V, dtype, row_stride)),
                                                        int(bool(has_draft)), int(bool(has_lens))))


# ---------------------------------------------------------------------------
# torch marshalling


def _torch():
    import torch
    return torch


def _dtype_code(t) -> int:
    torch = _torch()
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.bfloat16:
        return BF16
    raise TypeError(f"logits must be float32 or bfloat16, got {t.dtype}")


def _dev_ptr(t, dtype=None, what="tensor"):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError(f"{what} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    return t.data_ptr()


def _check_shapes(device, **named):
    """Every given tensor must have exactly its expected shape (the library
    reads that many elements through the raw pointer) and, when ``device`` is
    given, live on that device.  ``named`` maps a name to (tensor, shape);
    None tensors are skipped, a None shape checks the device only."""
    for what, (t, shape) in named.items():
        if t is None:
            continue
        if shape is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{what} must have shape {tuple(shape)}, got {tuple(t.shape)}")
        if device is not None and t.device != device:
            raise ValueError(f"{what} is on {t.device}, the logits on {device}")


def _stream_handle(stream):
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _options(stats_kernel=StatsKernel.AUTO, wait_timeout_us=0, events=None, lost_copy_request=0,
             lost_draw_request=0, draw_path=0):
    o = _Options()
    o.stats_kernel = int(stats_kernel)
    o.draw_path = int(draw_path)
    o.wait_timeout_us = int(wait_timeout_us)
    o.lost_copy_request = int(lost_copy_request)
    o.lost_draw_request = int(lost_draw_request)
    if events is not None:
        o.event_stats_begin = events[0].cuda_event
        o.event_stats_end = events[1].cuda_event
    return o


def _logit_shape(target, draft, V):
    if target.dim() != 3:
        raise ValueError("target logits must be [B, k_max+1, row_stride]")
    B, k1, row_stride = target.shape
    k_max = k1 - 1
    V = row_stride if V is None else int(V)
    dt = _dtype_code(target)
    if draft is not None:
        if draft.dtype != target.dtype or tuple(draft.shape) != (B, k_max, row_stride):
            raise ValueError("draft logits must be [B, k_max, row_stride] with the target dtype")
    return B, k_max, V, dt, row_stride


def spec_verify(target, draft, tokens, lens, uniforms, temperature=1.0, greedy=False, *, V=None,
                out=None, workspace=None, stream=None, stats_kernel=StatsKernel.AUTO,
                wait_timeout_us=0, events=None, lost_copy_request=0, lost_draw_request=0, draw_path=0):
    """Verify one batch on the GPU.  Returns ``(accept_len [B] int32,
    tokens [B, k_max+1] int32)`` (device tensors, valid once ``stream`` has
    run).  ``events=(begin, end)`` (torch.cuda.Event, already created)
    brackets the row-statistics kernel.  ``lost_copy_request`` and
    ``lost_draw_request`` are the test-only fault injections of
    ``sv_options`` (1 + the request whose first bulk copy in the
    row-statistics / draw kernel is never issued; 0 = off).  ``draw_path``
    picks how the final draws are made (DrawPath; AUTO by default)."""
    torch = _torch()
    B, k_max, V, dt, row_stride = _logit_shape(target, draft, V)
    dev = target.device
    if out is None:
        out = (torch.empty(B, dtype=torch.int32, device=dev),
               torch.empty(B, k_max + 1, dtype=torch.int32, device=dev))
    out_len, out_tok = out
    _check_shapes(dev, draft_tokens=(tokens, (B, k_max)), draft_lens=(lens, (B,)),
                  uniforms=(None if greedy else uniforms, (B, k_max + 1)),
                  out_accept_len=(out_len, (B,)), out_tokens=(out_tok, (B, k_max + 1)),
                  draft=(draft, None), workspace=(workspace, None))
    shape = _shape(B, k_max, V, dt, row_stride)
    lib = library()
    if workspace is None:
        workspace = torch.empty(max(lib.spec_verify_workspace_bytes(ctypes.byref(shape)), 256),
                                dtype=torch.uint8, device=dev)
    opts = _options(stats_kernel, wait_timeout_us, events, lost_copy_request, lost_draw_request, draw_path)
    st = lib.spec_verify_ex(
        ctypes.byref(shape), _dev_ptr(target, what="target"), _dev_ptr(draft, what="draft"),
        _dev_ptr(tokens, torch.int32, "draft_tokens"), _dev_ptr(lens, torch.int32, "draft_lens"),
        _dev_ptr(uniforms, torch.float32, "uniforms"), float(temperature), int(bool(greedy)),
        _dev_ptr(out_len, torch.int32, "out_accept_len"), _dev_ptr(out_tok, torch.int32, "out_tokens"),
        _dev_ptr(workspace, what="workspace"), workspace.numel() * workspace.element_size(),
        _stream_handle(stream), ctypes.byref(opts))
    _check(st, "spec_verify")
    return out_len, out_tok


def spec_verify_stats(target, draft, tokens, lens, temperature=1.0, *, V=None, workspace=None, stream=None,
                      stats_kernel=StatsKernel.AUTO):
    """Per-row natural-log lse of the target / draft rows and p, q at the
    drafted ids, as float32 device tensors ``(lse_t [B, k+1], lse_d [B, k],
    p [B, k], q [B, k])``; NaN where a row is unused."""
    torch = _torch()
    B, k_max, V, dt, row_stride = _logit_shape(target, draft, V)
    dev = target.device
    lse_t = torch.empty(B, k_max + 1, dtype=torch.float32, device=dev)
    lse_d = torch.empty(B, k_max, dtype=torch.float32, device=dev)
    p = torch.empty(B, k_max, dtype=torch.float32, device=dev)
    q = torch.empty(B, k_max, dtype=torch.float32, device=dev)
    _check_shapes(dev, draft_tokens=(tokens, (B, k_max)), draft_lens=(lens, (B,)))
    shape = _shape(B, k_max, V, dt, row_stride)
    lib = library()
    if workspace is None:
        workspace = torch.empty(max(lib.spec_verify_workspace_bytes(ctypes.byref(shape)), 256),
                                dtype=torch.uint8, device=dev)
    opts = _options(stats_kernel)
    st = lib.spec_verify_stats(
        ctypes.byref(shape), _dev_ptr(target, what="target"), _dev_ptr(draft, what="draft"),
        _dev_ptr(tokens, torch.int32, "draft_tokens"), _dev_ptr(lens, torch.int32, "draft_lens"),
        float(temperature), lse_t.data_ptr(), lse_d.data_ptr(), p.data_ptr(), q.data_ptr(),
        _dev_ptr(workspace, what="workspace"), workspace.numel() * workspace.element_size(),
        _stream_handle(stream), ctypes.byref(opts))
    _check(st, "spec_verify_stats")
    return lse_t, lse_d, p, q


def spec_verify_accept_sim(target, draft, tokens, lens, uniforms=None, temperature=1.0, decay=0.8, *, V=None,
                           workspace=None, stream=None):
    """Acceptance simulation (no draw): returns float32 / int32 device tensors
    ``(accept_prob [B, k], expected_len [B], first_reject [B], weights [B, k])``
    -- a_i = min(1, p_i/q_i) (NaN past the request's length), E[j], and, when
    ``uniforms`` is given, the first rejection j and the per-position weights
    (1 up to j, decay**(i - j) after, 0 past the length); the last two are
    None without uniforms."""
    torch = _torch()
    B, k_max, V, dt, row_stride = _logit_shape(target, draft, V)
    dev = target.device
    a = torch.empty(B, k_max, dtype=torch.float32, device=dev)
    e = torch.empty(B, dtype=torch.float32, device=dev)
    j = torch.empty(B, dtype=torch.int32, device=dev) if uniforms is not None else None
    w = torch.empty(B, k_max, dtype=torch.float32, device=dev) if uniforms is not None else None
    _check_shapes(dev, draft_tokens=(tokens, (B, k_max)), draft_lens=(lens, (B,)),
                  uniforms=(uniforms, (B, k_max + 1)))
    shape = _shape(B, k_max, V, dt, row_stride)
    lib = library()
    if workspace is None:
        workspace = torch.empty(max(lib.spec_verify_workspace_bytes(ctypes.byref(shape)), 256),
                                dtype=torch.uint8, device=dev)
    st = lib.spec_verify_accept_sim(
        ctypes.byref(shape), _dev_ptr(target, what="target"), _dev_ptr(draft, what="draft"),
        _dev_ptr(tokens, torch.int32, "draft_tokens"), _dev_ptr(lens, torch.int32, "draft_lens"),
        _dev_ptr(uniforms, torch.float32, "uniforms"), float(temperature), float(decay),
        a.data_ptr(), e.data_ptr(), None if j is None else j.data_ptr(), None if w is None else w.data_ptr(),
        _dev_ptr(workspace, what="workspace"), workspace.numel() * workspace.element_size(),
        _stream_handle(stream))
    _check(st, "spec_verify_accept_sim")
    return a, e, j, w


def _host_ptr(t, dtype=None, what="tensor"):
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError(f"{what} must be a host tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{what} must be {dtype}, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{what} must be contiguous")
    return t.data_ptr()


def spec_verify_host(target, draft, tokens, lens, uniforms, temperature=1.0, greedy=False, *, V=None,
                     out=None, staging=None, workspace=None, stream=None, device=None):
    """End-to-end call on HOST tensors (pin them for asynchronous copies):
    the library copies the inputs into ``staging`` (device), verifies, and
    copies the results back into ``out`` (host int32 tensors).  Results are
    valid after the stream is synchronised."""
    torch = _torch()
    B, k_max, V, dt, row_stride = _logit_shape(target, draft, V)
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    shape = _shape(B, k_max, V, dt, row_stride)
    lib = library()
    if out is None:
        out = (torch.empty(B, dtype=torch.int32, pin_memory=True),
               torch.empty(B, k_max + 1, dtype=torch.int32, pin_memory=True))
    _check_shapes(None, draft_tokens=(tokens, (B, k_max)), draft_lens=(lens, (B,)),
                  uniforms=(None if greedy else uniforms, (B, k_max + 1)),
                  out_accept_len=(out[0], (B,)), out_tokens=(out[1], (B, k_max + 1)))
    if staging is None:
        n = lib.spec_verify_host_staging_bytes(ctypes.byref(shape), int(draft is not None), int(lens is not None))
        staging = torch.empty(max(n, 256), dtype=torch.uint8, device=dev)
    if workspace is None:
        workspace = torch.empty(max(lib.spec_verify_workspace_bytes(ctypes.byref(shape)), 256),
                                dtype=torch.uint8, device=dev)
    st = lib.spec_verify_host(
        ctypes.byref(shape), _host_ptr(target, what="target"), _host_ptr(draft, what="draft"),
        _host_ptr(tokens, torch.int32, "draft_tokens"), _host_ptr(lens, torch.int32, "draft_lens"),
        _host_ptr(uniforms, torch.float32, "uniforms"), float(temperature), int(bool(greedy)),
        _host_ptr(out[0], torch.int32, "out_accept_len"), _host_ptr(out[1], torch.int32, "out_tokens"),
        _dev_ptr(staging, what="staging"), staging.numel(), _dev_ptr(workspace, what="workspace"),
        workspace.numel(), _stream_handle(stream))
    _check(st, "spec_verify_host")
    return out
