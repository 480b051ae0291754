"""ctypes binding of libgdn.so (declared in include/gdn.h).

Argument marshalling only: every step of the layer runs in the library's CUDA
kernels.  PyTorch provides device memory and the current stream.  There is no
fallback: if the library is missing, every call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

GDN_BF16, GDN_FP32 = 0, 1
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported configuration", 3: "misaligned pointer",
          4: "workspace missing or too small", 5: "CUDA runtime error",
          6: "device-side wait timed out"}
EXPORTS = ("gdn_version", "gdn_chunk_size", "gdn_fwd_workspace_size", "gdn_bwd_workspace_size",
           "gdn_fwd", "gdn_fwd_noalloc", "gdn_fwd_noalloc_status", "gdn_bwd", "gdn_decode",
           "gdn_device_status", "gdn_status_string", "gdn_trace_install", "gdn_kernel_name",
           "gdn_set_wait_limit", "gdn_set_test_hook")
GDN_TEST_STALL_COPY, GDN_TEST_FAIL_LAUNCH = 1, 2


class GdnError(RuntimeError):
    def __init__(self, code: int, what: str):
        super().__init__("%s: %s (status %d)" % (what, STATUS.get(code, "?"), code))
        self.code = code


class GdnDesc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int64), ("T", ctypes.c_int64), ("H", ctypes.c_int64),
                ("dk", ctypes.c_int64), ("dv", ctypes.c_int64), ("n_seqs", ctypes.c_int64),
                ("dtype", ctypes.c_int32), ("scale", ctypes.c_float), ("flags", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]

GDN_FLAG_PIECE_SCAN = 1
GDN_FLAG_QK_L2NORM = 2
GDN_FLAG_VALUE_SLICES = 4


_lock = threading.Lock()
_lib = None


def lib() -> ctypes.CDLL:
    """Load libgdn.so (raises if it was not built: there is no other path)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise ImportError("libgdn.so not built (run gated_delta_rule_99_b200.build)")
            L = ctypes.CDLL(LIB_PATH)
            vp, sz, i32p, fp = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_void_p
            dp = ctypes.POINTER(GdnDesc)
            L.gdn_version.restype = ctypes.c_int
            L.gdn_chunk_size.restype = ctypes.c_int
            for n in ("gdn_fwd_workspace_size", "gdn_bwd_workspace_size"):
                getattr(L, n).restype = sz
                getattr(L, n).argtypes = [dp]
            L.gdn_fwd.restype = ctypes.c_int
            L.gdn_fwd.argtypes = [dp, vp, vp, vp, fp, fp, i32p, i32p, fp, vp, fp, vp, sz, vp]
            L.gdn_fwd_noalloc.restype = ctypes.c_int
            L.gdn_fwd_noalloc.argtypes = [dp, vp, vp, vp, fp, fp, i32p, i32p, fp, vp, fp, vp]
            L.gdn_fwd_noalloc_status.restype = ctypes.c_int
            L.gdn_fwd_noalloc_status.argtypes = [vp]
            L.gdn_set_wait_limit.restype = None
            L.gdn_set_wait_limit.argtypes = [ctypes.c_uint32]
            L.gdn_set_test_hook.restype = None
            L.gdn_set_test_hook.argtypes = [ctypes.c_int32]
            L.gdn_bwd.restype = ctypes.c_int
            L.gdn_bwd.argtypes = [dp, vp, vp, vp, fp, fp, i32p, i32p, fp, vp, fp, vp, vp, vp, fp,
                                  fp, fp, vp, sz, vp]
            L.gdn_decode.restype = ctypes.c_int
            L.gdn_decode.argtypes = [dp, vp, vp, vp, fp, fp, fp, vp, vp]
            L.gdn_device_status.restype = ctypes.c_int
            L.gdn_device_status.argtypes = [vp, vp]
            L.gdn_status_string.restype = ctypes.c_char_p
            L.gdn_status_string.argtypes = [ctypes.c_int]
            L.gdn_trace_install.restype = None
            L.gdn_trace_install.argtypes = [ctypes.c_void_p]
            L.gdn_kernel_name.restype = ctypes.c_char_p
            L.gdn_kernel_name.argtypes = [ctypes.c_int32]
            _lib = L
    return _lib


def make_desc(B, T, H, dk, dv, n_seqs=0, dtype=GDN_BF16, scale=1.0, flags=0) -> GdnDesc:
    return GdnDesc(int(B), int(T), int(H), int(dk), int(dv), int(n_seqs), int(dtype), float(scale),
                   int(flags), 0)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _check(t, name, dtype=None, shape=None):
    if t is None:
        return
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)
    if dtype is not None and t.dtype != dtype:
        raise ValueError("%s must be %s, got %s" % (name, dtype, t.dtype))
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def _desc_from(q, v, cu_host, scale, flags=0):
    B, T, H, K = q.shape
    V = v.shape[-1]
    n_seqs = 0 if cu_host is None else cu_host.numel() - 1
    dt = {torch.bfloat16: GDN_BF16, torch.float32: GDN_FP32}.get(q.dtype)
    if dt is None:
        raise ValueError("q must be bf16 or fp32")
    return make_desc(B, T, H, K, V, n_seqs, dt, scale, flags), (B, T, H, K, V, n_seqs)


def _seqlens(cu_seqlens, cu_seqlens_host, device):
    if cu_seqlens is None and cu_seqlens_host is None:
        return None, None
    host = cu_seqlens_host if cu_seqlens_host is not None else cu_seqlens.cpu()
    host = host.to(torch.int32).contiguous()
    dev = cu_seqlens if cu_seqlens is not None and cu_seqlens.is_cuda else host.to(device)
    return dev.to(torch.int32).contiguous(), host


def fwd_workspace_size(desc: GdnDesc) -> int:
    return int(lib().gdn_fwd_workspace_size(ctypes.byref(desc)))


def bwd_workspace_size(desc: GdnDesc) -> int:
    return int(lib().gdn_bwd_workspace_size(ctypes.byref(desc)))


def alloc_workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 256), dtype=torch.uint8, device=device)


def gdn_fwd(q, k, v, g, beta, cu_seqlens=None, h0=None, scale=1.0, output_final_state=True,
            o=None, hT=None, workspace=None, cu_seqlens_host=None, stream=None, piece_scan=False,
            qk_l2norm=False, value_slices=False):
    """Forward of the gated delta rule through the C ABI.  Returns (o, hT);
    hT is None when output_final_state is False.  piece_scan sets
    GDN_FLAG_PIECE_SCAN (parallel pieces of long dense rows, joined exactly);
    qk_l2norm sets GDN_FLAG_QK_L2NORM (q and k rows divided by their norms);
    value_slices sets GDN_FLAG_VALUE_SLICES (chains split by value columns)."""
    L = lib()
    cu_dev, cu_host = _seqlens(cu_seqlens, cu_seqlens_host, q.device)
    flags = ((GDN_FLAG_PIECE_SCAN if piece_scan else 0) | (GDN_FLAG_QK_L2NORM if qk_l2norm else 0)
             | (GDN_FLAG_VALUE_SLICES if value_slices else 0))
    desc, (B, T, H, K, V, n_seqs) = _desc_from(q, v, cu_host, scale, flags)
    N = n_seqs if n_seqs else B
    _check(q, "q", q.dtype, (B, T, H, K)); _check(k, "k", q.dtype, (B, T, H, K))
    _check(v, "v", q.dtype, (B, T, H, V))
    _check(g, "g", torch.float32, (B, T, H)); _check(beta, "beta", torch.float32, (B, T, H))
    _check(h0, "h0", torch.float32, (N, H, K, V))
    if o is None:
        o = torch.empty(B, T, H, V, dtype=q.dtype, device=q.device)
    if hT is None and output_final_state:
        hT = torch.empty(N, H, K, V, dtype=torch.float32, device=q.device)
    _check(o, "o", q.dtype, (B, T, H, V)); _check(hT, "hT", torch.float32, (N, H, K, V))
    need = L.gdn_fwd_workspace_size(ctypes.byref(desc))
    if need == 0:
        raise GdnError(2, "gdn_fwd_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    rc = L.gdn_fwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                   _ptr(cu_dev), None if cu_host is None else ctypes.c_void_p(cu_host.data_ptr()),
                   _ptr(h0), _ptr(o), _ptr(hT), _ptr(workspace), workspace.numel(),
                   _stream(stream))
    if rc:
        raise GdnError(rc, "gdn_fwd")
    return o, hT


def gdn_bwd(q, k, v, g, beta, do, cu_seqlens=None, h0=None, dhT=None, scale=1.0, grads=None,
            workspace=None, cu_seqlens_host=None, stream=None, want_dh0=True, qk_l2norm=False,
            piece_scan=False):
    """Backward through the C ABI.  Returns (dq, dk, dv, dg, dbeta, dh0); with
    qk_l2norm, dq and dk are the gradients w.r.t. the raw (unnormalised) q and k;
    piece_scan sets GDN_FLAG_PIECE_SCAN (both chains of long dense rows in
    parallel pieces, joined exactly)."""
    L = lib()
    cu_dev, cu_host = _seqlens(cu_seqlens, cu_seqlens_host, q.device)
    flags = (GDN_FLAG_QK_L2NORM if qk_l2norm else 0) | (GDN_FLAG_PIECE_SCAN if piece_scan else 0)
    desc, (B, T, H, K, V, n_seqs) = _desc_from(q, v, cu_host, scale, flags)
    N = n_seqs if n_seqs else B
    _check(q, "q", q.dtype, (B, T, H, K)); _check(k, "k", q.dtype, (B, T, H, K))
    _check(v, "v", q.dtype, (B, T, H, V)); _check(do, "do", q.dtype, (B, T, H, V))
    _check(g, "g", torch.float32, (B, T, H)); _check(beta, "beta", torch.float32, (B, T, H))
    _check(h0, "h0", torch.float32, (N, H, K, V)); _check(dhT, "dhT", torch.float32, (N, H, K, V))
    if grads is None:
        e = lambda *s, dt=q.dtype: torch.empty(*s, dtype=dt, device=q.device)
        grads = (e(B, T, H, K), e(B, T, H, K), e(B, T, H, V), e(B, T, H, dt=torch.float32),
                 e(B, T, H, dt=torch.float32),
                 e(N, H, K, V, dt=torch.float32) if want_dh0 else None)
    dq, dk, dv, dg, dbeta, dh0 = grads
    need = L.gdn_bwd_workspace_size(ctypes.byref(desc))
    if need == 0:
        raise GdnError(2, "gdn_bwd_workspace_size")
    if workspace is None:
        workspace = alloc_workspace(need, q.device)
    rc = L.gdn_bwd(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                   _ptr(cu_dev), None if cu_host is None else ctypes.c_void_p(cu_host.data_ptr()),
                   _ptr(h0), _ptr(do), _ptr(dhT), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg),
                   _ptr(dbeta), _ptr(dh0), _ptr(workspace), workspace.numel(), _stream(stream))
    if rc:
        raise GdnError(rc, "gdn_bwd")
    return dq, dk, dv, dg, dbeta, dh0


def gdn_decode(q, k, v, g, beta, state, scale=1.0, o=None, stream=None, qk_l2norm=False):
    """Recurrent decode through the C ABI: advances ``state`` ([B][H][dk][dv]
    fp32, updated in place) through the T tokens of q, k, v ([B][T][H][D]) and
    returns o."""
    L = lib()
    desc, (B, T, H, K, V, _) = _desc_from(q, v, None, scale,
                                         GDN_FLAG_QK_L2NORM if qk_l2norm else 0)
    _check(q, "q", q.dtype, (B, T, H, K)); _check(k, "k", q.dtype, (B, T, H, K))
    _check(v, "v", q.dtype, (B, T, H, V))
    _check(g, "g", torch.float32, (B, T, H)); _check(beta, "beta", torch.float32, (B, T, H))
    _check(state, "state", torch.float32, (B, H, K, V))
    if o is None:
        o = torch.empty(B, T, H, V, dtype=q.dtype, device=q.device)
    _check(o, "o", q.dtype, (B, T, H, V))
    rc = L.gdn_decode(ctypes.byref(desc), _ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                      _ptr(state), _ptr(o), _stream(stream))
    if rc:
        raise GdnError(rc, "gdn_decode")
    return o


def device_status(workspace, stream=None) -> int:
    return int(lib().gdn_device_status(_ptr(workspace), _stream(stream)))


def set_wait_limit(polls: int) -> None:
    """Testing hook: device-side waits of later calls from this thread give up
    after ``polls`` polls (0 restores the built-in limit)."""
    lib().gdn_set_wait_limit(int(polls))


def set_test_hook(hook: int) -> None:
    """Testing hook: plant GDN_TEST_STALL_COPY or GDN_TEST_FAIL_LAUNCH in later
    calls from this thread (0 removes it)."""
    lib().gdn_set_test_hook(int(hook))


class GdnTrace(ctypes.Structure):
    _fields_ = [("capacity", ctypes.c_int32), ("count", ctypes.c_int32),
                ("dropped", ctypes.c_int32), ("pad", ctypes.c_int32),
                ("events", ctypes.POINTER(ctypes.c_void_p)),
                ("kernel_ids", ctypes.POINTER(ctypes.c_int32))]


class LaunchTrace:
    """Records a pair of CUDA events around every library kernel launch made
    from this thread while active (``with LaunchTrace(n) as t: ...``).
    ``per_kernel()`` returns {name: (launches, total_ms)} after a sync."""

    def __init__(self, capacity: int):
        self.capacity = int(capacity)
        self.torch_events = [torch.cuda.Event(enable_timing=True)
                             for _ in range(2 * self.capacity)]
        for e in self.torch_events:  # torch creates the CUDA event on first record
            e.record()
        torch.cuda.current_stream().synchronize()
        self._ev = (ctypes.c_void_p * (2 * self.capacity))(
            *[e.cuda_event for e in self.torch_events])
        self._ids = (ctypes.c_int32 * self.capacity)()
        self.trace = GdnTrace(self.capacity, 0, 0, 0, self._ev, self._ids)

    def __enter__(self):
        lib().gdn_trace_install(ctypes.byref(self.trace))
        return self

    def __exit__(self, *exc):
        lib().gdn_trace_install(None)
        return False

    def reset(self):
        self.trace.count = 0
        self.trace.dropped = 0

    @property
    def count(self):
        return int(self.trace.count)

    def per_kernel(self):
        out = {}
        for i in range(self.trace.count):
            name = lib().gdn_kernel_name(self._ids[i]).decode()
            ms = self.torch_events[2 * i].elapsed_time(self.torch_events[2 * i + 1])
            n, t = out.get(name, (0, 0.0))
            out[name] = (n + 1, t + ms)
        return out
