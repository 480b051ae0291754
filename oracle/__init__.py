"""fp64 CPU oracle for the Gated DeltaNet layer (forward and backward).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's CPU
baseline leg are the only callers.  The product package never imports this
module and this module never imports the product package; the two share only
the seeded input generator, which holds none of the method's arithmetic.

``gdn_ref.c`` holds the token-by-token recurrence (the definition the pages
hold every kernel to: jax-linear-attention 0.1.0, "How it works").  This
module gathers per-(document, head) units out of (B, T, H, D) arrays, runs the
C code over them in threads and scatters the results back.  ``chunked.py`` is
an independent fp64 restatement of the chunkwise algebra, used only to pin the
algebra against the token recurrence.

Parity pins: every function here is pinned by the ``-m "not gpu"`` tests in
``tests/test_oracle_pins.py`` (closed forms, invariants, brute force, finite
differences).  The pages print no worked numeric example for this method.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_ref.c")
_SO = os.path.join(_HERE, "libgdn_ref.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile gdn_ref.c into libgdn_ref.so next to it (plain gcc, IEEE fp64)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + ".tmp%d" % os.getpid()
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-pthread",
                               "-ffp-contract=off", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


class _Unit(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int64)] + [
        (n, ctypes.c_void_p) for n in
        ("q", "k", "v", "g", "beta", "h0", "o", "hT", "do_", "dhT",
         "dq", "dk", "dv", "dg", "dbeta", "dh0")]


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            for name in ("gdn_ref_fwd", "gdn_ref_bwd"):
                f = getattr(lib, name)
                f.restype = ctypes.c_int
                f.argtypes = [ctypes.POINTER(_Unit), ctypes.c_int, ctypes.c_int64,
                              ctypes.c_int64, ctypes.c_double, ctypes.c_int]
            _lib = lib
    return _lib


def default_threads() -> int:
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:  # pragma: no cover
        return os.cpu_count() or 1


def _segments(B, T, cu_seqlens):
    """List of (row b, token start, token end) per sequence; dense rows when cu_seqlens is None."""
    if cu_seqlens is None:
        return [(b, 0, T) for b in range(B)]
    cu = [int(x) for x in np.asarray(cu_seqlens).reshape(-1)]
    assert B == 1 and cu[0] == 0 and cu[-1] == T
    assert all(cu[i] <= cu[i + 1] for i in range(len(cu) - 1))
    return [(0, cu[i], cu[i + 1]) for i in range(len(cu) - 1)]


def _f64(x):
    """Contiguous fp64 numpy copy of a numpy array or a CPU torch tensor (bf16 upcasts exactly)."""
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _shape(x):
    return tuple(x.shape)


def _ptr(a):
    return None if a is None else a.ctypes.data


def _l2norm_rows(x):
    """Rows of x divided by their Euclidean norm (a zero row stays zero), and the norms.

    The optional normalisation of q and k per token and head that the layer
    applies itself when asked (jax-linear-attention 0.1.0, "Quick start":
    ``use_qk_l2norm=True``); the pages give no formula, so this is the plain
    x / sqrt(sum x^2)."""
    n = np.sqrt(np.sum(x * x, axis=-1, keepdims=True))
    return np.where(n > 0, x / np.where(n > 0, n, 1.0), 0.0), n


def _l2norm_back(xh, n, dxh):
    """Gradient w.r.t. the raw rows from the gradient w.r.t. the normalised rows
    xh = x / |x|:  dx = (dxh - xh (xh . dxh)) / |x|  (zero for a zero row)."""
    proj = dxh - xh * np.sum(xh * dxh, axis=-1, keepdims=True)
    return np.where(n > 0, proj / np.where(n > 0, n, 1.0), 0.0)


def gdn_fwd(q, k, v, g, beta, cu_seqlens=None, h0=None, scale=1.0, units=None, nthreads=None,
            qk_l2norm=False):
    """Token-by-token forward.  q,k: (B,T,H,K); v: (B,T,H,V); g, beta: (B,T,H);
    h0: (N,H,K,V) or None.  Returns o (B,T,H,V) and hT (N,H,K,V) in fp64.

    ``units``: optional iterable of (sequence, head) pairs to compute; the
    other entries of o and hT are left NaN (used for sampled parity).
    ``qk_l2norm``: normalise every q and k row first (see ``_l2norm_rows``)."""
    B, T, H, K = _shape(q)
    V = _shape(v)[-1]
    segs = _segments(B, T, cu_seqlens)
    N = len(segs)
    o = np.full((B, T, H, V), np.nan)
    hT = np.full((N, H, K, V), np.nan)
    sel = [(n, h) for n in range(N) for h in range(H)] if units is None else list(units)
    keep, arr = [], (_Unit * max(1, len(sel)))()
    for i, (n, h) in enumerate(sel):
        b, t0, t1 = segs[n]
        L = t1 - t0
        qu, ku = _f64(q[b, t0:t1, h]), _f64(k[b, t0:t1, h])
        if qk_l2norm:
            qu, ku = np.ascontiguousarray(_l2norm_rows(qu)[0]), np.ascontiguousarray(_l2norm_rows(ku)[0])
        bufs = dict(q=qu, k=ku, v=_f64(v[b, t0:t1, h]),
                    g=_f64(g[b, t0:t1, h]), beta=_f64(beta[b, t0:t1, h]),
                    h0=None if h0 is None else _f64(h0[n, h]),
                    o=np.zeros((max(L, 1), V)), hT=np.zeros((K, V)))
        keep.append(bufs)
        arr[i] = _Unit(L, *[_ptr(bufs.get(f)) for f in
                            ("q", "k", "v", "g", "beta", "h0", "o", "hT")], *([None] * 8))
    rc = _load().gdn_ref_fwd(arr, len(sel), K, V, float(scale), nthreads or default_threads())
    if rc:
        raise MemoryError("oracle forward failed (%d)" % rc)
    for (n, h), bufs in zip(sel, keep):
        b, t0, t1 = segs[n]
        o[b, t0:t1, h] = bufs["o"][: t1 - t0]
        hT[n, h] = bufs["hT"]
    return o, hT


def gdn_bwd(q, k, v, g, beta, do, cu_seqlens=None, h0=None, dhT=None, scale=1.0, units=None,
            nthreads=None, qk_l2norm=False):
    """Token-by-token backward of o and hT with upstream gradients do (B,T,H,V)
    and dhT (N,H,K,V) or None.  Returns dq, dk, dv, dg, dbeta, dh0 in fp64.
    With ``qk_l2norm`` dq and dk are the gradients w.r.t. the raw (unnormalised)
    q and k."""
    B, T, H, K = _shape(q)
    V = _shape(v)[-1]
    segs = _segments(B, T, cu_seqlens)
    N = len(segs)
    out = dict(dq=np.full((B, T, H, K), np.nan), dk=np.full((B, T, H, K), np.nan),
               dv=np.full((B, T, H, V), np.nan), dg=np.full((B, T, H), np.nan),
               dbeta=np.full((B, T, H), np.nan), dh0=np.full((N, H, K, V), np.nan))
    sel = [(n, h) for n in range(N) for h in range(H)] if units is None else list(units)
    keep, arr = [], (_Unit * max(1, len(sel)))()
    for i, (n, h) in enumerate(sel):
        b, t0, t1 = segs[n]
        L = max(t1 - t0, 1)
        c = _f64
        qu, ku = c(q[b, t0:t1, h]), c(k[b, t0:t1, h])
        if qk_l2norm:
            (qu, qn), (ku, kn) = _l2norm_rows(qu), _l2norm_rows(ku)
            qu, ku = np.ascontiguousarray(qu), np.ascontiguousarray(ku)
        bufs = dict(q=qu, k=ku, v=c(v[b, t0:t1, h]),
                    g=c(g[b, t0:t1, h]), beta=c(beta[b, t0:t1, h]),
                    h0=None if h0 is None else c(h0[n, h]),
                    do_=c(do[b, t0:t1, h]), dhT=None if dhT is None else c(dhT[n, h]),
                    dq=np.zeros((L, K)), dk=np.zeros((L, K)), dv=np.zeros((L, V)),
                    dg=np.zeros(L), dbeta=np.zeros(L), dh0=np.zeros((K, V)))
        if qk_l2norm:
            bufs["norms"] = (qn, kn)
        keep.append(bufs)
        arr[i] = _Unit(t1 - t0, _ptr(bufs["q"]), _ptr(bufs["k"]), _ptr(bufs["v"]), _ptr(bufs["g"]),
                       _ptr(bufs["beta"]), _ptr(bufs["h0"]), None, None, _ptr(bufs["do_"]),
                       _ptr(bufs["dhT"]), _ptr(bufs["dq"]), _ptr(bufs["dk"]), _ptr(bufs["dv"]),
                       _ptr(bufs["dg"]), _ptr(bufs["dbeta"]), _ptr(bufs["dh0"]))
    rc = _load().gdn_ref_bwd(arr, len(sel), K, V, float(scale), nthreads or default_threads())
    if rc:
        raise MemoryError("oracle backward failed (%d)" % rc)
    for (n, h), bufs in zip(sel, keep):
        b, t0, t1 = segs[n]
        L = t1 - t0
        if qk_l2norm and L > 0:
            qn, kn = bufs["norms"]
            bufs["dq"][:L] = _l2norm_back(bufs["q"], qn, bufs["dq"][:L])
            bufs["dk"][:L] = _l2norm_back(bufs["k"], kn, bufs["dk"][:L])
        for name in ("dq", "dk", "dv"):
            out[name][b, t0:t1, h] = bufs[name][:L]
        out["dg"][b, t0:t1, h] = bufs["dg"][:L]
        out["dbeta"][b, t0:t1, h] = bufs["dbeta"][:L]
        out["dh0"][n, h] = bufs["dh0"]
    return out["dq"], out["dk"], out["dv"], out["dg"], out["dbeta"], out["dh0"]
