"""Helpers shared by the tests (comparison metrics and oracle calls on sampled units)."""
import numpy as np
import torch

import oracle


def np64(t):
    if t is None:
        return None
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").double().numpy()
    return np.asarray(t, dtype=np.float64)


def maxnorm_err(x, ref):
    """max_i |x_i - ref_i| / max_i |ref_i| over the finite entries of ref."""
    x, ref = np64(x), np64(ref)
    m = np.isfinite(ref)
    assert m.any()
    assert np.isfinite(x[m]).all(), "non-finite values in the CUDA result"
    den = np.max(np.abs(ref[m]))
    return float(np.max(np.abs(x[m] - ref[m])) / (den if den > 0 else 1.0))


def oracle_fwd(inp, units=None):
    return oracle.gdn_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, cu_seqlens=inp.cu_seqlens,
                          h0=inp.h0, scale=inp.scale, units=units)


def oracle_bwd(inp, units=None):
    return oracle.gdn_bwd(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.do, cu_seqlens=inp.cu_seqlens,
                          h0=inp.h0, dhT=inp.dhT, scale=inp.scale, units=units)


def unit_mask(inp, units, kind):
    """Boolean mask over a (B,T,H,...) or (N,H,...) array selecting the sampled units."""
    B, T, H = inp.q.shape[:3]
    if inp.cu_seqlens is None:
        segs = [(b, 0, T) for b in range(B)]
    else:
        cu = inp.cu_seqlens.tolist()
        segs = [(0, cu[i], cu[i + 1]) for i in range(len(cu) - 1)]
    if kind == "state":
        m = np.zeros((len(segs), H), dtype=bool)
        for n, h in units:
            m[n, h] = True
        return m
    m = np.zeros((B, T, H), dtype=bool)
    for n, h in units:
        b, t0, t1 = segs[n]
        m[b, t0:t1, h] = True
    return m
