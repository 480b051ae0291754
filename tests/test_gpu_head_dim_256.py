"""GPU parity at head dim 256 (the key dim of the gdn-1p3b preset, whose K = 256
kernels jax-linear-attention 0.1.0 names in "Benchmarks", note (d)): these
shapes run on the fp32 CUDA-core kernels for both dtypes, whose chunk tiles
then have 256-float rows.  Every element is compared with the fp64 oracle, forward and backward,
on ragged lengths (a partial last chunk), packed documents (lengths 0, 1, 63,
64, 65), mixed head dims and strong decay, with initial and final states.
"""
import pytest
import torch

import gated_delta_rule_99_b200 as gdn
from gated_delta_rule_99_b200.inputs import make_inputs

from _util import maxnorm_err, oracle_bwd, oracle_fwd

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _check(inp, tol, bwd=True):
    d = inp.to("cuda")
    cu = d.cu_seqlens
    with gdn.LaunchTrace(64) as tr:
        o, hT = gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, cu_seqlens=cu, h0=d.h0, scale=d.scale)
        got = None
        if bwd:
            got = gdn.gdn_bwd(d.q, d.k, d.v, d.g, d.beta, d.do, cu_seqlens=cu, h0=d.h0,
                              dhT=d.dhT, scale=d.scale)
        torch.cuda.synchronize()
    names = set(tr.per_kernel())
    assert names and all(n.startswith(("simt_", "build_chunks")) for n in names), names
    ro, rh = oracle_fwd(inp)
    errs = {"o": maxnorm_err(o, ro), "hT": maxnorm_err(hT, rh)}
    if bwd:
        for name, a, b in zip(("dq", "dk", "dv", "dg", "dbeta", "dh0"), got, oracle_bwd(inp)):
            errs[name] = maxnorm_err(a, b)
    print("parity d256 %s: %s" % (inp.meta.get("dtype"), " ".join("%s=%.2e" % kv for kv in errs.items())))
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, (errs, tol)


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_head_dim_256_forward_backward(dtype):
    inp = make_inputs(B=2, T=200, H=2, K=256, V=256, dtype=dtype, seed=40)
    _check(inp, TOL[dtype])


@pytest.mark.parametrize("dtype,K,V", [("bf16", 256, 128), ("fp32", 128, 256), ("bf16", 64, 256)])
def test_head_dim_256_mixed_with_smaller_dims(dtype, K, V):
    inp = make_inputs(B=1, T=150, H=3, K=K, V=V, dtype=dtype, seed=41, scale=0.0625)
    _check(inp, TOL[dtype])


def test_head_dim_256_packed_documents():
    lengths = [1, 0, 63, 64, 65, 130]
    inp = make_inputs(B=1, T=sum(lengths), H=2, K=256, V=256, dtype="bf16", seed=42,
                      lengths=lengths)
    _check(inp, TOL["bf16"])


def test_head_dim_256_strong_decay_over_several_chunks():
    inp = make_inputs(B=1, T=300, H=1, K=256, V=256, dtype="fp32", seed=43, gate_scale=3.0)
    _check(inp, TOL["fp32"])


def test_head_dim_256_ignores_the_tensor_core_options():
    """The value-slices and piece-scan options apply to the tensor-core kernels
    only: at head dim 256 the results are bitwise those of the default call."""
    inp = make_inputs(B=1, T=1100, H=2, K=256, V=256, dtype="bf16", seed=44)
    d = inp.to("cuda")
    base = gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, h0=d.h0)
    for kw in (dict(value_slices=True), dict(piece_scan=True)):
        o, hT = gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, h0=d.h0, **kw)
        assert torch.equal(o, base[0]) and torch.equal(hT, base[1]), kw
    g0 = gdn.gdn_bwd(d.q, d.k, d.v, d.g, d.beta, d.do, h0=d.h0, dhT=d.dhT)
    g1 = gdn.gdn_bwd(d.q, d.k, d.v, d.g, d.beta, d.do, h0=d.h0, dhT=d.dhT, piece_scan=True)
    assert all(torch.equal(a, b) for a, b in zip(g0, g1))
