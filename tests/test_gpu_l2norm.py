"""The layer's own q/k normalisation (GDN_FLAG_QK_L2NORM; the pages' API
option use_qk_l2norm, read as x / |x| per token and head) against the fp64
oracle with the same option: the fused tensor-core path (bf16, d = 128), the
normalisation/projection passes of the other paths, decode, and full size."""
import pytest
import torch

import gated_delta_rule_99_b200 as gdn
import oracle
from gated_delta_rule_99_b200.inputs import WORKLOADS, make_inputs

from _util import maxnorm_err

pytestmark = pytest.mark.gpu
TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _check(inp, tol, units=None):
    d = inp.to("cuda")
    cu = d.cu_seqlens
    o, hT = gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, cu_seqlens=cu, h0=d.h0, scale=d.scale,
                        qk_l2norm=True)
    got = gdn.gdn_bwd(d.q, d.k, d.v, d.g, d.beta, d.do, cu_seqlens=cu, h0=d.h0, dhT=d.dhT,
                      scale=d.scale, qk_l2norm=True)
    torch.cuda.synchronize()
    kw = dict(cu_seqlens=inp.cu_seqlens, h0=inp.h0, scale=inp.scale, units=units, qk_l2norm=True)
    ro, rh = oracle.gdn_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, **kw)
    ref = oracle.gdn_bwd(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.do, dhT=inp.dhT, **kw)
    errs = {"o": maxnorm_err(o, ro), "hT": maxnorm_err(hT, rh)}
    for name, a, b in zip(("dq", "dk", "dv", "dg", "dbeta", "dh0"), got, ref):
        errs[name] = maxnorm_err(a, b)
    print("l2norm parity:", " ".join("%s=%.2e" % kv for kv in errs.items()))
    assert all(e <= tol for e in errs.values()), errs
    return o, got


def test_tensor_core_path_packed_ragged():
    lengths = [1, 0, 63, 64, 65, 130, 7, 200]
    inp = make_inputs(B=1, T=sum(lengths), H=3, K=128, V=128, dtype="bf16", seed=61,
                      lengths=lengths, raw_qk=True, scale=0.5)
    _check(inp, TOL["bf16"])


@pytest.mark.parametrize("dtype,K,V", [("fp32", 64, 128), ("bf16", 64, 64), ("fp32", 128, 64),
                                       ("bf16", 128, 64), ("bf16", 256, 256), ("fp32", 256, 128)])
def test_other_head_dims_and_fp32(dtype, K, V):
    inp = make_inputs(B=2, T=150, H=2, K=K, V=V, dtype=dtype, seed=62, raw_qk=True)
    _check(inp, TOL[dtype])


def test_many_units_per_cta_head_dim_64():
    """Packed ragged documents with more (chunk, head) units than SMs at d_k = 64:
    the persistent gradient kernel's prefetched q/k tiles are normalised and
    padded per unit."""
    import numpy as np
    lengths = [int(x) for x in np.random.default_rng(65).integers(1, 151, size=48)]
    inp = make_inputs(B=1, T=sum(lengths), H=8, K=64, V=128, dtype="bf16", seed=65,
                      lengths=lengths, raw_qk=True)
    _check(inp, TOL["bf16"])


def test_zero_rows_and_gradients_orthogonal_to_rows():
    inp = make_inputs(B=1, T=130, H=2, K=128, V=128, dtype="bf16", seed=63, raw_qk=True)
    inp.q[0, 5] = 0
    inp.k[0, 9] = 0
    o, (dq, dk, *_) = _check(inp, TOL["bf16"])
    assert torch.count_nonzero(o[0, 5]) == 0
    assert torch.count_nonzero(dq[0, 5]) == 0 and torch.count_nonzero(dk[0, 9]) == 0
    # a gradient row is orthogonal to its input row (the output is scale invariant)
    q, k = inp.q.float().cuda(), inp.k.float().cuda()
    rel = lambda g, x: ((g.float() * x).sum(-1).abs() /
                        (g.float().norm(dim=-1) * x.norm(dim=-1) + 1e-30)).max().item()
    assert rel(dq, q) < 2e-2 and rel(dk, k) < 2e-2


def test_decode():
    inp = make_inputs(B=8, T=3, H=4, K=128, V=128, dtype="bf16", seed=64, h0_std=0.3,
                      bwd=False, raw_qk=True)
    d = inp.to("cuda")
    state = d.h0.clone()
    o = gdn.gdn_decode(d.q, d.k, d.v, d.g, d.beta, state, qk_l2norm=True)
    torch.cuda.synchronize()
    ro, rh = oracle.gdn_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, h0=inp.h0, qk_l2norm=True)
    assert maxnorm_err(o, ro) <= TOL["bf16"] and maxnorm_err(state, rh) <= TOL["bf16"]


def test_full_size_sampled():
    w = dict(WORKLOADS[2], raw_qk=True, bwd=True)  # B=4 T=4096 H=16 d=128 bf16, raw q and k
    _check(make_inputs(**w), TOL["bf16"], units=[(0, 0), (3, 15), (2, 9)])
