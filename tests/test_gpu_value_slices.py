"""The forward chains by value slices (GDN_FLAG_VALUE_SLICES: each (sequence,
head) chain split over two CTAs of 64 value columns, the d_v slicing the
chunkwise form allows because the rows of S evolve independently).  Checked
against the fp64 oracle on every element of small ragged and packed cases and
of both head-dim mixes, on sampled units of the full-size forward workload,
with the piece scan, and bitwise for chained halves and run-to-run."""
import pytest
import torch

import gated_delta_rule_99_b200 as gdn
from gated_delta_rule_99_b200.inputs import make_inputs, workload

from _util import maxnorm_err, oracle_fwd

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _fwd(inp, **kw):
    d = inp.to("cuda")
    cu = None if d.cu_seqlens is None else d.cu_seqlens
    o, hT = gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, cu_seqlens=cu, h0=d.h0, scale=d.scale,
                        value_slices=True, **kw)
    torch.cuda.synchronize()
    return o, hT


def _check(inp, units=None, **kw):
    o, hT = _fwd(inp, **kw)
    ro, rh = oracle_fwd(inp, units)
    errs = {"o": maxnorm_err(o, ro), "hT": maxnorm_err(hT, rh)}
    print("value slices %s: %s" % (inp.meta.get("name", ""), errs))
    assert max(errs.values()) <= TOL, errs


@pytest.mark.parametrize("K,V", [(128, 128), (64, 128), (128, 64), (64, 64)])
def test_value_slices_packed_ragged(K, V):
    lengths = [1, 0, 63, 64, 65, 130, 7, 200]
    _check(make_inputs(B=1, T=sum(lengths), H=3, K=K, V=V, dtype="bf16", seed=70 + K + V,
                       lengths=lengths, scale=0.25, bwd=False))


def test_value_slices_dense_rows_with_tail_and_strong_decay():
    inp = make_inputs(B=2, T=300, H=2, K=128, V=128, dtype="bf16", seed=71, gate_scale=3.0,
                      bwd=False)
    inp.g[:, 77] = -30.0
    _check(inp)


def test_value_slices_full_size_forward_sampled():
    _check(workload(1), units=[(0, 0), (3, 15), (1, 7)])


def test_value_slices_with_piece_scan():
    _check(make_inputs(B=1, T=16384, H=2, K=128, V=128, dtype="bf16", seed=72, bwd=False),
           piece_scan=True)


def test_value_slices_chained_halves_and_reruns_bitwise():
    inp = make_inputs(B=2, T=1024, H=3, K=128, V=128, dtype="bf16", seed=73, bwd=False)
    d = inp.to("cuda")
    sl = lambda x, a, b: x[:, a:b].contiguous()
    f = lambda q, k, v, g, b, h0: gdn.gdn_fwd(q, k, v, g, b, h0=h0, value_slices=True)
    o, hT = f(d.q, d.k, d.v, d.g, d.beta, d.h0)
    o2, hT2 = f(d.q, d.k, d.v, d.g, d.beta, d.h0)
    oa, ha = f(sl(d.q, 0, 512), sl(d.k, 0, 512), sl(d.v, 0, 512), sl(d.g, 0, 512),
               sl(d.beta, 0, 512), d.h0)
    ob, hb = f(sl(d.q, 512, 1024), sl(d.k, 512, 1024), sl(d.v, 512, 1024), sl(d.g, 512, 1024),
               sl(d.beta, 512, 1024), ha)
    torch.cuda.synchronize()
    assert torch.equal(o, o2) and torch.equal(hT, hT2)
    assert torch.equal(o[:, :512], oa) and torch.equal(o[:, 512:], ob) and torch.equal(hT, hb)
