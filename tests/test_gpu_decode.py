"""Recurrent decode (gdn_decode) against the fp64 oracle: one and several
tokens per call, carried state, bf16 and fp32, both head dims; a prefill by
gdn_fwd followed by decode steps equals one forward over the whole row."""
import pytest
import torch

import gated_delta_rule_99_b200 as gdn
import oracle
from gated_delta_rule_99_b200.inputs import make_inputs

from _util import maxnorm_err

pytestmark = pytest.mark.gpu
TOL = {"fp32": 1e-4, "bf16": 2e-2}


@pytest.mark.parametrize("dtype,K,V,T", [("bf16", 128, 128, 1), ("fp32", 128, 128, 1),
                                         ("bf16", 64, 128, 3), ("fp32", 128, 64, 5)])
def test_decode_matches_oracle(dtype, K, V, T):
    inp = make_inputs(B=8, T=T, H=4, K=K, V=V, dtype=dtype, seed=40 + T, h0_std=0.3, bwd=False,
                      scale=0.5)
    d = inp.to("cuda")
    state = d.h0.clone()
    o = gdn.gdn_decode(d.q, d.k, d.v, d.g, d.beta, state, scale=0.5)
    torch.cuda.synchronize()
    ro, rh = oracle.gdn_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, h0=inp.h0, scale=0.5)
    assert maxnorm_err(o, ro) <= TOL[dtype]
    assert maxnorm_err(state, rh) <= TOL[dtype]


def test_prefill_then_decode_equals_one_forward():
    T0, T1 = 200, 3
    inp = make_inputs(B=2, T=T0 + T1, H=2, K=128, V=128, dtype="fp32", seed=44, bwd=False)
    d = inp.to("cuda")
    o_all, h_all = gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, h0=d.h0)
    sl = lambda x, a, b: x[:, a:b].contiguous()
    o0, h = gdn.gdn_fwd(sl(d.q, 0, T0), sl(d.k, 0, T0), sl(d.v, 0, T0), sl(d.g, 0, T0),
                        sl(d.beta, 0, T0), h0=d.h0)
    outs = []
    for t in range(T0, T0 + T1):
        outs.append(gdn.gdn_decode(sl(d.q, t, t + 1), sl(d.k, t, t + 1), sl(d.v, t, t + 1),
                                   sl(d.g, t, t + 1), sl(d.beta, t, t + 1), h))
    torch.cuda.synchronize()
    assert maxnorm_err(torch.cat(outs, 1), o_all[:, T0:]) <= 1e-5
    assert maxnorm_err(h, h_all) <= 1e-5
