"""Piece scan of long rows (GDN_FLAG_PIECE_SCAN): pieces of a dense row run in
parallel and are joined through each piece's exact affine map (transition and
offset).  Checked against the fp64 oracle and against the default sequential
path; the two paths differ only by the bf16 rounding of the transition
matrices."""
import numpy as np
import pytest
import torch

import gated_delta_rule_99_b200 as gdn
import oracle
from gated_delta_rule_99_b200.inputs import make_inputs, workload

from _util import maxnorm_err, np64

pytestmark = pytest.mark.gpu
TOL = 2e-2


def _fwd(d, piece_scan):
    o, hT = gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, h0=d.h0, scale=d.scale,
                        piece_scan=piece_scan)
    torch.cuda.synchronize()
    return o, hT


@pytest.mark.parametrize("B,T,H,gate", [(1, 16384, 2, 0.1), (2, 64 * 50 + 17, 1, 0.02),
                                        (1, 8192, 1, 0.005)])
def test_piece_scan_matches_oracle_and_default_path(B, T, H, gate):
    inp = make_inputs(B=B, T=T, H=H, K=128, V=128, dtype="bf16", seed=60 + H, gate_scale=gate,
                      bwd=False)
    d = inp.to("cuda")
    o_p, h_p = _fwd(d, True)
    o_s, h_s = _fwd(d, False)
    ro, rh = oracle.gdn_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, h0=inp.h0)
    errs = dict(o=maxnorm_err(o_p, ro), hT=maxnorm_err(h_p, rh),
                o_vs_seq=maxnorm_err(o_p, np64(o_s)), hT_vs_seq=maxnorm_err(h_p, np64(h_s)))
    print("piece scan B=%d T=%d H=%d: %s" % (B, T, H, errs))
    assert max(errs.values()) <= TOL, errs


def test_piece_scan_long_context_workload():
    """The long-row workload on the piece scan equals the default sequential
    path up to the bf16 rounding of the transition matrices (both are checked
    against the fp64 oracle over the whole row in
    test_gpu_parity.py::test_long_context_full_row_against_oracle)."""
    inp = workload(4, device="cuda")
    o_p, h_p = _fwd(inp, True)
    o_s, h_s = _fwd(inp, False)
    e_o = maxnorm_err(o_p.float(), o_s.float().cpu().numpy().astype(np.float64))
    e_h = maxnorm_err(h_p, h_s.cpu().numpy().astype(np.float64))
    print("piece scan long row: o vs sequential %.2e, hT vs sequential %.2e" % (e_o, e_h))
    assert e_o <= TOL and e_h <= TOL


def _bwd(d, piece_scan):
    r = gdn.gdn_bwd(d.q, d.k, d.v, d.g, d.beta, d.do, h0=d.h0, dhT=d.dhT, scale=d.scale,
                    piece_scan=piece_scan)
    torch.cuda.synchronize()
    return r


@pytest.mark.parametrize("B,T,H,gate", [(1, 16384, 2, 0.1), (2, 64 * 50 + 17, 1, 0.02),
                                        (1, 8192, 1, 0.005)])
def test_piece_scan_backward_matches_oracle_and_default_path(B, T, H, gate):
    """gdn_bwd with both chains split into pieces: every gradient against the
    fp64 oracle, and against the default backward (they differ only by the bf16
    rounding of the pieces' transition matrices)."""
    inp = make_inputs(B=B, T=T, H=H, K=128, V=128, dtype="bf16", seed=80 + H, gate_scale=gate,
                      scale=0.125)
    d = inp.to("cuda")
    got = _bwd(d, True)
    seq = _bwd(d, False)
    ref = oracle.gdn_bwd(inp.q, inp.k, inp.v, inp.g, inp.beta, inp.do, h0=inp.h0, dhT=inp.dhT,
                         scale=inp.scale)
    errs = {}
    for name, a, b, c in zip(("dq", "dk", "dv", "dg", "dbeta", "dh0"), got, ref, seq):
        errs[name] = maxnorm_err(a, b)
        errs[name + "_vs_seq"] = maxnorm_err(a, np64(c))
    print("piece scan backward B=%d T=%d H=%d: %s" % (B, T, H, errs))
    assert max(errs.values()) <= TOL, errs
