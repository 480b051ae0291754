"""Failure paths on the GPU, driven by the testing hooks of include/gdn.h and
never by a fault: a device-side wait that runs out (an input-copy mbarrier
armed for 16 bytes more than its copies bring, so it cannot complete although
every copy has landed) must come back as GDN_ERR_TIMEOUT through
gdn_device_status, and a failed launch (planted on the host: the launch is
skipped and reported as failed) as GDN_ERR_CUDA.  After either, the next
ordinary call on the same workspace must succeed and match the oracle (the
fail-closed behaviour of jax-linear-attention 0.1.0, "How it works")."""
import pytest
import torch

import gated_delta_rule_99_b200 as gdn
from gated_delta_rule_99_b200.inputs import make_inputs

from _util import maxnorm_err, oracle_bwd, oracle_fwd

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}
WHERE_PREP_COPIES = 31  # the tag the preparation step records when its copy wait gives up


def _calls(d, ws, cu_dev=None, cu_host=None):
    o, hT = gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, cu_seqlens=cu_dev, cu_seqlens_host=cu_host,
                        h0=d.h0, scale=d.scale, workspace=ws)
    grads = gdn.gdn_bwd(d.q, d.k, d.v, d.g, d.beta, d.do, cu_seqlens=cu_dev,
                        cu_seqlens_host=cu_host, h0=d.h0, dhT=d.dhT, scale=d.scale,
                        workspace=ws)
    return (o, hT) + tuple(grads)


def _check_against_oracle(inp, got, tol):
    ro, rh = oracle_fwd(inp)
    ref = (ro, rh) + tuple(oracle_bwd(inp))
    errs = {n: maxnorm_err(a, b) for n, a, b in
            zip(("o", "hT", "dq", "dk", "dv", "dg", "dbeta", "dh0"), got, ref)}
    assert max(errs.values()) <= tol, errs


def _workspace(inp):
    B, T, H, K = inp.q.shape
    n = 0 if inp.cu_seqlens is None else inp.n_seqs
    dt = gdn.GDN_BF16 if inp.q.dtype == torch.bfloat16 else gdn.GDN_FP32
    desc = gdn.make_desc(B, T, H, K, inp.v.shape[-1], n, dt, inp.scale)
    return gdn.alloc_workspace(max(gdn.fwd_workspace_size(desc), gdn.bwd_workspace_size(desc)),
                               "cuda")


@pytest.mark.parametrize("packed", [False, True])
def test_device_wait_runs_out_then_next_call_recovers(packed):
    lengths = [70, 0, 129, 101] if packed else None
    inp = make_inputs(B=1 if packed else 2, T=300, H=2, K=128, V=128, dtype="bf16", seed=41,
                      lengths=lengths)
    d = inp.to("cuda")
    cu_host = inp.cu_seqlens
    cu_dev = None if cu_host is None else cu_host.cuda()
    ws = _workspace(inp)
    gdn.set_wait_limit(1 << 14)
    gdn.set_test_hook(gdn.GDN_TEST_STALL_COPY)
    try:
        gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, cu_seqlens=cu_dev, cu_seqlens_host=cu_host,
                    h0=d.h0, workspace=ws)
        assert gdn.device_status(ws) == 6  # GDN_ERR_TIMEOUT
        assert int(ws[8:12].view(torch.int32).item()) == WHERE_PREP_COPIES
        assert gdn.device_status(ws) == 0  # read and cleared
        gdn.gdn_bwd(d.q, d.k, d.v, d.g, d.beta, d.do, cu_seqlens=cu_dev, cu_seqlens_host=cu_host,
                    h0=d.h0, dhT=d.dhT, workspace=ws)
        assert gdn.device_status(ws) == 6
        assert int(ws[8:12].view(torch.int32).item()) == WHERE_PREP_COPIES
    finally:
        gdn.set_test_hook(0)
        gdn.set_wait_limit(0)
    got = _calls(d, ws, cu_dev, cu_host)
    assert gdn.device_status(ws) == 0
    _check_against_oracle(inp, got, TOL["bf16"])


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_planted_launch_failure_returns_cuda_error_then_recovers(dtype):
    inp = make_inputs(B=1, T=150, H=2, K=64, V=128, dtype=dtype, seed=42, lengths=[40, 110])
    d = inp.to("cuda")
    cu_host = inp.cu_seqlens
    cu_dev = cu_host.cuda()
    ws = _workspace(inp)
    state = torch.zeros(1, 2, 64, 128, device="cuda")
    gdn.set_test_hook(gdn.GDN_TEST_FAIL_LAUNCH)
    try:
        with pytest.raises(gdn.GdnError) as e:
            gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, cu_seqlens=cu_dev, cu_seqlens_host=cu_host,
                        h0=d.h0, workspace=ws)
        assert e.value.code == 5  # GDN_ERR_CUDA
        with pytest.raises(gdn.GdnError) as e:
            gdn.gdn_bwd(d.q, d.k, d.v, d.g, d.beta, d.do, cu_seqlens=cu_dev,
                        cu_seqlens_host=cu_host, h0=d.h0, dhT=d.dhT, workspace=ws)
        assert e.value.code == 5
        with pytest.raises(gdn.GdnError) as e:
            gdn.gdn_decode(d.q[:, :1].contiguous(), d.k[:, :1].contiguous(),
                           d.v[:, :1].contiguous(), d.g[:, :1].contiguous(),
                           d.beta[:, :1].contiguous(), state)
        assert e.value.code == 5
    finally:
        gdn.set_test_hook(0)
    torch.cuda.synchronize()  # nothing was launched, so nothing failed on the device
    got = _calls(d, ws, cu_dev, cu_host)
    assert gdn.device_status(ws) == 0
    _check_against_oracle(inp, got, TOL[dtype])
