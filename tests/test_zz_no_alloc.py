"""gdn_fwd_noalloc: the forward for callers that cannot allocate device memory
(a process whose HBM is all held by a fixed pool, a plugin given only its
input and output buffers).  It runs on a static scratch array inside the
library; this test calls it through the C ABI twice in a row, on different
inputs, and checks each result against gdn_fwd with a caller workspace.  The
file sorts last so a failure here comes after every other test has run."""
import ctypes

import pytest
import torch

import gated_delta_rule_99_b200 as gdn
from gated_delta_rule_99_b200.inputs import make_inputs

from _util import maxnorm_err

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def _noalloc(d, cu_dev, cu_host, o, hT):
    L = gdn.lib()
    B, T, H, K = d.q.shape
    V = d.v.shape[-1]
    n = 0 if cu_host is None else cu_host.numel() - 1
    dt = gdn.GDN_BF16 if d.q.dtype == torch.bfloat16 else gdn.GDN_FP32
    desc = gdn.make_desc(B, T, H, K, V, n, dt, d.scale)
    p = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    return L.gdn_fwd_noalloc(ctypes.byref(desc), p(d.q), p(d.k), p(d.v), p(d.g), p(d.beta),
                             p(cu_dev), p(cu_host), p(d.h0), p(o), p(hT),
                             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


@pytest.mark.parametrize("dtype", ["bf16", "fp32"])
def test_noalloc_matches_workspace_forward_twice(dtype):
    cases = [make_inputs(B=1, T=333, H=2, K=128, V=128, dtype=dtype, seed=31,
                         lengths=[100, 0, 197, 36]),
             make_inputs(B=2, T=200, H=3, K=64, V=128, dtype=dtype, seed=32)]
    for inp in cases:
        d = inp.to("cuda")
        cu_host = inp.cu_seqlens
        cu_dev = None if cu_host is None else cu_host.cuda()
        ref_o, ref_h = gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, cu_seqlens=cu_dev,
                                   cu_seqlens_host=cu_host, h0=d.h0, scale=d.scale)
        o = torch.full_like(ref_o, float("nan"))
        hT = torch.full_like(ref_h, float("nan"))
        rc = _noalloc(d, cu_dev, cu_host, o, hT)
        assert rc == 0, gdn.lib().gdn_status_string(rc)
        torch.cuda.synchronize()
        assert maxnorm_err(o, ref_o) <= TOL[dtype]
        assert maxnorm_err(hT, ref_h) <= TOL[dtype]


def test_noalloc_rejects_problems_beyond_its_scratch():
    desc = gdn.make_desc(4, 4096, 16, 128, 128, 0, gdn.GDN_FP32)
    assert gdn.fwd_workspace_size(desc) > 64 * 1024 * 1024
    buf = torch.zeros(64, device="cuda")  # never read: the size check fails first
    p = ctypes.c_void_p(buf.data_ptr())
    rc = gdn.lib().gdn_fwd_noalloc(ctypes.byref(desc), p, p, p, p, p, None, None, None, p, None,
                                   ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 4  # GDN_ERR_WORKSPACE, returned before any launch


def test_noalloc_status_reports_and_clears_device_side_failures():
    """The device-side status of gdn_fwd_noalloc lives in the library's static
    scratch; gdn_fwd_noalloc_status reads and clears it.  A device copy of
    cu_seqlens that disagrees with the host mirror is caught on the device."""
    inp = make_inputs(B=1, T=200, H=1, K=64, V=64, dtype="bf16", seed=19, lengths=[100, 100])
    d = inp.to("cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    L = gdn.lib()
    o = torch.empty_like(d.v)
    hT = torch.empty(2, 1, 64, 64, device="cuda")
    bad_dev = torch.tensor([0, 201, 200], dtype=torch.int32, device="cuda")
    assert _noalloc(d, bad_dev, inp.cu_seqlens, o, hT) == 0  # accepted on the host
    assert L.gdn_fwd_noalloc_status(stream) == 1             # GDN_ERR_INVALID_ARG on the device
    assert L.gdn_fwd_noalloc_status(stream) == 0             # cleared by the read
    assert _noalloc(d, inp.cu_seqlens.cuda(), inp.cu_seqlens, o, hT) == 0
    assert L.gdn_fwd_noalloc_status(stream) == 0
    ref_o, ref_h = gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, cu_seqlens=inp.cu_seqlens.cuda(),
                               cu_seqlens_host=inp.cu_seqlens, h0=d.h0)
    torch.cuda.synchronize()
    assert maxnorm_err(o, ref_o) <= TOL["bf16"] and maxnorm_err(hT, ref_h) <= TOL["bf16"]
