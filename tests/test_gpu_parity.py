"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances (max-normalised error per tensor, max|x - ref| / max|ref|): 1e-4
for fp32 inputs and 2e-2 for bf16 inputs with fp32 state and accumulation.
Small cases compare every element; the full-size workloads compare the
sampled (sequence, head) units the oracle computes one by one.
"""
import numpy as np
import pytest
import torch

import gated_delta_rule_99_b200 as gdn
import oracle
from gated_delta_rule_99_b200.inputs import make_inputs, workload

from _util import maxnorm_err, np64, oracle_bwd, oracle_fwd, unit_mask

pytestmark = pytest.mark.gpu

TOL = {"fp32": 1e-4, "bf16": 2e-2}


def run_fwd(inp, **kw):
    d = inp.to("cuda")
    cu = None if d.cu_seqlens is None else d.cu_seqlens
    o, hT = gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, cu_seqlens=cu, h0=d.h0, scale=d.scale, **kw)
    torch.cuda.synchronize()
    return o, hT


def run_bwd(inp, **kw):
    d = inp.to("cuda")
    cu = None if d.cu_seqlens is None else d.cu_seqlens
    r = gdn.gdn_bwd(d.q, d.k, d.v, d.g, d.beta, d.do, cu_seqlens=cu, h0=d.h0, dhT=d.dhT,
                    scale=d.scale, **kw)
    torch.cuda.synchronize()
    return r


def check_all(inp, tol, units=None, bwd=True):
    o, hT = run_fwd(inp)
    ro, rh = oracle_fwd(inp, units)
    errs = {"o": maxnorm_err(o, ro), "hT": maxnorm_err(hT, rh)}
    if bwd:
        got = run_bwd(inp)
        ref = oracle_bwd(inp, units)
        for name, a, b in zip(("dq", "dk", "dv", "dg", "dbeta", "dh0"), got, ref):
            errs[name] = maxnorm_err(a, b)
    print("parity %s: %s" % (inp.meta.get("name", inp.meta.get("dtype")),
                             " ".join("%s=%.2e" % kv for kv in errs.items())))
    bad = {k: v for k, v in errs.items() if not v <= tol}
    assert not bad, (errs, tol)
    return errs


def test_tiny_fp32_forward_config():
    inp = workload(0)
    errs = check_all(inp, TOL["fp32"], bwd=False)
    assert errs["o"] < 1e-5


def test_fp32_forward_backward_with_states():
    inp = make_inputs(B=2, T=200, H=2, K=64, V=64, dtype="fp32", seed=10)
    check_all(inp, TOL["fp32"])


def test_fp32_scale_and_mixed_head_dims():
    inp = make_inputs(B=1, T=150, H=3, K=64, V=128, dtype="fp32", seed=11, scale=0.125)
    check_all(inp, TOL["fp32"])
    inp = make_inputs(B=1, T=90, H=1, K=128, V=64, dtype="fp32", seed=12)
    check_all(inp, TOL["fp32"])


@pytest.mark.parametrize("dtype", ["fp32", "bf16"])
def test_packed_ragged_documents(dtype):
    lengths = [1, 0, 63, 64, 65, 130, 7, 200]
    inp = make_inputs(B=1, T=sum(lengths), H=3, K=64, V=128, dtype=dtype, seed=13,
                      lengths=lengths)
    check_all(inp, TOL[dtype])


def test_bf16_ragged_dense_rows():
    inp = make_inputs(B=2, T=300, H=2, K=128, V=128, dtype="bf16", seed=14)
    check_all(inp, TOL["bf16"])


def test_fp32_strong_decay_and_unit_strength():
    inp = make_inputs(B=1, T=256, H=2, K=64, V=64, dtype="fp32", seed=15, gate_scale=3.0)
    inp.beta.fill_(1.0)
    check_all(inp, TOL["fp32"])


def _sampled(idx, units, bwd):
    inp = workload(idx, bwd=bwd)
    errs = check_all(inp, TOL[inp.meta["dtype"]], units=units, bwd=bwd)
    return errs


def test_full_size_forward_bf16_sampled():
    _sampled(1, [(0, 0), (3, 15), (1, 7)], bwd=False)


def test_full_size_forward_backward_bf16_sampled():
    _sampled(2, [(0, 0), (3, 15), (2, 9)], bwd=True)


def test_full_size_packed_forward_backward_sampled():
    inp = workload(3)
    n = inp.n_seqs
    _sampled(3, [(0, 0), (n - 1, 15), (n // 2, 5)], bwd=True)


def test_long_context_chained_halves_bitwise():
    """One call over the 1,048,576-token row equals two chained calls (the
    first half's hT as the second's h0) bitwise (jax-linear-attention 0.1.0,
    "Highlights")."""
    inp = workload(4, device="cuda")
    Th = inp.q.shape[1] // 2
    o, hT = gdn.gdn_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, h0=inp.h0)
    oa, ha = gdn.gdn_fwd(inp.q[:, :Th].contiguous(), inp.k[:, :Th].contiguous(),
                         inp.v[:, :Th].contiguous(), inp.g[:, :Th].contiguous(),
                         inp.beta[:, :Th].contiguous(), h0=inp.h0)
    ob, hb = gdn.gdn_fwd(inp.q[:, Th:].contiguous(), inp.k[:, Th:].contiguous(),
                         inp.v[:, Th:].contiguous(), inp.g[:, Th:].contiguous(),
                         inp.beta[:, Th:].contiguous(), h0=ha)
    torch.cuda.synchronize()
    assert torch.equal(o[:, :Th], oa) and torch.equal(o[:, Th:], ob)
    assert torch.equal(hT, hb)
    del o, oa, ob
    torch.cuda.empty_cache()


@pytest.mark.slow
def test_long_context_full_row_against_oracle():
    """The long-row workload (B=1, T=1,048,576, H=8, slow decay) against the fp64
    oracle over the whole row for two heads (the first and the last): every
    output element of those heads and their final states, on the default path
    and on the piece scan (the outputs match the token-by-token reference:
    jax-linear-attention 0.1.0, "FAQ").  The error is also checked on
    4,096-token windows at the start, the middle and the end of the row, so
    that build-up over the 16,384 chunk steps shows where it happens."""
    inp = workload(4, device="cuda")
    heads = [0, inp.q.shape[2] - 1]
    sel = lambda x: x[:, :, heads].cpu()
    ro, rh = oracle.gdn_fwd(sel(inp.q), sel(inp.k), sel(inp.v), sel(inp.g), sel(inp.beta),
                            h0=inp.h0[:, heads].cpu())
    T, W = inp.q.shape[1], 4096
    windows = [(0, W), (T // 2 - W // 2, T // 2 + W // 2), (T - W, T)]
    for piece in (False, True):
        o, hT = gdn.gdn_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, h0=inp.h0, piece_scan=piece)
        torch.cuda.synchronize()
        got_o = np64(o[:, :, heads].cpu())
        got_h = np64(hT[:, heads].cpu())
        del o, hT
        errs = {"o": maxnorm_err(got_o, ro), "hT": maxnorm_err(got_h, rh)}
        for a, b in windows:
            errs["o[%d:%d]" % (a, b)] = maxnorm_err(got_o[:, a:b], ro[:, a:b])
        print("long row vs oracle (%s): %s" % ("piece scan" if piece else "default",
                                               " ".join("%s=%.2e" % kv for kv in errs.items())))
        assert max(errs.values()) <= TOL["bf16"], errs
    torch.cuda.empty_cache()


def test_packed_equals_per_document_runs_bitwise():
    lengths = [70, 1, 128, 0, 33]
    inp = make_inputs(B=1, T=sum(lengths), H=2, K=128, V=128, dtype="bf16", seed=16,
                      lengths=lengths)
    o, hT = run_fwd(inp)
    got = run_bwd(inp)
    cu = inp.cu_seqlens.tolist()
    for n in range(len(lengths)):
        t0, t1 = cu[n], cu[n + 1]
        sl = lambda x: x[:, t0:t1].contiguous()
        sub = inp.to("cpu")
        sub.q, sub.k, sub.v, sub.g, sub.beta, sub.do = map(sl, (inp.q, inp.k, inp.v, inp.g,
                                                                 inp.beta, inp.do))
        sub.h0 = inp.h0[n:n + 1].contiguous()
        sub.dhT = inp.dhT[n:n + 1].contiguous()
        sub.cu_seqlens = None
        on, hn = run_fwd(sub)
        assert torch.equal(o[:, t0:t1], on)
        assert torch.equal(hT[n:n + 1], hn)
        gn = run_bwd(sub)
        for a, b in zip(got[:5], gn[:5]):
            assert torch.equal(a[:, t0:t1], b)
        assert torch.equal(got[5][n:n + 1], gn[5])


def _ragged_lengths(n, seed):
    rng = np.random.default_rng(seed)
    return [int(x) for x in rng.integers(1, 151, size=n)]


@pytest.mark.parametrize("case", ["packed", "dense"])
def test_tc_many_units_per_cta(case):
    """More (chunk, head) units than SMs, so every persistent CTA of the gradient
    kernel walks several units and prefetches the next one's inputs; short chunks
    (packed documents of 1-150 tokens, or a 40-token tail per dense row) take the
    row-store path between full ones.  Every element against the oracle."""
    if case == "packed":
        lengths = _ragged_lengths(56, 27)
        inp = make_inputs(B=1, T=sum(lengths), H=8, K=128, V=128, dtype="bf16", seed=27,
                          lengths=lengths)
    else:
        inp = make_inputs(B=3, T=1000, H=16, K=128, V=128, dtype="bf16", seed=28)
    check_all(inp, TOL["bf16"])


def test_tc_many_units_split_call_bitwise():
    """The same documents in one packed call and in two calls (first half, second
    half): each document's outputs are bitwise equal, whichever CTA and slot of
    the persistent kernel handled its units."""
    lengths = _ragged_lengths(40, 29)
    inp = make_inputs(B=1, T=sum(lengths), H=8, K=128, V=128, dtype="bf16", seed=29,
                      lengths=lengths)
    o, hT = run_fwd(inp)
    got = run_bwd(inp)
    cu = inp.cu_seqlens.tolist()
    half = len(lengths) // 2
    for n0, n1 in ((0, half), (half, len(lengths))):
        t0, t1 = cu[n0], cu[n1]
        sub = inp.to("cpu")
        sl = lambda x: x[:, t0:t1].contiguous()
        sub.q, sub.k, sub.v, sub.g, sub.beta, sub.do = map(sl, (inp.q, inp.k, inp.v, inp.g,
                                                                 inp.beta, inp.do))
        sub.h0 = inp.h0[n0:n1].contiguous()
        sub.dhT = inp.dhT[n0:n1].contiguous()
        sub.cu_seqlens = torch.tensor([c - t0 for c in cu[n0:n1 + 1]], dtype=torch.int32)
        on, hn = run_fwd(sub)
        assert torch.equal(o[:, t0:t1], on)
        assert torch.equal(hT[n0:n1], hn)
        gn = run_bwd(sub)
        for a, b in zip(got[:5], gn[:5]):
            assert torch.equal(a[:, t0:t1], b)
        assert torch.equal(got[5][n0:n1], gn[5])


def test_run_to_run_determinism():
    inp = make_inputs(B=2, T=500, H=4, K=128, V=128, dtype="bf16", seed=17)
    a = run_fwd(inp) + run_bwd(inp)
    b = run_fwd(inp) + run_bwd(inp)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


def test_empty_inputs_pass_state_through():
    inp = make_inputs(B=2, T=0, H=2, K=64, V=64, dtype="bf16", seed=18)
    o, hT = run_fwd(inp)
    assert o.numel() == 0 and torch.equal(hT.cpu(), inp.h0)
    *_, dh0 = run_bwd(inp)
    assert torch.equal(dh0.cpu(), inp.dhT)


def test_device_side_seqlens_check():
    lengths = [100, 100]
    inp = make_inputs(B=1, T=200, H=1, K=64, V=64, dtype="bf16", seed=19, lengths=lengths)
    d = inp.to("cuda")
    bad_dev = torch.tensor([0, 201, 200], dtype=torch.int32, device="cuda")
    ws = gdn.alloc_workspace(gdn.fwd_workspace_size(gdn.make_desc(1, 200, 1, 64, 64, 2)), "cuda")
    gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, cu_seqlens=bad_dev,
                cu_seqlens_host=inp.cu_seqlens, h0=d.h0, workspace=ws)
    assert gdn.device_status(ws) == 1
    gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, cu_seqlens=d.cu_seqlens.cuda(),
                cu_seqlens_host=inp.cu_seqlens, h0=d.h0, workspace=ws)
    assert gdn.device_status(ws) == 0


# ---- the tensor-core path (bf16, d_k = d_v = 128) on the small edge cases
def test_tc_packed_ragged_documents_with_scale():
    lengths = [1, 0, 63, 64, 65, 130, 7, 200]
    inp = make_inputs(B=1, T=sum(lengths), H=3, K=128, V=128, dtype="bf16", seed=21,
                      lengths=lengths, scale=0.125)
    check_all(inp, TOL["bf16"])


def test_tc_strong_decay_unit_strength_and_reset_gate():
    inp = make_inputs(B=2, T=190, H=2, K=128, V=128, dtype="bf16", seed=22, gate_scale=3.0)
    inp.beta.fill_(1.0)
    inp.g[:, 77] = -30.0  # decay to ~1e-13 inside a chunk
    check_all(inp, TOL["bf16"])


def test_tc_zero_write_strength_and_no_initial_state():
    inp = make_inputs(B=1, T=129, H=2, K=128, V=128, dtype="bf16", seed=23, h0_std=0.0)
    inp.beta[:, 40:90] = 0.0
    check_all(inp, TOL["bf16"])


# ---- head dims of 64 on the tensor-core path (the 128-wide tiles zero-padded)
@pytest.mark.parametrize("K,V", [(64, 64), (64, 128), (128, 64)])
def test_tc_head_dim_64_packed_ragged(K, V):
    lengths = [1, 0, 63, 64, 65, 130, 7, 200]
    inp = make_inputs(B=1, T=sum(lengths), H=3, K=K, V=V, dtype="bf16", seed=24 + K + V,
                      lengths=lengths, scale=0.25)
    check_all(inp, TOL["bf16"])


def test_tc_head_dim_64_dense_rows_full_size_sampled():
    inp = make_inputs(B=4, T=4096, H=16, K=64, V=64, dtype="bf16", seed=25)
    check_all(inp, TOL["bf16"], units=[(0, 0), (3, 15), (1, 8)])


def test_tc_head_dim_64_chained_halves_bitwise():
    inp = make_inputs(B=2, T=1024, H=2, K=64, V=128, dtype="bf16", seed=26, bwd=False)
    d = inp.to("cuda")
    o, hT = gdn.gdn_fwd(d.q, d.k, d.v, d.g, d.beta, h0=d.h0)
    sl = lambda x, a, b: x[:, a:b].contiguous()
    oa, ha = gdn.gdn_fwd(sl(d.q, 0, 512), sl(d.k, 0, 512), sl(d.v, 0, 512), sl(d.g, 0, 512),
                         sl(d.beta, 0, 512), h0=d.h0)
    ob, hb = gdn.gdn_fwd(sl(d.q, 512, 1024), sl(d.k, 512, 1024), sl(d.v, 512, 1024),
                         sl(d.g, 512, 1024), sl(d.beta, 512, 1024), h0=ha)
    torch.cuda.synchronize()
    assert torch.equal(o[:, :512], oa) and torch.equal(o[:, 512:], ob) and torch.equal(hT, hb)
