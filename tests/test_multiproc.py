"""Multi-process host logic of the benchmark, on CPU with the gloo backend
(world size 2): every rank runs its own seeded, independent problem (no data
exchange), the job time is the MAX over ranks, and the job throughput counts
every rank's tokens.  The per-rank problem here is a tiny oracle forward (the
CUDA path needs a GPU; these tests cover the rank plumbing)."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import bench
import oracle
from gated_delta_rule_99_b200.inputs import make_inputs


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_problem(rank):
    return make_inputs(B=1, T=40, H=2, K=8, V=6, dtype="fp32", seed=bench.rank_seed(rank),
                       bwd=False)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        inp = _rank_problem(rank)
        o, _ = oracle.gdn_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, h0=inp.h0, nthreads=1)
        fake_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        mx = bench.max_over_ranks(fake_ms, world, "cpu")
        val = bench.job_tokens_per_s(40, world, 3, mx)
        out[rank] = (float(np.abs(o).sum()), mx, val)
    finally:
        dist.destroy_process_group()


def test_two_ranks_independent_problems_and_max_time():
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, out)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    (s0, m0, v0), (s1, m1, v1) = out[0], out[1]
    assert m0 == m1 == 15.0                       # every rank reports the slowest rank's time
    assert v0 == v1 == pytest.approx(2 * 40 * 3 / 0.015)
    # each rank ran its own seeded problem, and equals the same problem run alone
    for r, s in ((0, s0), (1, s1)):
        inp = _rank_problem(r)
        o, _ = oracle.gdn_fwd(inp.q, inp.k, inp.v, inp.g, inp.beta, h0=inp.h0)
        assert float(np.abs(o).sum()) == s
    assert s0 != s1


def test_single_rank_is_identity():
    assert bench.max_over_ranks(12.5, 1, "cpu") == 12.5
    assert bench.job_tokens_per_s(16384, 1, 10, 1000.0) == pytest.approx(163840.0)
