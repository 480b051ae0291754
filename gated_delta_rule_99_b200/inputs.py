"""Seeded synthetic inputs for the Gated DeltaNet layer.

This module is shared by the CUDA path's tests and benchmark and by the oracle
checks.  It holds none of the layer's arithmetic: it only draws random numbers
in a fixed order and applies the input preparation the workloads state
(L2-normalised q and k per token and head, sigmoid write strength, negative
softplus log-decay), then casts.  It imports nothing else from this package.

Draw order (one ``torch.Generator`` seeded with ``seed``, all draws fp32):
q, k, v, g_raw, beta_raw, h0, do, dhT.  Packed document lengths come from a
second generator seeded ``seed + 1000``: integers uniform in [lo, hi]
(inclusive) are drawn until their sum reaches T; the last is cut to fit.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

# The five workloads the layer is measured and checked on.  Sizes are B, T, H,
# d_k, d_v; ``gate_scale`` multiplies -softplus(N(0,1)) in the log-decay.
WORKLOADS = {
    0: dict(name="gdn_fwd_fp32_B1_T256_H2_d64", B=1, T=256, H=2, K=64, V=64, dtype="fp32",
            gate_scale=0.1, h0_std=0.0, packed=None, seed=0, bwd=False),
    1: dict(name="gdn_fwd_bf16_B4_T4096_H16_d128", B=4, T=4096, H=16, K=128, V=128, dtype="bf16",
            gate_scale=0.1, h0_std=0.02, packed=None, seed=1, bwd=False),
    2: dict(name="gdn_fwdbwd_bf16_B4_T4096_H16_d128", B=4, T=4096, H=16, K=128, V=128,
            dtype="bf16", gate_scale=0.1, h0_std=0.02, packed=None, seed=2, bwd=True),
    3: dict(name="gdn_fwdbwd_bf16_packed_T16384_H16_d128", B=1, T=16384, H=16, K=128, V=128,
            dtype="bf16", gate_scale=0.1, h0_std=0.02, packed=(64, 4096), seed=3, bwd=True),
    4: dict(name="gdn_fwd_bf16_B1_T1048576_H8_d128", B=1, T=1 << 20, H=8, K=128, V=128,
            dtype="bf16", gate_scale=0.02, h0_std=0.02, packed=None, seed=4, bwd=False),
}


def doc_lengths(T: int, lo: int, hi: int, seed: int) -> list[int]:
    """Document lengths uniform in [lo, hi] until they cover T; the last is cut to fit."""
    gen = torch.Generator(device="cpu").manual_seed(seed + 1000)
    out, tot = [], 0
    while tot < T:
        n = int(torch.randint(lo, hi + 1, (1,), generator=gen).item())
        n = min(n, T - tot)
        out.append(n)
        tot += n
    return out


def cu_from_lengths(lengths) -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


@dataclass
class Inputs:
    q: torch.Tensor
    k: torch.Tensor
    v: torch.Tensor
    g: torch.Tensor
    beta: torch.Tensor
    h0: torch.Tensor | None
    cu_seqlens: torch.Tensor | None  # int32 on the CPU, or None for dense rows
    do: torch.Tensor | None = None
    dhT: torch.Tensor | None = None
    scale: float = 1.0
    meta: dict = field(default_factory=dict)

    @property
    def n_seqs(self) -> int:
        return self.q.shape[0] if self.cu_seqlens is None else self.cu_seqlens.numel() - 1

    def to(self, device):
        f = lambda x: None if x is None else x.to(device)
        return Inputs(f(self.q), f(self.k), f(self.v), f(self.g), f(self.beta), f(self.h0),
                      self.cu_seqlens, f(self.do), f(self.dhT), self.scale, dict(self.meta))


def _l2norm(x: torch.Tensor) -> torch.Tensor:
    return x / torch.sqrt((x * x).sum(-1, keepdim=True))


def make_inputs(B: int, T: int, H: int, K: int, V: int, dtype: str = "bf16", seed: int = 0,
                gate_scale: float = 0.1, h0_std: float = 0.02, lengths=None, packed=None,
                bwd: bool = True, dhT_std: float = 0.01, scale: float = 1.0,
                device: str = "cpu", raw_qk: bool = False, **_ignored) -> Inputs:
    """Draw one workload.  ``lengths`` (explicit document lengths) or ``packed``
    ((lo, hi) for random lengths) make a packed row; this needs B == 1.
    ``device`` picks where the generator runs (the draws differ between CPU
    and CUDA generators, so the oracle must be fed the same tensors).
    ``raw_qk`` leaves q and k unnormalised, each row scaled by its own factor
    exp(N(0, 1)) (inputs for the layer's own normalisation option); the other
    tensors are the same draws as without it."""
    tdt = {"bf16": torch.bfloat16, "fp32": torch.float32}[dtype]
    if packed is not None and lengths is None:
        lengths = doc_lengths(T, packed[0], packed[1], seed)
    cu = None
    if lengths is not None:
        assert B == 1 and sum(lengths) == T
        cu = cu_from_lengths(lengths)
    N = B if cu is None else cu.numel() - 1
    gen = torch.Generator(device=device).manual_seed(seed)
    f32 = dict(generator=gen, device=device, dtype=torch.float32)
    q = torch.randn(B, T, H, K, **f32)
    k = torch.randn(B, T, H, K, **f32)
    if not raw_qk:
        q, k = _l2norm(q).to(tdt), _l2norm(k).to(tdt)
    v = torch.randn(B, T, H, V, **f32).to(tdt)
    g = -torch.nn.functional.softplus(torch.randn(B, T, H, **f32)) * gate_scale
    beta = torch.sigmoid(torch.randn(B, T, H, **f32))
    h0 = torch.randn(N, H, K, V, **f32) * h0_std if h0_std > 0 else None
    do = dhT = None
    if bwd:
        do = torch.randn(B, T, H, V, **f32).to(tdt)
        dhT = torch.randn(N, H, K, V, **f32) * dhT_std if dhT_std > 0 else None
    if raw_qk:
        q = (q * torch.exp(torch.randn(B, T, H, 1, **f32))).to(tdt)
        k = (k * torch.exp(torch.randn(B, T, H, 1, **f32))).to(tdt)
    return Inputs(q, k, v, g, beta, h0, cu, do, dhT, scale,
                  dict(B=B, T=T, H=H, K=K, V=V, dtype=dtype, seed=seed))


def workload(idx: int, device: str = "cpu", bwd: bool | None = None) -> Inputs:
    w = dict(WORKLOADS[idx])
    if bwd is not None:
        w["bwd"] = bwd
    inp = make_inputs(device=device, **w)
    inp.meta["name"] = w["name"]
    return inp
