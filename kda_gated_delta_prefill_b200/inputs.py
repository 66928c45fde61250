"""Seeded synthetic inputs for the KDA chunk-prefill forward.

This module only draws random numbers in the shapes, dtypes and
distributions of the workloads; it holds none of the method's arithmetic.
Both the CUDA path's tests/benchmark and the CPU oracle consume what it
returns, so it must stay free of anything either side computes.

Tensor contract ("KDA Chunk Prefill on Ascend A3", section "Function and
tensor contract", plus the readings listed in the design notes):
    q, k  [B, T, H, K]   bf16        v     [B, T, HV, V]  bf16
    g     [B, T, HV, K]  fp32        beta  [B, T, HV]     fp32
    initial_state [N, HV, K, V] fp32 or None
    cu_seqlens    [N + 1] int32 or None (packed varlen batch, B == 1)

Draw order is q, k, v, g, beta, state from one ``torch.Generator`` seeded
per case.  ``device`` selects where the generator runs: CPU for the sizes
the oracle handles, CUDA for the large benchmark tensors (same recipe).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import torch
import torch.nn.functional as F


@dataclass
class Case:
    name: str
    B: int
    T: int
    H: int
    HV: int
    K: int = 128
    V: int = 128
    lengths: Optional[list] = None      # varlen: per-sequence lengths (B must be 1)
    gate: str = "softplus8"             # softplus8 | uniform5 | logsig128 | logsig8 | logsig1 | zero
    beta: str = "sigmoid1"              # sigmoid1 | sigmoid2 | zero | one | edge
    state: str = "none"                 # none | n01 (std 0.1) | quarter (std 0.25) | zeros
    qk_mode: str = "normal"             # normal | gain | tiny | zero_rows
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def N(self) -> int:
        return len(self.lengths) if self.lengths is not None else self.B

    @property
    def tokens(self) -> int:
        return self.B * self.T


# The five workloads the method is measured on (K = V = 128, chunk 64).
SMALLEST = Case("smallest_T128", B=1, T=128, H=1, HV=1, seed=1)
TAIL_STATE = Case("tail_T1000_H4_state", B=1, T=1000, H=4, HV=4, state="n01", seed=2)
WIDE_HEADS = Case("wide_B2_T4096_H96", B=2, T=4096, H=96, HV=96, seed=3)
VARLEN_GQA = Case("varlen_gqa_H8_HV32", B=1, T=11210, H=8, HV=32,
                  lengths=[1, 63, 64, 65, 777, 2048, 8192], gate="uniform5", beta="sigmoid2",
                  state="n01", seed=4)
LONG_PREFILL = Case("long_T65536_H64_state", B=1, T=65536, H=64, HV=64, state="n01", seed=5)

WORKLOADS = [SMALLEST, TAIL_STATE, WIDE_HEADS, VARLEN_GQA, LONG_PREFILL]


def cu_seqlens_of(lengths) -> torch.Tensor:
    cu = [0]
    for n in lengths:
        cu.append(cu[-1] + int(n))
    return torch.tensor(cu, dtype=torch.int32)


def make_inputs(case: Case, device: str | torch.device = "cpu") -> dict:
    """Draw one case.  Returns a dict of tensors on ``device`` (plus ``cu_seqlens`` or None)."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(case.seed)
    B, T, H, HV, K, V = case.B, case.T, case.H, case.HV, case.K, case.V
    if case.lengths is not None:
        assert B == 1 and sum(case.lengths) == T, "varlen cases pack into B == 1"

    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=dev, dtype=torch.float32)

    def qk():
        if case.qk_mode == "normal":
            x = randn(B, T, H, K)
        else:
            gain = torch.exp(randn(B, T, H, 1) * 0.6)
            x = gain * randn(B, T, H, K)
            if case.qk_mode == "tiny":
                x = (x.to(torch.bfloat16).float() * 1e-5)
        return x.to(torch.bfloat16)

    q = qk()
    k = qk()
    if case.qk_mode == "zero_rows":
        q[:, 0::3] = 0
        k[:, 1::3] = 0
    v = randn(B, T, HV, V).to(torch.bfloat16)

    if case.gate == "softplus8":
        g = -F.softplus(randn(B, T, HV, K)) / 8.0
    elif case.gate == "uniform5":
        g = torch.rand(B, T, HV, K, generator=gen, device=dev, dtype=torch.float32) * -5.0
    elif case.gate.startswith("logsig"):
        div = float(case.gate[len("logsig"):])
        g = F.logsigmoid(randn(B, T, HV, K)) / div
    elif case.gate == "zero":
        g = torch.zeros(B, T, HV, K, device=dev)
    else:
        raise ValueError(case.gate)

    if case.beta == "sigmoid1":
        beta = torch.sigmoid(randn(B, T, HV))
    elif case.beta == "sigmoid2":
        beta = torch.sigmoid(randn(B, T, HV) * 2.0)
    else:
        beta = torch.sigmoid(randn(B, T, HV))
        if case.beta == "zero":
            beta.zero_()
        elif case.beta == "one":
            beta.fill_(1.0)
        elif case.beta == "edge":
            pattern = torch.tensor([0.0, 1.0, 1e-4, 1.0 - 1e-4], device=dev)
            beta = pattern[torch.arange(T, device=dev) % 4].view(1, T, 1).expand(B, T, HV).contiguous()
        else:
            raise ValueError(case.beta)

    N = case.N
    if case.state == "none":
        s0 = None
    elif case.state == "n01":
        s0 = randn(N, HV, K, V) * 0.1
    elif case.state == "quarter":
        s0 = randn(N, HV, K, V) * 0.25
    elif case.state == "zeros":
        s0 = torch.zeros(N, HV, K, V, device=dev)
    else:
        raise ValueError(case.state)

    cu = None if case.lengths is None else cu_seqlens_of(case.lengths).to(dev)
    return {"q": q.contiguous(), "k": k.contiguous(), "v": v.contiguous(), "g": g.contiguous(),
            "beta": beta.contiguous(), "initial_state": s0, "cu_seqlens": cu}


def worked_example(T: int = 128, K: int = 128, V: int = 128) -> dict:
    """The page's worked example: q = k = e0 at every token, v = 1, g = 0, beta = 1, no state."""
    q = torch.zeros(1, T, 1, K)
    q[..., 0] = 1.0
    return {"q": q.to(torch.bfloat16), "k": q.clone().to(torch.bfloat16),
            "v": torch.ones(1, T, 1, V).to(torch.bfloat16), "g": torch.zeros(1, T, 1, K),
            "beta": torch.ones(1, T, 1), "initial_state": None, "cu_seqlens": None}


# ---------------------------------------------------------------------------------------------- backward
def make_backward_grads(case: Case, device: str | torch.device = "cpu") -> dict:
    """Seeded loss gradients for a backward of ``case``: dout ~ N(0,1) bf16 [B,T,HV,V] and dht ~ N(0, 0.1^2)
    fp32 [N,HV,K,V] (drawn in that order from their own generator, seed + 7919)."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(case.seed + 7919)
    dout = torch.randn(case.B, case.T, case.HV, case.V, generator=gen, device=dev).to(torch.bfloat16)
    dht = 0.1 * torch.randn(case.N, case.HV, case.K, case.V, generator=gen, device=dev)
    return {"dout": dout, "dht": dht}


# ---------------------------------------------------------------------------------------------- decode step
@dataclass
class DecodeCase:
    """One decode step of B rows on a pool of ``slots`` bf16 states; ``pad`` of the rows are -1 padding."""
    name: str
    B: int
    H: int
    HV: int
    slots: int
    pad: float = 0.0
    seed: int = 0


# The decode page's serving shape (H = 12, K = V = 128) at a large batch.
DECODE_SERVING = DecodeCase("decode_B1024_H12", B=1024, H=12, HV=12, slots=2048, seed=11)


def make_decode_inputs(case: DecodeCase, device: str | torch.device = "cpu") -> dict:
    """Draw q, k, v, g, beta, the state pool and the slot indices (in that order) for one decode step."""
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(case.seed)
    B, H, HV = case.B, case.H, case.HV

    def randn(*shape):
        return torch.randn(*shape, generator=gen, device=dev, dtype=torch.float32)

    q = randn(B, H, 128).to(torch.bfloat16)
    k = randn(B, H, 128).to(torch.bfloat16)
    v = randn(B, HV, 128).to(torch.bfloat16)
    g = -F.softplus(randn(B, HV, 128)) / 8.0
    beta = torch.sigmoid(randn(B, HV))
    state = (0.1 * randn(case.slots, HV, 128, 128)).to(torch.bfloat16)
    slots = torch.randperm(case.slots, generator=gen, device=dev)[:B].to(torch.int32)
    drop = torch.rand(B, generator=gen, device=dev) < case.pad
    idx = torch.where(drop, torch.full_like(slots, -1), slots)
    return {"q": q, "k": k, "v": v, "g": g, "beta": beta, "state": state, "state_indices": idx}
