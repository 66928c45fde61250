"""Shared helpers of the GPU parity tests: run the CUDA path and the oracle on
the same seeded inputs and compare with the stated tolerances.

Tolerances (written here once, used by every parity test):
  o            |gpu - ref| <= 2e-2 * max(1, |ref|)      (element-wise)
  final_state  ||gpu - ref||_F / ||ref||_F <= 5e-3     (per sequence and head)
  normalised Q/K: at most one bf16 ulp from the oracle
plus the page's own acceptance rule ("KDA Chunk Prefill on Ascend A3",
section "Public examples and full evaluation"): |a - g| <= 0.02 + 0.02|g|
and relative L2 <= 0.02 for both outputs, and no NaN/Inf.
"""
from __future__ import annotations

import numpy as np
import torch

O_TOL = 2e-2
STATE_REL_FRO = 5e-3


def to_cuda(x: dict) -> dict:
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}


def gpu_forward(x: dict, **kw):
    import kda_gated_delta_prefill_b200 as kda
    xc = to_cuda(x)
    o, s = kda.forward(xc["q"], xc["k"], xc["v"], xc["g"], xc["beta"], xc["initial_state"], xc["cu_seqlens"], **kw)
    torch.cuda.synchronize()
    return o, s


def oracle_forward(x: dict):
    import oracle
    return oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"], x["cu_seqlens"])


def compare(o_gpu: torch.Tensor, s_gpu: torch.Tensor, ref: dict, *, o_rows=None) -> dict:
    """Check the bars; returns measured error figures.  o_rows: optional boolean mask over [B,T]."""
    og = o_gpu.float().cpu().numpy().astype(np.float64)
    sg = s_gpu.float().cpu().numpy().astype(np.float64)
    orf, srf = ref["o64"], ref["state"]
    if o_rows is not None:
        og, orf = og[o_rows], orf[o_rows]
    assert np.isfinite(og).all() and np.isfinite(sg).all(), "NaN/Inf in GPU output"
    d = np.abs(og - orf)
    o_ratio = float((d / np.maximum(1.0, np.abs(orf))).max()) if d.size else 0.0
    assert o_ratio <= O_TOL, f"o error {o_ratio:.4g} > {O_TOL}"
    # page rule, o
    assert (d <= 0.02 + 0.02 * np.abs(orf)).all()
    if np.any(orf != 0):
        assert np.linalg.norm(og - orf) / np.linalg.norm(orf) <= 0.02
    # final state, per (sequence, head)
    worst = 0.0
    for n in range(srf.shape[0]):
        for h in range(srf.shape[1]):
            den = np.linalg.norm(srf[n, h])
            num = np.linalg.norm(sg[n, h] - srf[n, h])
            if den == 0:
                assert num == 0 or num < 1e-6, f"state ({n},{h}) should be zero"
                continue
            worst = max(worst, num / den)
    assert worst <= STATE_REL_FRO, f"final_state rel Frobenius {worst:.4g} > {STATE_REL_FRO}"
    sd = np.abs(sg - srf)
    assert (sd <= 0.02 + 0.02 * np.abs(srf)).all()
    return {"o_max_ratio": o_ratio, "state_rel_fro": worst}


def select_heads(x: dict, heads) -> dict:
    """Inputs restricted to value heads `heads` (and the Q/K heads they read)."""
    H, HV = x["q"].shape[2], x["v"].shape[2]
    group = HV // H
    qk_heads = sorted({h // group for h in heads})
    assert all(h // group == qk_heads[0] for h in heads) or group == 1
    out = dict(x)
    if group == 1:
        idx = torch.tensor(heads)
        out["q"] = x["q"][:, :, idx].contiguous()
        out["k"] = x["k"][:, :, idx].contiguous()
    else:
        out["q"] = x["q"][:, :, qk_heads].contiguous()
        out["k"] = x["k"][:, :, qk_heads].contiguous()
    hv = torch.tensor(heads)
    out["v"] = x["v"][:, :, hv].contiguous()
    out["g"] = x["g"][:, :, hv].contiguous()
    out["beta"] = x["beta"][:, :, hv].contiguous()
    if x["initial_state"] is not None:
        out["initial_state"] = x["initial_state"][:, hv].contiguous()
    return out
