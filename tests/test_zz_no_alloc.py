"""The allocation-free entry point (kda_prefill_forward_noalloc).

It exists for callers that may not allocate device memory during a call, so
its workspace is the library's fixed device array.  This file is collected
last so that a failure here cannot hide the result of any other test.

Both entry points run the same kernels over the same workspace layout, so
each no-allocation call must equal kda_prefill_forward on the same inputs bit
for bit.  The array keeps whatever the previous call left in it: the calls
below first fill it with a larger packed batch (more sequences, longer ones),
then run a smaller packed batch and a plain batch, so a kernel that read
stale chunk offsets, sequence order or chunk blocks from an earlier call
would break the equality.  One case is also compared with the oracle.
"""
import ctypes

import numpy as np
import pytest
import torch

from kda_gated_delta_prefill_b200 import inputs as gen
from tests.parity_util import O_TOL, STATE_REL_FRO, compare, oracle_forward, to_cuda

pytestmark = pytest.mark.gpu


def _call_noalloc(L, x, o, s):
    """kda_prefill_forward_noalloc straight through ctypes."""
    f = L.kda_prefill_forward_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P]
    f.restype = I
    ptr = lambda t: None if t is None else ctypes.c_void_p(t.data_ptr())
    B, T, H, K = x["q"].shape
    HV = x["v"].shape[2]
    cu = x["cu_seqlens"]
    num_seqs = cu.numel() - 1 if cu is not None else 0
    return f(ptr(x["q"]), ptr(x["k"]), ptr(x["v"]), ptr(x["g"]), ptr(x["beta"]), ptr(x["initial_state"]),
             ptr(cu), num_seqs, B, T, H, HV, K, 128, ptr(o), ptr(s),
             ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _close(o, s, o_ref, s_ref):
    o, o_ref = o.float().cpu().numpy(), o_ref.float().cpu().numpy()
    d = np.abs(o - o_ref) / np.maximum(1.0, np.abs(o_ref))
    assert np.isfinite(o).all() and d.max() <= O_TOL
    s, s_ref = s.cpu().numpy().astype(np.float64), s_ref.cpu().numpy().astype(np.float64)
    for n in range(s.shape[0]):
        for h in range(s.shape[1]):
            den = np.linalg.norm(s_ref[n, h])
            num = np.linalg.norm(s[n, h] - s_ref[n, h])
            assert num <= STATE_REL_FRO * den + 1e-6


def _run_noalloc(L, x, case):
    o = torch.full((case.B, case.T, case.HV, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    s = torch.full((case.N, case.HV, 128, 128), float("nan"), device="cuda")
    assert _call_noalloc(L, x, o, s) == 0
    torch.cuda.synchronize()
    return o, s


def test_noalloc_matches_forward_on_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kda_gated_delta_prefill_b200 as kda
    L = kda.lib()
    poison = gen.Case("noalloc_poison", B=1, T=1201, H=2, HV=8, lengths=[300, 2, 129, 64, 500, 1, 205], state="n01",
                      seed=90)
    small = gen.Case("noalloc_varlen", B=1, T=400, H=2, HV=8, lengths=[130, 1, 64, 205], state="n01", seed=91)
    cases = [poison, small, gen.TAIL_STATE]
    for i, case in enumerate(cases):
        x_cpu = gen.make_inputs(case)
        x = to_cuda(x_cpu)
        o_ref, s_ref = kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"], x["cu_seqlens"])
        torch.cuda.synchronize()
        o, s = _run_noalloc(L, x, case)
        _close(o, s, o_ref, s_ref)
        assert torch.equal(o, o_ref), case.name
        assert torch.equal(s, s_ref), case.name
        if case is small:  # the packed batch after the larger one, also against the oracle
            compare(o, s, oracle_forward(x_cpu))
    # the same small packed batch once more right after the plain batch
    x = to_cuda(gen.make_inputs(small))
    o_ref, s_ref = kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"], x["cu_seqlens"])
    o, s = _run_noalloc(L, x, small)
    assert torch.equal(o, o_ref) and torch.equal(s, s_ref)


def test_noalloc_rejects_sizes_over_its_limit():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kda_gated_delta_prefill_b200 as kda
    L = kda.lib()
    f = L.kda_prefill_forward_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P]
    f.restype = I
    # B=1, T=65536, H=HV=64 needs about 4.9 GB of workspace: rejected on the host, before any launch,
    # so the (small, never dereferenced) buffers below are never touched.
    buf = torch.empty(1 << 20, dtype=torch.uint8, device="cuda")
    a = lambda off: ctypes.c_void_p(buf.data_ptr() + off)
    rc = f(a(0), a(1 << 16), a(2 << 16), a(3 << 16), a(4 << 16), None, None, 0, 1, 65536, 64, 64, 128, 128,
           a(5 << 16), a(6 << 16), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 4  # KDA_ERR_WORKSPACE
