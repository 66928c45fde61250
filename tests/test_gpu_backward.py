"""GPU parity of the backward (kda_prefill_backward through the C ABI) against the oracle's float64 reverse mode.

Bar, per gradient tensor (dq, dk, dv, dg, dbeta, dh0):
  ||gpu - ref||_F / ||ref||_F <= 1e-2   and   max |gpu - ref| <= 2e-2 * max |ref|.
Where it comes from: the recomputed forward's chunk start states carry the forward's own error (its bar is a
relative Frobenius error of 5e-3 on the state); the reverse carry multiplies by the forward's fp16 blocks (2^-11
relative per operand); dq, dk and dv are returned in bf16 (2^-9 relative).  Single gradient elements can cancel
to near zero, so the element-wise bound is taken relative to the tensor's scale.
"""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

REL_FRO = 1e-2
MAX_REL = 2e-2


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kda_gated_delta_prefill_b200 as kda
    kda.lib()


def _case(B, T, H, HV, seed, state=True, dht=True, cu=None, gate=8.0, beta_zero=False):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(B, T, H, 128, generator=gen).bfloat16()
    k = torch.randn(B, T, H, 128, generator=gen).bfloat16()
    v = torch.randn(B, T, HV, 128, generator=gen).bfloat16()
    g = -torch.nn.functional.softplus(torch.randn(B, T, HV, 128, generator=gen)) / gate
    beta = torch.sigmoid(torch.randn(B, T, HV, generator=gen))
    if beta_zero:
        beta.zero_()
    N = B if cu is None else len(cu) - 1
    s0 = 0.1 * torch.randn(N, HV, 128, 128, generator=gen) if state else None
    dout = torch.randn(B, T, HV, 128, generator=gen).bfloat16()
    dh = 0.1 * torch.randn(N, HV, 128, 128, generator=gen) if dht else None
    cu_t = None if cu is None else torch.tensor(cu, dtype=torch.int32)
    return q, k, v, g, beta, s0, dout, dh, cu_t


def _run(q, k, v, g, beta, s0, dout, dh, cu):
    import kda_gated_delta_prefill_b200 as kda
    c = lambda t: None if t is None else t.cuda()
    out = kda.backward(c(q), c(k), c(v), c(g), c(beta), c(dout), c(s0), c(dh), c(cu), want_dh0=True)
    torch.cuda.synchronize()
    assert kda.device_error(clear=True) == 0
    ref = oracle.backward(q, k, v, g, beta, s0, dout.float().numpy(), None if dh is None else dh.numpy(), cu)
    return [t.float().cpu().numpy().astype(np.float64) for t in out[:5]] + [out[5].cpu().numpy()], ref


def _compare(got, ref, rows=None):
    names = ["dq", "dk", "dv", "dg", "dbeta", "dh0"]
    report = {}
    for name, a, b in zip(names, got, ref):
        if b is None:
            b = np.zeros_like(a)
        if rows is not None and name != "dh0":
            a, b = a[rows], b[rows]
        assert np.isfinite(a).all(), f"{name}: NaN/Inf"
        scale = np.abs(b).max()
        if scale == 0:
            assert np.abs(a).max() <= 1e-6, name
            continue
        fro = np.linalg.norm(a - b) / np.linalg.norm(b)
        mx = np.abs(a - b).max() / scale
        report[name] = (fro, mx)
        assert fro <= REL_FRO and mx <= MAX_REL, f"{name}: rel Frobenius {fro:.3g}, max {mx:.3g}"
    return report


@pytest.mark.parametrize("B,T,H,HV", [(1, 128, 1, 1), (2, 150, 1, 2), (1, 64, 2, 2), (1, 1, 1, 1),
                                      (1, 333, 2, 4)])
def test_backward_parity(B, T, H, HV):
    got, ref = _run(*_case(B, T, H, HV, seed=900 + T + HV))
    _compare(got, ref)


def test_backward_no_state_no_dht():
    q, k, v, g, beta, s0, dout, dh, cu = _case(1, 200, 1, 2, seed=931, state=False, dht=False)
    got, ref = _run(q, k, v, g, beta, s0, dout, dh, cu)
    ref = list(ref)
    # the initial state's gradient exists even without a state passed (zeros are a state)
    ref[5] = oracle.backward_f64(
        oracle.bits_to_f32(oracle.l2norm_bf16(q)).astype(np.float64),
        oracle.bits_to_f32(oracle.l2norm_bf16(k)).astype(np.float64),
        v.float().numpy().astype(np.float64), g.numpy().astype(np.float64), beta.numpy().astype(np.float64),
        None, dout.float().numpy().astype(np.float64), None)[5]
    _compare(got, ref)


def test_backward_beta_zero():
    got, ref = _run(*_case(1, 130, 1, 1, seed=941, beta_zero=True))
    _compare(got, ref)


def test_backward_varlen():
    cu = [0, 1, 64, 65, 65, 300]  # one token, exactly a chunk, one token, empty, a ragged multi-chunk sequence
    q, k, v, g, beta, s0, dout, dh, cu_t = _case(1, 300, 2, 4, seed=951, cu=cu)
    got, ref = _run(q, k, v, g, beta, s0, dout, dh, cu_t)
    _compare(got, ref)


def test_backward_strong_gates():
    """Gates down to about -5 per token (softplus without the /8): the factored gate terms stay in range."""
    got, ref = _run(*_case(1, 192, 1, 1, seed=961, gate=1.0))
    _compare(got, ref)


def test_backward_config2_shape():
    """The 4-head, 1000-token shape with a ragged tail (15 full chunks and one of 40 tokens)."""
    got, ref = _run(*_case(1, 1000, 4, 4, seed=2))
    _compare(got, ref)


def test_backward_full_workload_sampled():
    """The backward of the benchmark's workload (B=1, H=HV=64, T=65536, fp32 state; dout and dht from the
    benchmark's generator), computed for all heads on the GPU in the launch shape the benchmark times; heads are
    independent (H == HV), so the oracle checks two heads over the whole sequence."""
    import kda_gated_delta_prefill_b200 as kda
    from kda_gated_delta_prefill_b200 import inputs as gen
    case = gen.LONG_PREFILL
    x = gen.make_inputs(case, device="cuda")
    gr = gen.make_backward_grads(case, device="cuda")
    out = kda.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], gr["dout"], x["initial_state"], gr["dht"])
    torch.cuda.synchronize()
    assert kda.device_error(clear=True) == 0
    heads = [3, 62]
    sel = lambda t, dim: t.index_select(dim, torch.tensor(heads, device=t.device)).contiguous().cpu()
    ref = oracle.backward(sel(x["q"], 2), sel(x["k"], 2), sel(x["v"], 2), sel(x["g"], 2), sel(x["beta"], 2),
                          sel(x["initial_state"], 1), sel(gr["dout"], 2).float().numpy(), sel(gr["dht"], 1).numpy())
    got = [sel(out[i], 2).float().numpy().astype(np.float64) for i in range(5)] + [sel(out[5], 1).numpy()]
    report = _compare(got, ref)
    assert report["dq"][0] < REL_FRO


@pytest.mark.parametrize("B,T,H,HV,cu,exact", [
    (2, 150, 1, 2, None, True),      # one carry launch
    (1, 2048, 4, 4, None, True),     # the forward cut into parts (side-stream carries)
    (1, 8192, 1, 1, None, False),    # one unit, long: the segmented carry (affine maps and a scan)
    (1, 300, 2, 4, [0, 1, 64, 65, 65, 300], True),  # packed sequences
])
def test_saved_forward_then_backward(B, T, H, HV, cu, exact):
    """forward_save + backward(saved=...) against the oracle, against the recomputing backward (bit for bit
    where the saved forward's carry is the same computation) and with o/final_state equal to the forward's."""
    import kda_gated_delta_prefill_b200 as kda
    q, k, v, g, beta, s0, dout, dh, cu_t = _case(B, T, H, HV, seed=970 + T, cu=cu)
    c = lambda t: None if t is None else t.cuda()
    xs = [c(t) for t in (q, k, v, g, beta)]
    o1, sN1, saved = kda.forward_save(*xs, c(s0), c(cu_t))
    o2, sN2 = kda.forward(*xs, c(s0), c(cu_t))
    torch.cuda.synchronize()
    if cu is None:
        assert torch.equal(o1, o2)
    else:
        assert torch.equal(o1[:, :cu[-1]], o2[:, :cu[-1]])
    assert torch.equal(sN1, sN2)
    got_s = kda.backward(*xs, c(dout), c(s0), c(dh), c(cu_t), want_dh0=True, saved=saved)
    got_r = kda.backward(*xs, c(dout), c(s0), c(dh), c(cu_t), want_dh0=True)
    torch.cuda.synchronize()
    assert kda.device_error(clear=True) == 0
    if exact:
        for a, b in zip(got_s, got_r):
            assert torch.equal(a, b)
    ref = oracle.backward(q, k, v, g, beta, s0, dout.float().numpy(), dh.numpy(), cu_t)
    _compare([t.float().cpu().numpy().astype(np.float64) for t in got_s[:5]] + [got_s[5].cpu().numpy()], ref)


def test_saved_forward_with_head_groups():
    """2 x 80 units (between one and two waves of carry CTAs): forward_save splits the value heads into two
    groups, while the recomputing backward runs its forward in one launch of each kernel.  Heads are independent,
    so the saved forward's outputs and the two backwards must agree bit for bit."""
    import kda_gated_delta_prefill_b200 as kda
    B, T, H, HV = 2, 1024, 80, 80
    assert kda.kernel_launches(B, T, H, HV) == 4  # the two head groups
    q, k, v, g, beta, s0, dout, dh, _ = _case(B, T, H, HV, seed=991)
    c = lambda t: None if t is None else t.cuda()
    xs = [c(t) for t in (q, k, v, g, beta)]
    o1, sN1, saved = kda.forward_save(*xs, c(s0))
    o2, sN2 = kda.forward(*xs, c(s0))
    got_s = kda.backward(*xs, c(dout), c(s0), c(dh), want_dh0=True, saved=saved)
    got_r = kda.backward(*xs, c(dout), c(s0), c(dh), want_dh0=True)
    torch.cuda.synchronize()
    assert kda.device_error(clear=True) == 0
    assert torch.equal(o1, o2) and torch.equal(sN1, sN2)
    for a, b in zip(got_s, got_r):
        assert torch.equal(a, b)


def _gen_run(x, gr, want_dh0):
    import kda_gated_delta_prefill_b200 as kda
    c = lambda t: None if t is None else t.cuda()
    out = kda.backward(c(x["q"]), c(x["k"]), c(x["v"]), c(x["g"]), c(x["beta"]), c(gr["dout"]),
                       c(x["initial_state"]), c(gr["dht"]), c(x["cu_seqlens"]), want_dh0=want_dh0)
    torch.cuda.synchronize()
    assert kda.device_error(clear=True) == 0
    return out


@pytest.mark.parametrize("mode", [dict(qk_mode="gain"), dict(qk_mode="tiny"), dict(qk_mode="zero_rows"),
                                  dict(gate="logsig128"), dict(gate="logsig1"), dict(gate="zero"),
                                  dict(gate="uniform5"), dict(beta="one"), dict(beta="edge"),
                                  dict(beta="zero", state="quarter"), dict(state="quarter"), dict(state="zeros")],
                         ids=lambda m: "-".join(f"{k}={v}" for k, v in m.items()))
def test_backward_generator_modes(mode):
    """The forward's input modes (Q/K gain, tiny and all-zero rows; gates from -log(1+e^x)/128 down to
    U[-5, 0] per token; beta of one, zero and the repeating edge pattern; state scales) through the backward."""
    from kda_gated_delta_prefill_b200 import inputs as gen
    case = gen.Case("mode", B=1, T=300, H=2, HV=2, seed=17, **mode)
    x = gen.make_inputs(case)
    gr = gen.make_backward_grads(case)
    has_state = x["initial_state"] is not None
    out = _gen_run(x, gr, want_dh0=has_state)
    ref = oracle.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"],
                          gr["dout"].float().numpy(), gr["dht"].numpy())
    got = [t.float().cpu().numpy().astype(np.float64) for t in out[:5]]
    if has_state:
        got.append(out[5].cpu().numpy())
    _compare(got, list(ref[:len(got)]))


def test_backward_gqa_group_8():
    got, ref = _run(*_case(1, 257, 2, 16, seed=977))
    _compare(got, ref)


def test_backward_varlen_gqa_workload_sampled():
    """The packed-sequence GQA workload (lengths 1, 63, 64, 65, 777, 2048, 8192; H=8, HV=32; gates U[-5, 0];
    beta = sigmoid(N(0, 4)); per-sequence states) on the GPU for all heads; the oracle checks Q/K head 5 and
    its four value heads over every sequence."""
    from kda_gated_delta_prefill_b200 import inputs as gen
    case = gen.VARLEN_GQA
    x = gen.make_inputs(case)
    gr = gen.make_backward_grads(case)
    out = _gen_run(x, gr, want_dh0=True)
    hq, grp = 5, case.HV // case.H
    hv = torch.arange(hq * grp, (hq + 1) * grp)
    sel = lambda t, dim, idx: t.index_select(dim, idx).contiguous()
    hqi = torch.tensor([hq])
    ref = oracle.backward(sel(x["q"], 2, hqi), sel(x["k"], 2, hqi), sel(x["v"], 2, hv), sel(x["g"], 2, hv),
                          sel(x["beta"], 2, hv), sel(x["initial_state"], 1, hv),
                          sel(gr["dout"], 2, hv).float().numpy(), sel(gr["dht"], 1, hv).numpy(), x["cu_seqlens"])
    got = [sel(out[0].cpu(), 2, hqi), sel(out[1].cpu(), 2, hqi)] + \
          [sel(out[i].cpu(), 2, hv) for i in (2, 3, 4)] + [sel(out[5].cpu(), 1, hv)]
    _compare([t.float().numpy().astype(np.float64) for t in got], ref)
