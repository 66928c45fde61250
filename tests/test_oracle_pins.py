"""Pins of the CPU oracle against facts fixed outside it.

Every check here compares the oracle with something it does not compute
itself: the worked example printed on "KDA Chunk Prefill on Ascend A3"
(section "Example"), closed forms of the recurrence in that page's section
"Mathematical definition", a transition-matrix restatement of the same
recurrence, the page's chunk construction evaluated independently in numpy
(with ``numpy.linalg.solve`` as the triangular solve), and the tail /
varlen / GQA / resume invariances the contract implies.
"""
import json
import os

import numpy as np
import pytest
import torch

from kda_gated_delta_prefill_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def f32(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32)


def rel_fro(a, b):
    den = max(np.linalg.norm(b), 1e-300)
    return np.linalg.norm(a - b) / den


def small_case(B=1, T=37, H=1, HV=1, K=128, V=128, seed=0, state=True, gate=8.0):
    g_ = torch.Generator().manual_seed(seed)
    q = torch.randn(B, T, H, K, generator=g_).to(torch.bfloat16)
    k = torch.randn(B, T, H, K, generator=g_).to(torch.bfloat16)
    v = torch.randn(B, T, HV, V, generator=g_).to(torch.bfloat16)
    g = -torch.nn.functional.softplus(torch.randn(B, T, HV, K, generator=g_)) / gate
    beta = torch.sigmoid(torch.randn(B, T, HV, generator=g_))
    s0 = torch.randn(B, HV, K, V, generator=g_) * 0.1 if state else None
    return dict(q=q, k=k, v=v, g=g, beta=beta, initial_state=s0)


# ---------------------------------------------------------------- worked example

def test_worked_example_exact_bits(oracle):
    with open(os.path.join(GOLDEN, "worked_example.json")) as fh:
        gold = json.load(fh)
    x = gen.worked_example()
    out = oracle.forward(x["q"], x["k"], x["v"], x["g"], x["beta"])
    bits = int(gold["o_every_element_bf16_bits"], 16)
    assert np.all(out["o16"] == bits)
    assert f32(np.array([bits], np.uint16))[0] == gold["o_every_element"]
    S = out["state"][0, 0]
    assert np.all(S[0] == gold["final_state_row0"])
    assert np.all(S[1:] == gold["final_state_other_rows"])


def test_worked_example_beta_zero(oracle):
    x = gen.worked_example()
    out = oracle.forward(x["q"], x["k"], x["v"], x["g"], torch.zeros_like(x["beta"]))
    assert np.all(out["o64"] == 0.0) and np.all(out["state"] == 0.0)


def test_beta_zero_random_inputs_zero_state(oracle):
    c = small_case(state=False)
    out = oracle.forward(c["q"], c["k"], c["v"], c["g"], torch.zeros_like(c["beta"]))
    assert np.all(out["o64"] == 0.0) and np.all(out["state"] == 0.0)


# ---------------------------------------------------------------- normalisation

def test_norm_e0_stays_e0(oracle):
    x = torch.zeros(3, 128)
    x[:, 0] = 1.0
    out = oracle.l2norm_bf16(x.to(torch.bfloat16))
    assert np.all(f32(out) == x.numpy())


def test_norm_zero_row_is_zero(oracle):
    out = oracle.l2norm_bf16(torch.zeros(2, 128, dtype=torch.bfloat16))
    assert np.all(out == 0)


def test_norm_all_ones_row(oracle):
    # 1/sqrt(128 + 1e-6) rounds to bf16 0x3DB5, the same bits as 1/sqrt(128).
    out = oracle.l2norm_bf16(torch.ones(1, 128, dtype=torch.bfloat16))
    assert np.all(out == 0x3DB5)


def test_norm_eps_inside_sqrt(oracle):
    # |x|^2 = 1e-10 << 1e-6: with eps inside the root the result is ~x/1e-3 = 0.01,
    # while eps outside (x / (|x| + eps)) would give ~0.91 and no eps would give 1.
    x = torch.zeros(1, 128)
    x[0, 0] = 1e-5
    xb = x.to(torch.bfloat16)
    out = f32(oracle.l2norm_bf16(xb))[0, 0]
    xv = float(xb.float()[0, 0])
    expect = xv / np.sqrt(xv * xv + 1e-6)
    assert abs(out - expect) <= 2 ** -8 * expect
    assert 0.009 < out < 0.011


def test_norm_within_one_ulp_of_exact_quotient(oracle):
    # Rounding the real-number quotient to bf16 and the page's float32 evaluation order
    # can differ by at most one bf16 ulp, and only on rare near-ties.
    g_ = torch.Generator().manual_seed(7)
    gain = torch.exp(torch.randn(4096, 1, generator=g_) * 0.6)
    x = (gain * torch.randn(4096, 128, generator=g_)).to(torch.bfloat16)
    got = oracle.l2norm_bf16(x).astype(np.int32)
    xf = x.double().numpy()
    exact = xf / np.sqrt((xf * xf).sum(-1, keepdims=True) + float(np.float32(1e-6)))
    ref = torch.from_numpy(exact).to(torch.bfloat16).view(torch.int16).numpy().astype(np.int32)
    # same sign, compare magnitudes as integers
    diff = np.abs((got & 0x7FFF) - (ref & 0x7FFF))
    assert diff.max() <= 1
    assert (diff == 0).mean() > 0.995


def test_f64_to_bf16_rounding(oracle):
    assert oracle.f64_to_bf16_bits(1.0 / np.sqrt(128.0)) == 0x3DB5
    assert oracle.f64_to_bf16_bits(1.0) == 0x3F80
    # ties to even: 1 + 2^-8 lies exactly between 0x3F80 and 0x3F81 -> even 0x3F80
    assert oracle.f64_to_bf16_bits(1.0 + 2.0 ** -8) == 0x3F80
    assert oracle.f64_to_bf16_bits(1.0 + 3 * 2.0 ** -8) == 0x3F82
    # just above the tie rounds up (a float32 intermediate would lose this)
    assert oracle.f64_to_bf16_bits(1.0 + 2.0 ** -8 + 2.0 ** -40) == 0x3F81
    assert oracle.f64_to_bf16_bits(-2.5) == 0xC020


# ---------------------------------------------------------------- closed forms

def test_closed_form_beta_zero_with_state(oracle):
    # beta = 0: S_T = diag(exp(sum_t g_t)) S0 and o_t = K^-1/2 (q_t * exp(G_t))^T S0.
    c = small_case(T=29)
    out = oracle.forward(c["q"], c["k"], c["v"], c["g"], torch.zeros_like(c["beta"]), c["initial_state"],
                         return_normalized=True)
    g = c["g"].double().numpy()[0, :, 0]
    S0 = c["initial_state"].double().numpy()[0, 0]
    qn = f32(out["qn"])[0, :, 0].astype(np.float64)
    G = np.cumsum(g, axis=0)
    S_T = np.exp(G[-1])[:, None] * S0
    o_ref = (qn * np.exp(G)) @ S0 / np.sqrt(128.0)
    assert rel_fro(out["state"][0, 0], S_T) < 1e-12
    assert rel_fro(out["o64"][0, :, 0], o_ref) < 1e-12


def test_closed_form_orthonormal_keys(oracle):
    # g = 0, beta = 1, k_t = e_t: token t overwrites state row t with v_t, so the final
    # state rows are the v_t and o_t = K^-1/2 sum_{j<=t} q_t[j] v_j.
    T = 100
    g_ = torch.Generator().manual_seed(3)
    q = torch.randn(1, T, 1, 128, generator=g_).to(torch.bfloat16)
    k = torch.zeros(1, T, 1, 128)
    k[0, torch.arange(T), 0, torch.arange(T)] = 1.0
    v = torch.randn(1, T, 1, 128, generator=g_).to(torch.bfloat16)
    out = oracle.forward(q, k.to(torch.bfloat16), v, torch.zeros(1, T, 1, 128), torch.ones(1, T, 1),
                         return_normalized=True)
    vv = v.double().numpy()[0, :, 0]
    S = out["state"][0, 0]
    assert np.array_equal(S[:T], vv) and np.all(S[T:] == 0)
    qn = f32(out["qn"])[0, :, 0].astype(np.float64)
    o_ref = np.stack([(qn[t, :t + 1] @ vv[:t + 1]) for t in range(T)]) / np.sqrt(128.0)
    assert np.max(np.abs(out["o64"][0, :, 0] - o_ref)) < 1e-12


def test_closed_form_single_token(oracle):
    # T = 1, S0 = 0: o = K^-1/2 beta (q.k) v and S = beta k v^T.
    c = small_case(T=1, state=False)
    out = oracle.forward(c["q"], c["k"], c["v"], c["g"], c["beta"], return_normalized=True)
    qn = f32(out["qn"])[0, 0, 0].astype(np.float64)
    kn = f32(out["kn"])[0, 0, 0].astype(np.float64)
    vv = c["v"].double().numpy()[0, 0, 0]
    b = float(c["beta"][0, 0, 0])
    assert rel_fro(out["state"][0, 0], b * np.outer(kn, vv)) < 1e-13
    assert rel_fro(out["o64"][0, 0, 0], b * (qn @ kn) * vv / np.sqrt(128.0)) < 1e-12


def test_transition_matrix_form(oracle):
    # The update is S_t = (I - beta_t k_t k_t^T) diag(exp g_t) S_{t-1} + beta_t k_t v_t^T.
    rng = np.random.default_rng(11)
    T, K, V = 23, 128, 128
    qn = rng.standard_normal((1, T, 1, K)); qn /= np.linalg.norm(qn, axis=-1, keepdims=True)
    kn = rng.standard_normal((1, T, 1, K)); kn /= np.linalg.norm(kn, axis=-1, keepdims=True)
    v = rng.standard_normal((1, T, 1, V))
    g = -np.log1p(np.exp(rng.standard_normal((1, T, 1, K)))) / 4
    beta = 1 / (1 + np.exp(-rng.standard_normal((1, T, 1))))
    S0 = rng.standard_normal((1, 1, K, V)) * 0.3
    o, sN = oracle.recurrence_f64(qn, kn, v, g, beta, S0)
    S = S0[0, 0].copy()
    for t in range(T):
        kt = kn[0, t, 0]
        M = (np.eye(K) - beta[0, t, 0] * np.outer(kt, kt)) @ np.diag(np.exp(g[0, t, 0]))
        S = M @ S + beta[0, t, 0] * np.outer(kt, v[0, t, 0])
        assert rel_fro(o[0, t, 0], (qn[0, t, 0] / np.sqrt(K)) @ S) < 1e-12
    assert rel_fro(sN[0, 0], S) < 1e-12


# ---------------------------------------------------------------- chunk form

@pytest.mark.parametrize("chunk", [64, 16, 1])
def test_chunk_form_matches_recurrence(oracle, chunk):
    from oracle import chunk_form
    rng = np.random.default_rng(chunk)
    B, T, H, HV, K, V = 2, 150, 1, 2, 128, 128
    qn = rng.standard_normal((B, T, H, K)); qn /= np.linalg.norm(qn, axis=-1, keepdims=True)
    kn = rng.standard_normal((B, T, H, K)); kn /= np.linalg.norm(kn, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, HV, V))
    g = -np.log1p(np.exp(rng.standard_normal((B, T, HV, K)))) / 8
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, HV))))
    S0 = rng.standard_normal((B, HV, K, V)) * 0.1
    o1, s1 = oracle.recurrence_f64(qn, kn, v, g, beta, S0)
    o2, s2 = chunk_form.forward_f64(qn, kn, v, g, beta, S0, chunk=chunk)
    assert rel_fro(o1, o2) < 1e-10
    assert rel_fro(s1, s2) < 1e-10


def test_chunk_solve_residual():
    from oracle import chunk_form
    rng = np.random.default_rng(5)
    C, K, V = 64, 128, 128
    k = rng.standard_normal((C, K)); k /= np.linalg.norm(k, axis=-1, keepdims=True)
    q = rng.standard_normal((C, K)); q /= np.linalg.norm(q, axis=-1, keepdims=True)
    g = -np.abs(rng.standard_normal((C, K))) / 8
    beta = rng.uniform(0, 1, C)
    _, _, parts = chunk_form.chunk_step(q, k, rng.standard_normal((C, V)), g, beta, np.zeros((K, V)))
    A, L = parts["A"], parts["L"]
    assert np.max(np.abs((np.eye(C) + L) @ A - np.diag(beta))) < 1e-12
    assert np.all(np.triu(A, 1) == 0) or np.max(np.abs(np.triu(A, 1))) < 1e-14


# ---------------------------------------------------------------- invariances

def test_tail_padding_is_neutral(oracle):
    # A partial chunk padded with q = k = v = 0, g = 0, beta = 0 gives the same output rows
    # and the same final state ("zero-padding ... trimming output while preserving state").
    c = small_case(T=100)
    pad = 28
    def padt(x, val=0.0):
        z = torch.full((x.shape[0], pad) + tuple(x.shape[2:]), val, dtype=x.dtype)
        return torch.cat([x, z], dim=1)
    a = oracle.forward(c["q"], c["k"], c["v"], c["g"], c["beta"], c["initial_state"])
    b = oracle.forward(padt(c["q"]), padt(c["k"]), padt(c["v"]), padt(c["g"]), padt(c["beta"]),
                       c["initial_state"])
    assert np.array_equal(a["o64"], b["o64"][:, :100])
    assert np.array_equal(a["state"], b["state"])


def test_varlen_equals_separate_runs(oracle):
    lengths = [1, 17, 64, 65, 3]
    T = sum(lengths)
    c = small_case(T=T, H=2, HV=4, state=False, seed=9)
    s0 = torch.randn(len(lengths), 4, 128, 128, generator=torch.Generator().manual_seed(1)) * 0.1
    cu = gen.cu_seqlens_of(lengths)
    packed = oracle.forward(c["q"], c["k"], c["v"], c["g"], c["beta"], s0, cu_seqlens=cu)
    for n in range(len(lengths)):
        t0, t1 = int(cu[n]), int(cu[n + 1])
        sl = slice(t0, t1)
        one = oracle.forward(c["q"][:, sl], c["k"][:, sl], c["v"][:, sl], c["g"][:, sl], c["beta"][:, sl],
                             s0[n:n + 1])
        assert np.array_equal(packed["o64"][:, sl], one["o64"])
        assert np.array_equal(packed["state"][n], one["state"][0])


def test_gqa_equals_repeated_heads(oracle):
    # value head h reads Q/K head h // (HV/H)
    c = small_case(T=40, H=2, HV=6, seed=4)
    a = oracle.forward(c["q"], c["k"], c["v"], c["g"], c["beta"], c["initial_state"])
    rep = lambda x: x.repeat_interleave(3, dim=2)
    b = oracle.forward(rep(c["q"]), rep(c["k"]), c["v"], c["g"], c["beta"], c["initial_state"])
    assert np.array_equal(a["o64"], b["o64"]) and np.array_equal(a["state"], b["state"])


def test_split_resume_invariance(oracle):
    c = small_case(T=90, seed=12)
    full = oracle.forward(c["q"], c["k"], c["v"], c["g"], c["beta"], c["initial_state"])
    t1 = 53
    first = oracle.forward(*(c[n][:, :t1] for n in ("q", "k", "v", "g", "beta")), c["initial_state"])
    second = oracle.forward(*(c[n][:, t1:] for n in ("q", "k", "v", "g", "beta")),
                            torch.from_numpy(first["state"]).float())
    # the carried state passes through float32 once, hence a rounding-level tolerance
    assert rel_fro(second["state"], full["state"]) < 1e-6
    assert np.array_equal(first["o64"], full["o64"][:, :t1])
    assert rel_fro(second["o64"], full["o64"][:, t1:]) < 1e-6


def test_generator_is_deterministic():
    a = gen.make_inputs(gen.TAIL_STATE)
    b = gen.make_inputs(gen.TAIL_STATE)
    for key in ("q", "k", "v", "g", "beta", "initial_state"):
        assert torch.equal(a[key], b[key])
    assert a["g"].max() <= 0 and a["beta"].min() >= 0 and a["beta"].max() <= 1
    assert a["initial_state"].shape == (1, 4, 128, 128)
