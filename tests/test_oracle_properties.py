"""Property-based pins of the oracle (CPU): structural facts of the token recurrence of "KDA Chunk Prefill on
Ascend A3" (section "Mathematical definition"), checked on randomly drawn shapes, packings and gate strengths
instead of a few fixed cases.

* Packed sequences are independent: a packed batch equals its sequences run one by one (bit for bit).
* GQA: value head h reads Q/K head h // (HV/H), so repeating each Q/K head HV/H times changes nothing.
* The recurrence is a chain: running a sequence in two pieces, the second from the first's float64 end state,
  equals one run (bit for bit).
* The chunk form (the page's construction, in the independent numpy evaluator) equals the recurrence for any
  chunk size, including a ragged last chunk.
* The reverse mode is linear in the loss's cotangents (do, dht), independent across packed sequences, and
  unchanged when shared Q/K heads are repeated.
"""
import numpy as np
from hypothesis import given, settings
from hypothesis import strategies as st

import oracle
from oracle import chunk_form

K = V = 128
SETTINGS = dict(max_examples=12, deadline=None, derandomize=True)


def _draw(seed, B, T, H, HV, N, gate_div):
    rng = np.random.default_rng(seed)
    qn = rng.standard_normal((B, T, H, K))
    qn /= np.linalg.norm(qn, axis=-1, keepdims=True)
    kn = rng.standard_normal((B, T, H, K))
    kn /= np.linalg.norm(kn, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, HV, V))
    g = -np.log1p(np.exp(rng.standard_normal((B, T, HV, K)))) / gate_div
    beta = 1 / (1 + np.exp(-rng.standard_normal((B, T, HV))))
    s0 = rng.standard_normal((N, HV, K, V)) * 0.1
    return qn, kn, v, g, beta, s0


@settings(**SETTINGS)
@given(lengths=st.lists(st.integers(0, 40), min_size=1, max_size=4), H=st.integers(1, 2), grp=st.integers(1, 3),
       gate_div=st.sampled_from([1.0, 8.0, 128.0]), seed=st.integers(0, 2 ** 16))
def test_packed_batch_equals_separate_runs(lengths, H, grp, gate_div, seed):
    T, N, HV = sum(lengths), len(lengths), H * grp
    if T == 0:
        return
    qn, kn, v, g, beta, s0 = _draw(seed, 1, T, H, HV, N, gate_div)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    o, sN = oracle.recurrence_f64(qn, kn, v, g, beta, s0, cu)
    for n in range(N):
        sl = slice(int(cu[n]), int(cu[n + 1]))
        if cu[n] == cu[n + 1]:
            assert np.array_equal(sN[n], s0[n])  # an empty sequence passes its state through
            continue
        o1, s1 = oracle.recurrence_f64(qn[:, sl], kn[:, sl], v[:, sl], g[:, sl], beta[:, sl], s0[n:n + 1])
        assert np.array_equal(o[:, sl], o1)
        assert np.array_equal(sN[n], s1[0])


@settings(**SETTINGS)
@given(T=st.integers(1, 50), H=st.integers(1, 2), grp=st.integers(2, 4), seed=st.integers(0, 2 ** 16))
def test_gqa_equals_repeated_heads(T, H, grp, seed):
    HV = H * grp
    qn, kn, v, g, beta, s0 = _draw(seed, 1, T, H, HV, 1, 8.0)
    o, sN = oracle.recurrence_f64(qn, kn, v, g, beta, s0)
    rep = lambda x: np.repeat(x, grp, axis=2)
    o2, s2 = oracle.recurrence_f64(rep(qn), rep(kn), v, g, beta, s0)
    assert np.array_equal(o, o2) and np.array_equal(sN, s2)


@settings(**SETTINGS)
@given(T=st.integers(2, 60), cut=st.floats(0.05, 0.95), seed=st.integers(0, 2 ** 16))
def test_two_pieces_equal_one_run(T, cut, seed):
    qn, kn, v, g, beta, s0 = _draw(seed, 1, T, 1, 2, 1, 8.0)
    t1 = min(T - 1, max(1, int(T * cut)))
    o, sN = oracle.recurrence_f64(qn, kn, v, g, beta, s0)
    a = lambda x: x[:, :t1]
    b = lambda x: x[:, t1:]
    oa, sa = oracle.recurrence_f64(a(qn), a(kn), a(v), a(g), a(beta), s0)
    ob, sb = oracle.recurrence_f64(b(qn), b(kn), b(v), b(g), b(beta), sa)
    assert np.array_equal(o[:, :t1], oa) and np.array_equal(o[:, t1:], ob)
    assert np.array_equal(sN, sb)


@settings(**SETTINGS)
@given(T=st.integers(1, 70), chunk=st.sampled_from([1, 3, 16, 64]), gate_div=st.sampled_from([1.0, 8.0]),
       seed=st.integers(0, 2 ** 16))
def test_chunk_form_equals_recurrence_for_any_chunk_size(T, chunk, gate_div, seed):
    qn, kn, v, g, beta, s0 = _draw(seed, 1, T, 1, 1, 1, gate_div)
    o1, s1 = oracle.recurrence_f64(qn, kn, v, g, beta, s0)
    o2, s2 = chunk_form.forward_f64(qn, kn, v, g, beta, s0, chunk=chunk)
    rel = lambda a, b: np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300)
    assert rel(o2, o1) < 1e-9 and rel(s2, s1) < 1e-9


# ------------------------------------------------------------------------------------------------ backward
# The reverse mode (oracle.backward_f64) for the loss sum(o * do) + sum(final_state * dht).

@settings(**SETTINGS)
@given(T=st.integers(1, 45), H=st.integers(1, 2), grp=st.integers(1, 2), a=st.floats(-2, 2), b=st.floats(-2, 2),
       seed=st.integers(0, 2 ** 16))
def test_backward_is_linear_in_the_cotangents(T, H, grp, a, b, seed):
    """Gradients are linear in (do, dht) for fixed inputs."""
    HV = H * grp
    qn, kn, v, g, beta, s0 = _draw(seed, 1, T, H, HV, 1, 8.0)
    rng = np.random.default_rng(seed + 1)
    do1, do2 = rng.standard_normal((2, 1, T, HV, V))
    dh1, dh2 = rng.standard_normal((2, 1, HV, K, V))
    g1 = oracle.backward_f64(qn, kn, v, g, beta, s0, do1, dh1)
    g2 = oracle.backward_f64(qn, kn, v, g, beta, s0, do2, dh2)
    g12 = oracle.backward_f64(qn, kn, v, g, beta, s0, a * do1 + b * do2, a * dh1 + b * dh2)
    for x1, x2, x12 in zip(g1, g2, g12):
        want = a * x1 + b * x2
        assert np.abs(x12 - want).max() <= 1e-9 * max(1.0, np.abs(want).max())


@settings(**SETTINGS)
@given(lengths=st.lists(st.integers(0, 40), min_size=1, max_size=3), grp=st.integers(1, 2),
       seed=st.integers(0, 2 ** 16))
def test_backward_of_a_packed_batch_equals_separate_runs(lengths, grp, seed):
    T, N, H = sum(lengths), len(lengths), 1
    HV = H * grp
    if T == 0:
        return
    qn, kn, v, g, beta, s0 = _draw(seed, 1, T, H, HV, N, 8.0)
    rng = np.random.default_rng(seed + 2)
    do = rng.standard_normal((1, T, HV, V))
    dht = rng.standard_normal((N, HV, K, V))
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    packed = oracle.backward_f64(qn, kn, v, g, beta, s0, do, dht, cu)
    for n in range(N):
        sl = slice(int(cu[n]), int(cu[n + 1]))
        if cu[n] == cu[n + 1]:
            assert np.array_equal(packed[5][n], dht[n])  # an empty sequence passes the state gradient through
            continue
        one = oracle.backward_f64(qn[:, sl], kn[:, sl], v[:, sl], g[:, sl], beta[:, sl], s0[n:n + 1], do[:, sl],
                                  dht[n:n + 1])
        for x, y in zip(packed[:5], one[:5]):
            np.testing.assert_allclose(x[:, sl], y, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(packed[5][n], one[5][0], rtol=1e-12, atol=1e-14)


@settings(**SETTINGS)
@given(T=st.integers(1, 40), grp=st.integers(2, 3), seed=st.integers(0, 2 ** 16))
def test_backward_gqa_equals_repeated_heads(T, grp, seed):
    """The per-value-head gradients at the normalised rows do not depend on whether Q/K heads are shared."""
    qn, kn, v, g, beta, s0 = _draw(seed, 1, T, 1, grp, 1, 8.0)
    rng = np.random.default_rng(seed + 3)
    do = rng.standard_normal((1, T, grp, V))
    dht = rng.standard_normal((1, grp, K, V))
    a = oracle.backward_f64(qn, kn, v, g, beta, s0, do, dht)
    rep = lambda x: np.repeat(x, grp, axis=2)
    b = oracle.backward_f64(rep(qn), rep(kn), v, g, beta, s0, do, dht)
    for x, y in zip(a, b):
        assert np.array_equal(x, y)
