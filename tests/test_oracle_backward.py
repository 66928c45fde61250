"""Pins of the oracle's backward (the reverse mode of the token recurrence of "KDA Chunk Prefill on Ascend A3",
section "Mathematical definition", for the loss sum(o * do) + sum(final_state * dht) that the page's section
"Timing and required submission" names) against facts fixed outside it:

* central finite differences of the oracle's float64 FORWARD recurrence (a different code path: the forward
  never forms an adjoint), on small inputs that cross the backward's 32-token checkpoint blocks, with GQA,
  varlen batches and an absent initial state;
* closed forms of the gradients for one token from a zero state, and for beta = 0 (pure decay);
* finite differences of the float64 L2 normalisation for its Jacobian.
"""
import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def _unit_rows(rng, shape):
    x = rng.standard_normal(shape)
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def _case(rng, B, T, H, HV, K=128, V=128, state=True, N=None):
    N = B if N is None else N
    qn = _unit_rows(rng, (B, T, H, K))
    kn = _unit_rows(rng, (B, T, H, K))
    v = rng.standard_normal((B, T, HV, V))
    g = -rng.random((B, T, HV, K)) * 0.4
    beta = rng.random((B, T, HV))
    s0 = rng.standard_normal((N, HV, K, V)) * 0.1 if state else None
    do = rng.standard_normal((B, T, HV, V))
    dht = rng.standard_normal((N, HV, K, V))
    return qn, kn, v, g, beta, s0, do, dht


def _loss(oracle, args, do, dht, cu):
    o, sN = oracle.recurrence_f64(*args, cu_seqlens=cu)
    return float((o * do).sum() + (sN * dht).sum())


def _fd_check(oracle, qn, kn, v, g, beta, s0, do, dht, cu=None, picks=3, seed=0, eps=1e-6):
    H, HV = qn.shape[2], v.shape[2]
    dqn, dkn, dv, dg, db, ds0 = oracle.backward_f64(qn, kn, v, g, beta, s0, do, dht, cu)
    grads = [dqn.reshape(*qn.shape[:3], HV // H, -1).sum(3), dkn.reshape(*kn.shape[:3], HV // H, -1).sum(3),
             dv, dg, db, ds0]
    args = [qn, kn, v, g, beta, s0]
    rng = np.random.default_rng(seed)
    worst = 0.0
    for i, (arr, grad) in enumerate(zip(args, grads)):
        if arr is None:
            continue
        for _ in range(picks):
            idx = tuple(int(rng.integers(0, s)) for s in arr.shape)
            p = [a if a is None else a.copy() for a in args]
            m = [a if a is None else a.copy() for a in args]
            p[i][idx] += eps
            m[i][idx] -= eps
            fd = (_loss(oracle, p, do, dht, cu) - _loss(oracle, m, do, dht, cu)) / (2 * eps)
            err = abs(fd - grad[idx]) / max(1.0, abs(fd))
            worst = max(worst, err)
            assert err < 1e-6, (i, idx, fd, grad[idx])
    return worst


def test_fd_single_head(oracle):
    rng = np.random.default_rng(1)
    _fd_check(oracle, *_case(rng, 1, 40, 1, 1), seed=2)  # 40 tokens: two checkpoint blocks


def test_fd_gqa_batch(oracle):
    rng = np.random.default_rng(3)
    _fd_check(oracle, *_case(rng, 2, 9, 1, 3), seed=4)


def test_fd_no_initial_state(oracle):
    rng = np.random.default_rng(5)
    qn, kn, v, g, beta, s0, do, dht = _case(rng, 1, 7, 1, 2, state=False)
    _fd_check(oracle, qn, kn, v, g, beta, None, do, dht, seed=6)
    _, _, _, _, _, ds0 = oracle.backward_f64(qn, kn, v, g, beta, None, do, dht)
    # the initial state's gradient does not depend on whether a state was passed (zeros == None)
    _, _, _, _, _, ds0z = oracle.backward_f64(qn, kn, v, g, beta, np.zeros_like(dht), do, dht)
    assert np.array_equal(ds0, ds0z)


def test_fd_varlen(oracle):
    rng = np.random.default_rng(7)
    cu = np.array([0, 3, 3, 11, 36], np.int32)  # includes an empty sequence and one crossing a checkpoint
    qn, kn, v, g, beta, s0, do, dht = _case(rng, 1, 36, 2, 4, N=4)
    _fd_check(oracle, qn, kn, v, g, beta, s0, do, dht, cu=cu, seed=8)
    # the empty sequence passes the state gradient straight through
    _, _, _, _, _, ds0 = oracle.backward_f64(qn, kn, v, g, beta, s0, do, dht, cu)
    assert np.array_equal(ds0[1], dht[1])


def test_one_token_from_zero_state_closed_form(oracle):
    """T = 1, S0 = 0: o = s beta (q.k) v and S = beta k v^T, so
    dv = s beta (q.k) do + beta dht^T k,  dbeta = s (q.k)(v.do) + k^T dht v,  dq = s beta (v.do) k,
    dk = s beta (v.do) q + beta dht v,  dg = 0,
    ds0 = diag(e^g) (D - beta k k^T D) with D = dht + s q do^T."""
    rng = np.random.default_rng(9)
    K = V = 128
    s = 1 / np.sqrt(K)
    qn, kn, v, g, beta, _, do, dht = _case(rng, 1, 1, 1, 1, state=False)
    q, k, vv, gg, b, dd = qn[0, 0, 0], kn[0, 0, 0], v[0, 0, 0], g[0, 0, 0], beta[0, 0, 0], do[0, 0, 0]
    Dh = dht[0, 0]
    dqn, dkn, dv, dg, db, ds0 = oracle.backward_f64(qn, kn, v, g, beta, None, do, dht)
    qk, vd = q @ k, vv @ dd
    np.testing.assert_allclose(dv[0, 0, 0], s * b * qk * dd + b * (Dh.T @ k), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(db[0, 0, 0], s * qk * vd + k @ Dh @ vv, rtol=1e-12)
    np.testing.assert_allclose(dqn[0, 0, 0], s * b * vd * k, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(dkn[0, 0, 0], s * b * vd * q + b * (Dh @ vv), rtol=1e-12, atol=1e-12)
    assert np.all(dg == 0)
    D = Dh + s * np.outer(q, dd)
    ref = np.exp(gg)[:, None] * (D - b * np.outer(k, k @ D))
    np.testing.assert_allclose(ds0[0, 0], ref, rtol=1e-12, atol=1e-13)


def test_pure_decay_closed_form(oracle):
    """beta = 0: S_t = diag(e^{G_t}) S0 with G the inclusive cumulative gate, o_t = s q_t^T diag(e^{G_t}) S0.
    Then dv = dk = 0, dq_t = s diag(e^{G_t}) S0 do_t,
    ds0 = sum_t s diag(e^{G_t}) q_t do_t^T + diag(e^{G_T}) dht,
    dg_t = sum_{t' >= t} s q_t' * e^{G_t'} * (S0 do_t') + e^{G_T} * rowsum(S0 * dht)."""
    rng = np.random.default_rng(10)
    T, K = 6, 128
    s = 1 / np.sqrt(K)
    qn, kn, v, g, beta, s0, do, dht = _case(rng, 1, T, 1, 1)
    beta[:] = 0.0
    dqn, dkn, dv, dg, db, ds0 = oracle.backward_f64(qn, kn, v, g, beta, s0, do, dht)
    S0, Dh = s0[0, 0], dht[0, 0]
    G = np.cumsum(g[0, :, 0], axis=0)
    assert np.all(dv == 0) and np.all(dkn == 0)
    term = np.stack([s * qn[0, t, 0] * np.exp(G[t]) * (S0 @ do[0, t, 0]) for t in range(T)])
    last = np.exp(G[-1]) * (S0 * Dh).sum(1)
    for t in range(T):
        np.testing.assert_allclose(dqn[0, t, 0], s * np.exp(G[t]) * (S0 @ do[0, t, 0]), rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(dg[0, t, 0], term[t:].sum(0) + last, rtol=1e-10, atol=1e-12)
    ref = sum(s * np.outer(np.exp(G[t]) * qn[0, t, 0], do[0, t, 0]) for t in range(T)) + np.exp(G[-1])[:, None] * Dh
    np.testing.assert_allclose(ds0[0, 0], ref, rtol=1e-11, atol=1e-13)
    # dbeta is the derivative of switching the write on: k_t^T dS_t r_t, checked by differences
    _fd_check(oracle, qn, kn, v, g, beta, s0, do, dht, picks=2, seed=11)


def test_l2norm_jacobian(oracle):
    rng = np.random.default_rng(12)
    x = rng.standard_normal((3, 128)) * np.array([[1.0], [1e-3], [10.0]])
    dy = rng.standard_normal((3, 128))
    dx = oracle.l2norm_backward_f64(x, dy)

    def f(xx):
        return float((xx / np.sqrt((xx * xx).sum(-1, keepdims=True) + 1e-6) * dy).sum())

    for r, c in [(0, 5), (1, 77), (2, 127)]:
        h = 1e-6 * max(1e-3, abs(x[r, c]))
        p, m = x.copy(), x.copy()
        p[r, c] += h
        m[r, c] -= h
        fd = (f(p) - f(m)) / (2 * h)
        assert abs(fd - dx[r, c]) <= 1e-6 * max(1.0, abs(fd)), (r, c, fd, dx[r, c])


def test_raw_input_backward_matches_differences_loosely(oracle):
    """The raw-input wrapper (bf16 normalisation passed straight through) against differences of the smooth
    float64 forward with unrounded normalisation: equal up to the bf16 rounding of the normalised rows."""
    import torch
    rng = np.random.default_rng(13)
    B, T, H, HV, K = 1, 5, 1, 2, 128
    q = torch.from_numpy(rng.standard_normal((B, T, H, K))).to(torch.bfloat16)
    k = torch.from_numpy(rng.standard_normal((B, T, H, K))).to(torch.bfloat16)
    v = torch.from_numpy(rng.standard_normal((B, T, HV, K))).to(torch.bfloat16)
    g = torch.from_numpy(-rng.random((B, T, HV, K)) * 0.4).float()
    beta = torch.from_numpy(rng.random((B, T, HV))).float()
    s0 = torch.from_numpy(rng.standard_normal((B, HV, K, K)) * 0.1).float()
    do = rng.standard_normal((B, T, HV, K))
    dht = rng.standard_normal((B, HV, K, K))
    dq, dk, dv, dg, db, dh0 = oracle.backward(q, k, v, g, beta, s0, do, dht)
    qf, kf = q.float().numpy().astype(np.float64), k.float().numpy().astype(np.float64)
    args = [v.float().numpy().astype(np.float64), g.numpy().astype(np.float64),
            beta.numpy().astype(np.float64), s0.numpy().astype(np.float64)]

    def nrm(x):
        return x / np.sqrt((x * x).sum(-1, keepdims=True) + 1e-6)

    def loss(qq, kk):
        o, sN = oracle.recurrence_f64(nrm(qq), nrm(kk), *args)
        return float((o * do).sum() + (sN * dht).sum())

    fd_q, fd_k = np.zeros(K), np.zeros(K)
    for c in range(K):
        p, m = qf.copy(), qf.copy()
        p[0, 2, 0, c] += 1e-6
        m[0, 2, 0, c] -= 1e-6
        fd_q[c] = (loss(p, kf) - loss(m, kf)) / 2e-6
        p, m = kf.copy(), kf.copy()
        p[0, 1, 0, c] += 1e-6
        m[0, 1, 0, c] -= 1e-6
        fd_k[c] = (loss(qf, p) - loss(qf, m)) / 2e-6
    rel = np.linalg.norm(dq[0, 2, 0] - fd_q) / np.linalg.norm(fd_q)
    assert rel < 2e-2, rel
    rel = np.linalg.norm(dk[0, 1, 0] - fd_k) / np.linalg.norm(fd_k)
    assert rel < 2e-2, rel
