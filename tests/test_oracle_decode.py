"""Pins of the oracle's decode step (one token per row on a state pool) against closed forms and against
the token recurrence over two tokens; CPU only."""
import numpy as np
import pytest
import torch

import oracle

SCALE = 128 ** -0.5


def _inputs(B, H, HV, N, seed, zero_state=False, zero_beta=False):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, 128, generator=gen).bfloat16()
    k = torch.randn(B, H, 128, generator=gen).bfloat16()
    v = torch.randn(B, HV, 128, generator=gen).bfloat16()
    g = -torch.nn.functional.softplus(torch.randn(B, HV, 128, generator=gen)) / 8
    beta = torch.zeros(B, HV) if zero_beta else torch.sigmoid(torch.randn(B, HV, generator=gen))
    pool = torch.zeros(N, HV, 128, 128) if zero_state else (0.1 * torch.randn(N, HV, 128, 128, generator=gen)).bfloat16().float()
    return q, k, v, g, beta, pool


def _normalized(x):
    return oracle.bits_to_f32(oracle.l2norm_bf16(x)).astype(np.float64)


def test_zero_state_closed_form():
    # S = 0: the new state is beta kn v^T and o = K^-0.5 beta (qn . kn) v
    q, k, v, g, beta, pool = _inputs(3, 2, 4, 5, seed=1, zero_state=True)
    idx = torch.tensor([4, 0, 2], dtype=torch.int32)
    o, new = oracle.decode_step(q, k, v, g, beta, pool, idx)
    qn, kn = _normalized(q), _normalized(k)
    vv, bb = v.float().numpy().astype(np.float64), beta.numpy().astype(np.float64)
    for b in range(3):
        for h in range(4):
            hq = h // 2
            exp_state = bb[b, h] * np.outer(kn[b, hq], vv[b, h])
            np.testing.assert_allclose(new[idx[b], h], exp_state, rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(o[b, h], SCALE * bb[b, h] * qn[b, hq] @ kn[b, hq] * vv[b, h], rtol=1e-10,
                                       atol=1e-13)


def test_zero_beta_closed_form():
    # beta = 0: the state only decays, S' = diag(exp(g)) S, and o = K^-0.5 qn^T S'
    q, k, v, g, beta, pool = _inputs(2, 1, 2, 3, seed=2, zero_beta=True)
    idx = torch.tensor([1, 2], dtype=torch.int32)
    o, new = oracle.decode_step(q, k, v, g, beta, pool, idx)
    qn = _normalized(q)
    for b in range(2):
        for h in range(2):
            s1 = np.exp(g[b, h].numpy().astype(np.float64))[:, None] * pool[idx[b], h].numpy().astype(np.float64)
            np.testing.assert_allclose(new[idx[b], h], s1, rtol=1e-12, atol=1e-15)
            np.testing.assert_allclose(o[b, h], SCALE * qn[b, 0] @ s1, rtol=1e-10, atol=1e-12)


def test_padding_rows_and_untouched_slots():
    q, k, v, g, beta, pool = _inputs(4, 2, 2, 6, seed=3)
    idx = torch.tensor([-1, 3, -1, 0], dtype=torch.int32)
    o, new = oracle.decode_step(q, k, v, g, beta, pool, idx)
    assert np.all(o[0] == 0) and np.all(o[2] == 0)
    for s in (1, 2, 4, 5):
        assert np.array_equal(new[s], pool[s].numpy().astype(np.float64))
    assert not np.array_equal(new[3], pool[3].numpy().astype(np.float64))


def test_two_steps_equal_the_two_token_recurrence():
    # two decode steps on a pool (state kept unrounded between them) == the recurrence over T = 2
    q, k, v, g, beta, pool = _inputs(4, 1, 2, 3, seed=4)  # rows 0,1 = step 1 and rows 2,3 = step 2
    idx = torch.tensor([2, 0], dtype=torch.int32)
    o1, p1 = oracle.decode_step(q[:2], k[:2], v[:2], g[:2], beta[:2], pool, idx)
    o2, p2 = oracle.decode_step(q[2:], k[2:], v[2:], g[2:], beta[2:], p1.astype(np.float32), idx)
    # the same two sequences as a plain batch of two sequences of two tokens
    stack = lambda x: torch.stack([x[:2], x[2:]], dim=1)  # [2 sequences, 2 tokens, ...]
    ref = oracle.forward(stack(q), stack(k), stack(v), stack(g), stack(beta), pool[idx.long()])
    np.testing.assert_allclose(o1, ref["o64"][:, 0], rtol=1e-12, atol=1e-13)
    # step 2 started from p1 rounded to float32, so it agrees to float32 rounding of the state
    np.testing.assert_allclose(o2, ref["o64"][:, 1], rtol=1e-5, atol=1e-6)
    np.testing.assert_allclose(p2[idx.long()], ref["state"], rtol=1e-5, atol=1e-7)
