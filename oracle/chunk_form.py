"""Float64 numpy evaluation of the KDA chunk construction -- TEST INFRASTRUCTURE ONLY.

Written from "KDA Chunk Prefill on Ascend A3", section "Mathematical
definition" (the chunk construction and the paragraph on chunk size and
tail padding).  For one sequence, one value head and a chunk of C tokens
(zero-based, in token order), with G the inclusive per-channel cumulative
gate:

    L_ij   = beta_i * sum_d k_id k_jd exp(G_id - G_jd)     (j < i, else 0)
    A      = solve(I + L, diag(beta))
    W      = A @ (exp(G) * k)          U = A @ v
    Qg_i   = K^-0.5 q_i exp(G_i)       Kg_i = k_i exp(G_last - G_i)
    Aqk_ij = K^-0.5 sum_d q_id k_jd exp(G_id - G_jd)    (j <= i, else 0)
    Vnew   = U - W @ S_in
    O      = Qg @ S_in + Aqk @ Vnew
    S_out  = exp(G_last)[:, None] * S_in + Kg.T @ Vnew

The last partial chunk is zero-padded in q/k/v/g/beta; output rows of the
padding are dropped and the state is kept.  Inputs here are the already
normalised Q/K; this module never normalises.  It shares no code with the
C recurrence oracle and is used only to pin it.
"""
from __future__ import annotations

import numpy as np


def chunk_step(q, k, v, g, beta, S_in):
    """One chunk, literally as the equations read.  q,k,g [C,K]; v [C,V]; beta [C]; S_in [K,V]."""
    C, K = q.shape
    scale = K ** -0.5
    G = np.cumsum(g, axis=0)                       # G_i = sum_{u<=i} g_u
    diff = G[:, None, :] - G[None, :, :]           # [i, j, d] = G_id - G_jd
    lower_strict = np.tril(np.ones((C, C), dtype=bool), k=-1)
    causal = np.tril(np.ones((C, C), dtype=bool), k=0)
    # exp is only evaluated where the mask keeps the entry (j <= i), where G_i - G_j <= 0 for g <= 0.
    e = np.where(causal[:, :, None], np.exp(np.where(causal[:, :, None], diff, 0.0)), 0.0)
    kk = np.einsum("id,jd,ijd->ij", k, k, e)
    qk = np.einsum("id,jd,ijd->ij", q, k, e)
    L = np.where(lower_strict, beta[:, None] * kk, 0.0)
    A = np.linalg.solve(np.eye(C) + L, np.diag(beta))
    W = A @ (np.exp(G) * k)
    U = A @ v
    Qg = scale * q * np.exp(G)
    Kg = k * np.exp(G[-1][None, :] - G)
    Aqk = np.where(causal, scale * qk, 0.0)
    Vnew = U - W @ S_in
    O = Qg @ S_in + Aqk @ Vnew
    S_out = np.exp(G[-1])[:, None] * S_in + Kg.T @ Vnew
    return O, S_out, {"G": G, "L": L, "A": A, "W": W, "U": U, "Qg": Qg, "Kg": Kg, "Aqk": Aqk, "Vnew": Vnew}


def sequence_forward(q, k, v, g, beta, S0, chunk):
    """One (sequence, value head): q,k,g [T,K]; v [T,V]; beta [T]; S0 [K,V] -> (o [T,V], S [K,V])."""
    T, K = q.shape
    V = v.shape[1]
    S = np.array(S0, dtype=np.float64, copy=True)
    o = np.zeros((T, V), np.float64)
    for c0 in range(0, T, chunk):
        n = min(chunk, T - c0)
        pad = chunk - n

        def padded(x):
            x = np.asarray(x[c0:c0 + n], dtype=np.float64)
            if pad:
                x = np.concatenate([x, np.zeros((pad,) + x.shape[1:], np.float64)], axis=0)
            return x

        O, S, _ = chunk_step(padded(q), padded(k), padded(v), padded(g), padded(beta), S)
        o[c0:c0 + n] = O[:n]
    return o, S


def forward_f64(qn, kn, v, g, beta, initial_state=None, cu_seqlens=None, chunk=64):
    """Whole forward in the chunk form.  Shapes as the C oracle's recurrence_f64."""
    qn, kn, v, g, beta = (np.asarray(a, dtype=np.float64) for a in (qn, kn, v, g, beta))
    B, T, H, K = qn.shape
    HV, V = v.shape[2], v.shape[3]
    group = HV // H
    if cu_seqlens is None:
        seqs = [(b, 0, T) for b in range(B)]
    else:
        cu = [int(x) for x in cu_seqlens]
        seqs = [(0, cu[n], cu[n + 1]) for n in range(len(cu) - 1)]
    o = np.zeros((B, T, HV, V), np.float64)
    sN = np.zeros((len(seqs), HV, K, V), np.float64)
    for n, (b, t0, t1) in enumerate(seqs):
        for h in range(HV):
            hq = h // group
            S0 = np.zeros((K, V)) if initial_state is None else initial_state[n, h]
            on, Sn = sequence_forward(qn[b, t0:t1, hq], kn[b, t0:t1, hq], v[b, t0:t1, h],
                                      g[b, t0:t1, h], beta[b, t0:t1, h], S0, chunk)
            o[b, t0:t1, h] = on
            sN[n, h] = Sn
    return o, sN
