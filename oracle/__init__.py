"""CPU oracle for the KDA chunk-prefill forward -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import this package.  The
product library never links, loads or calls it, and it shares no code with
the CUDA path.

Two independent evaluators live here:

* ``kda_oracle.c`` (loaded through ctypes): the exact-rounding bf16 Q/K
  normalisation followed by the float64 token-by-token gated delta
  recurrence ("KDA Chunk Prefill on Ascend A3", section "Mathematical
  definition").  This is the definition the GPU path is compared against.
* ``chunk_form.py``: a numpy float64 evaluation of the page's chunk
  construction (G, L, A = solve(I+L, diag(beta)), W, U, Qg, Kg, Aqk, Vnew,
  O, S_out), used only to pin the recurrence from a second direction.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "libkda_oracle.so")
_lock = threading.Lock()
_lib = None

GCC_FLAGS = ["-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared", "-fPIC", "-std=c11"]


def build(force: bool = False) -> str:
    """Compile ``kda_oracle.c`` into ``oracle/_build/libkda_oracle.so``."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    subprocess.run(["gcc", *GCC_FLAGS, _SRC, "-o", tmp, "-lm"], check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        lib = ctypes.CDLL(build())
        P = ctypes.c_void_p
        I = ctypes.c_int
        lib.kda_oracle_l2norm_bf16.argtypes = [P, ctypes.c_int64, I, P]
        lib.kda_oracle_l2norm_bf16.restype = None
        lib.kda_oracle_recurrence_f64.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P]
        lib.kda_oracle_recurrence_f64.restype = I
        lib.kda_oracle_forward.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P]
        lib.kda_oracle_forward.restype = I
        lib.kda_oracle_backward_f64.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P]
        lib.kda_oracle_backward_f64.restype = I
        lib.kda_oracle_max_threads.argtypes = []
        lib.kda_oracle_max_threads.restype = I
        lib.kda_oracle_f64_to_bf16.argtypes = [ctypes.c_double]
        lib.kda_oracle_f64_to_bf16.restype = ctypes.c_uint16
        _lib = lib
        return lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _bf16_bits(x) -> np.ndarray:
    """Accept a torch bf16 tensor or a numpy uint16 array of bf16 bit patterns."""
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return np.ascontiguousarray(x)
    import torch
    assert x.dtype == torch.bfloat16, x.dtype
    return np.ascontiguousarray(x.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _f32(x) -> np.ndarray | None:
    if x is None:
        return None
    if isinstance(x, np.ndarray):
        return np.ascontiguousarray(x, dtype=np.float32)
    return np.ascontiguousarray(x.detach().cpu().float().numpy())


def bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact widening)."""
    return (bits.astype(np.uint32) << 16).view(np.float32)


def max_threads() -> int:
    return int(_load().kda_oracle_max_threads())


def f64_to_bf16_bits(x: float) -> int:
    return int(_load().kda_oracle_f64_to_bf16(float(x)))


def l2norm_bf16(x) -> np.ndarray:
    """Normalise rows of the last dimension; returns bf16 bit patterns (uint16)."""
    bits = _bf16_bits(x)
    K = bits.shape[-1]
    rows = bits.size // K if K else 0
    out = np.empty_like(bits)
    _load().kda_oracle_l2norm_bf16(_ptr(bits), rows, K, _ptr(out))
    return out


def recurrence_f64(qn, kn, v, g, beta, initial_state=None, cu_seqlens=None):
    """Float64 recurrence on already-normalised float64 arrays.

    Shapes: qn/kn [B,T,H,K], v [B,T,HV,V], g [B,T,HV,K], beta [B,T,HV],
    initial_state [N,HV,K,V] or None, cu_seqlens [N+1] int or None.
    Returns (o [B,T,HV,V], final_state [N,HV,K,V]) as float64.
    """
    qn = np.ascontiguousarray(qn, dtype=np.float64)
    kn = np.ascontiguousarray(kn, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    g = np.ascontiguousarray(g, dtype=np.float64)
    beta = np.ascontiguousarray(beta, dtype=np.float64)
    B, T, H, K = qn.shape
    HV, V = v.shape[2], v.shape[3]
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    N = B if cu is None else len(cu) - 1
    s0 = None if initial_state is None else np.ascontiguousarray(initial_state, dtype=np.float64)
    o = np.zeros((B, T, HV, V), np.float64)
    sN = np.empty((N, HV, K, V), np.float64)
    rc = _load().kda_oracle_recurrence_f64(_ptr(qn), _ptr(kn), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0),
                                           _ptr(cu), N, B, T, H, HV, K, V, _ptr(o), _ptr(sN))
    if rc != 0:
        raise ValueError("oracle recurrence rejected the shapes")
    return o, sN


def forward(q, k, v, g, beta, initial_state=None, cu_seqlens=None, return_normalized=False):
    """Oracle forward from raw inputs (bf16 q/k/v, f32 g/beta/state).

    Returns a dict with ``o64`` (float64), ``o16`` (bf16 bit patterns),
    ``state`` (float64) and optionally ``qn``/``kn`` (bf16 bit patterns).
    """
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    gf, bf = _f32(g), _f32(beta)
    s0 = _f32(initial_state)
    B, T, H, K = qb.shape
    HV, V = vb.shape[2], vb.shape[3]
    if cu_seqlens is not None:
        cu = np.ascontiguousarray(np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens),
                                  dtype=np.int32)
        N = len(cu) - 1
    else:
        cu, N = None, B
    o64 = np.empty((B, T, HV, V), np.float64)
    o16 = np.empty((B, T, HV, V), np.uint16)
    sN = np.empty((N, HV, K, V), np.float64)
    qn = np.empty_like(qb) if return_normalized else None
    kn = np.empty_like(kb) if return_normalized else None
    rc = _load().kda_oracle_forward(_ptr(qb), _ptr(kb), _ptr(vb), _ptr(gf), _ptr(bf), _ptr(s0), _ptr(cu),
                                    N, B, T, H, HV, K, V, _ptr(o64), _ptr(o16), _ptr(sN), _ptr(qn), _ptr(kn))
    if rc != 0:
        raise ValueError("oracle forward rejected the shapes")
    out = {"o64": o64, "o16": o16, "state": sN}
    if return_normalized:
        out["qn"], out["kn"] = qn, kn
    return out


def backward_f64(qn, kn, v, g, beta, initial_state, do, dht, cu_seqlens=None):
    """Reverse mode of ``recurrence_f64`` (same shapes and conventions) for the loss
    sum(o * do) + sum(final_state * dht) of the backward left optional on "KDA Chunk Prefill on Ascend A3"
    (section "Timing and required submission").  ``dht`` may be None (zero).

    Returns float64 arrays (dqn, dkn [B,T,HV,K] -- the gradient reaching the normalised q/k row that value
    head h read, not yet summed over a Q/K head's group --, dv [B,T,HV,V], dg [B,T,HV,K], dbeta [B,T,HV],
    ds0 [N,HV,K,V]).
    """
    qn = np.ascontiguousarray(qn, dtype=np.float64)
    kn = np.ascontiguousarray(kn, dtype=np.float64)
    v = np.ascontiguousarray(v, dtype=np.float64)
    g = np.ascontiguousarray(g, dtype=np.float64)
    beta = np.ascontiguousarray(beta, dtype=np.float64)
    do = np.ascontiguousarray(do, dtype=np.float64)
    B, T, H, K = qn.shape
    HV, V = v.shape[2], v.shape[3]
    cu = None if cu_seqlens is None else np.ascontiguousarray(cu_seqlens, dtype=np.int32)
    N = B if cu is None else len(cu) - 1
    s0 = None if initial_state is None else np.ascontiguousarray(initial_state, dtype=np.float64)
    dh = None if dht is None else np.ascontiguousarray(dht, dtype=np.float64)
    dqn = np.zeros((B, T, HV, K), np.float64)
    dkn = np.zeros((B, T, HV, K), np.float64)
    dv = np.zeros((B, T, HV, V), np.float64)
    dg = np.zeros((B, T, HV, K), np.float64)
    dbeta = np.zeros((B, T, HV), np.float64)
    ds0 = np.zeros((N, HV, K, V), np.float64)
    rc = _load().kda_oracle_backward_f64(_ptr(qn), _ptr(kn), _ptr(v), _ptr(g), _ptr(beta), _ptr(s0), _ptr(cu),
                                         N, B, T, H, HV, K, V, _ptr(do), _ptr(dh), _ptr(dqn), _ptr(dkn),
                                         _ptr(dv), _ptr(dg), _ptr(dbeta), _ptr(ds0))
    if rc != 0:
        raise ValueError("oracle backward rejected the shapes")
    return dqn, dkn, dv, dg, dbeta, ds0


def l2norm_backward_f64(x, dy, eps=1e-6):
    """Gradient through y = x / sqrt(sum(x^2) + eps) along the last axis, in float64:
    dx = dy / n - x (x . dy) / n^3 with n = sqrt(sum(x^2) + eps)."""
    x = np.asarray(x, dtype=np.float64)
    dy = np.asarray(dy, dtype=np.float64)
    n = np.sqrt((x * x).sum(-1, keepdims=True) + eps)
    return dy / n - x * (x * dy).sum(-1, keepdims=True) / n ** 3


def backward(q, k, v, g, beta, initial_state, do, dht, cu_seqlens=None):
    """Oracle backward from the raw inputs the library's forward takes.

    The forward's normalised q/k are the bf16-rounded values it uses; the rounding is passed through (its
    derivative taken as one), so dq = J_norm(q)^T sum_h dqn_h over the value heads h of q's group, with the
    normalisation's Jacobian at the raw float values.  Returns float64 (dq, dk [B,T,H,K], dv [B,T,HV,V],
    dg [B,T,HV,K], dbeta [B,T,HV], dh0 [N,HV,K,V] or None when ``initial_state`` is None).
    """
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    qn = bits_to_f32(l2norm_bf16(qb)).astype(np.float64)
    kn = bits_to_f32(l2norm_bf16(kb)).astype(np.float64)
    vf = bits_to_f32(vb).astype(np.float64)
    gf = _f32(g).astype(np.float64)
    bf = _f32(beta).astype(np.float64)
    s0 = None if initial_state is None else _f32(initial_state).astype(np.float64)
    dof = _f32(do).astype(np.float64) if not isinstance(do, np.ndarray) or do.dtype != np.uint16 else \
        bits_to_f32(do).astype(np.float64)
    dh = None if dht is None else _f32(dht).astype(np.float64)
    cu = None
    if cu_seqlens is not None:
        cu = np.asarray(cu_seqlens.cpu() if hasattr(cu_seqlens, "cpu") else cu_seqlens).astype(np.int32)
    dqn, dkn, dv, dg, dbeta, ds0 = backward_f64(qn, kn, vf, gf, bf, s0, dof, dh, cu)
    B, T, H, K = qb.shape
    HV = vb.shape[2]
    grp = HV // H
    dqn = dqn.reshape(B, T, H, grp, K).sum(3)
    dkn = dkn.reshape(B, T, H, grp, K).sum(3)
    dq = l2norm_backward_f64(bits_to_f32(qb), dqn)
    dk = l2norm_backward_f64(bits_to_f32(kb), dkn)
    return dq, dk, dv, dg, dbeta, (None if initial_state is None else ds0)


def decode_step(q, k, v, g, beta, state, state_indices):
    """One recurrent decode step per row on a state pool ("flashinfer.kda_decode.packed_kda_decode" page; the
    recurrence of "KDA Chunk Prefill on Ascend A3", section "Mathematical definition", for one token).

    q, k [B,H,K] and v [B,HV,V] (bf16 values), g [B,HV,K], beta [B,HV] (float32 values), state [N,HV,K,V]
    (the pool's values, e.g. bf16 held in float32), state_indices [B] (slot per row, -1 = padding row).
    Returns (o [B,HV,V] float64, zero on padding rows; new_state [N,HV,K,V] float64, where the slots of the
    active rows hold the updated state before any rounding and the other slots are unchanged).
    """
    qb, kb, vb = _bf16_bits(q), _bf16_bits(k), _bf16_bits(v)
    gf, bf = _f32(g), _f32(beta)
    pool = np.array(state.float().cpu().numpy() if hasattr(state, "cpu") else state, dtype=np.float64)
    idx = np.asarray(state_indices.cpu() if hasattr(state_indices, "cpu") else state_indices).astype(np.int64)
    B, H, K = qb.shape
    HV, V = vb.shape[1], vb.shape[2]
    o = np.zeros((B, HV, V), np.float64)
    rows = np.nonzero(idx >= 0)[0]
    if len(rows) == 0:
        return o, pool
    # the active rows as a batch of one-token sequences, each starting from its slot
    s0 = np.ascontiguousarray(pool[idx[rows]], dtype=np.float32)
    if not np.array_equal(s0.astype(np.float64), pool[idx[rows]]):
        raise ValueError("pool values must be float32-representable")
    res = forward(np.ascontiguousarray(qb[rows][:, None]), np.ascontiguousarray(kb[rows][:, None]),
                  np.ascontiguousarray(vb[rows][:, None]), np.ascontiguousarray(gf[rows][:, None]),
                  np.ascontiguousarray(bf[rows][:, None]), s0)
    o[rows] = res["o64"][:, 0]
    pool[idx[rows]] = res["state"]
    return o, pool

