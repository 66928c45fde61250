"""KDA chunk-prefill forward for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI in ``include/kda_prefill.h``: argument
marshalling only.  Every step of the forward runs in the CUDA kernels of
``libkda_prefill.so``; there is no CPU path.  If the library is missing the
calls raise, they never fall back.

    o, final_state = forward(q, k, v, g, beta, initial_state=None, cu_seqlens=None)

Shapes ("KDA Chunk Prefill on Ascend A3", section "Function and tensor
contract"): q, k [B,T,H,128] bf16; v [B,T,HV,128] bf16; g [B,T,HV,128]
fp32; beta [B,T,HV] fp32; initial_state [N,HV,128,128] fp32 or None;
cu_seqlens [N+1] int32 or None (then B must be 1).  Returns o
[B,T,HV,128] bf16 and final_state [N,HV,128,128] fp32.
"""
from __future__ import annotations

import ctypes
import os
import threading

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "_lib", "libkda_prefill.so")

STATUS = {0: "KDA_OK", 1: "KDA_ERR_INVALID_ARG", 2: "KDA_ERR_UNSUPPORTED", 3: "KDA_ERR_MISALIGNED",
          4: "KDA_ERR_WORKSPACE", 5: "KDA_ERR_CUDA"}

EXPORTED = ("kda_status_string", "kda_prefill_workspace_size", "kda_prefill_forward",
            "kda_prefill_host_staging_size", "kda_prefill_forward_host", "kda_prefill_device_error",
            "kda_l2norm_bf16", "kda_prefill_kernel_launches", "kda_decode_step",
            "kda_prefill_backward_workspace_size", "kda_prefill_backward_kernel_launches", "kda_prefill_backward",
            "kda_prefill_state_bf16_workspace_size", "kda_prefill_forward_state_bf16",
            "kda_prefill_forward_save", "kda_prefill_backward_saved", "kda_prefill_forward_varlen",
            "kda_prefill_varlen_kernel_launches")


class KdaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


_lock = threading.Lock()
_lib = None


def lib():
    """Load libkda_prefill.so (raises if it has not been built)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"CUDA library not built: {LIB_PATH} is missing "
                               "(run python -m kda_gated_delta_prefill_b200.build)")
        L = ctypes.CDLL(LIB_PATH)
        P, I, Z, I64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t, ctypes.c_int64
        L.kda_status_string.argtypes = [I]
        L.kda_status_string.restype = ctypes.c_char_p
        L.kda_prefill_workspace_size.argtypes = [I] * 7
        L.kda_prefill_workspace_size.restype = Z
        L.kda_prefill_forward.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, Z, P]
        L.kda_prefill_forward.restype = I
        L.kda_prefill_host_staging_size.argtypes = [I] * 9
        L.kda_prefill_host_staging_size.restype = Z
        L.kda_prefill_forward_host.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, Z, P]
        L.kda_prefill_forward_host.restype = I
        L.kda_prefill_device_error.argtypes = [P, I]
        L.kda_prefill_device_error.restype = I
        L.kda_l2norm_bf16.argtypes = [P, I64, I, P, P]
        L.kda_l2norm_bf16.restype = I
        L.kda_prefill_kernel_launches.argtypes = [I] * 7
        L.kda_prefill_kernel_launches.restype = I
        L.kda_decode_step.argtypes = [P, I64, P, I64, P, I64, P, P, P, I64, I, P, I, I, I, I, I, P, P]
        L.kda_decode_step.restype = I
        L.kda_prefill_backward_workspace_size.argtypes = [I] * 7
        L.kda_prefill_backward_workspace_size.restype = Z
        L.kda_prefill_backward_kernel_launches.argtypes = [I] * 7
        L.kda_prefill_backward_kernel_launches.restype = I
        L.kda_prefill_backward.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, Z, P]
        L.kda_prefill_backward.restype = I
        L.kda_prefill_state_bf16_workspace_size.argtypes = [I] * 7
        L.kda_prefill_state_bf16_workspace_size.restype = Z
        L.kda_prefill_forward_state_bf16.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, Z, P]
        L.kda_prefill_forward_state_bf16.restype = I
        L.kda_prefill_forward_save.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, Z, P]
        L.kda_prefill_forward_save.restype = I
        L.kda_prefill_backward_saved.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P, P, P, P, P, P, P, Z, P]
        L.kda_prefill_backward_saved.restype = I
        L.kda_prefill_forward_varlen.argtypes = [P, P, P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, Z, P]
        L.kda_prefill_forward_varlen.restype = I
        L.kda_prefill_varlen_kernel_launches.argtypes = [I, I, I, I, I, I, P]
        L.kda_prefill_varlen_kernel_launches.restype = I
        _lib = L
        return L


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream_ptr(stream, device=None):
    import torch
    if stream is None:
        stream = torch.cuda.current_stream(device)
    return ctypes.c_void_p(stream.cuda_stream)


def _on(device):
    """The calls launch on the CUDA runtime's current device: make it the tensors' device for the call."""
    import torch
    return torch.cuda.device(device)


def _need_all(checks, device=None, *, host=False):
    """The library reads and writes raw pointers, so a tensor of another dtype or size would let its kernels run
    past the buffer.  ``checks``: (name, tensor or None, dtype, element count or None, contiguous); first every
    dtype and size, then placement (``device``, or host memory) and layout."""
    checks = [c for c in checks if c[1] is not None]
    for name, t, dtype, numel, _ in checks:
        if t.dtype != dtype:
            raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
        if numel is not None and t.numel() != numel:
            raise ValueError(f"{name} must hold {numel} elements, got {t.numel()}")
    for name, t, _, _, contiguous in checks:
        if host:
            if t.is_cuda:
                raise ValueError(f"{name} must be a host tensor")
        else:
            if not t.is_cuda:
                raise ValueError(f"{name} must be a CUDA tensor")
            if device is not None and t.device != device:
                raise ValueError(f"{name} is on {t.device}, the other tensors on {device}")
        if contiguous and not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")


def _need(name, t, dtype, numel, device=None, *, host=False, contiguous=True):
    _need_all([(name, t, dtype, numel, contiguous)], device, host=host)


def _need_inputs(q, k, v, g, beta, initial_state, cu_seqlens, state_dtype=None, host=False, more=None):
    """Checks of the forward's inputs, and of ``more(B, T, H, HV, K, V, N)``: further checks in ``_need_all``'s
    form.  Returns (B, T, H, HV, K, V, N, device)."""
    import torch
    if q.dim() != 4 or v.dim() != 4:
        raise ValueError("q must be [B,T,H,K] and v [B,T,HV,V]")
    B, T, H, HV, K, V, N = _dims(q, v, cu_seqlens)
    dev = None if host else q.device
    bt = B * T
    checks = [("q", q, torch.bfloat16, bt * H * K, True), ("k", k, torch.bfloat16, bt * H * K, True),
              ("v", v, torch.bfloat16, bt * HV * V, True), ("g", g, torch.float32, bt * HV * K, True),
              ("beta", beta, torch.float32, bt * HV, True),
              ("initial_state", initial_state, state_dtype or torch.float32, N * HV * K * V, True),
              ("cu_seqlens", cu_seqlens, torch.int32, None, True)]
    if more is not None:
        checks += more(B, T, H, HV, K, V, N)
    _need_all(checks, dev, host=host)
    return B, T, H, HV, K, V, N, dev


def _check(rc: int, where: str):
    if rc != 0:
        raise KdaError(rc, where)


def _dims(q, v, cu_seqlens):
    B, T, H, K = q.shape
    HV, V = v.shape[2], v.shape[3]
    N = B if cu_seqlens is None else cu_seqlens.numel() - 1
    return B, T, H, HV, K, V, N


def workspace_size(B, T, H, HV, K=128, V=128, num_seqs=0) -> int:
    return int(lib().kda_prefill_workspace_size(B, T, H, HV, K, V, num_seqs))


def kernel_launches(B, T, H, HV, K=128, V=128, num_seqs=0) -> int:
    """Kernel launches one forward makes for these sizes on the current CUDA device (0 if rejected)."""
    return int(lib().kda_prefill_kernel_launches(B, T, H, HV, K, V, num_seqs))


def _host_cu(cu_seqlens_host):
    """A host copy of cu_seqlens (sequence, numpy array or CPU tensor) as contiguous int32 numpy."""
    import numpy as np
    if hasattr(cu_seqlens_host, "detach"):
        if cu_seqlens_host.device.type != "cpu":
            raise ValueError("cu_seqlens_host must be in host memory")
        cu_seqlens_host = cu_seqlens_host.detach().numpy()
    return np.ascontiguousarray(np.asarray(cu_seqlens_host, dtype=np.int32))


def varlen_kernel_launches(T, H, HV, cu_seqlens_host, K=128, V=128) -> int:
    """Kernel launches forward(..., cu_seqlens_host=...) makes for these lengths (0 if rejected)."""
    cu = _host_cu(cu_seqlens_host)
    return int(lib().kda_prefill_varlen_kernel_launches(T, H, HV, K, V, cu.size - 1,
                                                        cu.ctypes.data_as(ctypes.c_void_p)))


def forward(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *, o=None, final_state=None,
            workspace=None, stream=None, cu_seqlens_host=None):
    """Run the forward on CUDA tensors; returns (o, final_state).

    cu_seqlens_host: optional host copy of cu_seqlens (same values).  With it the library knows the sequence
    lengths and can overlap a packed batch's state carry with its intra-chunk work (kda_prefill_forward_varlen).
    """
    import torch
    B, T, H, HV, K, V, N, dev = _need_inputs(q, k, v, g, beta, initial_state, cu_seqlens)
    if cu_seqlens_host is not None and cu_seqlens is None:
        raise ValueError("cu_seqlens_host needs cu_seqlens")
    if o is None:
        o = torch.empty(B, T, HV, V, dtype=torch.bfloat16, device=dev)
    if final_state is None:
        final_state = torch.empty(N, HV, K, V, dtype=torch.float32, device=dev)
    _need("o", o, torch.bfloat16, B * T * HV * V, dev)
    _need("final_state", final_state, torch.float32, N * HV * K * V, dev)
    num_seqs = N if cu_seqlens is not None else 0
    ws_bytes = workspace_size(B, T, H, HV, K, V, num_seqs)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    if workspace is not None:
        _need("workspace", workspace, torch.uint8, None, dev)
    ws_n = workspace.numel() if workspace is not None else 0
    with _on(dev):
        if cu_seqlens_host is not None:
            cu_h = _host_cu(cu_seqlens_host)
            if cu_h.size != N + 1:
                raise ValueError(f"cu_seqlens_host has {cu_h.size} entries, expected {N + 1}")
            rc = lib().kda_prefill_forward_varlen(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                                  _ptr(initial_state), _ptr(cu_seqlens),
                                                  cu_h.ctypes.data_as(ctypes.c_void_p), num_seqs, T, H, HV, K, V,
                                                  _ptr(o), _ptr(final_state), _ptr(workspace), ws_n,
                                                  _stream_ptr(stream, dev))
            _check(rc, "kda_prefill_forward_varlen")
            return o, final_state
        rc = lib().kda_prefill_forward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state),
                                       _ptr(cu_seqlens), num_seqs, B, T, H, HV, K, V, _ptr(o), _ptr(final_state),
                                       _ptr(workspace), ws_n, _stream_ptr(stream, dev))
    _check(rc, "kda_prefill_forward")
    return o, final_state


def forward_state_bf16(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *, o=None, final_state=None,
                       workspace=None, stream=None):
    """The forward with a bf16 state: initial_state bf16 [N,HV,K,V] or None; returns (o, final_state bf16)."""
    import torch
    B, T, H, HV, K, V, N, dev = _need_inputs(q, k, v, g, beta, initial_state, cu_seqlens,
                                             state_dtype=torch.bfloat16)
    if o is None:
        o = torch.empty(B, T, HV, V, dtype=torch.bfloat16, device=dev)
    if final_state is None:
        final_state = torch.empty(N, HV, K, V, dtype=torch.bfloat16, device=dev)
    _need("o", o, torch.bfloat16, B * T * HV * V, dev)
    _need("final_state", final_state, torch.bfloat16, N * HV * K * V, dev)
    num_seqs = N if cu_seqlens is not None else 0
    ws_bytes = int(lib().kda_prefill_state_bf16_workspace_size(B, T, H, HV, K, V, num_seqs))
    if workspace is None:
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    _need("workspace", workspace, torch.uint8, None, dev)
    with _on(dev):
        rc = lib().kda_prefill_forward_state_bf16(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta),
                                                  _ptr(initial_state), _ptr(cu_seqlens), num_seqs, B, T, H, HV, K,
                                                  V, _ptr(o), _ptr(final_state), _ptr(workspace), workspace.numel(),
                                                  _stream_ptr(stream, dev))
    _check(rc, "kda_prefill_forward_state_bf16")
    return o, final_state


def backward_workspace_size(B, T, H, HV, K=128, V=128, num_seqs=0) -> int:
    return int(lib().kda_prefill_backward_workspace_size(B, T, H, HV, K, V, num_seqs))


def backward_kernel_launches(B, T, H, HV, K=128, V=128, num_seqs=0) -> int:
    """Kernel launches one backward makes for these sizes (0 if rejected)."""
    return int(lib().kda_prefill_backward_kernel_launches(B, T, H, HV, K, V, num_seqs))


def forward_save(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *, o=None, final_state=None, saved=None,
                 stream=None):
    """The forward that also keeps what the backward needs; returns (o, final_state, saved).  Pass ``saved`` to
    ``backward(..., saved=saved)`` with the same inputs."""
    import torch
    B, T, H, HV, K, V, N, dev = _need_inputs(q, k, v, g, beta, initial_state, cu_seqlens)
    if o is None:
        o = torch.empty(B, T, HV, V, dtype=torch.bfloat16, device=dev)
    if final_state is None:
        final_state = torch.empty(N, HV, K, V, dtype=torch.float32, device=dev)
    _need("o", o, torch.bfloat16, B * T * HV * V, dev)
    _need("final_state", final_state, torch.float32, N * HV * K * V, dev)
    num_seqs = N if cu_seqlens is not None else 0
    if saved is None:
        saved = torch.empty(max(backward_workspace_size(B, T, H, HV, K, V, num_seqs), 1), dtype=torch.uint8,
                            device=dev)
    _need("saved", saved, torch.uint8, None, dev)
    with _on(dev):
        rc = lib().kda_prefill_forward_save(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state),
                                            _ptr(cu_seqlens), num_seqs, B, T, H, HV, K, V, _ptr(o),
                                            _ptr(final_state), _ptr(saved), saved.numel(), _stream_ptr(stream, dev))
    _check(rc, "kda_prefill_forward_save")
    return o, final_state, saved


def backward(q, k, v, g, beta, dout, initial_state=None, dht=None, cu_seqlens=None, *, want_dh0=None,
             workspace=None, saved=None, stream=None):
    """Gradients of sum(o * dout) + sum(final_state * dht) for the forward on the same inputs (CUDA).

    Returns (dq, dk [B,T,H,K] bf16, dv [B,T,HV,V] bf16, dg [B,T,HV,K] fp32, dbeta [B,T,HV] fp32,
    dh0 [N,HV,K,V] fp32, or None when there is no initial state and want_dh0 is not set).  With ``saved`` (from
    ``forward_save`` on the same inputs) the forward is not recomputed.
    """
    import torch
    B, T, H, HV, K, V, N, dev = _need_inputs(
        q, k, v, g, beta, initial_state, cu_seqlens,
        more=lambda B, T, H, HV, K, V, N: [("dout", dout, torch.bfloat16, B * T * HV * V, True),
                                           ("dht", dht, torch.float32, N * HV * K * V, True)])
    dq = torch.empty(B, T, H, K, dtype=torch.bfloat16, device=dev)
    dk = torch.empty(B, T, H, K, dtype=torch.bfloat16, device=dev)
    dv = torch.empty(B, T, HV, V, dtype=torch.bfloat16, device=dev)
    dg = torch.empty(B, T, HV, K, dtype=torch.float32, device=dev)
    dbeta = torch.empty(B, T, HV, dtype=torch.float32, device=dev)
    if want_dh0 is None:
        want_dh0 = initial_state is not None
    dh0 = torch.empty(N, HV, K, V, dtype=torch.float32, device=dev) if want_dh0 else None
    num_seqs = N if cu_seqlens is not None else 0
    fn, name = lib().kda_prefill_backward, "kda_prefill_backward"
    if saved is not None:
        workspace, fn, name = saved, lib().kda_prefill_backward_saved, "kda_prefill_backward_saved"
    elif workspace is None:
        ws_bytes = backward_workspace_size(B, T, H, HV, K, V, num_seqs)
        workspace = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=dev)
    _need("saved" if saved is not None else "workspace", workspace, torch.uint8, None, dev)
    with _on(dev):
        rc = fn(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state), _ptr(cu_seqlens), num_seqs,
                B, T, H, HV, K, V, _ptr(dout), _ptr(dht), _ptr(dq), _ptr(dk), _ptr(dv), _ptr(dg), _ptr(dbeta),
                _ptr(dh0), _ptr(workspace), workspace.numel(), _stream_ptr(stream, dev))
    _check(rc, name)
    return dq, dk, dv, dg, dbeta, dh0


def host_staging_size(B, T, H, HV, K=128, V=128, num_seqs=0, has_initial_state=False, has_cu_seqlens=False) -> int:
    return int(lib().kda_prefill_host_staging_size(B, T, H, HV, K, V, num_seqs, int(has_initial_state),
                                                    int(has_cu_seqlens)))


def forward_host(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *, o, final_state, staging, stream=None):
    """Forward on HOST (ideally pinned) tensors through a device staging buffer.

    Enqueues the host->device copies, the forward and the device->host copies
    of o and final_state on ``stream``; the caller synchronises.
    """
    import torch
    B, T, H, HV, K, V, N, _ = _need_inputs(
        q, k, v, g, beta, initial_state, cu_seqlens, host=True,
        more=lambda B, T, H, HV, K, V, N: [("o", o, torch.bfloat16, B * T * HV * V, True),
                                           ("final_state", final_state, torch.float32, N * HV * K * V, True)])
    _need("staging", staging, torch.uint8, None)
    dev = staging.device
    num_seqs = N if cu_seqlens is not None else 0
    with _on(dev):
        rc = lib().kda_prefill_forward_host(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state),
                                            _ptr(cu_seqlens), num_seqs, B, T, H, HV, K, V, _ptr(o),
                                            _ptr(final_state), _ptr(staging), staging.numel(),
                                            _stream_ptr(stream, dev))
    _check(rc, "kda_prefill_forward_host")
    return o, final_state


def device_error(clear: bool = True) -> int:
    """Bits set by kernel waits that gave up on the current device (0 when none); synchronises."""
    w = ctypes.c_uint(0)
    _check(lib().kda_prefill_device_error(ctypes.byref(w), int(clear)), "kda_prefill_device_error")
    return int(w.value)


def decode_step(q, k, v, g, beta, state, state_indices, *, o=None, stream=None):
    """One recurrent decode step on a bf16 state pool (CUDA); returns o [B, HV, V].

    q, k: bf16 [B, H, K] and v: bf16 [B, HV, V], each row compact but rows may be strided (e.g. views of a
    packed [B, (2H + HV) * 128] QKV tensor); g: fp32 [B, HV, K]; beta: fp32 [B, HV]; state: bf16 pool
    [num_slots, HV, K, V] (compact inside a slot), updated in place; state_indices: int32 [B], -1 = padding row.
    """
    import torch
    if q.dim() != 3 or k.shape != q.shape or v.dim() != 3 or v.shape[0] != q.shape[0]:
        raise ValueError("q and k must be [B,H,K] and v [B,HV,V]")
    if state.dim() != 4 or state.shape[1] != v.shape[1]:
        raise ValueError("state must be a pool [num_slots, HV, K, V]")
    B, H, K = q.shape
    HV, V = v.shape[1], v.shape[2]
    dev = q.device
    _need_all([("q", q, torch.bfloat16, None, False), ("k", k, torch.bfloat16, None, False),
               ("v", v, torch.bfloat16, None, False), ("g", g, torch.float32, B * HV * K, True),
               ("beta", beta, torch.float32, B * HV, True), ("state", state, torch.bfloat16, None, False),
               ("state_indices", state_indices, torch.int32, B, True)], dev)
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.stride(2) != 1 or t.stride(1) != t.shape[2]:
            raise ValueError(f"{name} must have compact rows")
    if tuple(state.shape[1:]) != (HV, K, V) or state[0].stride() != (K * V, V, 1):
        raise ValueError("state must be a pool [num_slots, HV, K, V] compact inside each slot")
    if o is None:
        o = torch.empty(B, HV, V, dtype=torch.bfloat16, device=dev)
    _need("o", o, torch.bfloat16, B * HV * V, dev)
    with _on(dev):
        rc = lib().kda_decode_step(_ptr(q), q.stride(0), _ptr(k), k.stride(0), _ptr(v), v.stride(0), _ptr(g),
                                   _ptr(beta), _ptr(state), state.stride(0), state.shape[0], _ptr(state_indices),
                                   B, H, HV, K, V, _ptr(o), _stream_ptr(stream, dev))
    _check(rc, "kda_decode_step")
    return o


def l2norm_bf16(x, out=None, stream=None):
    """Exact-rounding L2 normalisation of rows of 128 bf16 values (CUDA)."""
    import torch
    _need("x", x, torch.bfloat16, None, x.device)
    if out is None:
        out = torch.empty_like(x)
    _need("out", out, torch.bfloat16, x.numel(), x.device)
    rows = x.numel() // x.shape[-1]
    with _on(x.device):
        rc = lib().kda_l2norm_bf16(_ptr(x), rows, x.shape[-1], _ptr(out), _stream_ptr(stream, x.device))
    _check(rc, "kda_l2norm_bf16")
    return out


def forward_noalloc(q, k, v, g, beta, initial_state=None, cu_seqlens=None, *, o=None, final_state=None,
                    stream=None):
    """The forward through kda_prefill_forward_noalloc: no workspace argument.

    For callers that may not allocate device memory during the call; the
    library's fixed 64 MiB scratch array limits the problem size (larger
    inputs raise KdaError with KDA_ERR_WORKSPACE).  Calls must not overlap.
    """
    import torch
    L = lib()
    f = L.kda_prefill_forward_noalloc
    P, I = ctypes.c_void_p, ctypes.c_int
    f.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, I, P, P, P]
    f.restype = I
    B, T, H, HV, K, V, N, dev = _need_inputs(q, k, v, g, beta, initial_state, cu_seqlens)
    if o is None:
        o = torch.empty(B, T, HV, V, dtype=torch.bfloat16, device=dev)
    if final_state is None:
        final_state = torch.empty(N, HV, K, V, dtype=torch.float32, device=dev)
    _need("o", o, torch.bfloat16, B * T * HV * V, dev)
    _need("final_state", final_state, torch.float32, N * HV * K * V, dev)
    num_seqs = N if cu_seqlens is not None else 0
    with _on(dev):
        rc = f(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), _ptr(initial_state), _ptr(cu_seqlens), num_seqs,
               B, T, H, HV, K, V, _ptr(o), _ptr(final_state), _stream_ptr(stream, dev))
    _check(rc, "kda_prefill_forward_noalloc")
    return o, final_state
