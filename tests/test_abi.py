"""The C-ABI library builds, loads without a GPU, exports every symbol the
header declares, and rejects bad arguments on the host (no compute calls)."""
import ctypes
import os
import re

import pytest

import kda_gated_delta_prefill_b200 as kda
from kda_gated_delta_prefill_b200 import build as kbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    kbuild.build()
    return kda.lib()


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(kda_[a-z0-9_]+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(L):
    names = declared_symbols()
    assert names >= set(kda.EXPORTED) - set(), names
    for n in names:
        assert hasattr(L, n), f"{n} declared but not exported"


def test_status_strings(L):
    for code, name in kda.STATUS.items():
        assert L.kda_status_string(code).decode() == name
    assert L.kda_status_string(99).decode() == "KDA_ERR_UNKNOWN"


def test_workspace_size(L):
    item = 74240
    # plain batch: B * ceil(T/64) chunks x HV heads of item blocks
    assert L.kda_prefill_workspace_size(2, 4096, 96, 96, 128, 128, 0) == 2 * 64 * 96 * item
    assert L.kda_prefill_workspace_size(1, 1000, 4, 4, 128, 128, 0) == 16 * 4 * item
    # packed batch: offsets, order and 4 x (N + 1) chunk-window offsets, then (ceil(T/64) + N) chunks as an
    # upper bound
    n = L.kda_prefill_workspace_size(1, 11210, 8, 32, 128, 128, 7)
    assert n == 256 + 256 + 256 + (176 + 7) * 32 * item
    n = L.kda_prefill_workspace_size(1, 11210, 8, 32, 128, 128, 100)
    assert n == 512 + 512 + 1792 + (176 + 100) * 32 * item
    # rejected sizes
    assert L.kda_prefill_workspace_size(1, 64, 1, 1, 64, 128, 0) == 0
    assert L.kda_prefill_workspace_size(1, 64, 2, 3, 128, 128, 0) == 0


def test_host_staging_size(L):
    B, T, H, HV = 1, 1000, 4, 4
    n = L.kda_prefill_host_staging_size(B, T, H, HV, 128, 128, 0, 1, 0)
    expect = 2 * T * H * 128 * 2 + T * HV * 128 * 2 + T * HV * 128 * 4 + T * HV * 4 + 2 * HV * 128 * 128 * 4 \
        + T * HV * 128 * 2 + L.kda_prefill_workspace_size(B, T, H, HV, 128, 128, 0)
    assert expect <= n <= expect + 16 * 256


FAKE = 1 << 20  # a 16-byte aligned non-null address that is never dereferenced


def call_forward(L, **over):
    a = dict(q=FAKE, k=FAKE * 2, v=FAKE * 3, g=FAKE * 4, beta=FAKE * 5, s0=None, cu=None, num_seqs=0,
             B=1, T=64, H=1, HV=1, K=128, V=128, o=FAKE * 6, sN=FAKE * 7, ws=None, ws_bytes=0)
    a.update(over)
    return L.kda_prefill_forward(a["q"], a["k"], a["v"], a["g"], a["beta"], a["s0"], a["cu"], a["num_seqs"],
                                 a["B"], a["T"], a["H"], a["HV"], a["K"], a["V"], a["o"], a["sN"], a["ws"],
                                 a["ws_bytes"], None)


@pytest.mark.parametrize("over,code", [
    (dict(B=0), 1), (dict(T=0), 1), (dict(H=0), 1), (dict(HV=3, H=2), 1), (dict(K=64), 2), (dict(V=256), 2),
    (dict(q=None), 1), (dict(sN=None), 1), (dict(o=None), 1),
    (dict(q=FAKE + 2), 3), (dict(g=FAKE * 4 + 8), 3), (dict(beta=FAKE * 5 + 2), 3),
    (dict(cu=FAKE * 8, num_seqs=0), 1), (dict(cu=FAKE * 8, num_seqs=2, B=2), 1),
    (dict(cu=FAKE * 8, num_seqs=2), 4),                      # varlen needs a workspace
    (dict(cu=FAKE * 8, num_seqs=2, ws=FAKE * 9, ws_bytes=16), 4),
    (dict(cu=FAKE * 8, num_seqs=2, ws=FAKE * 64 + 16, ws_bytes=1 << 30), 3),
    (dict(ws=None), 4), (dict(ws=FAKE * 64, ws_bytes=1000), 4),
    (dict(ws=FAKE * 2, ws_bytes=1 << 30), 1),                # workspace overlaps k
    (dict(o=FAKE), 1),                                       # o overlaps q
    (dict(sN=FAKE * 4), 1),                                  # final_state overlaps g
])
def test_forward_rejects_bad_arguments(L, over, code):
    assert call_forward(L, **over) == code


@pytest.mark.parametrize("cu_host,num_seqs,code", [
    (None, 2, 1),              # no host copy
    ([1, 30, 64], 2, 1),       # does not start at 0
    ([0, 30, 63], 2, 1),       # does not end at T
    ([0, 40, 30, 64], 3, 1),   # decreasing
    ([0, 64], 0, 1),           # no sequences
])
def test_varlen_forward_checks_the_host_boundaries(L, cu_host, num_seqs, code):
    arr = None if cu_host is None else (ctypes.c_int32 * len(cu_host))(*cu_host)
    rc = L.kda_prefill_forward_varlen(FAKE, FAKE * 2, FAKE * 3, FAKE * 4, FAKE * 5, None, FAKE * 8, arr, num_seqs,
                                      64, 1, 1, 128, 128, FAKE * 6, FAKE * 7, FAKE * 64, 1 << 30, None)
    assert rc == code
    # the same boundaries size the launch plan; malformed ones give 0
    assert L.kda_prefill_varlen_kernel_launches(64, 1, 1, 128, 128, num_seqs, arr) == 0


def test_partial_state_overlap_rejected(L):
    s0 = FAKE * 16
    assert call_forward(L, s0=s0, sN=s0 + 4096, ws=FAKE * 64, ws_bytes=1 << 26) == 1


def test_l2norm_rejects_bad_arguments(L):
    assert L.kda_l2norm_bf16(FAKE, 4, 64, FAKE * 2, None) == 2
    assert L.kda_l2norm_bf16(FAKE, -1, 128, FAKE * 2, None) == 1
    assert L.kda_l2norm_bf16(None, 4, 128, FAKE * 2, None) == 1
    assert L.kda_l2norm_bf16(FAKE + 2, 4, 128, FAKE * 2, None) == 3
    assert L.kda_l2norm_bf16(FAKE, 4, 128, FAKE + 256, None) == 1
    assert L.kda_l2norm_bf16(FAKE, 0, 128, FAKE * 2, None) == 0


def test_host_forward_rejects_small_staging(L):
    P = ctypes.c_void_p
    rc = L.kda_prefill_forward_host(P(FAKE), P(FAKE), P(FAKE), P(FAKE), P(FAKE), None, None, 0, 1, 64, 1, 1, 128,
                                    128, P(FAKE), P(FAKE), P(FAKE * 4), 16, None)
    assert rc == 4


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(kda, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(kda, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        kda.lib()


def call_decode(L, B=4, H=2, HV=4, K=128, V=128, q=1, k=2, v=3, g=4, beta=5, state=6, idx=7, o=8,
                qs=None, ks=None, vs=None, slot_stride=None, slots=8):
    P = ctypes.c_void_p
    step = 1 << 32  # arguments live far apart unless a case moves one
    ptr = lambda i: None if i is None else P(FAKE + int(i * step))
    qs = H * K if qs is None else qs
    ks = H * K if ks is None else ks
    vs = HV * V if vs is None else vs
    slot_stride = HV * K * V if slot_stride is None else slot_stride
    return L.kda_decode_step(ptr(q), qs, ptr(k), ks, ptr(v), vs, ptr(g), ptr(beta), ptr(state), slot_stride, slots,
                             ptr(idx), B, H, HV, K, V, ptr(o), None)


@pytest.mark.parametrize("over,code", [
    (dict(K=64), 2), (dict(V=64), 2), (dict(HV=3), 1), (dict(H=0), 1), (dict(B=-1), 1), (dict(slots=0), 1),
    (dict(q=None), 1), (dict(idx=None), 1), (dict(o=None), 1), (dict(qs=128), 1), (dict(vs=100), 1),
    (dict(slot_stride=1000), 1), (dict(state=6 + 2 ** -32 * 8), 3), (dict(qs=258), 3), (dict(q=1 + 2 ** -32 * 2), 3),
    (dict(o=6), 1), (dict(o=1), 1), (dict(state=3), 1),
])
def test_decode_rejects_bad_arguments(L, over, code):
    assert call_decode(L, **over) == code


def test_decode_empty_batch_is_a_no_op(L):
    assert call_decode(L, B=0) == 0


def call_backward(L, B=1, T=64, H=1, HV=1, K=128, V=128, q=1, k=2, v=3, g=4, beta=5, s0=None, do=6, dht=None,
                  dq=7, dk=8, dv=9, dg=10, db=11, dh0=None, ws=12, ws_bytes=None, cu=None, num_seqs=0):
    P = ctypes.c_void_p
    step = 1 << 32  # arguments live far apart unless a case moves one
    ptr = lambda i: None if i is None else P(FAKE + int(i * step))
    if ws_bytes is None:
        ws_bytes = L.kda_prefill_backward_workspace_size(B, T, H, HV, K, V, num_seqs)
    return L.kda_prefill_backward(ptr(q), ptr(k), ptr(v), ptr(g), ptr(beta), ptr(s0), ptr(cu), num_seqs, B, T, H, HV,
                                  K, V, ptr(do), ptr(dht), ptr(dq), ptr(dk), ptr(dv), ptr(dg), ptr(db), ptr(dh0),
                                  ptr(ws), ws_bytes, None)


@pytest.mark.parametrize("over,code", [
    (dict(K=64), 2), (dict(V=256), 2), (dict(HV=3, H=2), 1), (dict(B=0), 1), (dict(T=-1), 1),
    (dict(q=None), 1), (dict(do=None), 1), (dict(dg=None), 1), (dict(db=None), 1),
    (dict(q=1 + 2 ** -32 * 8), 3), (dict(dv=9 + 2 ** -32 * 4), 3), (dict(ws=12 + 2 ** -32 * 16), 3),
    (dict(dq=1), 1), (dict(dg=4), 1), (dict(dk=7), 1), (dict(dh0=13, s0=13), 1), (dict(ws=6), 1), (dict(ws=7), 1),
    (dict(ws_bytes=16), 4), (dict(ws=None), 4), (dict(cu=14, B=2, num_seqs=2), 1),
])
def test_backward_rejects_bad_arguments(L, over, code):
    assert call_backward(L, **over) == code


def test_backward_workspace_and_launch_counts(L):
    # per chunk and value head: the forward's block, a start state and an end-state gradient (fp32 K x V each)
    one = L.kda_prefill_backward_workspace_size(1, 64, 1, 1, 128, 128, 0)
    two = L.kda_prefill_backward_workspace_size(1, 128, 1, 1, 128, 128, 0)
    assert two - one >= 74240 + 2 * 65536
    assert L.kda_prefill_backward_workspace_size(1, 64, 1, 1, 64, 128, 0) == 0
    # forward intra-chunk and carry, reverse carry, chunk gradients (+ chunk offsets when packed); with GQA
    # (H < HV) also the kernel that sums each Q/K head's group through the normalisation's Jacobian
    assert L.kda_prefill_backward_kernel_launches(1, 64, 1, 1, 128, 128, 0) == 4
    assert L.kda_prefill_backward_kernel_launches(1, 64, 1, 1, 128, 128, 3) == 5
    assert L.kda_prefill_backward_kernel_launches(1, 64, 1, 2, 128, 128, 0) == 5


def test_saved_forward_and_backward_reject_small_or_overlapping_buffers(L):
    P = ctypes.c_void_p
    step = 1 << 32
    ptr = lambda i: P(FAKE + int(i * step))
    need = L.kda_prefill_backward_workspace_size(1, 64, 1, 1, 128, 128, 0)
    assert need > L.kda_prefill_workspace_size(1, 64, 1, 1, 128, 128, 0)  # the forward's workspace, then more
    fwd = lambda saved, nbytes, o=8: L.kda_prefill_forward_save(ptr(1), ptr(2), ptr(3), ptr(4), ptr(5), None, None, 0,
                                                                1, 64, 1, 1, 128, 128, ptr(o), ptr(9), saved, nbytes,
                                                                None)
    assert fwd(ptr(12), need - 256) == 4           # too small
    assert fwd(None, need) == 4                    # missing
    assert fwd(P(FAKE + 12 * step + 8), need) == 3  # misaligned
    assert fwd(ptr(8), need) == 1                  # overlaps o
    assert L.kda_prefill_forward_save(ptr(1), ptr(2), ptr(3), ptr(4), ptr(5), None, None, 0, 1, 64, 1, 1, 64, 128,
                                      ptr(8), ptr(9), ptr(12), need, None) == 2
    bwd = lambda saved, nbytes: L.kda_prefill_backward_saved(ptr(1), ptr(2), ptr(3), ptr(4), ptr(5), None, None, 0, 1,
                                                             64, 1, 1, 128, 128, ptr(6), None, ptr(7), ptr(8), ptr(9),
                                                             ptr(10), ptr(11), None, saved, nbytes, None)
    assert bwd(ptr(12), need - 256) == 4
    assert bwd(ptr(6), need) == 1  # overlaps dout


def test_bf16_state_forward_rejects_bad_arguments(L):
    P = ctypes.c_void_p
    step = 1 << 32
    ptr = lambda i: P(FAKE + int(i * step))
    need = L.kda_prefill_state_bf16_workspace_size(1, 64, 1, 1, 128, 128, 0)
    # two fp32 states more than the forward's workspace
    assert need >= L.kda_prefill_workspace_size(1, 64, 1, 1, 128, 128, 0) + 2 * 128 * 128 * 4
    f = lambda s0, sN, ws, nbytes, K=128: L.kda_prefill_forward_state_bf16(
        ptr(1), ptr(2), ptr(3), ptr(4), ptr(5), s0, None, 0, 1, 64, 1, 1, K, 128, ptr(8), sN, ws, nbytes, None)
    assert f(ptr(6), ptr(9), ptr(12), need, K=64) == 2
    assert f(ptr(6), None, ptr(12), need) == 1                      # final_state required
    assert f(ptr(6), P(FAKE + 9 * step + 8), ptr(12), need) == 3    # final_state misaligned
    assert f(ptr(6), ptr(9), ptr(12), need - 256) == 4
    assert f(ptr(6), ptr(9), ptr(9), need) == 1                     # workspace overlaps final_state
    assert f(ptr(6), P(FAKE + 6 * step + 16384), ptr(12), need) == 1  # states partly overlap


def _small_inputs(dtype_overrides=None):
    import torch
    x = {"q": torch.zeros(1, 64, 2, 128, dtype=torch.bfloat16), "k": torch.zeros(1, 64, 2, 128, dtype=torch.bfloat16),
         "v": torch.zeros(1, 64, 4, 128, dtype=torch.bfloat16), "g": torch.zeros(1, 64, 4, 128),
         "beta": torch.zeros(1, 64, 4)}
    for name, t in (dtype_overrides or {}).items():
        x[name] = t
    return x


@pytest.mark.parametrize("name,bad,msg", [
    ("g", lambda t: t.g.bfloat16(), "g must be torch.float32"),
    ("beta", lambda t: t.beta.double(), "beta must be torch.float32"),
    ("q", lambda t: t.q.float(), "q must be torch.bfloat16"),
    ("k", lambda t: t.k[:, :32], "k must hold"),
    ("v", lambda t: t.v[:, :32], "v must hold"),
])
def test_binding_rejects_wrong_dtype_or_size_before_any_launch(name, bad, msg):
    """The binding checks dtypes and element counts: the library only sees raw pointers, and a wrong-size
    buffer would let the kernels read or write past it."""
    import types
    import kda_gated_delta_prefill_b200 as kda
    x = _small_inputs()
    x[name] = bad(types.SimpleNamespace(**x))
    with pytest.raises(ValueError, match=msg):
        kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"])
    with pytest.raises(ValueError, match=msg):
        kda.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], torch_zeros_dout())


def torch_zeros_dout():
    import torch
    return torch.zeros(1, 64, 4, 128, dtype=torch.bfloat16)


def test_binding_rejects_host_tensors_and_wrong_optional_buffers():
    import torch
    import kda_gated_delta_prefill_b200 as kda
    x = _small_inputs()
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"])
    with pytest.raises(ValueError, match="initial_state must hold"):
        kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], torch.zeros(1, 4, 128, 64))
    with pytest.raises(ValueError, match="initial_state must be torch.bfloat16"):
        kda.forward_state_bf16(x["q"], x["k"], x["v"], x["g"], x["beta"], torch.zeros(1, 4, 128, 128))
    with pytest.raises(ValueError, match="cu_seqlens must be torch.int32"):
        kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], None, torch.tensor([0, 64]))
    with pytest.raises(ValueError, match="dout must be torch.bfloat16"):
        kda.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], torch.zeros(1, 64, 4, 128))
    with pytest.raises(ValueError, match="dht must hold"):
        kda.backward(x["q"], x["k"], x["v"], x["g"], x["beta"], torch_zeros_dout(), None, torch.zeros(1, 4, 128))
    # the host-buffer entry point wants host inputs and outputs of the right types, and a device staging buffer
    o_h = torch.empty(1, 64, 4, 128, dtype=torch.bfloat16)
    s_h = torch.empty(1, 4, 128, 128)
    with pytest.raises(ValueError, match="final_state must be torch.float32"):
        kda.forward_host(x["q"], x["k"], x["v"], x["g"], x["beta"], o=o_h, final_state=s_h.bfloat16(),
                         staging=torch.empty(16, dtype=torch.uint8))
    with pytest.raises(ValueError, match="staging must be a CUDA tensor"):
        kda.forward_host(x["q"], x["k"], x["v"], x["g"], x["beta"], o=o_h, final_state=s_h,
                         staging=torch.empty(16, dtype=torch.uint8))
    # the decode step: a bf16 pool, int32 slot indices
    q1 = torch.zeros(3, 2, 128, dtype=torch.bfloat16)
    v1 = torch.zeros(3, 4, 128, dtype=torch.bfloat16)
    g1, b1 = torch.zeros(3, 4, 128), torch.zeros(3, 4)
    with pytest.raises(ValueError, match="state must be torch.bfloat16"):
        kda.decode_step(q1, q1, v1, g1, b1, torch.zeros(5, 4, 128, 128), torch.zeros(3, dtype=torch.int32))
    with pytest.raises(ValueError, match="state_indices must be torch.int32"):
        kda.decode_step(q1, q1, v1, g1, b1, torch.zeros(5, 4, 128, 128, dtype=torch.bfloat16),
                        torch.zeros(3, dtype=torch.int64))
    with pytest.raises(ValueError, match="x must be torch.bfloat16"):
        kda.l2norm_bf16(torch.zeros(4, 128))
