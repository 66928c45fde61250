"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle on the
same seeded inputs.  Tolerances live in parity_util."""
import numpy as np
import pytest
import torch

from kda_gated_delta_prefill_b200 import inputs as gen
from tests.parity_util import O_TOL, STATE_REL_FRO, compare, gpu_forward, oracle_forward, select_heads, to_cuda

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kda_gated_delta_prefill_b200 as kda
    kda.lib()  # fail loudly if the library is missing


# ------------------------------------------------------------------ normalisation
# kda_l2norm_bf16 runs l2norm_half_row, the routine the forward's intra-chunk prologue runs on every q and k
# row (same thread mapping: two lanes per row, 64 elements each), so these checks cover the forward's
# normalisation arithmetic.

def _ordered(b):  # bf16 bits -> integers ordered like the values (+0 and -0 both 0)
    return np.where(b & 0x8000, -(b & 0x7FFF), b & 0x7FFF)


def _norm_bits(x):
    import kda_gated_delta_prefill_b200 as kda
    return kda.l2norm_bf16(x.cuda()).cpu().view(torch.int16).numpy().astype(np.int32) & 0xFFFF


@pytest.mark.parametrize("mode", ["normal", "gain", "tiny", "zero_rows"])
@pytest.mark.parametrize("which", ["q", "k"])
def test_l2norm_within_one_ulp(mode, which):
    import oracle
    case = gen.Case("norm", B=1, T=4096 + 5, H=4, HV=4, qk_mode=mode, seed=21)  # a ragged last group of rows
    x = gen.make_inputs(case)[which]
    ref = oracle.l2norm_bf16(x).astype(np.int32)
    diff = np.abs(_ordered(_norm_bits(x)) - _ordered(ref))
    assert diff.max() <= 1
    assert (diff == 0).mean() > 0.99


def test_l2norm_worked_example_rows():
    # the page's example: q = k = e0 rows stay e0 exactly; an all-ones row gives bf16 0x3DB5 in every element
    x = gen.worked_example()
    for name in ("q", "k"):
        bits = _norm_bits(x[name])
        e0 = np.zeros_like(bits)
        e0[..., 0] = 0x3F80
        assert np.array_equal(bits, e0)
    ones = torch.ones(37, 128, dtype=torch.bfloat16)
    assert np.all(_norm_bits(ones) == 0x3DB5)


# ------------------------------------------------------------------ worked example

def test_worked_example_exact():
    x = gen.worked_example()
    o, s = gpu_forward(x)
    bits = o.cpu().view(torch.int16).numpy().astype(np.int32) & 0xFFFF
    assert np.all(bits == 0x3DB5)
    S = s.cpu().numpy()[0, 0]
    assert np.all(S[0] == 1.0) and np.all(S[1:] == 0.0)


def test_beta_zero_gives_zeros():
    x = gen.make_inputs(gen.SMALLEST)
    x["beta"] = torch.zeros_like(x["beta"])
    o, s = gpu_forward(x)
    assert torch.all(o == 0) and torch.all(s == 0)


# ------------------------------------------------------------------ the workloads

@pytest.mark.parametrize("case", [gen.SMALLEST, gen.TAIL_STATE, gen.VARLEN_GQA], ids=lambda c: c.name)
def test_workload_full_parity(case):
    x = gen.make_inputs(case)
    o, s = gpu_forward(x)
    ref = oracle_forward(x)
    compare(o, s, ref)


def test_wide_heads_sampled():
    # B=2, H=HV=96, T=4096: all heads on the GPU, oracle on a sample of heads.
    x = gen.make_inputs(gen.WIDE_HEADS)
    o, s = gpu_forward(x)
    heads = [0, 37, 95]
    sub = select_heads(x, heads)
    ref = oracle_forward(sub)
    compare(o[:, :, heads].contiguous(), s[:, heads].contiguous(), ref)


def test_head_groups_match_per_head_calls_bit_for_bit():
    # 2 x 96 units: between one and two waves of carry CTAs, so the forward splits the value heads into two
    # groups (the first group's carry beside the second group's intra-chunk work).  Heads are independent, so
    # the same batch run as two calls of 48 heads each (fewer units than SMs: another launch plan) must give
    # the same bits.
    import kda_gated_delta_prefill_b200 as kda
    B, T, H = 2, 1024, 96
    case = gen.Case("head_groups", B=B, T=T, H=H, HV=H, state="n01", seed=701)
    assert kda.kernel_launches(B, T, H, H) == 4  # intra and carry of each group
    x = to_cuda(gen.make_inputs(case))
    o, s = kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"])
    for h0 in (0, 48):
        hs = slice(h0, h0 + 48)
        oh, sh = kda.forward(x["q"][:, :, hs].contiguous(), x["k"][:, :, hs].contiguous(),
                             x["v"][:, :, hs].contiguous(), x["g"][:, :, hs].contiguous(),
                             x["beta"][:, :, hs].contiguous(), x["initial_state"][:, hs].contiguous())
        torch.cuda.synchronize()
        assert torch.equal(o[:, :, hs], oh)
        assert torch.equal(s[:, hs], sh)
    assert kda.device_error(clear=True) == 0


def test_long_prefill_sampled():
    # B=1, H=HV=64, T=65536 with state, generated on the device as the benchmark does.
    x = gen.make_inputs(gen.LONG_PREFILL, device="cuda")
    import kda_gated_delta_prefill_b200 as kda
    o, s = kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"])
    torch.cuda.synchronize()
    heads = [5, 63]
    xc = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    sub = select_heads(xc, heads)
    ref = oracle_forward(sub)
    compare(o[:, :, heads].contiguous(), s[:, heads].contiguous(), ref)


# ------------------------------------------------------------------ edges and modes

@pytest.mark.parametrize("T", [1, 2, 15, 16, 17, 63, 64, 65, 127, 129, 200])
def test_lengths(T):
    case = gen.Case(f"len{T}", B=2, T=T, H=2, HV=2, state="n01", seed=100 + T)
    x = gen.make_inputs(case)
    o, s = gpu_forward(x)
    compare(o, s, oracle_forward(x))


@pytest.mark.parametrize("mode", [dict(qk_mode="gain"), dict(qk_mode="tiny"), dict(qk_mode="zero_rows"),
                                  dict(gate="logsig128"), dict(gate="logsig8"), dict(gate="logsig1"),
                                  dict(gate="zero"), dict(gate="uniform5"), dict(beta="one"), dict(beta="edge"),
                                  dict(beta="zero", state="quarter"), dict(state="quarter"), dict(state="zeros")],
                         ids=lambda m: "-".join(f"{k}={v}" for k, v in m.items()))
def test_generator_modes(mode):
    case = gen.Case("mode", B=1, T=300, H=2, HV=2, seed=7, **mode)
    x = gen.make_inputs(case)
    o, s = gpu_forward(x)
    compare(o, s, oracle_forward(x))


def test_gqa_group_8():
    case = gen.Case("gqa8", B=1, T=257, H=2, HV=16, state="n01", seed=31)
    x = gen.make_inputs(case)
    o, s = gpu_forward(x)
    compare(o, s, oracle_forward(x))


def test_varlen_with_empty_sequences():
    lengths = [0, 5, 0, 64, 1, 130, 0]
    case = gen.Case("varlen0", B=1, T=sum(lengths), H=2, HV=4, lengths=lengths, state="n01", seed=41)
    x = gen.make_inputs(case)
    o, s = gpu_forward(x)
    ref = oracle_forward(x)
    compare(o, s, ref)
    # empty sequences pass their state through unchanged
    for n, L in enumerate(lengths):
        if L == 0:
            assert torch.equal(s[n].cpu(), x["initial_state"][n])


def test_in_place_state_update():
    case = gen.Case("inplace", B=1, T=150, H=2, HV=2, state="n01", seed=51)
    x = gen.make_inputs(case)
    ref = oracle_forward(x)
    xc = to_cuda(x)
    import kda_gated_delta_prefill_b200 as kda
    st = xc["initial_state"].clone()
    o, s = kda.forward(xc["q"], xc["k"], xc["v"], xc["g"], xc["beta"], st, final_state=st)
    torch.cuda.synchronize()
    assert s.data_ptr() == st.data_ptr()
    compare(o, s, ref)


def test_split_resume_matches_full():
    case = gen.Case("split", B=1, T=333, H=2, HV=2, state="n01", seed=61)
    x = gen.make_inputs(case)
    full_o, full_s = gpu_forward(x)
    t1 = 128 + 37
    a = {k: (v[:, :t1].contiguous() if k in ("q", "k", "v", "g", "beta") else v) for k, v in x.items()}
    oa, sa = gpu_forward(a)
    b = {k: (v[:, t1:].contiguous() if k in ("q", "k", "v", "g", "beta") else v) for k, v in x.items()}
    b["initial_state"] = sa.cpu()
    ob, sb = gpu_forward(b)
    ref = oracle_forward(x)
    compare(torch.cat([oa, ob], dim=1), sb, ref)
    # The first part's rows come from a shorter last chunk, whose block-local gate products round
    # differently, so the split and the full run agree to rounding, not bit for bit.
    assert (oa.float() - full_o[:, :t1].float()).abs().max() < 1e-2


def test_outputs_fully_written():
    # NaN canaries in o and final_state must all be overwritten.
    case = gen.Case("canary", B=2, T=100, H=2, HV=4, seed=71)
    x = to_cuda(gen.make_inputs(case))
    import kda_gated_delta_prefill_b200 as kda
    o = torch.full((2, 100, 4, 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    s = torch.full((2, 4, 128, 128), float("nan"), device="cuda")
    kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], None, o=o, final_state=s)
    torch.cuda.synchronize()
    assert torch.isfinite(o.float()).all() and torch.isfinite(s).all()


def test_stale_workspace_contents_are_ignored():
    # The workspace needs no initialisation: NaN bytes left in it must not reach the outputs.
    import kda_gated_delta_prefill_b200 as kda
    case = gen.Case("stale", B=1, T=200, H=2, HV=4, state="n01", seed=87)
    x = gen.make_inputs(case)
    xc = to_cuda(x)
    n = kda.workspace_size(1, 200, 2, 4)
    ws = torch.full((n,), 0xFF, dtype=torch.uint8, device="cuda")
    o, s = kda.forward(xc["q"], xc["k"], xc["v"], xc["g"], xc["beta"], xc["initial_state"], workspace=ws)
    torch.cuda.synchronize()
    compare(o, s, oracle_forward(x))


def test_inputs_not_mutated():
    case = gen.Case("mut", B=1, T=130, H=2, HV=2, state="n01", seed=81)
    x = to_cuda(gen.make_inputs(case))
    before = {k: v.clone() for k, v in x.items() if isinstance(v, torch.Tensor)}
    import kda_gated_delta_prefill_b200 as kda
    kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"])
    torch.cuda.synchronize()
    for k, v in before.items():
        assert torch.equal(v, x[k]), k


def test_host_entry_point_matches_device_entry_point():
    import kda_gated_delta_prefill_b200 as kda
    x = gen.make_inputs(gen.TAIL_STATE)
    o_dev, s_dev = gpu_forward(x)
    B, T, H, HV = 1, 1000, 4, 4
    staging = torch.empty(kda.host_staging_size(B, T, H, HV, has_initial_state=True), dtype=torch.uint8,
                          device="cuda")
    pin = {k: v.pin_memory() for k, v in x.items() if isinstance(v, torch.Tensor)}
    o_h = torch.empty(B, T, HV, 128, dtype=torch.bfloat16).pin_memory()
    s_h = torch.empty(B, HV, 128, 128).pin_memory()
    kda.forward_host(pin["q"], pin["k"], pin["v"], pin["g"], pin["beta"], pin["initial_state"], None,
                     o=o_h, final_state=s_h, staging=staging)
    torch.cuda.synchronize()
    assert torch.equal(o_h, o_dev.cpu()) and torch.equal(s_h, s_dev.cpu())


@pytest.mark.parametrize("B,T,H,HV,state", [(1, 2088, 8, 24, "n01"), (2, 2600, 2, 4, "n01"), (2, 2600, 2, 4, "none")])
def test_host_entry_point_part_by_part(B, T, H, HV, state):
    # Plain batches that the forward cuts into parts: the host-buffer entry point uploads and downloads each
    # part's rows beside the kernels (strided copies when B > 1); the results equal the device entry point's.
    import kda_gated_delta_prefill_b200 as kda
    case = gen.Case(f"host_parts{B}_{T}", B=B, T=T, H=H, HV=HV, state=state, seed=350 + B + T)
    assert kda.kernel_launches(B, T, H, HV) > 2  # cut into parts
    x = gen.make_inputs(case)
    o_dev, s_dev = gpu_forward(x)
    staging = torch.empty(kda.host_staging_size(B, T, H, HV, has_initial_state=x["initial_state"] is not None),
                          dtype=torch.uint8, device="cuda")
    pin = {k: (v.pin_memory() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    o_h = torch.full((B, T, HV, 128), float("nan"), dtype=torch.bfloat16).pin_memory()
    s_h = torch.full((case.N, HV, 128, 128), float("nan")).pin_memory()
    for _ in range(2):  # twice: the second call reuses the copy streams and the staging buffer
        kda.forward_host(pin["q"], pin["k"], pin["v"], pin["g"], pin["beta"], pin["initial_state"], None,
                         o=o_h, final_state=s_h, staging=staging)
        torch.cuda.synchronize()
        assert torch.equal(o_h, o_dev.cpu()) and torch.equal(s_h, s_dev.cpu())


def test_repeat_calls_are_deterministic():
    x = gen.make_inputs(gen.TAIL_STATE)
    o1, s1 = gpu_forward(x)
    o2, s2 = gpu_forward(x)
    assert torch.equal(o1, o2) and torch.equal(s1, s2)


# ------------------------------------------------------------------ sequence cut into parts
# A fixed-length batch with fewer (sequence, value head) units than SMs and at least 32 chunks per sequence is
# run as consecutive parts of the sequence, the state carry of one part overlapping the intra-chunk work of the
# next.  The cut points are whole chunks, so the arithmetic per chunk is that of the uncut run.

@pytest.mark.parametrize("T,state", [(2088, "n01"), (5120, "none"), (8209, "n01")])
def test_parts_full_parity(T, state):
    # 24 value heads (GQA groups of 3): enough units that the carry is overlapped rather than segmented
    case = gen.Case(f"parts{T}", B=1, T=T, H=8, HV=24, state=state, seed=300 + T)
    x = gen.make_inputs(case)
    o, s = gpu_forward(x)
    compare(o, s, oracle_forward(x))


def test_parts_match_the_uncut_run_bit_for_bit():
    # The same sequence passed as a packed batch of one sequence takes the uncut path.
    case = gen.Case("parts_vs_uncut", B=1, T=4160, H=8, HV=32, state="n01", seed=311)
    x = gen.make_inputs(case)
    o_cut, s_cut = gpu_forward(x)
    xv = dict(x)
    xv["cu_seqlens"] = torch.tensor([0, case.T], dtype=torch.int32)
    o_one, s_one = gpu_forward(xv)
    assert torch.equal(o_cut, o_one)
    assert torch.equal(s_cut, s_one)


# ------------------------------------------------------------------ packed batches cut into chunk windows
# Given a host copy of cu_seqlens (kda_prefill_forward_varlen), the library knows the lengths and may cut a packed
# batch into windows of chunk index within each sequence, carrying window j beside the intra-chunk work of window
# j+1.  Each window's carry starts from the float32 state the previous one left in final_state, so the results
# equal the uncut packed run bit for bit.

WINDOW_MIXES = {
    "gqa_mix": ([1, 63, 64, 65, 777, 2048, 8192], 8, 32),  # the packed GQA workload's lengths
    "empty_and_short": ([0, 2100, 0, 1, 129, 3000, 0], 2, 4),
    "one_long": ([5000], 2, 4),
    "two_equal": ([2048, 2048], 4, 8),
    "ragged_tail": ([2049, 63, 2111], 2, 2),
}


def _window_count(T, H, HV, cu_h):
    import kda_gated_delta_prefill_b200 as kda
    n = kda.varlen_kernel_launches(T, H, HV, cu_h)
    return (n - 3) // 2 if n > 4 else 1


@pytest.mark.parametrize("mix", list(WINDOW_MIXES))
def test_windows_match_the_uncut_packed_run_bit_for_bit(mix):
    lengths, H, HV = WINDOW_MIXES[mix]
    case = gen.Case(f"win_{mix}", B=1, T=sum(lengths), H=H, HV=HV, lengths=lengths, state="n01",
                    seed=600 + len(mix))
    x = gen.make_inputs(case)
    cu_h = x["cu_seqlens"]
    assert _window_count(case.T, H, HV, cu_h) >= 2  # the windowed path is taken
    o_w, s_w = gpu_forward(x, cu_seqlens_host=cu_h)
    o_u, s_u = gpu_forward(x)
    assert torch.equal(o_w, o_u)
    assert torch.equal(s_w, s_u)
    import kda_gated_delta_prefill_b200 as kda
    assert kda.device_error(clear=True) == 0


def test_windows_with_many_sequences():
    # 1500 sequences (more than one block of the window-offset scan) around one long one, in a shuffled order
    rng = np.random.default_rng(7)
    lengths = [int(x) for x in rng.integers(0, 12, size=1500)]
    lengths[911] = 3000
    case = gen.Case("win_many", B=1, T=sum(lengths), H=1, HV=2, lengths=lengths, state="n01", seed=691)
    x = gen.make_inputs(case)
    assert _window_count(case.T, 1, 2, x["cu_seqlens"]) >= 2
    o_w, s_w = gpu_forward(x, cu_seqlens_host=x["cu_seqlens"])
    o_u, s_u = gpu_forward(x)
    assert torch.equal(o_w, o_u)
    assert torch.equal(s_w, s_u)


def test_windows_full_parity():
    lengths = [2049, 63, 0, 2111]
    case = gen.Case("win_oracle", B=1, T=sum(lengths), H=2, HV=2, lengths=lengths, state="n01", seed=641)
    x = gen.make_inputs(case)
    assert _window_count(case.T, 2, 2, x["cu_seqlens"]) >= 2
    o, s = gpu_forward(x, cu_seqlens_host=x["cu_seqlens"])
    compare(o, s, oracle_forward(x))


def test_windows_short_batch_runs_uncut():
    lengths = [300, 1900, 64]  # the longest has 30 chunks: too short to cut
    case = gen.Case("win_short", B=1, T=sum(lengths), H=2, HV=4, lengths=lengths, state="n01", seed=651)
    x = gen.make_inputs(case)
    import kda_gated_delta_prefill_b200 as kda
    assert kda.varlen_kernel_launches(case.T, 2, 4, x["cu_seqlens"]) == 4
    o_w, s_w = gpu_forward(x, cu_seqlens_host=x["cu_seqlens"])
    o_u, s_u = gpu_forward(x)
    assert torch.equal(o_w, o_u) and torch.equal(s_w, s_u)


def test_windows_in_place_state_update():
    lengths = [3000, 0, 700]
    case = gen.Case("win_inplace", B=1, T=sum(lengths), H=2, HV=2, lengths=lengths, state="n01", seed=661)
    x = gen.make_inputs(case)
    xc = to_cuda(x)
    import kda_gated_delta_prefill_b200 as kda
    st = xc["initial_state"].clone()
    o, s = kda.forward(xc["q"], xc["k"], xc["v"], xc["g"], xc["beta"], st, xc["cu_seqlens"], final_state=st,
                       cu_seqlens_host=x["cu_seqlens"])
    o_u, s_u = gpu_forward(x)
    torch.cuda.synchronize()
    assert s.data_ptr() == st.data_ptr()
    assert torch.equal(o, o_u) and torch.equal(s, s_u)


def test_windows_host_entry_point():
    # kda_prefill_forward_host passes its host cu_seqlens on, so a packed batch takes the windowed path there
    lengths = [2500, 17, 900]
    case = gen.Case("win_host", B=1, T=sum(lengths), H=2, HV=4, lengths=lengths, state="n01", seed=671)
    x = gen.make_inputs(case)
    import kda_gated_delta_prefill_b200 as kda
    assert _window_count(case.T, 2, 4, x["cu_seqlens"]) >= 2
    N, T, HV = case.N, case.T, case.HV
    pin = {k: v.pin_memory() for k, v in x.items() if isinstance(v, torch.Tensor)}
    o_h = torch.empty(1, T, HV, 128, dtype=torch.bfloat16).pin_memory()
    s_h = torch.empty(N, HV, 128, 128).pin_memory()
    staging = torch.empty(kda.host_staging_size(1, T, 2, HV, num_seqs=N, has_initial_state=True,
                                                has_cu_seqlens=True), dtype=torch.uint8, device="cuda")
    kda.forward_host(pin["q"], pin["k"], pin["v"], pin["g"], pin["beta"], pin["initial_state"], pin["cu_seqlens"],
                     o=o_h, final_state=s_h, staging=staging)
    torch.cuda.synchronize()
    o_u, s_u = gpu_forward(x)
    assert torch.equal(o_h, o_u.cpu()) and torch.equal(s_h, s_u.cpu())


def test_windows_captured_in_a_cuda_graph():
    import kda_gated_delta_prefill_b200 as kda
    lengths = [2300, 5, 0, 1200]
    cases = [gen.Case(f"wgraph{i}", B=1, T=sum(lengths), H=2, HV=4, lengths=lengths, state="n01", seed=681 + i)
             for i in range(2)]
    xs = [gen.make_inputs(c) for c in cases]
    cu_h = xs[0]["cu_seqlens"]
    assert _window_count(cases[0].T, 2, 4, cu_h) >= 2
    xcs = [to_cuda(x) for x in xs]
    N, T = cases[0].N, cases[0].T
    buf = {k: v.clone() for k, v in xcs[0].items() if isinstance(v, torch.Tensor)}
    ws = torch.empty(kda.workspace_size(1, T, 2, 4, 128, 128, N), dtype=torch.uint8, device="cuda")
    o = torch.empty(1, T, 4, 128, dtype=torch.bfloat16, device="cuda")
    s = torch.empty(N, 4, 128, 128, device="cuda")

    def call():
        kda.forward(buf["q"], buf["k"], buf["v"], buf["g"], buf["beta"], buf["initial_state"], buf["cu_seqlens"],
                    o=o, final_state=s, workspace=ws, cu_seqlens_host=cu_h)

    call()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for xc in xcs:
        for k, t in buf.items():
            t.copy_(xc[k])
        o.fill_(float("nan"))
        s.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        o_ref, s_ref = kda.forward(xc["q"], xc["k"], xc["v"], xc["g"], xc["beta"], xc["initial_state"],
                                   xc["cu_seqlens"])
        torch.cuda.synchronize()
        assert torch.equal(o, o_ref) and torch.equal(s, s_ref)
    del graph
    assert kda.device_error(clear=True) == 0


def test_parts_in_place_state_update():
    case = gen.Case("parts_inplace", B=1, T=3000, H=2, HV=2, state="n01", seed=321)
    x = gen.make_inputs(case)
    ref = oracle_forward(x)
    xc = to_cuda(x)
    import kda_gated_delta_prefill_b200 as kda
    st = xc["initial_state"].clone()
    o, s = kda.forward(xc["q"], xc["k"], xc["v"], xc["g"], xc["beta"], st, final_state=st)
    torch.cuda.synchronize()
    assert s.data_ptr() == st.data_ptr()
    compare(o, s, ref)


def test_parts_on_a_non_default_stream():
    case = gen.Case("parts_stream", B=1, T=2600, H=2, HV=2, state="n01", seed=331)
    x = gen.make_inputs(case)
    ref = oracle_forward(x)
    xc = to_cuda(x)
    import kda_gated_delta_prefill_b200 as kda
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        o, s = kda.forward(xc["q"], xc["k"], xc["v"], xc["g"], xc["beta"], xc["initial_state"])
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    compare(o, s, ref)


def test_parts_from_concurrent_host_threads():
    # Forwards cut into parts, issued at the same time from several host threads on their own streams: each
    # takes its own side stream (or waits for one) and must equal the single-threaded result bit for bit.
    import threading
    import kda_gated_delta_prefill_b200 as kda
    case = gen.Case("parts_threads", B=1, T=2600, H=4, HV=8, state="n01", seed=361)
    x = to_cuda(gen.make_inputs(case))
    assert kda.kernel_launches(1, case.T, case.H, case.HV) > 2
    o_ref, s_ref = kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"])
    torch.cuda.synchronize()
    results, errors = [None] * 6, []

    def run(i):
        try:
            st = torch.cuda.Stream()
            st.wait_stream(torch.cuda.default_stream())
            with torch.cuda.stream(st):
                outs = [kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"]) for _ in range(3)]
            st.synchronize()
            results[i] = outs
        except Exception as e:  # reported below
            errors.append(repr(e))

    threads = [threading.Thread(target=run, args=(i,)) for i in range(6)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for outs in results:
        for o, s in outs:
            assert torch.equal(o, o_ref) and torch.equal(s, s_ref)
    assert kda.device_error(clear=True) == 0


def test_parts_repeatable_under_load():
    # The carry of each part runs beside the next part's intra-chunk kernel.  Repeated calls must agree bit for
    # bit with the uncut run and leave the device error word clear: a pipeline wait that gave up (for
    # instance on a barrier that had already moved two phases on) sets a bit there and corrupts the result.
    import kda_gated_delta_prefill_b200 as kda
    case = gen.Case("parts_load", B=1, T=16384, H=32, HV=32, state="n01", seed=341)
    x = gen.make_inputs(case, device="cuda")
    assert kda.kernel_launches(1, case.T, case.H, case.HV) == 16
    cu = torch.tensor([0, case.T], dtype=torch.int32, device="cuda")
    o_ref, s_ref = kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"], cu)
    torch.cuda.synchronize()
    kda.device_error(clear=True)
    o = torch.empty_like(o_ref)
    s = torch.empty_like(s_ref)
    for _ in range(12):
        kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"], o=o, final_state=s)
    torch.cuda.synchronize()
    assert kda.device_error(clear=True) == 0
    assert torch.equal(o, o_ref)
    assert torch.equal(s, s_ref)



# ------------------------------------------------------------------ segmented carry
# A plain batch with few (sequence, value head) units and long sequences carries segments of every sequence
# at once: per segment its linear map and its image of zero, a scan of the segment start states, then all
# segments with outputs.  The results follow the same recurrence with different rounding, so they are compared
# with the oracle at the usual tolerances.

@pytest.mark.parametrize("B,T,H,HV,state", [(1, 5120, 2, 2, "none"), (1, 8209, 2, 2, "n01"), (2, 4096, 1, 1, "n01"),
                                            (1, 6000, 1, 2, "n01")])
def test_segmented_full_parity(B, T, H, HV, state):
    import kda_gated_delta_prefill_b200 as kda
    case = gen.Case(f"seg{T}", B=B, T=T, H=H, HV=HV, state=state, seed=400 + T + HV)
    assert kda.kernel_launches(B, T, H, HV) == 4
    x = gen.make_inputs(case)
    o, s = gpu_forward(x)
    compare(o, s, oracle_forward(x))


def test_segmented_in_place_state_update():
    case = gen.Case("seg_inplace", B=1, T=5120, H=2, HV=2, state="n01", seed=431)
    x = gen.make_inputs(case)
    ref = oracle_forward(x)
    xc = to_cuda(x)
    import kda_gated_delta_prefill_b200 as kda
    st = xc["initial_state"].clone()
    o, s = kda.forward(xc["q"], xc["k"], xc["v"], xc["g"], xc["beta"], st, final_state=st)
    torch.cuda.synchronize()
    assert s.data_ptr() == st.data_ptr()
    assert kda.device_error(clear=True) == 0
    compare(o, s, ref)


def test_segmented_long_few_heads_sampled():
    # B=1, H=HV=4, T=65536 (14 segments per unit); the oracle checks one head.
    import kda_gated_delta_prefill_b200 as kda
    case = gen.Case("seg_long", B=1, T=65536, H=4, HV=4, state="n01", seed=441)
    x = gen.make_inputs(case, device="cuda")
    o, s = kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"])
    torch.cuda.synchronize()
    assert kda.device_error(clear=True) == 0
    xc = {k: (v.cpu() if isinstance(v, torch.Tensor) else v) for k, v in x.items()}
    sub = select_heads(xc, [3])
    compare(o[:, :, [3]].contiguous(), s[:, [3]].contiguous(), oracle_forward(sub))


@pytest.mark.parametrize("B,T,H,HV,varlen", [(1, 200, 2, 4, False), (2, 1000, 4, 4, False), (1, 300, 1, 2, True)])
def test_bf16_state_forward(B, T, H, HV, varlen):
    """bf16 state storage: the oracle runs from the bf16 initial state's values; the kernel's final state is the
    nearest-even bf16 of its fp32 state, so the state bar widens by one bf16 unit (2^-8 relative) of each element."""
    import kda_gated_delta_prefill_b200 as kda
    import oracle
    gen_ = torch.Generator().manual_seed(1700 + T)
    cu = torch.tensor([0, 37, 37, 300], dtype=torch.int32) if varlen else None
    N = 3 if varlen else B
    q = torch.randn(B, T, H, 128, generator=gen_).bfloat16()
    k = torch.randn(B, T, H, 128, generator=gen_).bfloat16()
    v = torch.randn(B, T, HV, 128, generator=gen_).bfloat16()
    g = -torch.nn.functional.softplus(torch.randn(B, T, HV, 128, generator=gen_)) / 8
    beta = torch.sigmoid(torch.randn(B, T, HV, generator=gen_))
    s0 = (0.1 * torch.randn(N, HV, 128, 128, generator=gen_)).bfloat16()
    c = lambda t: None if t is None else t.cuda()
    o, sN = kda.forward_state_bf16(c(q), c(k), c(v), c(g), c(beta), c(s0), c(cu))
    torch.cuda.synchronize()
    assert sN.dtype == torch.bfloat16
    ref = oracle.forward(q, k, v, g, beta, s0.float(), cu)
    og = o.float().cpu().numpy()
    if varlen:
        rows = np.zeros((B, T), bool)
        rows[0, :300] = True
        og, orf = og[rows], ref["o64"][rows]
    else:
        orf = ref["o64"]
    # o: the element-wise bar of every parity test, |d_i| <= 2e-2 * max(1, |ref_i|)
    assert np.isfinite(og).all()
    assert (np.abs(og - orf) <= O_TOL * np.maximum(1.0, np.abs(orf))).all()
    sg = sN.float().cpu().numpy().astype(np.float64)
    sr = ref["state"]
    for n in range(N):
        for h in range(HV):
            den = np.linalg.norm(sr[n, h])
            assert np.linalg.norm(sg[n, h] - sr[n, h]) <= (STATE_REL_FRO + 2 ** -8) * den
    assert (np.abs(sg - sr) <= 0.02 + 0.02 * np.abs(sr) + 2 ** -8 * np.abs(sr)).all()
    # in place: final_state may be the initial state's buffer
    s_io = c(s0.clone())
    kda.forward_state_bf16(c(q), c(k), c(v), c(g), c(beta), s_io, c(cu), final_state=s_io)
    torch.cuda.synchronize()
    assert torch.equal(s_io.cpu(), sN.cpu())


# ------------------------------------------------------------------ CUDA graphs
# The library allocates nothing and never synchronises, so a forward can be captured in a CUDA graph and
# replayed; the side stream of a sequence cut into parts becomes a fork and a join inside the graph.

@pytest.mark.parametrize("B,T,H,HV,lengths", [(1, 2600, 4, 8, None),      # cut into parts (side stream)
                                              (1, 5120, 2, 2, None),      # segmented carry
                                              (1, 1300, 2, 4, [700, 0, 64, 536]),  # packed sequences
                                              (2, 300, 2, 4, None),       # plain, uncut
                                              (2, 1024, 8, 96, None)],    # two head groups
                         ids=["parts", "segmented", "packed", "plain", "head_groups"])
def test_forward_captured_in_a_cuda_graph(B, T, H, HV, lengths):
    import kda_gated_delta_prefill_b200 as kda
    cases = [gen.Case(f"graph{i}", B=B, T=T, H=H, HV=HV, lengths=lengths, state="n01", seed=500 + 7 * i + T)
             for i in range(2)]
    xs = [to_cuda(gen.make_inputs(c)) for c in cases]
    N = cases[0].N
    num_seqs = N if lengths is not None else 0
    buf = {k: v.clone() for k, v in xs[0].items() if isinstance(v, torch.Tensor)}
    ws = torch.empty(kda.workspace_size(B, T, H, HV, 128, 128, num_seqs), dtype=torch.uint8, device="cuda")
    o = torch.empty(B, T, HV, 128, dtype=torch.bfloat16, device="cuda")
    s = torch.empty(N, HV, 128, 128, device="cuda")

    def call():
        kda.forward(buf["q"], buf["k"], buf["v"], buf["g"], buf["beta"], buf["initial_state"], buf.get("cu_seqlens"),
                    o=o, final_state=s, workspace=ws)

    call()  # eager warm-up before the capture
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call()
    for x in xs:  # replay on new inputs copied into the captured buffers
        for k, t in buf.items():
            t.copy_(x[k])
        o.fill_(float("nan"))
        s.fill_(float("nan"))
        graph.replay()
        torch.cuda.synchronize()
        o_ref, s_ref = kda.forward(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"], x["cu_seqlens"])
        torch.cuda.synchronize()
        if lengths is None:
            assert torch.equal(o, o_ref)
        else:  # rows outside every packed sequence are not written; here the sequences cover all rows
            assert torch.equal(o[:, :sum(lengths)], o_ref[:, :sum(lengths)])
        assert torch.equal(s, s_ref)
    del graph
    assert kda.device_error(clear=True) == 0
