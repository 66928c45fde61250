"""The benchmark's byte and FLOP model (the numerators of its roofline fractions), checked on CPU against figures
fixed outside it: hand-computed totals for the five workloads (per token and value head, q and k 256 bytes each
divided by the GQA group, v 256, g 512, beta 4, o 256; plus the fp32 state read and written; 180,224 dense
chunk-form FLOPs per token and value head), and the byte sizes of the very tensors the seeded generators produce
and the entry points read and write."""
import pytest
import torch

import bench
from kda_gated_delta_prefill_b200 import inputs as gen

# algorithmic bytes of the five workloads, worked out by hand
WORKLOAD_BYTES = {
    "smallest_T128": 262_656,
    "tail_T1000_H4_state": 6_684_288,
    "wide_B2_T4096_H96": 1_223_688_192,
    "varlen_gqa_H8_HV32": 444_040_448,
    "long_T65536_H64_state": 6_467_616_768,
}


@pytest.mark.parametrize("case", gen.WORKLOADS, ids=lambda c: c.name)
def test_forward_bytes_of_the_five_workloads(case):
    assert bench.algorithmic_bytes(case) == WORKLOAD_BYTES[case.name]


def test_forward_flops_of_the_long_prefill():
    assert bench.chunk_flops(gen.LONG_PREFILL) == 4_194_304 * 180_224  # 7.56e11


def _nbytes(*ts):
    return sum(t.numel() * t.element_size() for t in ts if t is not None)


@pytest.mark.parametrize("case", [
    gen.Case("f1", B=2, T=70, H=2, HV=6, state="n01", seed=1),
    gen.Case("f2", B=1, T=100, H=1, HV=1, seed=2),
    gen.Case("f3", B=1, T=90, H=2, HV=4, lengths=[10, 0, 80], state="n01", seed=3),
], ids=lambda c: c.name)
def test_forward_bytes_are_the_tensor_sizes(case):
    """Inputs read once, o and the final state written once (q and k once per Q/K head)."""
    x = gen.make_inputs(case)
    o = torch.empty(case.B, case.T, case.HV, case.V, dtype=torch.bfloat16)
    final = torch.empty(case.N, case.HV, case.K, case.V, dtype=torch.float32)
    want = _nbytes(x["q"], x["k"], x["v"], x["g"], x["beta"], x["initial_state"], o, final)
    assert bench.algorithmic_bytes(case) == want


@pytest.mark.parametrize("case", [
    gen.Case("b1", B=2, T=70, H=2, HV=6, state="n01", seed=1),
    gen.Case("b2", B=1, T=100, H=1, HV=1, seed=2),
], ids=lambda c: c.name)
def test_backward_bytes_are_the_tensor_sizes(case):
    """q, k, v, g, beta, dout and dht read; dq, dk, dv, dg, dbeta written; with an initial state, that state read
    and dh0 written (the benchmark's backward asks for dh0 only when there is an initial state)."""
    x = gen.make_inputs(case)
    gr = gen.make_backward_grads(case)
    s0 = x["initial_state"]
    outs = [torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"]), torch.empty_like(x["g"]),
            torch.empty_like(x["beta"]), None if s0 is None else torch.empty_like(s0)]
    want = _nbytes(x["q"], x["k"], x["v"], x["g"], x["beta"], gr["dout"], gr["dht"], s0, *outs)
    assert bench.backward_bytes(case) == want


def test_decode_bytes_are_the_tensor_sizes():
    """Every (row, value head) reads and writes its bf16 state; q, k, v, g, beta and the slot index read; o
    written."""
    case = gen.DecodeCase("d", B=5, H=2, HV=6, slots=9, seed=4)
    x = gen.make_decode_inputs(case)
    o = torch.empty_like(x["v"])
    state_rw = 2 * case.B * case.HV * 128 * 128 * 2
    want = state_rw + _nbytes(x["q"], x["k"], x["v"], x["g"], x["beta"], x["state_indices"], o)
    assert bench.decode_bytes(case) == want
