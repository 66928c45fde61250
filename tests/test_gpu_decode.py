"""GPU parity of the decode step (kda_decode_step through the C ABI) against the oracle's decode step."""
import numpy as np
import pytest
import torch

import oracle

pytestmark = pytest.mark.gpu

BF16_ULP = 2.0 ** -8  # relative spacing of bf16 values (one unit in the last place at most 2^-7, at least 2^-8)


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import kda_gated_delta_prefill_b200 as kda
    kda.lib()


def _case(B, H, HV, N, seed, pad=0.0):
    gen = torch.Generator().manual_seed(seed)
    q = torch.randn(B, H, 128, generator=gen).bfloat16()
    k = torch.randn(B, H, 128, generator=gen).bfloat16()
    v = torch.randn(B, HV, 128, generator=gen).bfloat16()
    g = -torch.nn.functional.softplus(torch.randn(B, HV, 128, generator=gen)) / 8
    beta = torch.sigmoid(torch.randn(B, HV, generator=gen))
    pool = (0.1 * torch.randn(N, HV, 128, 128, generator=gen)).bfloat16()
    slots = torch.randperm(N, generator=gen)[:B].to(torch.int32)
    drop = torch.rand(B, generator=gen) < pad
    idx = torch.where(drop, torch.full_like(slots, -1), slots)
    return q, k, v, g, beta, pool, idx


def _gpu(q, k, v, g, beta, pool, idx):
    import kda_gated_delta_prefill_b200 as kda
    d = [t.cuda() for t in (q, k, v, g, beta, pool, idx)]
    o = kda.decode_step(*d)
    torch.cuda.synchronize()
    return o.cpu(), d[5].cpu()


def _check(o, new_pool, ref_o, ref_pool, pool, idx, g):
    active = idx >= 0
    # o: bf16 of an fp32 computation against the float64 result
    err = (o.float().numpy() - ref_o).reshape(len(idx), -1)
    scale = np.abs(ref_o).reshape(len(idx), -1).max(axis=1, keepdims=True) + 1e-6
    assert np.all(np.abs(err) <= 2 * BF16_ULP * scale + 1e-6), np.abs(err / scale).max()
    assert torch.all(o[~active] == 0)
    # updated slots.  Each element is the bf16 rounding of an fp32 computation of S' + beta kn r, and the
    # kernel's normalised kn may differ from the oracle's by one bf16 unit in an element (the order of the
    # sum of squares is free), so the bound is two bf16 units of the element, one of the update beta kn r, and
    # the fp32 error of the 128-term dot products relative to the slot's scale.
    for b in np.nonzero(active.numpy())[0]:
        s = int(idx[b])
        exact = ref_pool[s]
        got = new_pool[s].float().numpy().astype(np.float64)
        decayed = np.exp(g[b].numpy().astype(np.float64))[:, :, None] * pool[s].float().numpy().astype(np.float64)
        tol = (2 * BF16_ULP * np.abs(exact) + 2 * BF16_ULP * np.abs(exact - decayed)
               + 1e-5 * np.abs(exact).max(axis=(1, 2), keepdims=True))
        assert np.all(np.abs(got - exact) <= tol), (s, np.abs(got - exact).max())
    # every other slot untouched, bit for bit
    touched = set(idx[active].tolist())
    for s in range(pool.shape[0]):
        if s not in touched:
            assert torch.equal(new_pool[s], pool[s]), s


# (400, 4, 8): 3200 (row, head) units, several per persistent CTA, with padding rows among them
@pytest.mark.parametrize("B,H,HV,N,pad", [(1, 1, 1, 1, 0.0), (37, 2, 4, 64, 0.25), (64, 12, 12, 96, 0.1),
                                          (5, 1, 8, 5, 0.0), (400, 4, 8, 512, 0.3)])
def test_decode_parity(B, H, HV, N, pad):
    q, k, v, g, beta, pool, idx = _case(B, H, HV, N, seed=500 + B + HV, pad=pad)
    o, new_pool = _gpu(q, k, v, g, beta, pool, idx)
    ref_o, ref_pool = oracle.decode_step(q, k, v, g, beta, pool.float(), idx)
    _check(o, new_pool, ref_o, ref_pool, pool, idx, g)


def test_decode_all_padding_touches_nothing():
    q, k, v, g, beta, pool, idx = _case(8, 2, 2, 8, seed=521)
    idx = torch.full_like(idx, -1)
    o, new_pool = _gpu(q, k, v, g, beta, pool, idx)
    assert torch.all(o == 0)
    assert torch.equal(new_pool, pool)


def test_decode_packed_qkv_rows():
    # q, k, v as views of one packed [B, (2H + HV) * 128] tensor (row stride (2H + HV) * 128)
    import kda_gated_delta_prefill_b200 as kda
    B, H, HV = 16, 3, 6
    q, k, v, g, beta, pool, idx = _case(B, H, HV, 20, seed=531, pad=0.2)
    packed = torch.cat([q.reshape(B, -1), k.reshape(B, -1), v.reshape(B, -1)], dim=1).cuda()
    qv = packed[:, : H * 128].view(B, H, 128)
    kv = packed[:, H * 128: 2 * H * 128].view(B, H, 128)
    vv = packed[:, 2 * H * 128:].view(B, HV, 128)
    assert qv.stride(0) == (2 * H + HV) * 128
    pool_a, pool_b = pool.cuda(), pool.cuda()
    o_a = kda.decode_step(qv, kv, vv, g.cuda(), beta.cuda(), pool_a, idx.cuda())
    o_b = kda.decode_step(q.cuda(), k.cuda(), v.cuda(), g.cuda(), beta.cuda(), pool_b, idx.cuda())
    torch.cuda.synchronize()
    assert torch.equal(o_a, o_b)
    assert torch.equal(pool_a, pool_b)


def test_decode_steps_follow_the_oracle():
    # eight steps feeding the pool back; the oracle rounds its states to bf16 between steps, as the pool does
    import kda_gated_delta_prefill_b200 as kda
    B, H, HV, N = 6, 2, 4, 10
    pool0 = _case(B, H, HV, N, seed=540)[5]
    pool_gpu = pool0.cuda()
    pool_ref = pool0.float()
    for step in range(8):
        q, k, v, g, beta, _, idx = _case(B, H, HV, N, seed=541 + step, pad=0.2)
        o = kda.decode_step(q.cuda(), k.cuda(), v.cuda(), g.cuda(), beta.cuda(), pool_gpu, idx.cuda())
        ref_o, ref_pool = oracle.decode_step(q, k, v, g, beta, pool_ref, idx)
        torch.cuda.synchronize()
        err = np.abs(o.cpu().float().numpy() - ref_o).max()
        assert err <= 2e-2 * (np.abs(ref_o).max() + 1e-3), (step, err)
        pool_ref = torch.from_numpy(ref_pool).bfloat16().float()
    diff = (pool_gpu.cpu().float() - pool_ref).abs().max().item()
    assert diff <= 4 * BF16_ULP * pool_ref.abs().max().item(), diff


def test_decode_full_workload_sampled():
    """The 1024-row, 12-head serving step on its 2048-slot pool, in the launch shape the benchmark times:
    rows are independent, so a sample of rows is checked against the oracle on just their slots."""
    import kda_gated_delta_prefill_b200 as kda
    from kda_gated_delta_prefill_b200.inputs import DECODE_SERVING, make_decode_inputs
    case = DECODE_SERVING
    d = make_decode_inputs(case, device="cuda")
    before = d["state"].clone()
    o = kda.decode_step(d["q"], d["k"], d["v"], d["g"], d["beta"], d["state"], d["state_indices"])
    torch.cuda.synchronize()
    assert kda.device_error(clear=True) == 0
    rows = torch.arange(0, case.B, 33)  # 32 rows spread over the batch (and so over the CTAs' unit lists)
    idx = d["state_indices"][rows].cpu()
    slots = idx.clamp(min=0).long()
    mini = before[slots.cuda()].cpu()
    mini_idx = torch.where(idx >= 0, torch.arange(len(rows), dtype=torch.int32), idx)
    sub = [d[n][rows.cuda()].cpu() for n in ("q", "k", "v", "g", "beta")]
    ref_o, ref_pool = oracle.decode_step(*sub, mini.float(), mini_idx)
    got_pool = d["state"][slots.cuda()].cpu()
    _check(o[rows.cuda()].cpu(), got_pool, ref_o, ref_pool, mini, mini_idx, sub[3])
    # slots no row selects keep their bytes
    unused = torch.ones(case.slots, dtype=torch.bool)
    unused[d["state_indices"][d["state_indices"] >= 0].long().cpu()] = False
    free = torch.nonzero(unused).flatten()[:64].cuda()
    assert torch.equal(d["state"][free], before[free])
