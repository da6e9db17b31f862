"""CUDA path (through the C ABI) against the fp64 oracle, element by element.

Small problems are compared in full; they span several 128-row/128-key tiles
and ragged tails. Full-size workloads run in the same launch configuration
the benchmark times and are compared on a deterministic row sample that the
oracle computes one row at a time, plus properties that hold at any size.
"""
import numpy as np
import pytest
import torch

from exact_softmax_attention_04_b200 import synth
from parity import assert_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_softmax_attention_04_b200 import build_lib
    build_lib.build()
    import exact_softmax_attention_04_b200 as pkg
    return pkg


def _gpu(attn, q, k, v, causal, window, scale=None):
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), scale, causal, window)
    assert attn.sync_status() == attn.ATTN_OK
    return o, lse


def _full_check(attn, oracle_mod, q, k, v, causal, window, scale=None, what=""):
    d = q.shape[-1]
    sc = scale if scale is not None else 1.0 / np.sqrt(d)
    o, lse = _gpu(attn, q, k, v, causal, window, scale)
    o_ref, lse_ref = oracle_mod.attn_fwd(q, k, v, sc, causal, window)
    return assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, what)


def _sampled_check(attn, oracle_mod, wl, rows, o=None, lse=None):
    q, k, v = synth.make_inputs(wl)
    if o is None:
        o, lse = _gpu(attn, q, k, v, wl.causal, wl.window, wl.scale)
    o_s = o.view(-1, wl.d)[torch.as_tensor(rows, device=o.device)].float().cpu().numpy()
    l_s = lse.view(-1)[torch.as_tensor(rows, device=o.device)].cpu().numpy()
    o_ref, lse_ref, _ = oracle_mod.attn_rows(q, k, v, wl.scale, wl.causal, wl.window, rows)
    return assert_close(o_s, l_s, o_ref, lse_ref, wl.name), o, lse


def test_small_causal_workload_in_full(attn, oracle_mod):
    wl = synth.SMALL_CAUSAL
    q, k, v = synth.make_inputs(wl)
    _full_check(attn, oracle_mod, q, k, v, wl.causal, wl.window, wl.scale, wl.name)


MASKS = [(False, -1), (True, -1), (True, 0), (True, 1), (True, 127), (True, 128), (True, 129),
         (True, 300), (True, 100000), (False, 0), (False, 1), (False, 127), (False, 200), (False, 100000)]


@pytest.fixture(params=["per_item", "persistent"])
def schedule(request, attn):
    """Run the test under one forward work schedule (forced), then restore
    the automatic choice."""
    mode = {"per_item": attn.SCHEDULE_PER_ITEM, "persistent": attn.SCHEDULE_PERSISTENT}[request.param]
    attn.set_fwd_schedule(mode)
    yield request.param
    attn.set_fwd_schedule(attn.SCHEDULE_AUTO)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n", [1, 77, 128, 129, 256, 383, 640])
@pytest.mark.parametrize("causal,window", MASKS)
def test_small_shapes_all_masks_in_full(attn, oracle_mod, schedule, d, n, causal, window):
    q_std = 4.0 if (n + d + window) % 2 else 1.0
    q, k, v = synth.make_qkv(1, 2, n, d, seed=n * 7 + d, q_std=q_std)
    _full_check(attn, oracle_mod, q, k, v, causal, window, what=f"{schedule} n{n} d{d} c{causal} w{window}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("B,H,Hkv,n,causal,window,block", [
    (3, 5, 5, 700, True, 200, 0), (2, 8, 2, 1000, True, -1, 0), (1, 6, 3, 2100, False, 300, 0),
    (2, 4, 4, 1500, False, -1, 0), (1, 8, 8, 3000, True, -1, 512), (2, 4, 1, 999, False, -1, 256)])
def test_schedules_agree_bit_for_bit(attn, d, B, H, Hkv, n, causal, window, block):
    """The persistent form walks the same work items with the same per-tile
    arithmetic as one CTA per item: equal outputs, bit for bit (many items
    per persistent CTA here: grouped heads, block masks, ragged tails)."""
    q, k, v = synth.make_qkv(B, H, n, d, seed=B * 100 + n + d, q_std=3.0, Hkv=Hkv)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    outs = []
    try:
        for mode in (attn.SCHEDULE_PER_ITEM, attn.SCHEDULE_PERSISTENT):
            attn.set_fwd_schedule(mode)
            o, lse = attn.attn_fwd(qd, kd, vd, None, causal, window, block=block)
            assert attn.sync_status() == attn.ATTN_OK
            outs.append((o, lse))
    finally:
        attn.set_fwd_schedule(attn.SCHEDULE_AUTO)
    assert torch.equal(outs[0][0], outs[1][0]) and torch.equal(outs[0][1], outs[1][1])


def test_persistent_schedule_many_items_per_cta(attn, oracle_mod):
    """64 heads x 24 query-tile pairs = 1536 items over the SMs (about ten per
    persistent CTA), window 256, both head sizes; sampled rows against the
    oracle."""
    try:
        attn.set_fwd_schedule(attn.SCHEDULE_PERSISTENT)
        for d in (64, 128):
            wl = synth.Workload(f"persist-B4-H16-n6000-d{d}-window256", 4, 16, 6000, d, True, 256, q_std=4.0)
            rows = synth.sample_rows(wl.B, wl.H, wl.n, per_head_random=64, seed=5)
            _sampled_check(attn, oracle_mod, wl, rows)
    finally:
        attn.set_fwd_schedule(attn.SCHEDULE_AUTO)


def test_batch_and_many_heads(attn, oracle_mod):
    q, k, v = synth.make_qkv(3, 5, 200, 64, seed=21)
    for causal, window in [(False, -1), (True, -1), (True, 50)]:
        _full_check(attn, oracle_mod, q, k, v, causal, window, what=f"B3H5 c{causal} w{window}")


def test_non_default_scale(attn, oracle_mod):
    q, k, v = synth.make_qkv(1, 2, 300, 128, seed=22)
    for scale in (0.01, 0.3):
        _full_check(attn, oracle_mod, q, k, v, True, -1, scale=scale, what=f"scale {scale}")


@pytest.mark.parametrize("d", [64, 128])
def test_zero_queries_give_mean_of_allowed_values(attn, d):
    n = 333
    _, k, v = synth.make_qkv(1, 2, n, d, seed=30)
    q = torch.zeros_like(k)
    vf = v.double()
    for causal, window in [(False, -1), (True, -1), (True, 40)]:
        o, lse = _gpu(attn, q, k, v, causal, window)
        o, lse = o.double().cpu(), lse.double().cpu()
        for i in (0, 1, 39, 40, 41, 127, 128, 200, n - 1):
            lo = max(0, i - window) if window >= 0 else 0
            hi = i + 1 if causal else n
            ref = vf[..., lo:hi, :].mean(dim=-2)
            assert (o[..., i, :] - ref).abs().max() <= 2e-2
            assert (lse[..., i] - np.log(hi - lo)).abs().max() <= 1e-3


@pytest.mark.parametrize("d", [64, 128])
def test_window_zero_returns_values_exactly(attn, d):
    q, k, v = synth.make_qkv(2, 2, 257, d, seed=31, q_std=4.0)
    o, lse = _gpu(attn, q, k, v, True, 0)
    assert torch.equal(o.cpu(), v)
    ref = (q.double() * k.double()).sum(-1) / np.sqrt(d)
    assert (lse.double().cpu() - ref).abs().max() <= 1e-3


def _allowed(i, j, n, causal, window, block):
    """Key j is attended by query i (the mask's plain definition)."""
    if block > 0:
        lo, hi = max(0, (i // block - 1) * block), (i if causal else min(n - 1, (i // block + 1) * block - 1))
    else:
        lo = max(0, i - window) if window >= 0 else 0
        hi = i if causal else (min(n - 1, i + window) if window >= 0 else n - 1)
    return lo <= j <= hi


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal,window,block,J", [(True, -1, 0, [200, 250, 299]), (True, 100, 0, [5, 130, 299]),
                                                   (False, 100, 0, [5, 299]), (True, -1, 96, [20, 250])])
def test_masked_keys_carry_exactly_zero_weight(attn, schedule, d, causal, window, block, J):
    """A masked key reaches no output: with V at the keys J set to the largest
    finite bf16 value, every row that attends none of J gives the same bits
    as before (a weight of even 2^-125 on a masked key would show), and LSE
    does not change at all."""
    n = 300
    q, k, v = synth.make_qkv(1, 2, n, d, seed=36, q_std=4.0)
    v2 = v.clone()
    v2[..., J, :] = torch.finfo(torch.bfloat16).max
    o1, l1 = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), None, causal, window, block=block)
    o2, l2 = attn.attn_fwd(q.cuda(), k.cuda(), v2.cuda(), None, causal, window, block=block)
    assert attn.sync_status() == attn.ATTN_OK
    rows = [i for i in range(n) if not any(_allowed(i, j, n, causal, window, block) for j in J)]
    assert len(rows) > 50
    assert torch.equal(o1[..., rows, :], o2[..., rows, :])
    assert torch.equal(l1, l2)


def test_key_value_permutation_invariance(attn):
    q, k, v = synth.make_qkv(1, 2, 512, 128, seed=32, q_std=4.0)
    perm = torch.randperm(512, generator=torch.Generator().manual_seed(1))
    o1, l1 = _gpu(attn, q, k, v, False, -1)
    o2, l2 = _gpu(attn, q, k[..., perm, :].contiguous(), v[..., perm, :].contiguous(), False, -1)
    assert (o1.float() - o2.float()).abs().max().item() <= 2e-2
    assert (l1 - l2).abs().max().item() <= 1e-3


def test_runs_are_deterministic(attn):
    q, k, v = synth.make_qkv(1, 4, 1000, 64, seed=33)
    o1, l1 = _gpu(attn, q, k, v, True, 300)
    o2, l2 = _gpu(attn, q, k, v, True, 300)
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_host_entry_point_matches_device_entry_point(attn):
    q, k, v = synth.make_qkv(2, 3, 700, 128, seed=34)
    o_d, l_d = _gpu(attn, q, k, v, True, 200)
    qp, kp, vp = q.pin_memory(), k.pin_memory(), v.pin_memory()
    o_h, l_h = attn.attn_fwd_host(qp, kp, vp, causal=True, window=200)
    assert attn.sync_status() == attn.ATTN_OK
    assert torch.equal(o_h, o_d.cpu()) and torch.equal(l_h, l_d.cpu())


def test_host_entry_pipelined_chunks_equal_device(attn):
    """Large enough for the host entry point to pipeline its copies over
    chunks of heads (13 heads: a ragged last chunk), called twice back to
    back into different outputs with no synchronisation in between."""
    qa, ka, va = synth.make_qkv(1, 13, 4096, 128, seed=91)
    qb, kb, vb = synth.make_qkv(1, 13, 4096, 128, seed=92)
    o_a, l_a = _gpu(attn, qa, ka, va, True, 1000)
    o_b, l_b = _gpu(attn, qb, kb, vb, True, 1000)
    pinned = [t.pin_memory() for t in (qa, ka, va, qb, kb, vb)]
    o1, l1 = attn.attn_fwd_host(*pinned[:3], causal=True, window=1000)
    o2, l2 = attn.attn_fwd_host(*pinned[3:], causal=True, window=1000)
    assert attn.sync_status() == attn.ATTN_OK
    assert torch.equal(o1, o_a.cpu()) and torch.equal(l1, l_a.cpu())
    assert torch.equal(o2, o_b.cpu()) and torch.equal(l2, l_b.cpu())


@pytest.mark.parametrize("wl", synth.sweep(), ids=lambda w: w.name)
def test_sweep_cells_sampled(attn, oracle_mod, wl):
    rows = synth.sample_rows(wl.B, wl.H, wl.n, per_head_random=24, bound_every=16)
    _sampled_check(attn, oracle_mod, wl, rows)


@pytest.mark.parametrize("wl", [synth.Workload("B1-H2-n50001-d128-causal", 1, 2, 50001, 128, True, q_std=2.0, seed=3),
                                synth.Workload("B1-H3-n40007-d64-window1000", 1, 3, 40007, 64, True, 1000, seed=4)],
                         ids=lambda w: w.name)
def test_large_ragged_lengths_sampled(attn, oracle_mod, wl):
    """Long sequences whose length is no multiple of the 128-row tile: the
    last, partly filled query and key tiles among the sampled rows."""
    rows = synth.sample_rows(wl.B, wl.H, wl.n, per_head_random=24, bound_every=64, edge=40)
    _sampled_check(attn, oracle_mod, wl, rows)


@pytest.mark.parametrize("wl", [synth.FULL_N8192, synth.WINDOW_N32768, synth.CAUSAL_N131072,
                                synth.SYM_N16384], ids=lambda w: w.name)
def test_full_size_workloads_sampled(attn, oracle_mod, wl):
    per_head = 16 if wl.n >= 65536 else 24
    rows = synth.sample_rows(wl.B, wl.H, wl.n, per_head_random=per_head, bound_every=64, edge=32)
    _, o, lse = _sampled_check(attn, oracle_mod, wl, rows)
    assert bool(torch.isfinite(lse).all()) and bool(torch.isfinite(o.float()).all())
    q, k, v = synth.make_inputs(wl)
    o2, l2 = _gpu(attn, q, k, v, wl.causal, wl.window, wl.scale)
    assert torch.equal(o, o2) and torch.equal(lse, l2)


# ---------------------------------------------------------------- grouped-query attention

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,Hkv", [(4, 2), (6, 3), (8, 1)])
@pytest.mark.parametrize("causal,window", [(False, -1), (True, -1), (True, 100)])
def test_gqa_small_shapes_in_full(attn, oracle_mod, d, H, Hkv, causal, window):
    n = 300
    q, k, v = synth.make_qkv(2, H, n, d, seed=H * 10 + Hkv, q_std=2.0, Hkv=Hkv)
    sc = 1.0 / np.sqrt(d)
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), sc, causal, window)
    assert attn.sync_status() == attn.ATTN_OK
    rows = np.arange(2 * H * n)
    o_ref, lse_ref = oracle_mod.attn_rows_gqa(q, k, v, sc, causal, window, rows)
    assert_close(o.float().cpu().numpy().reshape(-1, d), lse.cpu().numpy().reshape(-1), o_ref, lse_ref,
                 f"gqa H{H} Hkv{Hkv} d{d} c{causal} w{window}")


def test_gqa_equals_multi_head_on_repeated_kv_bit_for_bit(attn):
    B, H, Hkv, n, d = 2, 8, 2, 777, 128
    q, k, v = synth.make_qkv(B, H, n, d, seed=70, Hkv=Hkv)
    o_g, l_g = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), None, True, -1)
    kr = k.repeat_interleave(H // Hkv, dim=1).contiguous().cuda()
    vr = v.repeat_interleave(H // Hkv, dim=1).contiguous().cuda()
    o_m, l_m = attn.attn_fwd(q.cuda(), kr, vr, None, True, -1)
    assert attn.sync_status() == attn.ATTN_OK
    assert torch.equal(o_g, o_m) and torch.equal(l_g, l_m)


def test_gqa_workload_sampled(attn, oracle_mod):
    wl = synth.GQA_N8192
    q, k, v = synth.make_inputs(wl)
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), wl.scale, wl.causal, wl.window)
    assert attn.sync_status() == attn.ATTN_OK
    rows = synth.sample_rows(wl.B, wl.H, wl.n, per_head_random=8, bound_every=16, edge=8)
    idx = torch.as_tensor(rows, device=o.device)
    o_s = o.view(-1, wl.d)[idx].float().cpu().numpy()
    l_s = lse.view(-1)[idx].cpu().numpy()
    o_ref, lse_ref = oracle_mod.attn_rows_gqa(q, k, v, wl.scale, wl.causal, wl.window, rows)
    assert_close(o_s, l_s, o_ref, lse_ref, wl.name)


@pytest.mark.parametrize("d", [64, 128])
def test_symmetric_window_closed_forms(attn, d):
    """Symmetric window: w = 0 returns V exactly; zero queries give the mean of
    the values in [max(0, i-w), min(n-1, i+w)] with LSE = ln(count)."""
    n, w = 333, 40
    q, k, v = synth.make_qkv(1, 2, n, d, seed=90, q_std=4.0)
    o, _ = _gpu(attn, q, k, v, False, 0)
    assert torch.equal(o.cpu(), v)
    z = torch.zeros_like(q)
    o, lse = _gpu(attn, z, k, v, False, w)
    o, lse, vf = o.double().cpu(), lse.double().cpu(), v.double()
    for i in (0, 1, 39, 40, 41, 127, 128, 200, 292, 293, n - 1):
        lo, hi = max(0, i - w), min(n - 1, i + w)
        assert (o[..., i, :] - vf[..., lo:hi + 1, :].mean(dim=-2)).abs().max() <= 2e-2
        assert (lse[..., i] - np.log(hi - lo + 1)).abs().max() <= 1e-3


# ---------------------------------------------------------------- block-local mask

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block", [1, 64, 100, 128, 256])
@pytest.mark.parametrize("causal", [False, True])
def test_block_mask_small_in_full(attn, oracle_mod, d, block, causal):
    n = 600
    q, k, v = synth.make_qkv(1, 2, n, d, seed=block + d, q_std=4.0 if causal else 1.0)
    sc = 1.0 / np.sqrt(d)
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), sc, causal, -1, block=block)
    assert attn.sync_status() == attn.ATTN_OK
    o_ref, lse_ref = oracle_mod.attn_fwd(q, k, v, sc, causal, -1, block)
    assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, f"block{block} d{d} c{causal}")


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("causal", [False, True])
def test_block_of_n_tokens_or_more_is_no_mask(attn, oracle_mod, d, causal):
    """One block covers the sequence: the keys of attn_fwd without a window,
    bit for bit; one token fewer leaves a second block of one token."""
    n = 333
    q, k, v = synth.make_qkv(1, 2, n, d, seed=5 + d)
    qc, kc, vc = q.cuda(), k.cuda(), v.cuda()
    o0, l0 = attn.attn_fwd(qc, kc, vc, None, causal, -1)
    for block in (n, 4 * n):
        o, lse = attn.attn_fwd(qc, kc, vc, None, causal, -1, block=block)
        assert torch.equal(o, o0) and torch.equal(lse, l0)
    o, lse = attn.attn_fwd(qc, kc, vc, None, causal, -1, block=n - 1)
    assert attn.sync_status() == attn.ATTN_OK
    o_ref, lse_ref = oracle_mod.attn_fwd(q, k, v, 1.0 / np.sqrt(d), causal, -1, n - 1)
    assert_close(o.float().cpu().numpy(), lse.cpu().numpy(), o_ref, lse_ref, f"block n-1 d{d} c{causal}")


def test_block_mask_gqa(attn, oracle_mod):
    B, H, Hkv, n, d = 2, 8, 2, 500, 128
    q, k, v = synth.make_qkv(B, H, n, d, seed=95, Hkv=Hkv)
    sc = 1.0 / np.sqrt(d)
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), sc, True, -1, block=160)
    assert attn.sync_status() == attn.ATTN_OK
    rows = np.arange(B * H * n)
    o_ref, lse_ref = oracle_mod.attn_rows_gqa(q, k, v, sc, True, -1, rows, block=160)
    assert_close(o.float().cpu().numpy().reshape(-1, d), lse.cpu().numpy().reshape(-1), o_ref, lse_ref, "gqa block")


def test_block_workload_sampled(attn, oracle_mod):
    wl = synth.BLOCK_N16384
    q, k, v = synth.make_inputs(wl)
    o, lse = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), wl.scale, wl.causal, wl.window, block=wl.block)
    assert attn.sync_status() == attn.ATTN_OK
    rows = synth.sample_rows(wl.B, wl.H, wl.n, per_head_random=16, bound_every=4, edge=16)
    idx = torch.as_tensor(rows, device=o.device)
    o_ref, lse_ref, _ = oracle_mod.attn_rows(q, k, v, wl.scale, wl.causal, wl.window, rows, block=wl.block)
    assert_close(o.view(-1, wl.d)[idx].float().cpu().numpy(), lse.view(-1)[idx].cpu().numpy(), o_ref, lse_ref,
                 wl.name)
