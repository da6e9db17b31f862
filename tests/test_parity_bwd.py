"""Backward pass (through the C ABI) against the fp64 backward oracle.

The GPU side runs the product pipeline: attn_fwd gives O and LSE, attn_bwd
takes them with dO. The oracle computes dQ, dK, dV from Q, K, V and dO
alone. Small problems are compared in full (several 128-row tiles, ragged
tails, every mask); full-size workloads are compared on sampled query rows
(dQ) and sampled key rows of a few heads (dK, dV), plus invariants.
"""
import numpy as np
import pytest
import torch

from exact_softmax_attention_04_b200 import synth
from parity import assert_grads_close

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def attn():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from exact_softmax_attention_04_b200 import build_lib
    build_lib.build()
    import exact_softmax_attention_04_b200 as pkg
    return pkg


def _fwd_bwd(attn, q, k, v, do, causal, window, scale=None, workspace=None):
    qc, kc, vc, doc = (x.cuda() for x in (q, k, v, do))
    o, lse = attn.attn_fwd(qc, kc, vc, scale, causal, window)
    dq, dk, dv = attn.attn_bwd(qc, kc, vc, o, lse, doc, scale, causal, window, workspace=workspace)
    assert attn.sync_status() == attn.ATTN_OK
    return dq, dk, dv


def _np(t):
    return t.float().cpu().numpy()


MASKS = [(False, -1), (True, -1), (True, 0), (True, 1), (True, 127), (True, 128), (True, 129),
         (True, 300), (True, 100000), (False, 0), (False, 1), (False, 127), (False, 200)]


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("n", [1, 77, 128, 129, 256, 383, 640])
@pytest.mark.parametrize("causal,window", MASKS)
def test_bwd_small_shapes_all_masks_in_full(attn, oracle_mod, d, n, causal, window):
    q_std = 4.0 if (n + d + window) % 2 else 1.0
    q, k, v = synth.make_qkv(1, 2, n, d, seed=n * 7 + d, q_std=q_std)
    do = synth.make_dout(1, 2, n, d, seed=n * 7 + d)
    sc = 1.0 / np.sqrt(d)
    grads = _fwd_bwd(attn, q, k, v, do, causal, window)
    refs = oracle_mod.attn_bwd(q, k, v, do, sc, causal, window)
    assert_grads_close([_np(g) for g in grads], refs, f"n{n} d{d} c{causal} w{window}")


def test_bwd_batch_heads_and_scale(attn, oracle_mod):
    q, k, v = synth.make_qkv(3, 5, 200, 64, seed=60)
    do = synth.make_dout(3, 5, 200, 64, seed=60)
    for causal, window, scale in [(False, -1, 0.125), (True, -1, 0.3), (True, 50, 0.05)]:
        grads = _fwd_bwd(attn, q, k, v, do, causal, window, scale)
        refs = oracle_mod.attn_bwd(q, k, v, do, scale, causal, window)
        assert_grads_close([_np(g) for g in grads], refs, f"B3H5 c{causal} w{window} s{scale}")


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_window_zero(attn, d):
    """w = 0: P is the identity, so dV = dO exactly and dQ, dK vanish (up to
    the rounding of dO.v - dO.O, both of which equal dO.v)."""
    q, k, v = synth.make_qkv(2, 2, 257, d, seed=61, q_std=4.0)
    do = synth.make_dout(2, 2, 257, d, seed=61)
    dq, dk, dv = _fwd_bwd(attn, q, k, v, do, True, 0)
    assert torch.equal(dv.cpu(), do)
    assert dq.float().abs().max().item() <= 1e-3
    assert dk.float().abs().max().item() <= 1e-3


@pytest.mark.parametrize("causal,window", [(False, -1), (True, -1), (True, 200), (False, 150)])
def test_bwd_softmax_invariants(attn, causal, window):
    """sum_j dK_j = 0 and sum_j dV_j = sum_i dO_i per head (rows of P sum to 1)."""
    q, k, v = synth.make_qkv(1, 4, 1000, 128, seed=62, q_std=2.0)
    do = synth.make_dout(1, 4, 1000, 128, seed=62)
    dq, dk, dv = _fwd_bwd(attn, q, k, v, do, causal, window)
    dk64, dv64 = dk.double().cpu(), dv.double().cpu()
    ksum = dk64.sum(dim=2).abs().max().item()
    assert ksum <= 2e-2 * dk64.abs().sum(dim=2).max().item() / np.sqrt(1000), ksum
    vs = dv64.sum(dim=2) - do.double().sum(dim=2)
    assert vs.abs().max().item() <= 1e-2 * do.double().abs().sum(dim=2).max().item() / np.sqrt(1000)


@pytest.mark.parametrize("d", [64, 128])
def test_bwd_deterministic_and_dirty_workspace(attn, d):
    """dK and dV (both head sizes) and dQ (d = 128) are accumulated inside one
    CTA in a fixed order, so runs are bit-identical; at d = 64 dQ sums key
    tiles by reduce-adds in a varying order (equal up to fp32 rounding). A
    workspace full of garbage gives the same result (the prep kernel
    rewrites what it reads)."""
    q, k, v = synth.make_qkv(1, 4, 1000, d, seed=63)
    do = synth.make_dout(1, 4, 1000, d, seed=63)
    ws = torch.full((attn.bwd_workspace_bytes(1, 4, 1000, d),), 0x7f, dtype=torch.uint8, device="cuda")
    a = _fwd_bwd(attn, q, k, v, do, True, 300, workspace=ws)
    b = _fwd_bwd(attn, q, k, v, do, True, 300)
    assert torch.equal(a[1], b[1]) and torch.equal(a[2], b[2])
    if d == 128:
        assert torch.equal(a[0], b[0])
    else:
        assert (a[0].float() - b[0].float()).abs().max().item() <= 1e-2 * a[0].float().abs().max().item()


@pytest.mark.parametrize("wl", [synth.FULL_N8192, synth.WINDOW_N32768, synth.SYM_N16384,
                                # lengths that are no multiple of the 128-row tile
                                synth.Workload("B1-H2-n20011-d128-causal", 1, 2, 20011, 128, True, q_std=2.0, seed=7),
                                synth.Workload("B1-H2-n12345-d64-window2000", 1, 2, 12345, 64, True, 2000, seed=8)],
                         ids=lambda w: w.name)
def test_bwd_full_size_workloads_sampled(attn, oracle_mod, wl):
    q, k, v = synth.make_inputs(wl)
    do = synth.make_dout(wl.B, wl.H, wl.n, wl.d, seed=wl.seed)
    grads = _fwd_bwd(attn, q, k, v, do, wl.causal, wl.window, wl.scale)
    qrows = synth.sample_rows(wl.B, wl.H, wl.n, per_head_random=4, bound_every=1024, edge=4)
    # key rows of two heads (first and last): their columns need every row of
    # the head's softmax statistics in the oracle
    rng = np.random.default_rng(5)
    heads = [0, wl.B * wl.H - 1]
    krows = np.concatenate([h * wl.n + np.unique(np.concatenate(
        [rng.integers(0, wl.n, 48), [0, 127, 128, wl.n - 1]])) for h in heads])
    dq_ref, dk_ref, dv_ref = oracle_mod.attn_bwd_rows(q, k, v, do, wl.scale, wl.causal, wl.window,
                                                      qrows, krows)
    d = wl.d
    sel = lambda t, rows: t.view(-1, d)[torch.as_tensor(rows, device=t.device)].float().cpu().numpy()
    assert_grads_close([sel(grads[0], qrows), sel(grads[1], krows), sel(grads[2], krows)],
                       [dq_ref, dk_ref, dv_ref], wl.name)
    for g in grads:
        assert bool(torch.isfinite(g.float()).all())


# ---------------------------------------------------------------- grouped-query attention

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,Hkv", [(4, 2), (6, 3), (8, 1)])
@pytest.mark.parametrize("causal,window", [(False, -1), (True, -1), (True, 100), (False, 60)])
def test_gqa_bwd_small_in_full(attn, oracle_mod, d, H, Hkv, causal, window):
    B, n = 2, 300
    q, k, v = synth.make_qkv(B, H, n, d, seed=H * 10 + Hkv + d, q_std=2.0, Hkv=Hkv)
    do = synth.make_dout(B, H, n, d, seed=H * 10 + Hkv + d)
    sc = 1.0 / np.sqrt(d)
    grads = _fwd_bwd(attn, q, k, v, do, causal, window, sc)
    rows_q, rows_k = np.arange(B * H * n), np.arange(B * Hkv * n)
    refs = oracle_mod.attn_bwd_rows_gqa(q, k, v, do, sc, causal, window, rows_q, rows_k)
    assert_grads_close([g.float().cpu().numpy().reshape(-1, d) for g in grads], refs,
                       f"gqa H{H} Hkv{Hkv} d{d} c{causal} w{window}")


@pytest.mark.parametrize("d", [64, 128])
def test_gqa_bwd_equals_group_sums_of_multi_head(attn, d):
    """Grouped-query dK, dV equal the group sums of the multi-head gradients
    on repeated K/V (each rounded to bf16 separately, hence a tolerance);
    dQ is the same computation."""
    B, H, Hkv, n = 1, 8, 2, 500
    q, k, v = synth.make_qkv(B, H, n, d, seed=80 + d, Hkv=Hkv)
    do = synth.make_dout(B, H, n, d, seed=80 + d)
    g = _fwd_bwd(attn, q, k, v, do, True, -1)
    G = H // Hkv
    m = _fwd_bwd(attn, q, k.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1), do, True, -1)
    if d == 128:
        assert torch.equal(g[0], m[0])  # the dQ kernel does the same work in the same order
    else:
        assert (g[0].float() - m[0].float()).abs().max().item() <= 1e-2 * m[0].float().abs().max().item()
    for a, b in ((g[1], m[1]), (g[2], m[2])):
        ref = b.float().view(B, Hkv, G, n, d).sum(dim=2)
        assert (a.float() - ref).abs().max().item() <= 2e-2 * ref.abs().max().item()


# ---------------------------------------------------------------- block-local mask

@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("block,causal", [(1, True), (64, False), (100, True), (256, False), (300, True)])
@pytest.mark.parametrize("H,Hkv", [(2, 2), (4, 2)])
def test_block_mask_bwd_small_in_full(attn, oracle_mod, d, block, causal, H, Hkv):
    B, n = 1, 520
    q, k, v = synth.make_qkv(B, H, n, d, seed=block + d + H, q_std=2.0, Hkv=Hkv)
    do = synth.make_dout(B, H, n, d, seed=block + d + H)
    sc = 1.0 / np.sqrt(d)
    qc, kc, vc, doc = (x.cuda() for x in (q, k, v, do))
    o, lse = attn.attn_fwd(qc, kc, vc, sc, causal, -1, block=block)
    grads = attn.attn_bwd(qc, kc, vc, o, lse, doc, sc, causal, -1, block=block)
    assert attn.sync_status() == attn.ATTN_OK
    refs = oracle_mod.attn_bwd_rows_gqa(q, k, v, do, sc, causal, -1, np.arange(B * H * n),
                                        np.arange(B * Hkv * n), block=block)
    assert_grads_close([g.float().cpu().numpy().reshape(-1, d) for g in grads], refs,
                       f"block{block} c{causal} H{H} Hkv{Hkv} d{d}")
