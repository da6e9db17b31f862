"""Decode against rolling caches (through the C ABI) against the fp64 oracle.

Small problems cover every grouped-query ratio, head size, partially filled
and wrapped caches, cache sizes around multiples of the kernel's 128-slot
tile, mixed positions within a batch, splits of the slots that lie wholly
or partly past the cached positions, and caches whose unused slots hold
NaN; the full-size
workload (64 sequences at position 32767 against 4096-slot caches) is
compared on every row. The same for steps of a few new tokens per sequence
(attn_decode_multi): every column count of the kernel (query heads of a
group times tokens, 1 to 16), windows shorter than the cache, equality with
the forward pass's window rows, and its full-size workload (four tokens per
sequence).
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


def _gpu(attn, q, kc, vc, pos, scale=None):
    o, lse = attn.attn_decode(q.cuda(), kc.cuda(), vc.cuda(), torch.tensor(pos, dtype=torch.int32).cuda(),
                              scale)
    assert attn.sync_status() == attn.ATTN_OK
    return o, lse


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,Hkv", [(4, 4), (4, 2), (8, 2), (8, 1)])
@pytest.mark.parametrize("W", [1, 63, 64, 65, 127, 128, 129, 200, 1024])
def test_decode_small_in_full(attn, oracle_mod, d, H, Hkv, W):
    B = 4
    q, kc, vc = synth.make_decode(B, H, Hkv, W, d, seed=W * 3 + H + d, q_std=2.0)
    pos = [0, W // 2, W - 1, 3 * W + 7]  # one slot, half full, just full, wrapped
    sc = 1.0 / np.sqrt(d)
    o, lse = _gpu(attn, q, kc, vc, pos, sc)
    o_ref, lse_ref = oracle_mod.attn_decode(q, kc, vc, pos, sc)
    assert_close(o.float().cpu().numpy().reshape(-1, d), lse.cpu().numpy().reshape(-1),
                 o_ref.reshape(-1, d), lse_ref.reshape(-1), f"W{W} H{H} Hkv{Hkv} d{d}")


def test_decode_equals_forward_window_row(attn, oracle_mod):
    """Caches filled from a sequence by the write rule: the decode of the last
    position equals row T-1 of the forward pass with causal window W-1."""
    B, H, Hkv, T, W, d = 2, 8, 2, 300, 128, 128
    q, k, v = synth.make_qkv(B, H, T, d, seed=77, Hkv=Hkv)
    kc, vc = synth.ring_from_sequence(k, W), synth.ring_from_sequence(v, W)
    o_dec, l_dec = _gpu(attn, q[:, :, T - 1].contiguous(), kc, vc, [T - 1] * B)
    o_fwd, l_fwd = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), None, True, W - 1)
    assert attn.sync_status() == attn.ATTN_OK
    assert (o_dec.float() - o_fwd[:, :, T - 1].float()).abs().max().item() <= 2e-2
    assert (l_dec - l_fwd[:, :, T - 1]).abs().max().item() <= 1e-3


def test_decode_full_size_workload_every_row(attn, oracle_mod):
    wl = synth.DECODE_W4096
    q, kc, vc = synth.make_decode(wl.B, wl.H, wl.Hkv, wl.W, wl.d, seed=wl.seed, q_std=wl.q_std)
    o, lse = _gpu(attn, q, kc, vc, [wl.pos] * wl.B, wl.scale)
    o_ref, lse_ref = oracle_mod.attn_decode(q, kc, vc, [wl.pos] * wl.B, wl.scale)
    assert_close(o.float().cpu().numpy().reshape(-1, wl.d), lse.cpu().numpy().reshape(-1),
                 o_ref.reshape(-1, wl.d), lse_ref.reshape(-1), wl.name)
    o2, l2 = _gpu(attn, q, kc, vc, [wl.pos] * wl.B, wl.scale)
    assert torch.equal(o, o2) and torch.equal(lse, l2)


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("W,pos", [(300, [0, 130, 255, 299]), (4096, [5, 1000, 2047, 2048]),
                                   (2500, [1, 127, 128, 129])])
def test_decode_unused_slots_hold_nan(attn, oracle_mod, d, W, pos):
    """Slots no position has reached yet may hold anything, NaN included: the
    result depends on the cached positions only (several splits of the slots
    lie wholly or partly past them)."""
    B, H, Hkv = len(pos), 8, 2
    q, kc, vc = synth.make_decode(B, H, Hkv, W, d, seed=W + d, q_std=2.0)
    for b, t in enumerate(pos):
        kc[b, :, t + 1:] = float("nan")
        vc[b, :, t + 1:] = float("nan")
    sc = 1.0 / np.sqrt(d)
    o, lse = _gpu(attn, q, kc, vc, pos, sc)
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()
    o_ref, lse_ref = oracle_mod.attn_decode(q, kc, vc, pos, sc)
    assert_close(o.float().cpu().numpy().reshape(-1, d), lse.cpu().numpy().reshape(-1),
                 o_ref.reshape(-1, d), lse_ref.reshape(-1), f"nan-slots W{W} d{d}")


@pytest.mark.parametrize("H,Hkv", [(4, 4), (8, 1), (16, 2)])
def test_decode_d128_many_splits_mixed_positions(attn, oracle_mod, H, Hkv):
    """Few (sequence, kv head) pairs, so the 4096 slots are cut into many
    splits; positions from one slot to a wrapped cache."""
    B, W, d = 3, 4096, 128
    q, kc, vc = synth.make_decode(B, H, Hkv, W, d, seed=H * 7 + Hkv, q_std=3.0)
    pos = [0, 2049, 40000]
    sc = 1.0 / np.sqrt(d)
    o, lse = _gpu(attn, q, kc, vc, pos, sc)
    o_ref, lse_ref = oracle_mod.attn_decode(q, kc, vc, pos, sc)
    assert_close(o.float().cpu().numpy().reshape(-1, d), lse.cpu().numpy().reshape(-1),
                 o_ref.reshape(-1, d), lse_ref.reshape(-1), f"splits H{H} Hkv{Hkv}")


# ---------------------------------------------------------------------------
# A few new tokens per sequence (attn_decode_multi): token u at position
# pos - T + 1 + u attends to max(0, t_u - w) .. t_u.

def _gpu_multi(attn, q, kc, vc, pos, window, scale=None):
    o, lse = attn.attn_decode_multi(q.cuda(), kc.cuda(), vc.cuda(), torch.tensor(pos, dtype=torch.int32).cuda(),
                                    window, scale)
    assert attn.sync_status() == attn.ATTN_OK
    return o, lse


def _check_multi(attn, oracle_mod, q, kc, vc, pos, window, d, what):
    sc = 1.0 / np.sqrt(d)
    o, lse = _gpu_multi(attn, q, kc, vc, pos, window, sc)
    o_ref, lse_ref = oracle_mod.attn_decode_multi(q, kc, vc, pos, sc, window)
    assert_close(o.float().cpu().numpy().reshape(-1, d), lse.cpu().numpy().reshape(-1),
                 o_ref.reshape(-1, d), lse_ref.reshape(-1), what)
    return o, lse


@pytest.mark.parametrize("d", [64, 128])
@pytest.mark.parametrize("H,Hkv,T", [(4, 4, 4), (8, 2, 4), (8, 1, 2), (6, 2, 3), (12, 2, 2), (16, 1, 1),
                                     (3, 3, 2)])
@pytest.mark.parametrize("W,window", [(128, 124), (200, 50), (64, 0), (129, 100), (1024, 1020)])
def test_decode_multi_small_in_full(attn, oracle_mod, d, H, Hkv, T, W, window):
    if window + T > W:
        pytest.skip("window does not fit the cache")
    B = 4
    q, kc, vc = synth.make_decode_multi(B, H, Hkv, T, W, d, seed=W * 5 + H * 3 + T + d, q_std=2.0)
    pos = [T - 1, W // 2, W - 1, 3 * W + 7]  # first tokens, half full, just full, wrapped
    _check_multi(attn, oracle_mod, q, kc, vc, pos, window, d, f"multi W{W} w{window} H{H} Hkv{Hkv} T{T} d{d}")


def test_decode_multi_one_token_full_window_equals_decode(attn, oracle_mod):
    """attn_decode is attn_decode_multi with T = 1 and window W - 1: the same
    kernel, bit for bit."""
    B, H, Hkv, W, d = 3, 8, 2, 300, 128
    q, kc, vc = synth.make_decode(B, H, Hkv, W, d, seed=91, q_std=2.0)
    pos = [0, 150, 1000]
    o1, l1 = _gpu(attn, q, kc, vc, pos)
    o2, l2 = _gpu_multi(attn, q.unsqueeze(2).contiguous(), kc, vc, pos, W - 1)
    assert torch.equal(o1, o2.squeeze(2)) and torch.equal(l1, l2.squeeze(2))


@pytest.mark.parametrize("T,window", [(4, 124), (2, 60), (3, 0)])
def test_decode_multi_equals_forward_window_rows(attn, oracle_mod, T, window):
    """Caches filled from a sequence by the write rule: the last T positions
    decoded in one step equal rows N-T .. N-1 of the forward pass with causal
    window w (GPU forward and oracle)."""
    B, H, Hkv, N, W, d = 2, 8, 2, 300, 128, 128
    q, k, v = synth.make_qkv(B, H, N, d, seed=78 + T, Hkv=Hkv, q_std=2.0)
    kc, vc = synth.ring_from_sequence(k, W), synth.ring_from_sequence(v, W)
    qs = q[:, :, N - T:].contiguous()
    o_dec, l_dec = _gpu_multi(attn, qs, kc, vc, [N - 1] * B, window)
    o_fwd, l_fwd = attn.attn_fwd(q.cuda(), k.cuda(), v.cuda(), None, True, window)
    assert attn.sync_status() == attn.ATTN_OK
    assert (o_dec.float() - o_fwd[:, :, N - T:].float()).abs().max().item() <= 2e-2
    assert (l_dec - l_fwd[:, :, N - T:]).abs().max().item() <= 1e-3
    rows = [(b * H + h) * N + t for b in range(B) for h in range(H) for t in range(N - T, N)]
    o_ref, l_ref = oracle_mod.attn_rows_gqa(q, k, v, 1.0 / np.sqrt(d), True, window, rows)
    assert_close(o_dec.float().cpu().numpy().reshape(-1, d), l_dec.cpu().numpy().reshape(-1), o_ref, l_ref,
                 f"decode T{T} w{window} vs forward rows")


@pytest.mark.parametrize("d", [64, 128])
def test_decode_multi_unread_slots_hold_nan(attn, oracle_mod, d):
    """Slots outside every token's window (unwritten ones, and with a window
    shorter than the cache the oldest cached ones) may hold NaN."""
    B, H, Hkv, T, W, w = 4, 8, 2, 4, 600, 300
    q, kc, vc = synth.make_decode_multi(B, H, Hkv, T, W, d, seed=33 + d, q_std=2.0)
    pos = [3, 200, 599, 5000]
    for b, t in enumerate(pos):
        used = torch.zeros(W, dtype=torch.bool)
        for p in range(max(0, t - T + 1 - w), t + 1):
            used[p % W] = True
        kc[b, :, ~used] = float("nan")
        vc[b, :, ~used] = float("nan")
    o, lse = _check_multi(attn, oracle_mod, q, kc, vc, pos, w, d, f"multi nan-slots d{d}")
    assert torch.isfinite(o.float()).all() and torch.isfinite(lse).all()


def test_decode_multi_full_size_workload_every_row(attn, oracle_mod):
    wl = synth.DECODE_T4_W4096
    q, kc, vc = synth.make_decode_multi(wl.B, wl.H, wl.Hkv, wl.T, wl.W, wl.d, seed=wl.seed, q_std=wl.q_std)
    o, lse = _check_multi(attn, oracle_mod, q, kc, vc, [wl.pos] * wl.B, wl.w, wl.d, wl.name)
    o2, l2 = _gpu_multi(attn, q, kc, vc, [wl.pos] * wl.B, wl.w, wl.scale)
    assert torch.equal(o, o2) and torch.equal(lse, l2)
