"""Pins of the fp64 decode oracle (one query token against a rolling cache).

CPU only. The decode result is the sliding-window attention row of the
query's position; the pins build the rolling cache by the write rule (slot
p mod W) from a full sequence and compare with the window oracle's row, with
a textbook numpy computation on tiny inputs, and with invariances.
"""
import numpy as np
import pytest
import torch

from exact_softmax_attention_04_b200 import synth


def _seq(B, H, Hkv, T, d, seed):
    q, k, v = synth.make_qkv(B, H, T, d, seed=seed, q_std=2.0, Hkv=Hkv)
    return q, k, v


@pytest.mark.parametrize("T,W", [(1, 8), (5, 8), (8, 8), (9, 8), (30, 8), (100, 16), (64, 64)])
@pytest.mark.parametrize("H,Hkv", [(2, 2), (4, 1), (6, 3)])
def test_decode_equals_window_row_of_full_sequence(oracle_mod, T, W, H, Hkv):
    """Writing positions 0..T-1 into W slots (p mod W) and decoding the last
    position equals the causal window-(W-1) attention row T-1 of the full
    sequence: keys max(0, T-W) .. T-1."""
    B, d = 2, 16
    q, k, v = _seq(B, H, Hkv, T, d, seed=T * 31 + W)
    kc, vc = synth.ring_from_sequence(k, W), synth.ring_from_sequence(v, W)
    t = T - 1
    o, lse = oracle_mod.attn_decode(q[:, :, t].contiguous(), kc, vc, [t] * B, 0.3)
    rows = [(b * H + h) * T + t for b in range(B) for h in range(H)]
    o_ref, lse_ref = oracle_mod.attn_rows_gqa(q, k, v, 0.3, True, W - 1, rows)
    np.testing.assert_allclose(o.reshape(-1, d), o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(-1), lse_ref, rtol=0, atol=1e-12)


def test_decode_matches_textbook_on_tiny_inputs(oracle_mod):
    """Softmax over the cached slots written out in numpy: slots 0..pos when
    the cache is not full, all W slots otherwise."""
    B, H, Hkv, W, d = 3, 4, 2, 6, 8
    q, kc, vc = synth.make_decode(B, H, Hkv, W, d, seed=5, q_std=3.0)
    pos = [0, 3, 17]
    o, lse = oracle_mod.attn_decode(q, kc, vc, pos, 0.4)
    Q, K, V = (x.double().numpy() for x in (q, kc, vc))
    for b in range(B):
        n_valid = min(pos[b] + 1, W)
        for h in range(H):
            kh = h // (H // Hkv)
            s = 0.4 * K[b, kh, :n_valid] @ Q[b, h]
            w = np.exp(s - s.max())
            np.testing.assert_allclose(o[b, h], (w / w.sum()) @ V[b, kh, :n_valid], rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[b, h], s.max() + np.log(w.sum()), rtol=0, atol=1e-12)


def test_full_cache_is_invariant_to_slot_rotation(oracle_mod):
    """A full cache holds the same set of positions in any slot order."""
    B, H, Hkv, W, d = 2, 4, 2, 10, 16
    q, kc, vc = synth.make_decode(B, H, Hkv, W, d, seed=6)
    a = oracle_mod.attn_decode(q, kc, vc, [25, 9], 0.25)
    kr, vr = torch.roll(kc, 3, dims=2), torch.roll(vc, 3, dims=2)
    b = oracle_mod.attn_decode(q, kr, vr, [25, 9], 0.25)
    np.testing.assert_allclose(a[0], b[0], rtol=0, atol=1e-12)
    np.testing.assert_allclose(a[1], b[1], rtol=0, atol=1e-12)


def test_position_zero_returns_first_value(oracle_mod):
    q, kc, vc = synth.make_decode(2, 4, 4, 8, 16, seed=7, q_std=4.0)
    o, lse = oracle_mod.attn_decode(q, kc, vc, [0, 0], 0.25)
    np.testing.assert_array_equal(o, vc[:, :, 0].double().numpy())


def test_decode_oracle_rejects_bad_arguments(oracle_mod):
    q, kc, vc = synth.make_decode(1, 4, 2, 8, 16, seed=8)
    with pytest.raises(ValueError):
        oracle_mod.attn_decode(q, kc, vc, [-1], 0.25)
    q3, kc3, vc3 = synth.make_decode(1, 4, 3, 8, 16, seed=8)
    with pytest.raises(ValueError):
        oracle_mod.attn_decode(q3, kc3, vc3, [0], 0.25)  # 3 does not divide 4


def test_unused_slots_never_read(oracle_mod):
    """Slots no position has reached yet (slot >= pos + 1 while pos < W - 1)
    may hold anything: NaN there leaves the result bit for bit unchanged."""
    B, H, Hkv, W, d = 3, 4, 2, 40, 16
    q, kc, vc = synth.make_decode(B, H, Hkv, W, d, seed=21, q_std=1.5)
    pos = [0, 17, 38]
    o_ref, l_ref = oracle_mod.attn_decode(q, kc, vc, pos, 0.3)
    kn, vn = kc.clone(), vc.clone()
    for b, t in enumerate(pos):
        kn[b, :, t + 1:] = float("nan")
        vn[b, :, t + 1:] = float("nan")
    o, l = oracle_mod.attn_decode(q, kn, vn, pos, 0.3)
    assert np.array_equal(o, o_ref) and np.array_equal(l, l_ref)


# ---------------------------------------------------------------------------
# A few new tokens per sequence (T >= 1) with an explicit causal window w
# (w + T <= W): token u at position pos - T + 1 + u sees max(0, t_u - w) .. t_u.

@pytest.mark.parametrize("N,W,T,window", [(1, 8, 1, 7), (4, 8, 4, 4), (4, 8, 2, 3), (9, 8, 2, 6), (9, 8, 4, 4),
                                          (30, 8, 3, 5), (30, 8, 4, 0), (37, 16, 4, 12), (16, 16, 1, 15),
                                          (50, 16, 3, 2), (64, 64, 4, 60)])
@pytest.mark.parametrize("H,Hkv", [(2, 2), (4, 1), (6, 3)])
def test_multi_decode_equals_window_rows_of_full_sequence(oracle_mod, N, W, T, window, H, Hkv):
    """Writing positions 0..N-1 into W slots (p mod W) and decoding the last
    T positions equals rows N-T .. N-1 of the causal window-w attention of the
    full sequence."""
    B, d = 2, 16
    q, k, v = _seq(B, H, Hkv, N, d, seed=N * 7 + W * 3 + T)
    kc, vc = synth.ring_from_sequence(k, W), synth.ring_from_sequence(v, W)
    o, lse = oracle_mod.attn_decode_multi(q[:, :, N - T:].contiguous(), kc, vc, [N - 1] * B, 0.3, window)
    rows = [(b * H + h) * N + t for b in range(B) for h in range(H) for t in range(N - T, N)]
    o_ref, lse_ref = oracle_mod.attn_rows_gqa(q, k, v, 0.3, True, window, rows)
    np.testing.assert_allclose(o.reshape(-1, d), o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse.reshape(-1), lse_ref, rtol=0, atol=1e-12)


def test_multi_decode_of_one_token_with_the_full_window_is_decode(oracle_mod):
    B, H, Hkv, W, d = 3, 4, 2, 12, 16
    q, kc, vc = synth.make_decode(B, H, Hkv, W, d, seed=9, q_std=2.0)
    pos = [0, 7, 40]
    a = oracle_mod.attn_decode(q, kc, vc, pos, 0.3)
    b = oracle_mod.attn_decode_multi(q.unsqueeze(2).contiguous(), kc, vc, pos, 0.3, W - 1)
    assert np.array_equal(a[0], b[0].reshape(B, H, d)) and np.array_equal(a[1], b[1].reshape(B, H))


def test_multi_decode_matches_textbook_on_tiny_inputs(oracle_mod):
    """Softmax over each token's window, with slots located by the write rule,
    written out in numpy."""
    B, H, Hkv, T, W, d, w = 2, 4, 2, 3, 7, 8, 3
    g = torch.Generator().manual_seed(13)
    q = (2.0 * torch.randn((B, H, T, d), generator=g)).to(torch.bfloat16)
    kc = torch.randn((B, Hkv, W, d), generator=g).to(torch.bfloat16)
    vc = torch.randn((B, Hkv, W, d), generator=g).to(torch.bfloat16)
    pos = [2, 19]
    o, lse = oracle_mod.attn_decode_multi(q, kc, vc, pos, 0.4, w)
    Q, K, V = (x.double().numpy() for x in (q, kc, vc))
    for b in range(B):
        for h in range(H):
            kh = h // (H // Hkv)
            for u in range(T):
                t = pos[b] - T + 1 + u
                slots = [p % W for p in range(max(0, t - w), t + 1)]
                s = 0.4 * K[b, kh, slots] @ Q[b, h, u]
                e = np.exp(s - s.max())
                np.testing.assert_allclose(o[b, h, u], (e / e.sum()) @ V[b, kh, slots], rtol=0, atol=1e-12)
                np.testing.assert_allclose(lse[b, h, u], s.max() + np.log(e.sum()), rtol=0, atol=1e-12)


def test_multi_decode_reads_only_each_tokens_window(oracle_mod):
    """Slots holding no position of any token's window (unwritten, or with a
    window shorter than the cache) may hold anything: NaN there leaves the
    result bit for bit unchanged."""
    B, H, Hkv, T, W, d, w = 3, 4, 2, 4, 40, 16, 20
    g = torch.Generator().manual_seed(17)
    q = torch.randn((B, H, T, d), generator=g).to(torch.bfloat16)
    kc = torch.randn((B, Hkv, W, d), generator=g).to(torch.bfloat16)
    vc = torch.randn((B, Hkv, W, d), generator=g).to(torch.bfloat16)
    pos = [3, 30, 97]
    o_ref, l_ref = oracle_mod.attn_decode_multi(q, kc, vc, pos, 0.3, w)
    kn, vn = kc.clone(), vc.clone()
    for b, t in enumerate(pos):
        used = {p % W for p in range(max(0, t - T + 1 - w), t + 1)}
        for slot in range(W):
            if slot not in used:
                kn[b, :, slot] = float("nan")
                vn[b, :, slot] = float("nan")
    o, l = oracle_mod.attn_decode_multi(q, kn, vn, pos, 0.3, w)
    assert np.array_equal(o, o_ref) and np.array_equal(l, l_ref)


def test_multi_decode_oracle_rejects_bad_arguments(oracle_mod):
    g = torch.Generator().manual_seed(3)
    q = torch.randn((1, 4, 3, 16), generator=g).to(torch.bfloat16)
    kc = torch.randn((1, 2, 8, 16), generator=g).to(torch.bfloat16)
    with pytest.raises(ValueError):
        oracle_mod.attn_decode_multi(q, kc, kc, [1], 0.25, 3)   # pos < T - 1
    with pytest.raises(ValueError):
        oracle_mod.attn_decode_multi(q, kc, kc, [9], 0.25, 6)   # w + T > W: evicted positions needed
    with pytest.raises(ValueError):
        oracle_mod.attn_decode_multi(q, kc, kc, [9], 0.25, -1)  # a window is required
    oracle_mod.attn_decode_multi(q, kc, kc, [9], 0.25, 5)       # w + T = W is fine
