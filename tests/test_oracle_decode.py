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
