"""Pins of the fp64 oracle against facts that do not come from the oracle.

CPU only. Each test names what fixes its expected value: a brute-force
textbook computation on tiny inputs, a closed form, an invariant of the
definition, a library routine, or the values printed on the pages.
"""
import os

import numpy as np
import pytest
import torch

from exact_softmax_attention_04_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _f64(t):
    return t.to(torch.float64).numpy()


def _brute(q, k, v, scale, causal, window):
    """Textbook masked softmax attention over the full score matrix.

    Built the way the pages build it: the full S = Q K^T / sqrt(d), a boolean
    mask made like the sliding-window snippet (ones on [max(0, i-w), i]), the
    local-attention range max(0, i-w) ... min(n-1, i+w) when not causal, or
    the triu(1) causal mask, masked_fill with -inf, row softmax, then times V.
    """
    Q, K, V = _f64(q), _f64(k), _f64(v)
    n = Q.shape[-2]
    S = (Q @ np.swapaxes(K, -1, -2)) * scale
    if window >= 0:
        keep = np.zeros((n, n), dtype=bool)
        for i in range(n):
            last = i if causal else min(n - 1, i + window)
            keep[i, max(0, i - window): last + 1] = True
    elif causal:
        keep = ~np.triu(np.ones((n, n), dtype=bool), 1)
    else:
        keep = np.ones((n, n), dtype=bool)
    S = np.where(keep, S, -np.inf)
    M = S.max(axis=-1, keepdims=True)
    E = np.exp(S - M)
    Z = E.sum(axis=-1, keepdims=True)
    P = E / Z
    return P @ V, (M + np.log(Z))[..., 0], P


MASKS = [(False, -1), (True, -1), (True, 0), (True, 1), (True, 3), (True, 64),
         (False, 0), (False, 1), (False, 3), (False, 64)]


@pytest.mark.parametrize("n", [1, 7, 33, 64])
@pytest.mark.parametrize("causal,window", MASKS)
def test_oracle_matches_brute_force_on_tiny_inputs(oracle_mod, n, causal, window):
    q, k, v = synth.make_qkv(2, 2, n, 16, seed=3, q_std=2.0)
    scale = 1.0 / np.sqrt(16)
    o, lse = oracle_mod.attn_fwd(q, k, v, scale, causal, window)
    o_ref, lse_ref, _ = _brute(q, k, v, scale, causal, window)
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,window", MASKS)
def test_weights_rows_sum_to_one_and_reproduce_output(oracle_mod, causal, window):
    n = 40
    q, k, v = synth.make_qkv(1, 2, n, 32, seed=5)
    rows = np.arange(2 * n)
    o, lse, w = oracle_mod.attn_rows(q, k, v, 0.125, causal, window, rows, want_weights=True)
    np.testing.assert_allclose(w.sum(axis=1), 1.0, rtol=0, atol=1e-12)
    assert (w >= 0).all()
    # masked keys get exactly zero weight
    for r in rows:
        i = r % n
        allowed = oracle_mod.mask_row(n, i, causal, window)
        assert (w[r][~allowed] == 0).all()
        assert (w[r][allowed] > 0).all()
    V = _f64(v).reshape(2, n, 32)
    recon = np.stack([w[r] @ V[r // n] for r in rows])
    np.testing.assert_allclose(o, recon, rtol=0, atol=1e-12)
    _, _, P = _brute(q, k, v, 0.125, causal, window)
    np.testing.assert_allclose(w, P.reshape(2 * n, n), rtol=0, atol=1e-13)


@pytest.mark.parametrize("n", [5, 64, 130])
def test_mask_row_matches_page_window_snippet(oracle_mod, n):
    """The page's snippet sets ones on mask[i, max(0, i-w) : i+1]."""
    for w in [0, 1, 3, 17, n - 1, n, 2 * n]:
        for i in range(n):
            ref = np.zeros(n, dtype=bool)
            ref[max(0, i - w): i + 1] = True
            assert (oracle_mod.mask_row(n, i, True, w) == ref).all()
    for i in range(n):
        ref = ~np.triu(np.ones((n, n), dtype=bool), 1)[i]
        assert (oracle_mod.mask_row(n, i, True, -1) == ref).all()
        assert oracle_mod.mask_row(n, i, False, -1).all()


def test_window_at_least_n_equals_causal(oracle_mod):
    n = 96
    q, k, v = synth.make_qkv(1, 3, n, 32, seed=7, q_std=4.0)
    o_c, l_c = oracle_mod.attn_fwd(q, k, v, 0.2, True, -1)
    for w in (n - 1, n, 4 * n):
        o_w, l_w = oracle_mod.attn_fwd(q, k, v, 0.2, True, w)
        assert np.array_equal(o_w, o_c) and np.array_equal(l_w, l_c)
    # rows i <= w see the full causal prefix also when w < n
    o_w, l_w = oracle_mod.attn_fwd(q, k, v, 0.2, True, 40)
    assert np.array_equal(o_w[..., :41, :], o_c[..., :41, :])
    assert not np.allclose(o_w[..., 41:, :], o_c[..., 41:, :])


def test_window_zero_attends_to_self_only(oracle_mod):
    n, d = 50, 64
    q, k, v = synth.make_qkv(1, 2, n, d, seed=11)
    scale = 1.0 / 8.0
    o, lse = oracle_mod.attn_fwd(q, k, v, scale, True, 0)
    np.testing.assert_array_equal(o, _f64(v))
    qk = (_f64(q) * _f64(k)).sum(-1) * scale
    np.testing.assert_allclose(lse, qk, rtol=0, atol=1e-12)


def test_causal_row_zero_is_first_value(oracle_mod):
    q, k, v = synth.make_qkv(2, 2, 30, 16, seed=2, q_std=4.0)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.25, True, -1)
    np.testing.assert_array_equal(o[..., 0, :], _f64(v)[..., 0, :])
    np.testing.assert_allclose(lse[..., 0], (_f64(q)[..., 0, :] * _f64(k)[..., 0, :]).sum(-1) * 0.25,
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("causal,window", [(False, -1), (True, -1), (True, 5)])
def test_zero_queries_give_mean_of_allowed_values(oracle_mod, causal, window):
    n, d = 45, 32
    _, k, v = synth.make_qkv(1, 2, n, d, seed=4)
    q = torch.zeros_like(k)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.3, causal, window)
    V = _f64(v)
    for i in range(n):
        lo = max(0, i - window) if window >= 0 else 0
        hi = i + 1 if causal else n
        np.testing.assert_allclose(o[..., i, :], V[..., lo:hi, :].mean(axis=-2), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[..., i], np.log(hi - lo), rtol=0, atol=1e-14)


def test_equal_keys_give_uniform_weights(oracle_mod):
    n, d = 33, 16
    q, _, v = synth.make_qkv(1, 1, n, d, seed=8, q_std=3.0)
    k = torch.ones_like(q)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.5, False, -1)
    np.testing.assert_allclose(o[0, 0], np.broadcast_to(_f64(v)[0, 0].mean(0), (n, d)), rtol=0, atol=1e-14)
    s = _f64(q)[0, 0].sum(-1) * 0.5
    np.testing.assert_allclose(lse[0, 0], s + np.log(n), rtol=0, atol=1e-12)


def test_logit_shift_moves_lse_and_keeps_output(oracle_mod):
    """Adding t to the last coordinate of q_i, with that coordinate of every
    key set to 1, adds scale*t to every logit of row i."""
    n, d = 48, 32
    q, k, v = synth.make_qkv(1, 2, n, d, seed=9)
    k = k.clone()
    k[..., -1] = 1.0
    q0 = q.clone()
    q0[..., -1] = 0.0
    q1 = q0.clone()
    q1[..., -1] = 3.0
    for causal, window in [(False, -1), (True, -1), (True, 6)]:
        o0, l0 = oracle_mod.attn_fwd(q0, k, v, 0.25, causal, window)
        o1, l1 = oracle_mod.attn_fwd(q1, k, v, 0.25, causal, window)
        np.testing.assert_allclose(o1, o0, rtol=0, atol=1e-13)
        np.testing.assert_allclose(l1 - l0, 0.75, rtol=0, atol=1e-12)


def test_key_value_permutation_invariance_without_mask(oracle_mod):
    n, d = 64, 32
    q, k, v = synth.make_qkv(1, 2, n, d, seed=10, q_std=4.0)
    perm = torch.randperm(n, generator=torch.Generator().manual_seed(0))
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.2, False, -1)
    o_p, lse_p = oracle_mod.attn_fwd(q, k[..., perm, :].contiguous(), v[..., perm, :].contiguous(),
                                     0.2, False, -1)
    np.testing.assert_allclose(o_p, o, rtol=0, atol=1e-13)
    np.testing.assert_allclose(lse_p, lse, rtol=0, atol=1e-13)


def test_online_softmax_recurrence_equals_two_pass(oracle_mod):
    """The running-max / running-normaliser recurrence (FlashAttention's online
    softmax, with the output kept unnormalised and divided once at the end)
    over random chunkings reproduces the oracle's two-pass result."""
    n, d = 300, 32
    q, k, v = synth.make_qkv(1, 2, n, d, seed=12, q_std=4.0)
    scale = 1.0 / np.sqrt(d)
    rng = np.random.default_rng(0)
    for causal, window in [(False, -1), (True, -1), (True, 37)]:
        o_ref, lse_ref = oracle_mod.attn_fwd(q, k, v, scale, causal, window)
        Q, K, V = _f64(q)[0], _f64(k)[0], _f64(v)[0]
        for h in range(2):
            for i in rng.integers(0, n, 12):
                keys = [j for j in range(n) if (not causal or j <= i) and (window < 0 or j >= i - window)]
                cuts = sorted(set(rng.integers(1, len(keys), rng.integers(0, 6)).tolist())) if len(keys) > 1 else []
                m, l, acc = -np.inf, 0.0, np.zeros(d)
                for chunk in np.split(np.array(keys), cuts):
                    s = (K[h, chunk] @ Q[h, i]) * scale
                    m_new = max(m, s.max())
                    alpha = np.exp(m - m_new)
                    e = np.exp(s - m_new)
                    l = alpha * l + e.sum()
                    acc = alpha * acc + e @ V[h, chunk]
                    m = m_new
                np.testing.assert_allclose(acc / l, o_ref[0, h, i], rtol=0, atol=1e-12)
                np.testing.assert_allclose(m + np.log(l), lse_ref[0, h, i], rtol=0, atol=1e-12)


def _golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                key, val = line.split()
                vals[key] = val
    return vals


def test_associativity_identity_escape2(oracle_mod):
    """(Q K^T) V = Q (K^T V) with the oracle's contraction routine, at the
    page's N = 2000, d = 64, under numpy's default allclose; plus the page's
    printed float counts."""
    g = _golden("associativity_escape2.txt")
    N, d = int(g["N"]), int(g["d"])
    assert N * N == int(g["nxn_floats"]) and d * d == int(g["dxd_floats"])
    # three N x d standard-normal matrices (the worked example's sizes)
    Q, K, V = np.random.default_rng(0).standard_normal((3, N, d))
    A = oracle_mod.matmul(oracle_mod.matmul(Q, K, tb=True), V)
    Bm = oracle_mod.matmul(Q, oracle_mod.matmul(K, V, ta=True))
    assert str(bool(np.allclose(A, Bm))) == g["allclose"]


def test_identity_kernel_is_unnormalised_product(oracle_mod):
    """With the softmax weight replaced by the raw score and no mask, the
    attention rows give scale * (Q K^T) V, which must equal scale * Q (K^T V)."""
    n, d = 200, 64
    q, k, v = synth.make_qkv(1, 2, n, d, seed=13)
    rows = np.arange(2 * n)
    o, _, _ = oracle_mod.attn_rows(q, k, v, 0.125, False, -1, rows, kernel=oracle_mod.KERNEL_IDENTITY)
    Q, K, V = _f64(q)[0], _f64(k)[0], _f64(v)[0]
    ref = np.concatenate([Q[h] @ (K[h].T @ V[h]) for h in range(2)]) * 0.125
    np.testing.assert_allclose(o, ref, rtol=1e-10, atol=1e-9)


def test_matmul_routine_matches_library(oracle_mod):
    rng = np.random.default_rng(1)
    a = rng.standard_normal((7, 5))
    b = rng.standard_normal((5, 9))
    np.testing.assert_allclose(oracle_mod.matmul(a, b), a @ b, rtol=0, atol=1e-13)
    np.testing.assert_allclose(oracle_mod.matmul(a.T.copy(), b, ta=True), a @ b, rtol=0, atol=1e-13)
    np.testing.assert_allclose(oracle_mod.matmul(a, b.T.copy(), tb=True), a @ b, rtol=0, atol=1e-13)
    np.testing.assert_allclose(oracle_mod.matmul(a.T.copy(), b.T.copy(), ta=True, tb=True), a @ b,
                               rtol=0, atol=1e-13)


def test_row_subset_equals_full_run(oracle_mod):
    q, k, v = synth.make_qkv(2, 2, 70, 32, seed=14)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.17, True, 9)
    rows = np.array([0, 5, 69, 70, 139, 200, 279])
    o_r, lse_r, _ = oracle_mod.attn_rows(q, k, v, 0.17, True, 9, rows)
    np.testing.assert_array_equal(o_r, o.reshape(-1, 32)[rows])
    np.testing.assert_array_equal(lse_r, lse.reshape(-1)[rows])


def test_oracle_rejects_bad_arguments(oracle_mod):
    q, k, v = synth.make_qkv(1, 1, 8, 16)
    with pytest.raises(ValueError):
        oracle_mod.attn_rows(q, k, v, 0.25, True, -1, [8])  # row out of range
    _, k2, v2 = synth.make_qkv(1, 1, 8, 16, Hkv=1)
    q2, _, _ = synth.make_qkv(1, 2, 8, 16)
    with pytest.raises(ValueError):
        oracle_mod.attn_rows(q2, k2, v2, 0.25, True, -1, [0])  # fewer K/V heads: use attn_rows_gqa


def test_pair_count_matches_explicit_masks(oracle_mod):
    for n in (1, 2, 9, 130):
        for causal, window in [(False, -1), (True, -1), (True, 0), (True, 3), (True, 128), (True, 500),
                               (False, 0), (False, 3), (False, 128), (False, 500)]:
            cnt = sum(int(oracle_mod.mask_row(n, i, causal, window).sum()) for i in range(n))
            assert cnt == synth.attended_pairs_per_head(n, causal, window)


# ---------------------------------------------------------------- grouped-query attention

def _brute_gqa(q, k, v, scale, causal, window):
    """Textbook GQA: query head h uses key/value head h // (H // Hkv)."""
    H, Hkv = q.shape[1], k.shape[1]
    idx = torch.arange(H) // (H // Hkv)
    return _brute(q, k[:, idx], v[:, idx], scale, causal, window)


@pytest.mark.parametrize("H,Hkv", [(4, 4), (4, 2), (6, 3), (4, 1)])
@pytest.mark.parametrize("causal,window", [(False, -1), (True, -1), (True, 5)])
def test_gqa_oracle_matches_brute_force(oracle_mod, H, Hkv, causal, window):
    n, d = 37, 16
    q, _, _ = synth.make_qkv(2, H, n, d, seed=60)
    _, k, v = synth.make_qkv(2, Hkv, n, d, seed=61)
    rows = np.arange(2 * H * n)
    o, lse = oracle_mod.attn_rows_gqa(q, k, v, 0.3, causal, window, rows)
    o_ref, lse_ref, _ = _brute_gqa(q, k, v, 0.3, causal, window)
    np.testing.assert_allclose(o, o_ref.reshape(-1, d), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref.reshape(-1), rtol=0, atol=1e-12)


def test_gqa_equals_multi_head_with_repeated_kv(oracle_mod):
    """MQA/GQA is multi-head attention whose K/V heads are repeated within each
    group of H/Hkv consecutive query heads (not interleaved across groups)."""
    B, H, Hkv, n, d = 2, 8, 2, 50, 32
    q, _, _ = synth.make_qkv(B, H, n, d, seed=62)
    _, k, v = synth.make_qkv(B, Hkv, n, d, seed=63)
    rows = np.arange(B * H * n)
    o, lse = oracle_mod.attn_rows_gqa(q, k, v, 0.2, True, -1, rows)
    kr = k.repeat_interleave(H // Hkv, dim=1).contiguous()
    vr = v.repeat_interleave(H // Hkv, dim=1).contiguous()
    o_m, lse_m, _ = oracle_mod.attn_rows(q, kr, vr, 0.2, True, -1, rows)
    assert np.array_equal(o, o_m) and np.array_equal(lse, lse_m)
    # the other plausible mapping (h % Hkv) gives a different answer
    kw = k.repeat(1, H // Hkv, 1, 1).contiguous()
    vw = v.repeat(1, H // Hkv, 1, 1).contiguous()
    o_w, _, _ = oracle_mod.attn_rows(q, kw, vw, 0.2, True, -1, rows)
    assert not np.allclose(o, o_w)


def test_gqa_rejects_non_dividing_heads(oracle_mod):
    q, _, _ = synth.make_qkv(1, 4, 8, 16)
    _, k, v = synth.make_qkv(1, 3, 8, 16)
    with pytest.raises(ValueError):
        oracle_mod.attn_rows_gqa(q, k, v, 0.25, False, -1, [0])


# ---------------------------------------------------------------- symmetric window

def test_symmetric_window_matches_page_range(oracle_mod):
    """Local attention: token i attends to max(0, i-w) ... min(n-1, i+w)."""
    n = 50
    for w in (0, 1, 7, 49, 60):
        for i in range(n):
            m = oracle_mod.mask_row(n, i, False, w)
            assert np.flatnonzero(m).tolist() == list(range(max(0, i - w), min(n - 1, i + w) + 1))


def test_symmetric_window_at_least_n_minus_1_equals_no_mask(oracle_mod):
    q, k, v = synth.make_qkv(1, 2, 40, 16, seed=80, q_std=3.0)
    a = oracle_mod.attn_fwd(q, k, v, 0.25, False, -1)
    for w in (39, 100):
        b = oracle_mod.attn_fwd(q, k, v, 0.25, False, w)
        np.testing.assert_array_equal(a[0], b[0])
        np.testing.assert_array_equal(a[1], b[1])


def test_symmetric_window_zero_and_zero_queries(oracle_mod):
    q, k, v = synth.make_qkv(1, 2, 30, 16, seed=81, q_std=4.0)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.25, False, 0)
    np.testing.assert_array_equal(o, _f64(v))
    z = torch.zeros_like(q)
    o, lse = oracle_mod.attn_fwd(z, k, v, 0.25, False, 4)
    V = _f64(v)
    for i in range(30):
        lo, hi = max(0, i - 4), min(29, i + 4)
        np.testing.assert_allclose(o[:, :, i], V[:, :, lo:hi + 1].mean(axis=2), rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, :, i], np.log(hi - lo + 1), rtol=0, atol=1e-12)


def test_symmetric_pair_count_closed_form():
    """sum_i (min(n-1, i+w) - max(0, i-w) + 1) = n(2w+1) - w(w+1) for w < n."""
    for n in (1, 2, 5, 130, 1000):
        for w in (0, 1, 3, n - 1, n, 5 * n):
            direct = sum(min(n - 1, i + w) - max(0, i - w) + 1 for i in range(n))
            assert synth.attended_pairs_per_head(n, False, w) == direct


# ---------------------------------------------------------------- block-local (block-sparse) mask

def _block_keep(n, block, causal):
    """The page's block-sparse pattern written with block indices: key j in
    the query's block or the block before it (and j <= i if causal)."""
    i = np.arange(n)[:, None] // block
    j = np.arange(n)[None, :] // block
    keep = (j == i) | (j == i - 1)
    if causal:
        keep &= np.arange(n)[None, :] <= np.arange(n)[:, None]
    return keep


@pytest.mark.parametrize("n,block", [(1, 4), (10, 1), (37, 4), (64, 16), (70, 128)])
@pytest.mark.parametrize("causal", [False, True])
def test_block_mask_matches_block_indices_and_brute_force(oracle_mod, n, block, causal):
    keep = _block_keep(n, block, causal)
    for i in range(n):
        np.testing.assert_array_equal(oracle_mod.mask_row(n, i, causal, -1, block), keep[i])
    q, k, v = synth.make_qkv(1, 2, n, 16, seed=n + block, q_std=2.0)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.25, causal, -1, block)
    Q, K, V = _f64(q), _f64(k), _f64(v)
    S = np.where(keep, (Q @ np.swapaxes(K, -1, -2)) * 0.25, -np.inf)
    M = S.max(axis=-1, keepdims=True)
    E = np.exp(S - M)
    np.testing.assert_allclose(o, (E / E.sum(-1, keepdims=True)) @ V, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, (M + np.log(E.sum(-1, keepdims=True)))[..., 0], rtol=0, atol=1e-12)
    assert int(keep.sum()) == synth.attended_pairs_block(n, block, causal)


def test_block_mask_special_cases(oracle_mod):
    """b >= n: one block, so the mask is no mask (or causal); b = 1: keys i-1
    and i, the causal window 1."""
    q, k, v = synth.make_qkv(1, 2, 40, 16, seed=91, q_std=3.0)
    for causal in (False, True):
        a = oracle_mod.attn_fwd(q, k, v, 0.25, causal, -1, 64)
        b = oracle_mod.attn_fwd(q, k, v, 0.25, causal, -1)
        np.testing.assert_array_equal(a[0], b[0])
        c = oracle_mod.attn_fwd(q, k, v, 0.25, causal, -1, 1)
        d = oracle_mod.attn_fwd(q, k, v, 0.25, True, 1)
        np.testing.assert_array_equal(c[0], d[0])
    with pytest.raises(ValueError):
        oracle_mod.attn_fwd(q, k, v, 0.25, True, 3, 8)  # a block mask takes no window
