"""Pins of the fp64 backward-pass oracle against facts that do not come from it.

CPU only. The gradients are fixed by the forward definition and calculus;
each test names what fixes its expected value: reverse-mode differentiation
of the textbook forward by a library (torch.autograd in fp64), central finite
differences of the textbook forward, invariants of the softmax, or closed
forms of special masks and inputs.
"""
import numpy as np
import pytest
import torch

from exact_softmax_attention_04_b200 import synth

MASKS = [(False, -1), (True, -1), (True, 0), (True, 1), (True, 3), (True, 64),
         (False, 0), (False, 2), (False, 64)]


def _textbook_forward(q, k, v, scale, causal, window):
    """O = softmax(masked(scale Q K^T)) V over the full score matrix (torch ops,
    differentiable): the triu(1) causal mask, ones on [max(0, i-w), i] for a
    window, masked_fill with -inf, row softmax."""
    n = q.shape[-2]
    s = (q @ k.transpose(-1, -2)) * scale
    i = torch.arange(n).view(n, 1)
    j = torch.arange(n).view(1, n)
    drop = torch.zeros(n, n, dtype=torch.bool)
    if causal:
        drop |= j > i
    if window >= 0:
        drop |= j < i - window
        if not causal:
            drop |= j > i + window
    return s.masked_fill(drop, float("-inf")).softmax(-1) @ v


def _rand(shape, seed, std=1.0):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(shape, generator=g, dtype=torch.float64) * std


@pytest.mark.parametrize("n", [1, 7, 33, 64])
@pytest.mark.parametrize("causal,window", MASKS)
def test_bwd_matches_autograd_of_textbook_forward(oracle_mod, n, causal, window):
    shape = (2, 2, n, 8)
    q, k, v, do = (_rand(shape, s, std) for s, std in ((1, 2.0), (2, 1.0), (3, 1.0), (4, 1.0)))
    scale = 0.35
    qa, ka, va = (x.clone().requires_grad_(True) for x in (q, k, v))
    o = _textbook_forward(qa, ka, va, scale, causal, window)
    (o * do).sum().backward()
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, do, scale, causal, window)
    for got, ref in ((dq, qa.grad), (dk, ka.grad), (dv, va.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)


def test_bwd_matches_central_finite_differences(oracle_mod):
    """dL/dx for L = sum(O * dO), by (L(x + h e) - L(x - h e)) / 2h on the
    textbook forward evaluated in fp64 numpy, for random coordinates of Q,
    K and V under each mask."""
    rng = np.random.default_rng(7)
    n, d, scale = 9, 4, 0.6
    for causal, window in ((False, -1), (True, -1), (True, 2), (False, 2)):
        q, k, v, do = (_rand((1, 1, n, d), s) for s in (11, 12, 13, 14))
        dq, dk, dv = oracle_mod.attn_bwd(q, k, v, do, scale, causal, window)

        def loss(qq, kk, vv):
            with torch.no_grad():
                return float((_textbook_forward(qq, kk, vv, scale, causal, window) * do).sum())

        h = 1e-5
        for which, grad in ((0, dq), (1, dk), (2, dv)):
            for _ in range(8):
                i, c = int(rng.integers(n)), int(rng.integers(d))
                xs = [q.clone(), k.clone(), v.clone()]
                xs[which][0, 0, i, c] += h
                up = loss(*xs)
                xs[which][0, 0, i, c] -= 2 * h
                dn = loss(*xs)
                fd = (up - dn) / (2 * h)
                assert abs(fd - grad[0, 0, i, c]) <= 1e-8 * max(1.0, abs(fd)), (which, i, c, fd)


@pytest.mark.parametrize("causal,window", MASKS)
def test_key_gradients_sum_to_zero_and_value_gradients_to_sum_of_dout(oracle_mod, causal, window):
    """Each row of the softmax sums to 1 over A(i), so adding one vector to
    every key changes no output (sum_j dK_j = 0) and sum_j dV_j = sum_i dO_i."""
    q, k, v = synth.make_qkv(2, 3, 50, 16, seed=40, q_std=3.0)
    do = _rand(q.shape, 41).to(torch.bfloat16)
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, do, 0.25, causal, window)
    assert np.abs(dk.sum(axis=2)).max() <= 1e-12 * max(1.0, np.abs(dk).max()) * 50
    np.testing.assert_allclose(dv.sum(axis=2), do.double().numpy().sum(axis=2), rtol=0, atol=1e-12)


def test_window_zero_gradients(oracle_mod):
    """w = 0: each query attends to itself only, P is the identity, so O = V,
    dV = dO and the scores receive no gradient (dQ = dK = 0)."""
    q, k, v = synth.make_qkv(1, 2, 40, 16, seed=42, q_std=4.0)
    do = _rand(q.shape, 43).to(torch.bfloat16)
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, do, 0.25, True, 0)
    assert np.abs(dq).max() == 0.0 and np.abs(dk).max() == 0.0
    np.testing.assert_array_equal(dv, do.double().numpy())


@pytest.mark.parametrize("causal,window", [(False, -1), (True, -1), (True, 5)])
def test_zero_queries_value_gradient_closed_form(oracle_mod, causal, window):
    """Q = 0: every allowed weight of row i is 1/|A(i)|, so
    dV_j = sum over queries i that attend to j of dO_i / |A(i)|."""
    n, d = 30, 8
    _, k, v = synth.make_qkv(1, 1, n, d, seed=44)
    q = torch.zeros_like(k)
    do = _rand(q.shape, 45).to(torch.bfloat16)
    _, _, dv = oracle_mod.attn_bwd(q, k, v, do, 0.3, causal, window)
    D = do.double().numpy()[0, 0]
    ref = np.zeros((n, d))
    for i in range(n):
        lo = max(0, i - window) if window >= 0 else 0
        hi = i + 1 if causal else n
        ref[lo:hi] += D[i] / (hi - lo)
    np.testing.assert_allclose(dv[0, 0], ref, rtol=0, atol=1e-12)


def test_gradients_are_linear_in_dout(oracle_mod):
    q, k, v = synth.make_qkv(1, 2, 20, 8, seed=46)
    do1 = _rand(q.shape, 47)
    do2 = _rand(q.shape, 48)
    qd, kd, vd = (x.double() for x in (q, k, v))
    g1 = oracle_mod.attn_bwd(qd, kd, vd, do1, 0.3, True, -1)
    g2 = oracle_mod.attn_bwd(qd, kd, vd, do2, 0.3, True, -1)
    g12 = oracle_mod.attn_bwd(qd, kd, vd, 2.0 * do1 - do2, 0.3, True, -1)
    for a, b, c in zip(g1, g2, g12):
        np.testing.assert_allclose(c, 2.0 * a - b, rtol=0, atol=1e-12)


def test_bf16_inputs_read_as_their_exact_values(oracle_mod):
    """bf16 tensors and the same values widened to fp64 give identical
    gradients (bf16 -> fp64 is exact)."""
    q, k, v = synth.make_qkv(1, 2, 25, 16, seed=49)
    do = _rand(q.shape, 50).to(torch.bfloat16)
    a = oracle_mod.attn_bwd(q, k, v, do, 0.25, True, 4)
    b = oracle_mod.attn_bwd(q.double(), k.double(), v.double(), do.double(), 0.25, True, 4)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_bwd_row_subsets_equal_full_run(oracle_mod):
    q, k, v = synth.make_qkv(2, 2, 40, 8, seed=51)
    do = _rand(q.shape, 52).to(torch.bfloat16)
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, do, 0.3, True, 7)
    qrows = [0, 5, 39, 40, 77, 159]
    krows = [3, 41, 120, 159]
    sq, sk, sv = oracle_mod.attn_bwd_rows(q, k, v, do, 0.3, True, 7, qrows, krows)
    np.testing.assert_array_equal(sq, dq.reshape(-1, 8)[qrows])
    np.testing.assert_array_equal(sk, dk.reshape(-1, 8)[krows])
    np.testing.assert_array_equal(sv, dv.reshape(-1, 8)[krows])


def test_bwd_oracle_rejects_bad_arguments(oracle_mod):
    q, k, v = synth.make_qkv(1, 1, 8, 8, seed=53)
    do = q.clone()
    with pytest.raises(ValueError):
        oracle_mod.attn_bwd_rows(q, k, v, do, 0.3, True, -1, [8], [])   # row out of range
    with pytest.raises(ValueError):
        oracle_mod.attn_bwd_rows(q, k, v[:, :, :4], do, 0.3, True, -1, [0], [])
    with pytest.raises(TypeError):
        oracle_mod.attn_bwd_rows(q, k, v, do.double(), 0.3, True, -1, [0], [])


# ---------------------------------------------------------------- grouped-query attention

def _textbook_gqa_forward(q, k, v, scale, causal, window):
    """Grouped-query forward written with repeat_interleave: query head h
    reads key/value head h // (H // Hkv)."""
    H, Hkv = q.shape[1], k.shape[1]
    idx = torch.arange(H) // (H // Hkv)
    return _textbook_forward(q, k[:, idx], v[:, idx], scale, causal, window)


@pytest.mark.parametrize("H,Hkv", [(4, 2), (6, 3), (4, 1)])
@pytest.mark.parametrize("causal,window", [(False, -1), (True, -1), (True, 3), (False, 2)])
def test_gqa_bwd_matches_autograd(oracle_mod, H, Hkv, causal, window):
    """autograd through the repeat of K and V sums the group's gradients."""
    B, n, d = 2, 13, 8
    q, do = _rand((B, H, n, d), 61, 2.0), _rand((B, H, n, d), 62)
    k, v = _rand((B, Hkv, n, d), 63), _rand((B, Hkv, n, d), 64)
    qa, ka, va = (x.clone().requires_grad_(True) for x in (q, k, v))
    (_textbook_gqa_forward(qa, ka, va, 0.4, causal, window) * do).sum().backward()
    rows_q = np.arange(B * H * n)
    rows_k = np.arange(B * Hkv * n)
    dq, dk, dv = oracle_mod.attn_bwd_rows_gqa(q, k, v, do, 0.4, causal, window, rows_q, rows_k)
    np.testing.assert_allclose(dq, qa.grad.numpy().reshape(-1, d), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk, ka.grad.numpy().reshape(-1, d), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv, va.grad.numpy().reshape(-1, d), rtol=0, atol=1e-12)


def test_gqa_bwd_equals_group_sum_of_multi_head_gradients(oracle_mod):
    """With K, V repeated per query head, multi-head dK, dV summed over each
    group equal the grouped-query dK, dV; dQ is the same."""
    B, H, Hkv, n, d = 1, 6, 2, 20, 8
    q, k, v = synth.make_qkv(B, H, n, d, seed=65, Hkv=Hkv)
    do = _rand(q.shape, 66).to(torch.bfloat16)
    G = H // Hkv
    kr, vr = k.repeat_interleave(G, dim=1), v.repeat_interleave(G, dim=1)
    dq_m, dk_m, dv_m = oracle_mod.attn_bwd(q, kr, vr, do, 0.3, True, 5)
    rows_q, rows_k = np.arange(B * H * n), np.arange(B * Hkv * n)
    dq_g, dk_g, dv_g = oracle_mod.attn_bwd_rows_gqa(q, k, v, do, 0.3, True, 5, rows_q, rows_k)
    np.testing.assert_allclose(dq_g, dq_m.reshape(-1, d), rtol=0, atol=1e-12)
    np.testing.assert_allclose(dk_g.reshape(B, Hkv, n, d), dk_m.reshape(B, Hkv, G, n, d).sum(axis=2),
                               rtol=0, atol=1e-12)
    np.testing.assert_allclose(dv_g.reshape(B, Hkv, n, d), dv_m.reshape(B, Hkv, G, n, d).sum(axis=2),
                               rtol=0, atol=1e-12)


@pytest.mark.parametrize("block", [1, 3, 8])
@pytest.mark.parametrize("causal", [False, True])
def test_block_mask_bwd_matches_autograd(oracle_mod, block, causal):
    B, H, n, d = 1, 2, 21, 8
    q, k, v, do = (_rand((B, H, n, d), s) for s in (71, 72, 73, 74))
    i = torch.arange(n).view(n, 1)
    j = torch.arange(n).view(1, n)
    keep = ((j // block) == (i // block)) | ((j // block) == (i // block) - 1)
    if causal:
        keep &= j <= i
    qa, ka, va = (x.clone().requires_grad_(True) for x in (q, k, v))
    s = (qa @ ka.transpose(-1, -2)) * 0.5
    o = s.masked_fill(~keep, float("-inf")).softmax(-1) @ va
    (o * do).sum().backward()
    dq, dk, dv = oracle_mod.attn_bwd(q, k, v, do, 0.5, causal, -1, block)
    for got, ref in ((dq, qa.grad), (dk, ka.grad), (dv, va.grad)):
        np.testing.assert_allclose(got, ref.numpy(), rtol=0, atol=1e-12)
