"""Seeded synthetic inputs and workload descriptions.

This module is shared by the tests, the benchmark and the smoke check. It
draws random numbers and names workloads; it does none of the attention
arithmetic, so both the CUDA path and the CPU oracle can take their inputs
from here without sharing any computation.

Recipe (stated once, used everywhere): a CPU ``torch.Generator`` seeded with
``seed`` draws Q, then K, then V, each as fp32 standard normals of shape
[B, H, n, d]; Q is multiplied by ``q_std``; each tensor is then rounded to
bf16 (round to nearest even). Layout is contiguous [B, H, n, d], the
(batch, heads, tokens, head size) order of the naive-versus-fused timing
snippet on "Efficient Transformers: Sparse Attention, Linear Attention and
FlashAttention" (section "Family 3").
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Tuple

import torch


@dataclasses.dataclass(frozen=True)
class Workload:
    """One attention problem: shapes, mask and input distribution."""

    name: str
    B: int
    H: int
    n: int
    d: int
    causal: bool
    window: int = -1  # < 0: no window; >= 0: keys max(0, i - window) .. i
    q_std: float = 1.0
    seed: int = 0
    Hkv: int = 0      # key/value heads (grouped-query attention); 0 means H
    block: int = 0    # > 0: block-local mask (own block and the previous one)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def kv_heads(self) -> int:
        return self.Hkv if self.Hkv > 0 else self.H

    @property
    def mask(self) -> str:
        if self.block > 0:
            return f"block{self.block}" + ("-causal" if self.causal else "")
        if self.window >= 0:
            return f"window{self.window}" if self.causal else f"symwindow{self.window}"
        return "causal" if self.causal else "none"

    def describe(self) -> dict:
        return {
            "workload": self.name,
            "B": self.B,
            "H": self.H,
            "H_kv": self.kv_heads,
            "n": self.n,
            "d": self.d,
            "mask": self.mask,
            "scale": f"1/sqrt({self.d})",
            "q_std": self.q_std,
            "seed": self.seed,
        }


def attended_pairs_per_head(n: int, causal: bool, window: int) -> int:
    """Number of (query, key) pairs a mask allows in one head.

    none: n*n; causal: n(n+1)/2; causal window w: sum over i of
    min(i, w) + 1; symmetric window w (not causal): sum over i of
    min(n-1, i+w) - max(0, i-w) + 1 = n(2w+1) - w(w+1) for w < n. Used only
    to count the unmasked FLOPs (4*d per pair).
    """
    if window >= 0 and not causal:
        w = window
        if w >= n - 1:
            return n * n
        return n * (2 * w + 1) - w * (w + 1)
    if window >= 0:
        w = window
        if w >= n - 1:
            return n * (n + 1) // 2
        # rows 0..w attend i+1 keys, rows w+1..n-1 attend w+1 keys
        return (w + 1) * (w + 2) // 2 + (n - w - 1) * (w + 1)
    if causal:
        return n * (n + 1) // 2
    return n * n


def attended_pairs_block(n: int, block: int, causal: bool) -> int:
    """Pairs of the block-local mask in one head: query i attends to the keys
    of its own block floor(i/b) and of the previous block (j <= i as well
    when causal)."""
    total = 0
    for i in range(n):
        bi = i // block
        lo = max(0, (bi - 1) * block)
        hi = i if causal else min(n - 1, (bi + 1) * block - 1)
        total += hi - lo + 1
    return total


def workload_pairs_per_head(wl: "Workload") -> int:
    if wl.block > 0:
        return attended_pairs_block(wl.n, wl.block, wl.causal)
    return attended_pairs_per_head(wl.n, wl.causal, wl.window)


def unmasked_flops(wl: "Workload") -> int:
    """4*d FLOPs per attended pair (2*d for QK^T, 2*d for PV), times B*H."""
    return 4 * wl.d * workload_pairs_per_head(wl) * wl.B * wl.H


def make_qkv(B: int, H: int, n: int, d: int, seed: int = 0, q_std: float = 1.0, Hkv: int = 0
             ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Q as a contiguous bf16 CPU tensor [B, H, n, d] and K, V as [B, Hkv, n, d]
    (Hkv = H when 0), following the recipe above."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((B, H, n, d), generator=g, dtype=torch.float32)
    if q_std != 1.0:
        q.mul_(q_std)
    q = q.to(torch.bfloat16)
    kv_shape = (B, Hkv if Hkv > 0 else H, n, d)
    k = torch.randn(kv_shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    v = torch.randn(kv_shape, generator=g, dtype=torch.float32).to(torch.bfloat16)
    return q.contiguous(), k.contiguous(), v.contiguous()


def make_dout(B: int, H: int, n: int, d: int, seed: int = 0) -> torch.Tensor:
    """Upstream gradient dO for the backward pass: a contiguous bf16 CPU tensor
    [B, H, n, d] of N(0, 1) draws from a CPU generator seeded seed + 1 (fp32
    draws rounded to bf16)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed + 1)
    return torch.randn((B, H, n, d), generator=g, dtype=torch.float32).to(torch.bfloat16).contiguous()


def make_inputs(wl: Workload):
    return make_qkv(wl.B, wl.H, wl.n, wl.d, wl.seed, wl.q_std, wl.Hkv)


def sample_rows(B: int, H: int, n: int, per_head_random: int = 256, seed: int = 1,
                tile: int = 128, bound_every: int = 8, edge: int = 64) -> torch.Tensor:
    """Deterministic row subset (flat index bh*n + i) for large problems.

    Per head: the first and last ``edge`` rows, the two rows on both sides of
    every ``bound_every``-th tile boundary, and ``per_head_random`` uniform rows
    from a generator seeded with ``seed``. Sorted and unique.
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    rows = []
    fixed = list(range(min(edge, n))) + list(range(max(0, n - edge), n))
    for b0 in range(tile, n, tile * bound_every):
        fixed += [b0 - 1, b0]
    for bh in range(B * H):
        r = torch.randint(0, n, (per_head_random,), generator=g).tolist()
        base = bh * n
        rows.extend(base + i for i in fixed + r)
    return torch.unique(torch.tensor(rows, dtype=torch.int64))


# The workloads the pages' numbers and the target configurations describe.
SMALL_CAUSAL = Workload("B1-H2-n256-d64-causal", 1, 2, 256, 64, True)
FULL_N8192 = Workload("B8-H8-n8192-d64-none", 8, 8, 8192, 64, False)
WINDOW_N32768 = Workload("B1-H32-n32768-d128-window4096", 1, 32, 32768, 128, True, 4096)
CAUSAL_N131072 = Workload("B1-H8-n131072-d128-causal", 1, 8, 131072, 128, True)
# Grouped-query attention with the head layout the pages quote for LLaMA-2 70B
# (64 query heads sharing 8 key/value heads), causal, 8192 tokens.
GQA_N8192 = Workload("B1-H64-Hkv8-n8192-d128-causal", 1, 64, 8192, 128, True, Hkv=8)
# Symmetric local window (each token sees 256 neighbours on either side, the
# 512-token span of Longformer-style local attention), d = 64, 16k tokens.
SYM_N16384 = Workload("B2-H16-n16384-d64-symwindow256", 2, 16, 16384, 64, False, 256)
# Block-local mask (own block and the previous one) with 512-token blocks,
# d = 128, 16k tokens: the block-sparse pattern of the sub-quadratic page.
BLOCK_N16384 = Workload("B2-H16-n16384-d128-block512", 2, 16, 16384, 128, False, block=512)


@dataclasses.dataclass(frozen=True)
class DecodeWorkload:
    """One decode step against rolling key/value caches of W slots: T new
    query tokens per sequence, the last at position `pos` (every sequence at
    the same position), grouped-query heads, causal window `window` per token
    (-1: W - 1, the whole cache)."""

    name: str
    B: int
    H: int
    Hkv: int
    W: int
    d: int
    pos: int
    q_std: float = 1.0
    seed: int = 0
    T: int = 1
    window: int = -1

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d)

    @property
    def w(self) -> int:
        return self.W - 1 if self.window < 0 else self.window

    @property
    def keys(self) -> int:
        """Cached positions the step reads (every cached slot)."""
        return min(self.pos + 1, self.W)

    @property
    def attended(self) -> int:
        """Attended (token, position) pairs per query head: token u at
        position pos - T + 1 + u sees min(t_u, w) + 1 positions."""
        return sum(min(self.pos - self.T + 1 + u, self.w) + 1 for u in range(self.T))

    def describe(self) -> dict:
        return {"workload": self.name, "B": self.B, "H": self.H, "H_kv": self.Hkv, "cache_slots": self.W,
                "d": self.d, "tokens_per_sequence": self.T, "window": self.w, "position": self.pos,
                "cached_positions_read": self.keys, "scale": f"1/sqrt({self.d})", "q_std": self.q_std,
                "seed": self.seed}


def make_decode(B: int, H: int, Hkv: int, W: int, d: int, seed: int = 0, q_std: float = 1.0
                ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """q [B, H, d] and rolling caches k, v [B, Hkv, W, d], bf16, drawn like
    make_qkv (q, then k, then v from one generator seeded `seed`)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((B, H, d), generator=g, dtype=torch.float32)
    if q_std != 1.0:
        q.mul_(q_std)
    k = torch.randn((B, Hkv, W, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, W, d), generator=g, dtype=torch.float32)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def make_decode_multi(B: int, H: int, Hkv: int, T: int, W: int, d: int, seed: int = 0, q_std: float = 1.0
                      ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """q [B, H, T, d] and rolling caches k, v [B, Hkv, W, d], bf16, drawn like
    make_decode (q, then k, then v from one generator seeded `seed`)."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    q = torch.randn((B, H, T, d), generator=g, dtype=torch.float32)
    if q_std != 1.0:
        q.mul_(q_std)
    k = torch.randn((B, Hkv, W, d), generator=g, dtype=torch.float32)
    v = torch.randn((B, Hkv, W, d), generator=g, dtype=torch.float32)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def ring_from_sequence(seq: torch.Tensor, W: int) -> torch.Tensor:
    """The rolling cache after writing positions 0 .. T-1 of `seq` [B, Hkv,
    T, d] in order, position p into slot p mod W (unwritten slots zero)."""
    B, Hkv, T, d = seq.shape
    ring = torch.zeros((B, Hkv, W, d), dtype=seq.dtype)
    for p in range(T):
        ring[:, :, p % W] = seq[:, :, p]
    return ring


# Decode against a 4096-slot rolling cache at position 32767 (n = 32,768, the
# worked example's cache size), Mistral-7B-like heads (32 query heads sharing
# 8 key/value heads, d = 128), 64 sequences per step.
DECODE_W4096 = DecodeWorkload("decode-B64-H32-Hkv8-W4096-d128-pos32767", 64, 32, 8, 4096, 128, 32767)
# The same caches with four new tokens per sequence (a speculative step): the
# 4096-slot cache serves a window of 4092 earlier positions to each of them.
DECODE_T4_W4096 = DecodeWorkload("decode-B64-H32-Hkv8-T4-W4096-w4092-d128-pos32767", 64, 32, 8, 4096, 128,
                                 32767, T=4, window=4092)


def decode_by_name(name: str) -> Optional[DecodeWorkload]:
    for wl in (DECODE_W4096, DECODE_T4_W4096):
        if wl.name == name:
            return wl
    return None


def sweep() -> List[Workload]:
    """n in {1024, 4096, 16384, 65536} x d in {64, 128} x five masks;
    B*H*n = 262144 tokens (B=1); Q ~ N(0, 4^2) for large logits."""
    out = []
    for n in (1024, 4096, 16384, 65536):
        for d in (64, 128):
            H = 262144 // n
            for causal, window in ((False, -1), (True, -1), (True, 256), (True, 1024), (True, 4096)):
                m = f"window{window}" if window >= 0 else ("causal" if causal else "none")
                out.append(Workload(f"sweep-n{n}-d{d}-{m}", 1, H, n, d, causal, window, q_std=4.0))
    return out


def by_name(name: str) -> Optional[Workload]:
    for wl in [SMALL_CAUSAL, FULL_N8192, WINDOW_N32768, CAUSAL_N131072, GQA_N8192, SYM_N16384,
               BLOCK_N16384] + sweep():
        if wl.name == name:
            return wl
    return None
