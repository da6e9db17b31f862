"""fp64 CPU oracle for exact softmax attention, forward and backward (test
infrastructure only).

Only the tests, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package. The CUDA product path never does.

``attn_oracle.c`` holds the arithmetic; this module compiles it with gcc
(``build()``) and calls it through ctypes. Inputs are bf16 CPU tensors
[B, H, n, d]; outputs are fp64 numpy arrays.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Optional, Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

KERNEL_SOFTMAX = 0
KERNEL_IDENTITY = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        build()
        lib = ctypes.CDLL(_LIB)
        i64, dbl, vp, ip = ctypes.c_int64, ctypes.c_double, ctypes.c_void_p, ctypes.c_int
        lib.oracle_attn_rows_f64.argtypes = [vp, vp, vp, i64, i64, i64, i64, dbl, ip, i64, i64, ip,
                                             vp, i64, vp, vp, vp]
        lib.oracle_attn_rows_f64.restype = ip
        lib.oracle_attn_rows_gqa_f64.argtypes = [vp, vp, vp, i64, i64, i64, i64, i64, dbl, ip, i64,
                                                 i64, ip, vp, i64, vp, vp, vp]
        lib.oracle_attn_rows_gqa_f64.restype = ip
        lib.oracle_attn_fwd_f64.argtypes = [vp, vp, vp, i64, i64, i64, i64, dbl, ip, i64, i64, vp, vp]
        lib.oracle_attn_fwd_f64.restype = ip
        lib.oracle_matmul_f64.argtypes = [i64, i64, i64, vp, ip, vp, ip, vp]
        lib.oracle_matmul_f64.restype = ip
        lib.oracle_mask_row.argtypes = [i64, i64, ip, i64, i64, vp]
        lib.oracle_mask_row.restype = ip
        lib.oracle_attn_bwd_rows_f64.argtypes = [vp, vp, vp, vp, ip, i64, i64, i64, i64, dbl, ip,
                                                 i64, i64, vp, i64, vp, i64, vp, vp, vp]
        lib.oracle_attn_bwd_rows_f64.restype = ip
        lib.oracle_attn_bwd_rows_gqa_f64.argtypes = [vp, vp, vp, vp, ip, i64, i64, i64, i64, i64, dbl, ip,
                                                     i64, i64, vp, i64, vp, i64, vp, vp, vp]
        lib.oracle_attn_bwd_rows_gqa_f64.restype = ip
        lib.oracle_attn_decode_f64.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, dbl, vp, vp]
        lib.oracle_attn_decode_f64.restype = ip
        lib.oracle_attn_decode_multi_f64.argtypes = [vp, vp, vp, vp, i64, i64, i64, i64, i64, i64, i64, dbl,
                                                     vp, vp]
        lib.oracle_attn_decode_multi_f64.restype = ip
        lib.oracle_num_threads.argtypes = []
        lib.oracle_num_threads.restype = ip
        _lib = lib
    return _lib


def _bits(t) -> np.ndarray:
    """bf16 torch tensor -> contiguous uint16 numpy view of its bit patterns."""
    import torch
    if t.dtype != torch.bfloat16:
        raise TypeError("oracle inputs must be bf16")
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def attn_rows(q, k, v, scale: float, causal: bool, window: int, rows,
              kernel: int = KERNEL_SOFTMAX, want_weights: bool = False, block: int = 0
              ) -> Tuple[np.ndarray, np.ndarray, Optional[np.ndarray]]:
    """O (nrows x d), LSE (nrows) and optionally weights (nrows x n) for flat
    rows. block > 0 selects the block-local mask (own block and the previous
    one; window must then be < 0)."""
    lib = _load()
    if not (q.shape == k.shape == v.shape) or len(q.shape) != 4:
        raise ValueError("q, k and v must all be [B, H, n, d] (see attn_rows_gqa for fewer K/V heads)")
    B, H, n, d = q.shape
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.empty((rows.size, d), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64)
    w = np.empty((rows.size, n), dtype=np.float64) if want_weights else None
    rc = lib.oracle_attn_rows_f64(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, B, H, n, d,
                                  float(scale), int(bool(causal)), int(window), int(block), int(kernel),
                                  rows.ctypes.data, rows.size, o.ctypes.data, lse.ctypes.data,
                                  w.ctypes.data if w is not None else None)
    if rc != 0:
        raise ValueError(f"oracle_attn_rows_f64 rejected its arguments (rc={rc})")
    return o, lse, w


def attn_rows_gqa(q, k, v, scale: float, causal: bool, window: int, rows,
                  kernel: int = KERNEL_SOFTMAX, block: int = 0) -> Tuple[np.ndarray, np.ndarray]:
    """Grouped-query form: q [B, H, n, d], k and v [B, Hkv, n, d], Hkv | H.
    O (nrows x d) and LSE (nrows) for flat query rows (b*H + h)*n + i."""
    lib = _load()
    B, H, n, d = q.shape
    Hkv = k.shape[1]
    if k.shape != v.shape or k.shape[0] != B or k.shape[2:] != q.shape[2:]:
        raise ValueError("k and v must be [B, Hkv, n, d]")
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
    o = np.empty((rows.size, d), dtype=np.float64)
    lse = np.empty(rows.size, dtype=np.float64)
    rc = lib.oracle_attn_rows_gqa_f64(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, B, H, Hkv, n, d,
                                      float(scale), int(bool(causal)), int(window), int(block), int(kernel),
                                      rows.ctypes.data, rows.size, o.ctypes.data, lse.ctypes.data, None)
    if rc != 0:
        raise ValueError(f"oracle_attn_rows_gqa_f64 rejected its arguments (rc={rc})")
    return o, lse


def attn_fwd(q, k, v, scale: float, causal: bool, window: int = -1, block: int = 0
             ) -> Tuple[np.ndarray, np.ndarray]:
    """Full O [B,H,n,d] and LSE [B,H,n] in fp64."""
    lib = _load()
    if not (q.shape == k.shape == v.shape) or len(q.shape) != 4:
        raise ValueError("q, k and v must all be [B, H, n, d]")
    B, H, n, d = q.shape
    qb, kb, vb = _bits(q), _bits(k), _bits(v)
    o = np.empty((B, H, n, d), dtype=np.float64)
    lse = np.empty((B, H, n), dtype=np.float64)
    rc = lib.oracle_attn_fwd_f64(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, B, H, n, d,
                                 float(scale), int(bool(causal)), int(window), int(block),
                                 o.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_attn_fwd_f64 rejected its arguments (rc={rc})")
    return o, lse


IN_BF16 = 0
IN_F64 = 1


def _bwd_input(t):
    """(array, type) for the backward oracle: bf16 torch tensors as their bit
    patterns, anything else as contiguous fp64."""
    import torch
    if isinstance(t, torch.Tensor) and t.dtype == torch.bfloat16:
        return _bits(t), IN_BF16
    if isinstance(t, torch.Tensor):
        t = t.detach().cpu().numpy()
    return np.ascontiguousarray(np.asarray(t, dtype=np.float64)), IN_F64


def attn_bwd_rows(q, k, v, dout, scale: float, causal: bool, window: int, qrows=(), krows=(),
                  block: int = 0) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Backward pass for selected rows. q, k, v, dout: [B, H, n, d], all bf16
    torch tensors or all fp64 arrays. Returns dQ for the flat query rows
    ``qrows`` (len x d) and dK, dV for the flat key rows ``krows`` (len x d
    each), flat row = (b*H + h)*n + i, all fp64."""
    lib = _load()
    shapes = {tuple(x.shape) for x in (q, k, v, dout)}
    if len(shapes) != 1 or len(q.shape) != 4:
        raise ValueError("q, k, v and dout must all be [B, H, n, d]")
    B, H, n, d = q.shape
    ins = [_bwd_input(x) for x in (q, k, v, dout)]
    if len({t for _, t in ins}) != 1:
        raise TypeError("q, k, v and dout must be all bf16 or all floating point")
    typ = ins[0][1]
    qr = np.ascontiguousarray(np.asarray(qrows, dtype=np.int64).reshape(-1))
    kr = np.ascontiguousarray(np.asarray(krows, dtype=np.int64).reshape(-1))
    dq = np.empty((qr.size, d), dtype=np.float64)
    dk = np.empty((kr.size, d), dtype=np.float64)
    dv = np.empty((kr.size, d), dtype=np.float64)
    rc = lib.oracle_attn_bwd_rows_f64(ins[0][0].ctypes.data, ins[1][0].ctypes.data,
                                      ins[2][0].ctypes.data, ins[3][0].ctypes.data, typ,
                                      B, H, n, d, float(scale), int(bool(causal)), int(window), int(block),
                                      qr.ctypes.data, qr.size, kr.ctypes.data, kr.size,
                                      dq.ctypes.data, dk.ctypes.data, dv.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_attn_bwd_rows_f64 rejected its arguments (rc={rc})")
    return dq, dk, dv


def attn_bwd_rows_gqa(q, k, v, dout, scale: float, causal: bool, window: int, qrows=(), krows=(),
                      block: int = 0) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Grouped-query backward for selected rows: q, dout [B, H, n, d], k, v
    [B, Hkv, n, d] (all bf16 tensors or all fp64). dQ for flat query rows
    (b*H + h)*n + i, dK and dV for flat key rows (b*Hkv + g)*n + j."""
    lib = _load()
    if q.shape != dout.shape or k.shape != v.shape or len(q.shape) != 4 or len(k.shape) != 4:
        raise ValueError("q, dout must be [B, H, n, d] and k, v [B, Hkv, n, d]")
    B, H, n, d = q.shape
    Hkv = k.shape[1]
    if k.shape[0] != B or k.shape[2:] != q.shape[2:]:
        raise ValueError("k and v must be [B, Hkv, n, d]")
    ins = [_bwd_input(x) for x in (q, k, v, dout)]
    if len({t for _, t in ins}) != 1:
        raise TypeError("q, k, v and dout must be all bf16 or all floating point")
    qr = np.ascontiguousarray(np.asarray(qrows, dtype=np.int64).reshape(-1))
    kr = np.ascontiguousarray(np.asarray(krows, dtype=np.int64).reshape(-1))
    dq = np.empty((qr.size, d), dtype=np.float64)
    dk = np.empty((kr.size, d), dtype=np.float64)
    dv = np.empty((kr.size, d), dtype=np.float64)
    rc = lib.oracle_attn_bwd_rows_gqa_f64(ins[0][0].ctypes.data, ins[1][0].ctypes.data,
                                          ins[2][0].ctypes.data, ins[3][0].ctypes.data, ins[0][1],
                                          B, H, Hkv, n, d, float(scale), int(bool(causal)), int(window),
                                          int(block), qr.ctypes.data, qr.size, kr.ctypes.data, kr.size,
                                          dq.ctypes.data, dk.ctypes.data, dv.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_attn_bwd_rows_gqa_f64 rejected its arguments (rc={rc})")
    return dq, dk, dv


def attn_bwd(q, k, v, dout, scale: float, causal: bool, window: int = -1, block: int = 0
             ) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Full dQ, dK, dV [B, H, n, d] in fp64."""
    B, H, n, d = q.shape
    rows = np.arange(B * H * n, dtype=np.int64)
    dq, dk, dv = attn_bwd_rows(q, k, v, dout, scale, causal, window, rows, rows, block)
    return dq.reshape(B, H, n, d), dk.reshape(B, H, n, d), dv.reshape(B, H, n, d)


def attn_decode(q, k_cache, v_cache, pos, scale: float) -> Tuple[np.ndarray, np.ndarray]:
    """Decode against rolling caches: q bf16 [B, H, d], k_cache / v_cache bf16
    [B, Hkv, W, d] (position p at slot p mod W), pos [B] (>= 0). Returns O
    [B, H, d] and LSE [B, H] in fp64."""
    lib = _load()
    if len(q.shape) != 3 or len(k_cache.shape) != 4 or k_cache.shape != v_cache.shape:
        raise ValueError("q must be [B, H, d] and the caches [B, Hkv, W, d]")
    B, H, d = q.shape
    Bk, Hkv, W, dk = k_cache.shape
    if Bk != B or dk != d:
        raise ValueError("cache shape does not match q")
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    p = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(-1))
    if p.size != B:
        raise ValueError("pos must have B entries")
    o = np.empty((B, H, d), dtype=np.float64)
    lse = np.empty((B, H), dtype=np.float64)
    rc = lib.oracle_attn_decode_f64(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, p.ctypes.data,
                                    B, H, Hkv, W, d, float(scale), o.ctypes.data, lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_attn_decode_f64 rejected its arguments (rc={rc})")
    return o, lse


def attn_decode_multi(q, k_cache, v_cache, pos, scale: float, window: int) -> Tuple[np.ndarray, np.ndarray]:
    """Decode of T new tokens per sequence against rolling caches: q bf16
    [B, H, T, d] (token u at position pos[b] - T + 1 + u), k_cache / v_cache
    bf16 [B, Hkv, W, d] (position p at slot p mod W), pos [B] (>= T - 1, the
    last new token's position), causal window `window` (window + T <= W).
    Returns O [B, H, T, d] and LSE [B, H, T] in fp64."""
    lib = _load()
    if len(q.shape) != 4 or len(k_cache.shape) != 4 or k_cache.shape != v_cache.shape:
        raise ValueError("q must be [B, H, T, d] and the caches [B, Hkv, W, d]")
    B, H, T, d = q.shape
    Bk, Hkv, W, dk = k_cache.shape
    if Bk != B or dk != d:
        raise ValueError("cache shape does not match q")
    qb, kb, vb = _bits(q), _bits(k_cache), _bits(v_cache)
    p = np.ascontiguousarray(np.asarray(pos, dtype=np.int64).reshape(-1))
    if p.size != B:
        raise ValueError("pos must have B entries")
    o = np.empty((B, H, T, d), dtype=np.float64)
    lse = np.empty((B, H, T), dtype=np.float64)
    rc = lib.oracle_attn_decode_multi_f64(qb.ctypes.data, kb.ctypes.data, vb.ctypes.data, p.ctypes.data,
                                          B, H, Hkv, T, W, d, int(window), float(scale), o.ctypes.data,
                                          lse.ctypes.data)
    if rc != 0:
        raise ValueError(f"oracle_attn_decode_multi_f64 rejected its arguments (rc={rc})")
    return o, lse


def matmul(a: np.ndarray, b: np.ndarray, ta: bool = False, tb: bool = False) -> np.ndarray:
    """op(a) @ op(b) in fp64 through the oracle's own contraction routine."""
    lib = _load()
    a = np.ascontiguousarray(a, dtype=np.float64)
    b = np.ascontiguousarray(b, dtype=np.float64)
    m, k = (a.shape[1], a.shape[0]) if ta else a.shape
    k2, n = (b.shape[1], b.shape[0]) if tb else b.shape
    if k != k2:
        raise ValueError("inner dimensions differ")
    c = np.empty((m, n), dtype=np.float64)
    rc = lib.oracle_matmul_f64(m, n, k, a.ctypes.data, int(ta), b.ctypes.data, int(tb),
                               c.ctypes.data)
    if rc != 0:
        raise ValueError("oracle_matmul_f64 rejected its arguments")
    return c


def mask_row(n: int, i: int, causal: bool, window: int, block: int = 0) -> np.ndarray:
    lib = _load()
    out = np.empty(n, dtype=np.uint8)
    if lib.oracle_mask_row(n, i, int(bool(causal)), int(window), int(block), out.ctypes.data) != 0:
        raise ValueError("bad mask arguments")
    return out.astype(bool)


def num_threads() -> int:
    return _load().oracle_num_threads()
