"""Exact softmax attention forward for B200 (sm_100a): Python binding.

Argument marshalling only. Every step of the computation runs in the CUDA
kernels of ``libattn_b200.so`` (built in-tree by ``build_lib.py``); this module
checks tensor properties, allocates outputs with torch and passes raw
pointers and the current CUDA stream through the C ABI of ``include/attn.h``.
There is no CPU fallback: the first call that needs the library raises if
it is missing.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libattn_b200.so")

ATTN_OK = 0
ATTN_ERR_INVALID = 1
ATTN_ERR_UNSUPPORTED = 2
ATTN_ERR_CUDA = 3
ATTN_ERR_TIMEOUT = 4
ATTN_ERR_TOO_LARGE = 5

# Every symbol include/attn.h declares.
EXPORTS = ("attn_fwd", "attn_fwd_gqa", "attn_fwd_host", "attn_host_staging_release",
           "attn_sync_status", "attn_strerror", "attn_attended_pairs", "attn_fwd_host_noalloc",
           "attn_bwd", "attn_bwd_gqa", "attn_bwd_workspace_bytes", "attn_decode",
           "attn_decode_workspace_bytes", "attn_decode_multi", "attn_decode_multi_workspace_bytes",
           "attn_fwd_blocklocal", "attn_bwd_blocklocal", "attn_fwd_schedule", "attn_fwd_schedule_for")


class AttnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {strerror(code)} (status {code})")


def _load() -> ctypes.CDLL:
    return load_library(LIB_PATH)


def load_library(path: str) -> ctypes.CDLL:
    """ctypes handle of a libattn_b200 build at ``path`` with argument types set."""
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m exact_softmax_attention_04_b200.build_lib` "
            "(there is no CPU fallback)")
    lib = ctypes.CDLL(path)
    vp, i, f, i64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_int64
    fwd_args = [vp, vp, vp, vp, vp, i, i, i, i, f, i, i, vp]
    lib.attn_fwd.argtypes = fwd_args
    lib.attn_fwd.restype = i
    lib.attn_fwd_gqa.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
    lib.attn_fwd_gqa.restype = i
    lib.attn_fwd_blocklocal.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, i, i, vp]
    lib.attn_fwd_blocklocal.restype = i
    lib.attn_fwd_host.argtypes = fwd_args
    lib.attn_fwd_host.restype = i
    lib.attn_fwd_host_noalloc.argtypes = fwd_args
    lib.attn_fwd_host_noalloc.restype = i
    lib.attn_host_staging_release.argtypes = []
    lib.attn_host_staging_release.restype = i
    lib.attn_sync_status.argtypes = [vp]
    lib.attn_sync_status.restype = i
    lib.attn_strerror.argtypes = [i]
    lib.attn_strerror.restype = ctypes.c_char_p
    lib.attn_attended_pairs.argtypes = [i64, i, i64]
    lib.attn_attended_pairs.restype = i64
    lib.attn_bwd.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                             i, i, i, i, f, i, i, vp]
    lib.attn_bwd.restype = i
    lib.attn_bwd_gqa.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                                 i, i, i, i, i, f, i, i, vp]
    lib.attn_bwd_gqa.restype = i
    lib.attn_bwd_blocklocal.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t,
                                        i, i, i, i, i, f, i, i, vp]
    lib.attn_bwd_blocklocal.restype = i
    lib.attn_bwd_workspace_bytes.argtypes = [i, i, i, i]
    lib.attn_bwd_workspace_bytes.restype = i64
    lib.attn_decode.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, i, i, i, i, i, f, vp]
    lib.attn_decode.restype = i
    lib.attn_decode_workspace_bytes.argtypes = [i, i, i, i, i]
    lib.attn_decode_workspace_bytes.restype = i64
    lib.attn_fwd_schedule.argtypes = [i]
    lib.attn_fwd_schedule.restype = i
    lib.attn_fwd_schedule_for.argtypes = [i, i, i, i]
    lib.attn_fwd_schedule_for.restype = i
    lib.attn_decode_multi.argtypes = [vp, vp, vp, vp, vp, vp, vp, ctypes.c_size_t, i, i, i, i, i, i, i, f, vp]
    lib.attn_decode_multi.restype = i
    lib.attn_decode_multi_workspace_bytes.argtypes = [i, i, i, i, i, i, i]
    lib.attn_decode_multi_workspace_bytes.restype = i64
    return lib


_lib_handle: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    """The loaded libattn_b200.so (loaded on first use)."""
    global _lib_handle
    if _lib_handle is None:
        _lib_handle = _load()
    return _lib_handle


def strerror(code: int) -> str:
    return lib().attn_strerror(int(code)).decode()


def attended_pairs(n: int, causal: bool, window: int = -1) -> int:
    r = lib().attn_attended_pairs(int(n), int(bool(causal)), int(window))
    if r < 0:
        raise ValueError("bad mask arguments")
    return int(r)


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> Optional[int]:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _check_qkv(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, device: bool,
               grouped: bool = False) -> None:
    for name, t in (("q", q), ("k", k), ("v", v)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bf16")
        if t.dim() != 4:
            raise ValueError(f"{name} must be [B, H, n, d]")
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
        if device and not t.is_cuda:
            raise ValueError(f"{name} must be a CUDA tensor")
        if not device and t.is_cuda:
            raise ValueError(f"{name} must be a host tensor")
    if grouped:
        if not (k.shape == v.shape and k.shape[0] == q.shape[0] and k.shape[2:] == q.shape[2:]
                and q.shape[1] % k.shape[1] == 0):
            raise ValueError("k and v must be [B, Hkv, n, d] with Hkv dividing H")
    elif not (q.shape == k.shape == v.shape):
        raise ValueError("q, k and v must have the same shape")
    if device and not (q.device == k.device == v.device):
        raise ValueError("q, k and v must be on one device")


def attn_fwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: Optional[float] = None,
             causal: bool = False, window: int = -1, out: Optional[torch.Tensor] = None,
             lse: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
             block: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """O = softmax(scale * Q K^T) V and its per-row log-sum-exp, on the GPU.

    q: bf16 CUDA tensor [B, H, n, d]; k, v: [B, H, n, d], or [B, Hkv, n, d]
    with Hkv dividing H for grouped-query / multi-query attention (query
    head h reads key/value head h // (H // Hkv)). Contiguous, d in {64, 128}.
    causal / window: see include/attn.h (window >= 0 without causal is the
    symmetric window i - window .. i + window). block > 0 selects the
    block-local mask instead of a window (own block and the previous one).
    Returns (o bf16 [B, H, n, d], lse fp32 [B, H, n]); enqueued on ``stream``
    (default: the current stream), asynchronous like any CUDA op.
    """
    grouped = k.dim() == 4 and q.dim() == 4 and k.shape[1] != q.shape[1]
    _check_qkv(q, k, v, device=True, grouped=grouped)
    B, H, n, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, n), dtype=torch.float32, device=q.device)
    if out.shape != q.shape or out.dtype != torch.bfloat16 or not out.is_contiguous():
        raise ValueError("out must be a contiguous bf16 tensor shaped like q")
    if lse.shape != (B, H, n) or lse.dtype != torch.float32 or not lse.is_contiguous():
        raise ValueError("lse must be a contiguous fp32 tensor [B, H, n]")
    if block > 0 and window >= 0:
        raise ValueError("a block-local mask takes no window")
    with torch.cuda.device(q.device):
        if block > 0:
            rc = lib().attn_fwd_blocklocal(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                           lse.data_ptr(), B, H, k.shape[1], n, d, float(scale),
                                           int(bool(causal)), int(block), _stream_handle(stream))
        elif grouped:
            rc = lib().attn_fwd_gqa(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                    lse.data_ptr(), B, H, k.shape[1], n, d, float(scale),
                                    int(bool(causal)), int(window), _stream_handle(stream))
        else:
            rc = lib().attn_fwd(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                lse.data_ptr(), B, H, n, d, float(scale), int(bool(causal)),
                                int(window), _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_blocklocal" if block > 0 else ("attn_fwd_gqa" if grouped else "attn_fwd"))
    return out, lse


def bwd_workspace_bytes(B: int, H: int, n: int, d: int) -> int:
    r = int(lib().attn_bwd_workspace_bytes(int(B), int(H), int(n), int(d)))
    if r < 0:
        raise ValueError("unsupported or invalid shape for attn_bwd")
    return r


def attn_bwd(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, o: torch.Tensor,
             lse: torch.Tensor, dout: torch.Tensor, scale: Optional[float] = None,
             causal: bool = False, window: int = -1, workspace: Optional[torch.Tensor] = None,
             stream: Optional[torch.cuda.Stream] = None, block: int = 0
             ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Gradients (dq, dk, dv) of the attention forward pass on the GPU.

    q, o, dout: bf16 CUDA tensors [B, H, n, d]; k, v: [B, H, n, d], or
    [B, Hkv, n, d] with Hkv dividing H (grouped-query attention: dk, dv then
    have Hkv heads and sum over each group). Contiguous; o and lse are
    attn_fwd's outputs for q, k, v with the same scale and mask; dout is the
    upstream gradient dL/dO. ``workspace`` (optional) is a uint8 CUDA tensor
    of at least bwd_workspace_bytes(B, H, n, d) bytes. Enqueued on
    ``stream`` (default: the current stream).
    """
    grouped = k.dim() == 4 and q.dim() == 4 and k.shape[1] != q.shape[1]
    _check_qkv(q, k, v, device=True, grouped=grouped)
    for name, t in (("o", o), ("dout", dout)):
        if t.dtype != torch.bfloat16 or t.shape != q.shape or not t.is_contiguous() or \
                t.device != q.device:
            raise ValueError(f"{name} must be a contiguous bf16 tensor shaped like q on q's device")
    B, H, n, d = q.shape
    if lse.shape != (B, H, n) or lse.dtype != torch.float32 or not lse.is_contiguous() or \
            lse.device != q.device:
        raise ValueError("lse must be a contiguous fp32 tensor [B, H, n] on q's device")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    need = bwd_workspace_bytes(B, H, n, d)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    if workspace.device != q.device or not workspace.is_contiguous():
        raise ValueError("workspace must be a contiguous tensor on q's device")
    if block > 0 and window >= 0:
        raise ValueError("a block-local mask takes no window")
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    args = (q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(), lse.data_ptr(), dout.data_ptr(),
            dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), workspace.data_ptr(),
            workspace.numel() * workspace.element_size(), B, H, k.shape[1], n, d, float(scale),
            int(bool(causal)), int(block if block > 0 else window), _stream_handle(stream))
    with torch.cuda.device(q.device):
        rc = (lib().attn_bwd_blocklocal if block > 0 else lib().attn_bwd_gqa)(*args)
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_bwd_blocklocal" if block > 0 else "attn_bwd_gqa")
    return dq, dk, dv


def decode_workspace_bytes(B: int, H: int, Hkv: int, W: int, d: int) -> int:
    r = int(lib().attn_decode_workspace_bytes(int(B), int(H), int(Hkv), int(W), int(d)))
    if r < 0:
        raise ValueError("unsupported or invalid shape for attn_decode")
    return r


def attn_decode(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, pos: torch.Tensor,
                scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One decode step: q bf16 [B, H, d], rolling caches k_cache / v_cache bf16
    [B, Hkv, W, d] (position p in slot p mod W), pos int32 [B] on the device
    (each sequence's query position). Returns (o bf16 [B, H, d], lse fp32
    [B, H]); see include/attn.h."""
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if q.dim() != 3 or k_cache.dim() != 4 or k_cache.shape != v_cache.shape:
        raise ValueError("q must be [B, H, d] and the caches [B, Hkv, W, d]")
    B, H, d = q.shape
    if k_cache.shape[0] != B or k_cache.shape[3] != d:
        raise ValueError("cache shape does not match q")
    Hkv, W = k_cache.shape[1], k_cache.shape[2]
    if pos.dtype != torch.int32 or pos.shape != (B,) or not pos.is_cuda or not pos.is_contiguous():
        raise ValueError("pos must be a contiguous int32 CUDA tensor [B]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(decode_workspace_bytes(B, H, Hkv, W, d), dtype=torch.uint8, device=q.device)
    with torch.cuda.device(q.device):
        rc = lib().attn_decode(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), pos.data_ptr(),
                               out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                               workspace.numel() * workspace.element_size(), B, H, Hkv, W, d, float(scale),
                               _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_decode")
    return out, lse


SCHEDULE_AUTO, SCHEDULE_PER_ITEM, SCHEDULE_PERSISTENT = 0, 1, 2


def set_fwd_schedule(mode: int) -> int:
    """Process-wide forward work schedule (auto / one CTA per work item /
    persistent); returns the previous mode. See attn_fwd_schedule."""
    prev = int(lib().attn_fwd_schedule(int(mode)))
    if prev < 0:
        raise ValueError(f"unknown schedule {mode}")
    return prev


def fwd_schedule_for(n: int, causal: bool, window: int = -1, block: int = 0) -> str:
    """'per_item' or 'persistent': the form the forward takes for this
    problem under the current setting (see attn_fwd_schedule_for)."""
    r = int(lib().attn_fwd_schedule_for(int(n), int(bool(causal)), int(window), int(block)))
    if r < 0:
        raise ValueError("n must be >= 1")
    return "persistent" if r == SCHEDULE_PERSISTENT else "per_item"


def decode_multi_workspace_bytes(B: int, H: int, Hkv: int, T: int, W: int, window: int, d: int) -> int:
    r = int(lib().attn_decode_multi_workspace_bytes(int(B), int(H), int(Hkv), int(T), int(W), int(window),
                                                    int(d)))
    if r < 0:
        raise ValueError("unsupported or invalid shape for attn_decode_multi")
    return r


def attn_decode_multi(q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor, pos: torch.Tensor,
                      window: int, scale: Optional[float] = None, out: Optional[torch.Tensor] = None,
                      lse: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
                      stream: Optional[torch.cuda.Stream] = None) -> Tuple[torch.Tensor, torch.Tensor]:
    """A decode step of T new tokens per sequence: q bf16 [B, H, T, d] (token
    u at position pos[b] - T + 1 + u), rolling caches k_cache / v_cache bf16
    [B, Hkv, W, d], pos int32 [B] on the device (each sequence's last new
    token), causal window `window` (window + T <= W). Returns (o bf16
    [B, H, T, d], lse fp32 [B, H, T]); see include/attn.h."""
    for name, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        if t.dtype != torch.bfloat16 or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous bf16 CUDA tensor")
    if q.dim() != 4 or k_cache.dim() != 4 or k_cache.shape != v_cache.shape:
        raise ValueError("q must be [B, H, T, d] and the caches [B, Hkv, W, d]")
    B, H, T, d = q.shape
    if k_cache.shape[0] != B or k_cache.shape[3] != d:
        raise ValueError("cache shape does not match q")
    Hkv, W = k_cache.shape[1], k_cache.shape[2]
    if pos.dtype != torch.int32 or pos.shape != (B,) or not pos.is_cuda or not pos.is_contiguous():
        raise ValueError("pos must be a contiguous int32 CUDA tensor [B]")
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty((B, H, T), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = torch.empty(decode_multi_workspace_bytes(B, H, Hkv, T, W, window, d), dtype=torch.uint8,
                                device=q.device)
    with torch.cuda.device(q.device):
        rc = lib().attn_decode_multi(q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(), pos.data_ptr(),
                                     out.data_ptr(), lse.data_ptr(), workspace.data_ptr(),
                                     workspace.numel() * workspace.element_size(), B, H, Hkv, T, W, int(window), d,
                                     float(scale), _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_decode_multi")
    return out, lse


def attn_fwd_host(q: torch.Tensor, k: torch.Tensor, v: torch.Tensor, scale: Optional[float] = None,
                  causal: bool = False, window: int = -1, out: Optional[torch.Tensor] = None,
                  lse: Optional[torch.Tensor] = None, stream: Optional[torch.cuda.Stream] = None,
                  device: int = 0) -> Tuple[torch.Tensor, torch.Tensor]:
    """The same operation on host (ideally pinned) tensors: the library copies
    q, k, v to the device, runs the kernel and copies o and lse back, all on
    ``stream``. Synchronize the stream before reading the outputs."""
    _check_qkv(q, k, v, device=False)
    B, H, n, d = q.shape
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    pin = q.is_pinned()
    if out is None:
        out = torch.empty(q.shape, dtype=torch.bfloat16, pin_memory=pin)
    if lse is None:
        lse = torch.empty((B, H, n), dtype=torch.float32, pin_memory=pin)
    with torch.cuda.device(device):
        rc = lib().attn_fwd_host(q.data_ptr(), k.data_ptr(), v.data_ptr(), out.data_ptr(),
                                lse.data_ptr(), B, H, n, d, float(scale), int(bool(causal)),
                                int(window), _stream_handle(stream))
    if rc != ATTN_OK:
        raise AttnError(rc, "attn_fwd_host")
    return out, lse


def sync_status(stream: Optional[torch.cuda.Stream] = None) -> int:
    """Synchronize ``stream`` and return (and clear) the device status."""
    return int(lib().attn_sync_status(_stream_handle(stream)))


def host_staging_release() -> int:
    return int(lib().attn_host_staging_release())
