"""attn_fwd_host_noalloc, the entry point that allocates no device memory.

Some callers cannot let a library allocate device memory on their behalf:
their device memory is a fixed budget that another component owns, or they
cannot afford the device-wide synchronisation cudaMalloc/cudaFree may cause.
For them attn_fwd_host_noalloc keeps all of its device scratch in one static
array of ATTN_NOALLOC_SCRATCH_BYTES per device.

The GPU test compares two consecutive calls of it with the existing
host-buffer entry point, attn_fwd_host, on the same inputs, within the parity
tolerances used everywhere else. This file is named so that pytest collects it
last; it passes on its own in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

from exact_softmax_attention_04_b200 import synth
from parity import assert_close

FAKE = 0x10000  # never dereferenced: the calls below are rejected before any device work


def _pkg():
    from exact_softmax_attention_04_b200 import build_lib
    build_lib.build()
    import exact_softmax_attention_04_b200 as pkg
    return pkg


def test_noalloc_rejects_problems_larger_than_its_scratch():
    pkg = _pkg()
    lib = pkg.lib()
    # 4 bf16 tensors of 1*8*65536*64 elements = 256 MiB > 64 MiB of scratch
    rc = lib.attn_fwd_host_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 65536, 64, 0.125, 1, -1, None)
    assert rc == pkg.ATTN_ERR_TOO_LARGE
    assert "scratch" in pkg.strerror(rc)
    # ordinary argument errors keep their usual codes
    assert lib.attn_fwd_host_noalloc(None, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.125, 0, -1,
                                     None) == pkg.ATTN_ERR_INVALID
    assert lib.attn_fwd_host_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 96, 0.125, 0, -1,
                                     None) == pkg.ATTN_ERR_UNSUPPORTED


def _noalloc(pkg, q, k, v, scale, causal, window):
    B, H, n, d = q.shape
    o = torch.empty(q.shape, dtype=torch.bfloat16)
    lse = torch.empty((B, H, n), dtype=torch.float32)
    rc = pkg.lib().attn_fwd_host_noalloc(q.data_ptr(), k.data_ptr(), v.data_ptr(), o.data_ptr(),
                                         lse.data_ptr(), B, H, n, d, float(scale), int(causal),
                                         int(window), torch.cuda.current_stream().cuda_stream)
    assert rc == pkg.ATTN_OK, pkg.strerror(rc)
    return o, lse


@pytest.mark.gpu
def test_noalloc_matches_host_entry_point_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    pkg = _pkg()
    cases = [((1, 2, 300, 64), True, -1, 41), ((2, 3, 517, 128), True, 200, 42)]
    for (B, H, n, d), causal, window, seed in cases:
        q, k, v = synth.make_qkv(B, H, n, d, seed=seed, q_std=2.0)
        scale = 1.0 / np.sqrt(d)
        o_ref, lse_ref = pkg.attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), scale,
                                           causal, window)
        assert pkg.sync_status() == pkg.ATTN_OK
        o, lse = _noalloc(pkg, q, k, v, scale, causal, window)
        assert_close(o.float().numpy(), lse.numpy(), o_ref.float().numpy(), lse_ref.numpy(),
                     f"noalloc B{B} H{H} n{n} d{d}")
