"""attn_fwd_host_noalloc, the entry point that allocates no device memory.

Some callers cannot let a library allocate device memory on their behalf:
their device memory is a fixed budget that another component owns, or they
cannot afford the device-wide synchronisation cudaMalloc/cudaFree may cause.
For them attn_fwd_host_noalloc keeps all of its device scratch in one static
array of ATTN_NOALLOC_SCRATCH_BYTES per device.

The GPU test checks, for both head sizes, a causal window and a problem at the
size limit of the scratch array:
- two calls in a row on the same inputs, each compared with the fp64 oracle
  and with the existing host-buffer entry point, attn_fwd_host, within the
  parity tolerances used everywhere else (and equal to each other);
- the largest case runs first, so the smaller ones that follow find its
  leftover contents in the shared array;
- the device's free memory is the same before and after all of these calls
  (after one warm-up call per head size, which loads the kernels).
This file is named so that pytest collects it last; it passes on its own in
a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

from exact_softmax_attention_04_b200 import synth
from parity import assert_close

FAKE = 0x10000  # never dereferenced: the calls below are rejected before any device work
SCRATCH = 64 << 20


def _pkg():
    from exact_softmax_attention_04_b200 import build_lib
    build_lib.build()
    import exact_softmax_attention_04_b200 as pkg
    return pkg


def _need(B, H, n, d):
    """Scratch bytes of one call: status word, q, k, v, o, lse (each part
    rounded up to 256 bytes)."""
    up = lambda x: (x + 255) // 256 * 256
    return 256 + 4 * up(B * H * n * d * 2) + up(B * H * n * 4)


def test_noalloc_rejects_problems_larger_than_its_scratch():
    pkg = _pkg()
    lib = pkg.lib()
    # 4 bf16 tensors of 1*8*65536*64 elements = 256 MiB > 64 MiB of scratch
    rc = lib.attn_fwd_host_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 65536, 64, 0.125, 1, -1, None)
    assert rc == pkg.ATTN_ERR_TOO_LARGE
    assert "scratch" in pkg.strerror(rc)
    # one token past the largest d = 128 problem of four heads that fits
    assert _need(1, 4, 16320, 128) <= SCRATCH < _need(1, 4, 16321, 128)
    rc = lib.attn_fwd_host_noalloc(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 4, 16321, 128, 0.125, 1, -1, None)
    assert rc == pkg.ATTN_ERR_TOO_LARGE
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
def test_noalloc_matches_oracle_and_host_entry_point_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import oracle
    oracle.build()
    pkg = _pkg()
    # (shape, causal, window, seed, rows compared with the oracle: None = all)
    cases = [((1, 4, 16320, 128), True, -1, 40, "sample"),   # at the size limit, first
             ((2, 3, 517, 128), True, 200, 42, None),
             ((1, 2, 300, 64), True, -1, 41, None),
             ((2, 2, 333, 64), True, 77, 43, None)]
    assert _need(1, 4, 16320, 128) <= SCRATCH
    inputs, host_refs, oracle_refs = [], [], []
    for (B, H, n, d), causal, window, seed, rows in cases:
        q, k, v = synth.make_qkv(B, H, n, d, seed=seed, q_std=2.0)
        scale = 1.0 / np.sqrt(d)
        inputs.append((q, k, v, scale))
        # the existing host-buffer entry point (it allocates its staging here,
        # before the free-memory check below)
        o_h, l_h = pkg.attn_fwd_host(q.pin_memory(), k.pin_memory(), v.pin_memory(), scale, causal, window)
        assert pkg.sync_status() == pkg.ATTN_OK
        host_refs.append((o_h.clone(), l_h.clone()))
        idx = (synth.sample_rows(B, H, n, per_head_random=128, seed=seed).numpy() if rows == "sample"
               else np.arange(B * H * n))
        o_r, l_r = oracle.attn_rows(q, k, v, scale, causal, window, idx)[:2]
        oracle_refs.append((idx, o_r, l_r))
    # warm-up: one small call per head size loads both kernels and looks up
    # the scratch array's address
    for d in (64, 128):
        q, k, v = synth.make_qkv(1, 1, 64, d, seed=1)
        _noalloc(pkg, q, k, v, 0.125, True, -1)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    for ((B, H, n, d), causal, window, seed, _), (q, k, v, scale), (o_h, l_h), (idx, o_r, l_r) in zip(
            cases, inputs, host_refs, oracle_refs):
        first = None
        for call in range(2):
            o, lse = _noalloc(pkg, q, k, v, scale, causal, window)
            what = f"noalloc call {call + 1} B{B} H{H} n{n} d{d} w{window}"
            o_flat, l_flat = o.float().numpy().reshape(-1, d), lse.numpy().reshape(-1)
            assert_close(o_flat[idx], l_flat[idx], o_r, l_r, what + " vs oracle")
            assert_close(o.float().numpy(), lse.numpy(), o_h.float().numpy(), l_h.numpy(),
                         what + " vs attn_fwd_host")
            if first is None:
                first = (o, lse)
            else:  # the forward is deterministic: the second call repeats the first
                assert torch.equal(o, first[0]) and torch.equal(lse, first[1]), what
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before, "attn_fwd_host_noalloc changed free device memory"
    pkg.host_staging_release()
