"""Failure detection without faulting the GPU.

Every wait in the kernels is bounded (about one second). Builds with a
test-only hook never load one tile (forward: the first V tile; backward: the
first Q/dO stage; decode: the first K tile), so a wait for it must expire:
the kernel then sets the device status word, stops all roles, waits
(bounded) for what it issued, frees TMEM and returns. The host must read
ATTN_ERR_TIMEOUT, the status must clear, and the CUDA context must stay
usable for a correct computation afterwards.
"""
import time

import numpy as np
import pytest
import torch

from exact_softmax_attention_04_b200 import synth
from parity import assert_close

pytestmark = pytest.mark.gpu


def test_expired_wait_reports_timeout_and_context_survives(tmp_path, oracle_mod):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_softmax_attention_04_b200 as pkg
    from exact_softmax_attention_04_b200 import build_lib
    build_lib.build()
    fault_lib = pkg.load_library(build_lib.build_variant(tmp_path / "libattn_fault.so",
                                                         ["ATTN_FAULT_DROP_FIRST_V"]))
    # one CTA (n = 256: two 128-row tiles), several key tiles
    q, k, v = synth.make_qkv(1, 1, 256, 64, seed=50)
    qd, kd, vd = q.cuda(), k.cuda(), v.cuda()
    o = torch.empty_like(qd)
    lse = torch.empty((1, 1, 256), dtype=torch.float32, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.time()
    rc = fault_lib.attn_fwd(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(),
                            1, 1, 256, 64, 0.125, 0, -1, stream)
    assert rc == pkg.ATTN_OK
    st = fault_lib.attn_sync_status(stream)
    elapsed = time.time() - t0
    assert st == pkg.ATTN_ERR_TIMEOUT, pkg.strerror(st)
    assert elapsed < 30.0
    assert fault_lib.attn_sync_status(stream) == pkg.ATTN_OK  # read-and-clear
    # the context is intact: the normal library computes the same problem correctly
    o2, lse2 = pkg.attn_fwd(qd, kd, vd, 0.125, False, -1)
    assert pkg.sync_status() == pkg.ATTN_OK
    o_ref, lse_ref = oracle_mod.attn_fwd(q, k, v, 0.125, False, -1)
    assert_close(o2.float().cpu().numpy(), lse2.cpu().numpy(), o_ref, lse_ref, "after timeout")


def test_backward_expired_wait_reports_timeout_and_context_survives(tmp_path, oracle_mod):
    """The backward kernel's first Q/dO stage is never loaded (test-only
    ATTN_FAULT_BWD_DROP_FIRST_Q hook): its MMA warp's wait must expire, the
    call must report ATTN_ERR_TIMEOUT, and the context must stay usable."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_softmax_attention_04_b200 as pkg
    from exact_softmax_attention_04_b200 import build_lib
    from parity import assert_grads_close
    build_lib.build()
    fault_lib = pkg.load_library(build_lib.build_variant(tmp_path / "libattn_fault_bwd.so",
                                                         ["ATTN_FAULT_BWD_DROP_FIRST_Q"]))
    n, d = 384, 64
    q, k, v = synth.make_qkv(1, 1, n, d, seed=51)
    do = synth.make_dout(1, 1, n, d, seed=51)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = pkg.attn_fwd(qd, kd, vd, 0.125, True, -1)
    assert pkg.sync_status() == pkg.ATTN_OK
    dq, dk, dv = torch.empty_like(qd), torch.empty_like(qd), torch.empty_like(qd)
    ws = torch.empty(pkg.bwd_workspace_bytes(1, 1, n, d), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    t0 = time.time()
    rc = fault_lib.attn_bwd(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), o.data_ptr(), lse.data_ptr(),
                            dod.data_ptr(), dq.data_ptr(), dk.data_ptr(), dv.data_ptr(), ws.data_ptr(),
                            ws.numel(), 1, 1, n, d, 0.125, 1, -1, stream)
    assert rc == pkg.ATTN_OK
    st = fault_lib.attn_sync_status(stream)
    assert st == pkg.ATTN_ERR_TIMEOUT, pkg.strerror(st)
    assert time.time() - t0 < 30.0
    assert fault_lib.attn_sync_status(stream) == pkg.ATTN_OK
    grads = pkg.attn_bwd(qd, kd, vd, o, lse, dod, 0.125, True, -1)
    assert pkg.sync_status() == pkg.ATTN_OK
    refs = oracle_mod.attn_bwd(q, k, v, do, 0.125, True, -1)
    assert_grads_close([g.float().cpu().numpy() for g in grads], refs, "after backward timeout")


def test_decode_expired_wait_reports_timeout_and_context_survives(tmp_path, oracle_mod):
    """The decode kernel's first K tile is never loaded (test-only
    ATTN_FAULT_DEC_DROP_FIRST_K hook): the MMA warp's and the softmax warps'
    waits on it must expire, the call must report ATTN_ERR_TIMEOUT, and the
    context must stay usable."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_softmax_attention_04_b200 as pkg
    from exact_softmax_attention_04_b200 import build_lib
    build_lib.build()
    fault_lib = pkg.load_library(build_lib.build_variant(tmp_path / "libattn_fault_dec.so",
                                                         ["ATTN_FAULT_DEC_DROP_FIRST_K"]))
    # four CTAs (four splits of one 128-slot tile each), four query heads per K/V head
    B, H, Hkv, W, d = 1, 4, 1, 512, 128
    q, kc, vc = synth.make_decode(B, H, Hkv, W, d, seed=52, q_std=1.0)
    qd, kd, vd = q.cuda(), kc.cuda(), vc.cuda()
    pos = torch.tensor([W - 1], dtype=torch.int32, device="cuda")
    o = torch.empty_like(qd)
    lse = torch.empty((B, H), dtype=torch.float32, device="cuda")
    ws = torch.empty(pkg.decode_workspace_bytes(B, H, Hkv, W, d), dtype=torch.uint8, device="cuda")
    stream = torch.cuda.current_stream().cuda_stream
    sc = 1.0 / np.sqrt(d)
    t0 = time.time()
    rc = fault_lib.attn_decode(qd.data_ptr(), kd.data_ptr(), vd.data_ptr(), pos.data_ptr(), o.data_ptr(),
                               lse.data_ptr(), ws.data_ptr(), ws.numel(), B, H, Hkv, W, d, sc, stream)
    assert rc == pkg.ATTN_OK
    st = fault_lib.attn_sync_status(stream)
    assert st == pkg.ATTN_ERR_TIMEOUT, pkg.strerror(st)
    assert time.time() - t0 < 30.0
    assert fault_lib.attn_sync_status(stream) == pkg.ATTN_OK
    o2, lse2 = pkg.attn_decode(qd, kd, vd, pos, sc)
    assert pkg.sync_status() == pkg.ATTN_OK
    o_ref, lse_ref = oracle_mod.attn_decode(q, kc, vc, [W - 1], sc)
    assert_close(o2.float().cpu().numpy().reshape(-1, d), lse2.cpu().numpy().reshape(-1),
                 o_ref.reshape(-1, d), lse_ref.reshape(-1), "after decode timeout")
