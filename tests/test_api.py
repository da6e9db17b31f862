"""The C ABI boundary, checked without a GPU: the library builds and loads,
exports every function include/attn.h declares, and rejects bad arguments
before touching the device."""
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "attn.h")


@pytest.fixture(scope="module")
def attn():
    from exact_softmax_attention_04_b200 import build_lib
    build_lib.build()
    import exact_softmax_attention_04_b200 as pkg
    return pkg


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(attn_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = _declared_functions()
    assert "attn_fwd" in names and "attn_sync_status" in names
    import exact_softmax_attention_04_b200 as pkg
    assert sorted(pkg.EXPORTS) == names


def test_library_exports_every_declared_symbol(attn):
    out = subprocess.run(["nm", "-D", "--defined-only", attn.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\S+)$", out, flags=re.M))
    for name in _declared_functions():
        assert name in exported, name
        assert hasattr(attn.lib(), name)
    # nothing else leaks out as a C symbol of ours
    assert not [s for s in exported if s.startswith("attn_") and s not in _declared_functions()]


def test_header_compiles_as_c(tmp_path):
    src = tmp_path / "t.c"
    src.write_text('#include "attn.h"\n'
                   'int main(void){ const char *(*f)(int) = attn_strerror; (void)f;'
                   ' return ATTN_OK; }\n')
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), "-c",
                    str(src), "-o", str(tmp_path / "t.o")], check=True)


def test_strerror_covers_every_status(attn):
    texts = {attn.strerror(c) for c in range(5)}
    assert len(texts) == 5
    assert attn.strerror(99) == "unknown status"


def test_attended_pairs_matches_the_workload_counts(attn):
    from exact_softmax_attention_04_b200 import synth
    for n in (1, 2, 127, 128, 129, 1000, 131072):
        for causal, window in [(False, -1), (True, -1), (True, 0), (True, 1), (True, 256), (True, 4096),
                               (True, 10 ** 6), (False, 0), (False, 1), (False, 256), (False, 10 ** 6)]:
            assert attn.attended_pairs(n, causal, window) == synth.attended_pairs_per_head(n, causal, window)
    with pytest.raises(ValueError):
        attn.attended_pairs(-1, False, 3)


FAKE = 0x10000  # 16-byte aligned, never dereferenced: every case below fails validation first


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), 1), (dict(lse=0), 1), (dict(B=0), 1), (dict(H=-1), 1), (dict(n=0), 1),
    (dict(d=0), 1), (dict(scale=0.0), 1), (dict(scale=float("nan")), 1), (dict(scale=-1.0), 1),
    (dict(scale=float("inf")), 1), (dict(causal=2), 1), (dict(q=FAKE + 8), 1), (dict(lse=FAKE + 2), 1),
    (dict(d=96), 2), (dict(d=256), 2), (dict(n=(1 << 30) + 1), 2),
    (dict(B=1 << 16, H=1 << 16), 1),
])
def test_attn_fwd_rejects_bad_arguments_before_any_cuda_call(attn, kw, code):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, B=1, H=1, n=128, d=64, scale=0.125,
             causal=1, window=-1, stream=None)
    a.update(kw)
    rc = attn.lib().attn_fwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["B"], a["H"], a["n"],
                             a["d"], a["scale"], a["causal"], a["window"], a["stream"])
    assert rc == code


def test_host_entry_point_rejects_bad_arguments(attn):
    rc = attn.lib().attn_fwd_host(None, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 64, 0.125, 0, -1, None)
    assert rc == attn.ATTN_ERR_INVALID
    rc = attn.lib().attn_fwd_host(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 1, 128, 80, 0.125, 0, -1, None)
    assert rc == attn.ATTN_ERR_UNSUPPORTED


def test_python_binding_checks_tensors_before_calling(attn):
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn.attn_fwd(q, q, q)  # host tensors on the device entry point
    with pytest.raises(TypeError):
        attn.attn_fwd_host(q.float(), q, q)
    with pytest.raises(ValueError):
        attn.attn_fwd_host(q, q[..., :32].contiguous(), q)


def test_missing_library_fails_loudly(monkeypatch, attn):
    import exact_softmax_attention_04_b200 as pkg
    monkeypatch.setattr(pkg, "LIB_PATH", "/nonexistent/libattn_b200.so")
    with pytest.raises(ImportError):
        pkg._load()


def test_gqa_entry_point_rejects_bad_head_counts(attn):
    lib = attn.lib()
    for Hkv in (0, -2, 3, 16):
        rc = lib.attn_fwd_gqa(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, Hkv, 128, 64, 0.125, 1, -1, None)
        assert rc == attn.ATTN_ERR_INVALID, Hkv
    rc = lib.attn_fwd_gqa(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 2, 128, 80, 0.125, 1, -1, None)
    assert rc == attn.ATTN_ERR_UNSUPPORTED


def test_binding_checks_grouped_shapes(attn):
    import torch
    q = torch.zeros(1, 8, 16, 64, dtype=torch.bfloat16)
    kv = torch.zeros(1, 3, 16, 64, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        attn._check_qkv(q, kv, kv, device=False, grouped=True)
    kv2 = torch.zeros(1, 2, 16, 64, dtype=torch.bfloat16)
    attn._check_qkv(q, kv2, kv2, device=False, grouped=True)


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), 1), (dict(dout=0), 1), (dict(dq=0), 1), (dict(workspace=0), 1), (dict(lse=0), 1),
    (dict(B=0), 1), (dict(n=0), 1), (dict(scale=0.0), 1), (dict(scale=float("nan")), 1),
    (dict(causal=2), 1), (dict(dk=FAKE + 8), 1), (dict(workspace=FAKE + 4), 1), (dict(lse=FAKE + 2), 1),
    (dict(ws_bytes=0), 1), (dict(d=96), 2), (dict(n=(1 << 30) + 1), 2),
    (dict(B=1 << 16, H=1 << 16), 1),
])
def test_attn_bwd_rejects_bad_arguments_before_any_cuda_call(attn, kw, code):
    a = dict(q=FAKE, k=FAKE, v=FAKE, o=FAKE, lse=FAKE, dout=FAKE, dq=FAKE, dk=FAKE, dv=FAKE,
             workspace=FAKE, ws_bytes=1 << 40, B=1, H=1, n=128, d=64, scale=0.125, causal=1,
             window=-1, stream=None)
    a.update(kw)
    rc = attn.lib().attn_bwd(a["q"], a["k"], a["v"], a["o"], a["lse"], a["dout"], a["dq"], a["dk"],
                             a["dv"], a["workspace"], a["ws_bytes"], a["B"], a["H"], a["n"], a["d"],
                             a["scale"], a["causal"], a["window"], a["stream"])
    assert rc == code


def test_bwd_workspace_size(attn):
    # two fp32 per-row arrays padded to 128-row tiles, plus at d = 64 an fp32
    # dQ accumulator, each part rounded up to 256 bytes
    def expect(B, H, n, d):
        r = lambda x: (x + 255) // 256 * 256
        n_pad = (n + 127) // 128 * 128
        return (r(B * H * n * d * 4) if d == 64 else 0) + 2 * r(B * H * n_pad * 4)
    for shape in [(1, 1, 1, 64), (1, 2, 300, 64), (2, 3, 129, 128), (8, 8, 8192, 64)]:
        assert attn.bwd_workspace_bytes(*shape) == expect(*shape)
    assert attn.lib().attn_bwd_workspace_bytes(1, 1, 128, 80) == -1
    assert attn.lib().attn_bwd_workspace_bytes(0, 1, 128, 64) == -1


def test_bwd_binding_checks_tensors_before_calling(attn):
    import torch
    q = torch.zeros(1, 1, 8, 64, dtype=torch.bfloat16)
    lse = torch.zeros(1, 1, 8)
    with pytest.raises(ValueError):
        attn.attn_bwd(q, q, q, q, lse, q)  # host tensors


@pytest.mark.parametrize("kw,code", [
    (dict(q=0), 1), (dict(pos=0), 1), (dict(workspace=0), 1), (dict(B=0), 1), (dict(W=0), 1),
    (dict(scale=0.0), 1), (dict(Hkv=3), 1), (dict(q=FAKE + 8), 1), (dict(pos=FAKE + 2), 1),
    (dict(ws_bytes=0), 1), (dict(d=96), 2), (dict(H=34, Hkv=2), 2), (dict(H=32, Hkv=1), 2),
    (dict(B=70000, H=8, Hkv=1), 2),
])
def test_attn_decode_rejects_bad_arguments_before_any_cuda_call(attn, kw, code):
    a = dict(q=FAKE, k=FAKE, v=FAKE, pos=FAKE, o=FAKE, lse=FAKE, workspace=FAKE, ws_bytes=1 << 40,
             B=2, H=8, Hkv=2, W=4096, d=128, scale=0.125, stream=None)
    a.update(kw)
    rc = attn.lib().attn_decode(a["q"], a["k"], a["v"], a["pos"], a["o"], a["lse"], a["workspace"],
                                a["ws_bytes"], a["B"], a["H"], a["Hkv"], a["W"], a["d"], a["scale"],
                                a["stream"])
    assert rc == code


def test_decode_workspace_size(attn):
    # per-split partials: nsplit * B * H * (d + 2) fp32; the split rule cuts
    # the 128-slot tiles into splits minimising waves x (tiles per split + 1)
    # over 2 x 148 resident CTAs (first minimum, 1 to 64 splits)
    def expect(B, H, Hkv, W, d):
        tiles = (W + 127) // 128
        best = None
        for ns in range(1, min(tiles, 64) + 1):
            per = (tiles + ns - 1) // ns
            ctas = B * Hkv * ((tiles + per - 1) // per)
            cost = ((ctas + 295) // 296) * (per + 1)
            if best is None or cost < best[0]:
                best = (cost, per)
        chunk = best[1] * 128
        return ((W + chunk - 1) // chunk) * B * H * (d + 2) * 4
    for shape in [(1, 1, 1, 1, 64), (2, 8, 2, 4096, 128), (64, 32, 8, 4096, 128), (3, 4, 4, 200, 64)]:
        assert attn.decode_workspace_bytes(*shape) == expect(*shape)
    assert attn.lib().attn_decode_workspace_bytes(1, 34, 2, 64, 64) == -1  # 17 query heads per K/V head
    # several new tokens per sequence: T partial rows per (b, h)
    for B, H, Hkv, T, W, w, d in [(2, 8, 2, 4, 4096, 4092, 128), (64, 32, 8, 4, 4096, 4092, 128),
                                  (3, 6, 2, 3, 200, 50, 64), (1, 16, 1, 1, 128, 127, 64)]:
        assert attn.decode_multi_workspace_bytes(B, H, Hkv, T, W, w, d) == expect(B, H, Hkv, W, d) * T
    # T = 1 with the whole cache as the window is attn_decode
    assert attn.decode_multi_workspace_bytes(2, 8, 2, 1, 4096, 4095, 128) == attn.decode_workspace_bytes(
        2, 8, 2, 4096, 128)


@pytest.mark.parametrize("kw,code", [
    (dict(T=0), 1), (dict(window=-1), 1), (dict(window=4093), 1), (dict(T=5, window=4092), 1),
    (dict(H=20, Hkv=5, T=5, window=100), 2), (dict(H=8, Hkv=1, T=3, window=100), 2), (dict(q=0), 1),
    (dict(ws_bytes=0), 1), (dict(d=96), 2), (dict(Hkv=3), 1),
])
def test_attn_decode_multi_rejects_bad_arguments_before_any_cuda_call(attn, kw, code):
    a = dict(q=FAKE, k=FAKE, v=FAKE, pos=FAKE, o=FAKE, lse=FAKE, workspace=FAKE, ws_bytes=1 << 40,
             B=2, H=8, Hkv=2, T=4, W=4096, window=4092, d=128, scale=0.125, stream=None)
    a.update(kw)
    rc = attn.lib().attn_decode_multi(a["q"], a["k"], a["v"], a["pos"], a["o"], a["lse"], a["workspace"],
                                      a["ws_bytes"], a["B"], a["H"], a["Hkv"], a["T"], a["W"], a["window"],
                                      a["d"], a["scale"], a["stream"])
    assert rc == code


def test_bwd_gqa_entry_point_rejects_bad_head_counts(attn):
    lib = attn.lib()
    for Hkv in (0, -2, 3, 16):
        rc = lib.attn_bwd_gqa(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 40,
                              1, 8, Hkv, 128, 64, 0.125, 1, -1, None)
        assert rc == attn.ATTN_ERR_INVALID, Hkv


def test_blocklocal_entry_points_reject_bad_blocks(attn):
    lib = attn.lib()
    for block in (0, -5):
        assert lib.attn_fwd_blocklocal(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 8, 128, 64, 0.125, 1, block,
                                       None) == attn.ATTN_ERR_INVALID
        assert lib.attn_bwd_blocklocal(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 40,
                                       1, 8, 8, 128, 64, 0.125, 1, block, None) == attn.ATTN_ERR_INVALID
    assert lib.attn_fwd_blocklocal(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 3, 128, 64, 0.125, 1, 64,
                                   None) == attn.ATTN_ERR_INVALID   # 3 does not divide 8
    assert lib.attn_fwd_blocklocal(FAKE, FAKE, FAKE, FAKE, FAKE, 1, 8, 8, 128, 96, 0.125, 1, 64,
                                   None) == attn.ATTN_ERR_UNSUPPORTED


def test_block_pair_count_workload(attn):
    from exact_softmax_attention_04_b200 import synth
    wl = synth.BLOCK_N16384
    # 32 blocks of 512: block 0 sees itself (512 keys), later blocks 1024 keys
    assert synth.workload_pairs_per_head(wl) == 512 * 512 + 31 * 512 * 1024


def test_fwd_schedule_setting(attn):
    lib = attn.lib()
    assert lib.attn_fwd_schedule(attn.SCHEDULE_PERSISTENT) == attn.SCHEDULE_AUTO
    assert lib.attn_fwd_schedule(attn.SCHEDULE_PER_ITEM) == attn.SCHEDULE_PERSISTENT
    assert lib.attn_fwd_schedule(7) == -1                      # unknown: nothing changes
    assert lib.attn_fwd_schedule(attn.SCHEDULE_AUTO) == attn.SCHEDULE_PER_ITEM
    with pytest.raises(ValueError):
        attn.set_fwd_schedule(-3)


def test_fwd_schedule_for_reports_the_automatic_choice(attn):
    """Plain causal: persistent up to n = 16384; windows and no mask:
    persistent when a query tile walks few key tiles; a forced setting wins."""
    f = attn.fwd_schedule_for
    assert f(131072, True) == "per_item"          # the largest target workload
    assert f(16384, True) == "persistent"
    assert f(65536, True) == "per_item"
    assert f(8192, False) == "per_item"           # no mask, long rows
    assert f(1024, False) == "persistent"         # no mask, short rows
    assert f(65536, True, 256) == "persistent"    # narrow window
    assert f(32768, True, 4096) == "per_item"     # wide window
    assert f(4096, True, 4096) == "persistent"    # a window of n or more is plain causal
    assert f(16384, False, 256) == "persistent"   # symmetric window 256
    prev = attn.set_fwd_schedule(attn.SCHEDULE_PERSISTENT)
    try:
        assert f(131072, True) == "persistent"
    finally:
        attn.set_fwd_schedule(prev)
    assert attn.lib().attn_fwd_schedule_for(0, 1, -1, 0) == -1
