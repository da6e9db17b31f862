"""Host-side helpers of bench.py that decide what the JSON line reports:
the kernel-source hash behind roofline.traffic, the traffic record lookup,
and the summary of the clock samples taken during the timed region."""
import os
import shutil

import bench


def test_strip_comments_keeps_code_and_literals():
    src = (
        '#include "a.h"  // trailing\n'
        "\n"
        "/* block\n   comment */ int x = 1; /* inline */ int y = 2;\n"
        'const char *s = "not // a comment /* nor this */";\n'
        "char c = '\"'; char e = '\\'';  // quote characters\n"
        'const char *t = "escaped \\" quote // still string";\n'
        "   \n"
        "int z; // end\n"
    )
    out = bench.strip_comments(src)
    assert out.split("\n") == [
        '#include "a.h"',
        " int x = 1;  int y = 2;",
        'const char *s = "not // a comment /* nor this */";',
        "char c = '\"'; char e = '\\'';",
        'const char *t = "escaped \\" quote // still string";',
        "int z;",
    ]


def _copy_sources(tmp_path):
    src = os.path.join(bench.ROOT, "exact_softmax_attention_04_b200", "csrc")
    dst = tmp_path / "exact_softmax_attention_04_b200" / "csrc"
    dst.mkdir(parents=True)
    for f in bench.FWD_KERNEL_SOURCES:
        shutil.copy(os.path.join(src, f), dst / f)
    return dst


def test_kernel_hash_ignores_comments_but_not_code(tmp_path, monkeypatch):
    base = bench.kernel_source_hash()
    csrc = _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_source_hash() == base
    p = csrc / "attn_fwd_kernel.cuh"
    text = p.read_text()
    p.write_text("// a new comment\n\n/* and a block\n of them */\n" + text.replace("\n", "  \n", 3))
    assert bench.kernel_source_hash() == base
    p.write_text(text.replace("constexpr int QT = 2;", "constexpr int QT = 3;"))
    assert bench.kernel_source_hash() != base


def test_traffic_record_only_for_matching_sources(tmp_path, monkeypatch):
    _copy_sources(tmp_path)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    prof = tmp_path / "profiles"
    prof.mkdir()
    rec = prof / f"{bench.KERNEL_NAME}.W.traffic.txt"
    rec.write_text(f"# header: with a colon\nkernel_sources_sha256_16: {bench.kernel_source_hash()}\n"
                   "dram_bytes_per_launch: 12345\n")
    assert bench.recorded_traffic("W") == 12345
    rec.write_text("kernel_sources_sha256_16: 0000000000000000\ndram_bytes_per_launch: 12345\n")
    assert bench.recorded_traffic("W") is None
    assert bench.recorded_traffic("missing") is None


def test_clock_summary_uses_samples_inside_the_timed_region():
    import datetime
    t0 = datetime.datetime(2026, 1, 2, 3, 4, 5).timestamp()

    def line(dt, mhz, cap):
        ts = datetime.datetime.fromtimestamp(t0 + dt).strftime("%Y/%m/%d %H:%M:%S.%f")[:-3]
        act = "Active" if cap else "Not Active"
        return f"{ts}, {mhz}, 1965, 900.0, 0x0, Not Active, Not Active, Not Active, {act}"

    cs = bench.ClockSampler(-1)
    cs.out = "\n".join([line(-5.0, 1965, False), line(0.2, 1800, True), line(0.4, 1900, True),
                        line(0.6, 1850, False), line(9.0, 1000, False), "garbage"])
    s = cs.summary(t0, t0 + 1.0)
    assert s["samples"] == 3 and s["sm_mhz"] == 1850 and s["sm_max_mhz"] == 1965
    assert s["reasons"] == ["sw_power_cap"] and s["window"] == "timed region"
    s_all = cs.summary(t0 + 100, t0 + 101)  # no sample inside: all of them, labelled so
    assert s_all["samples"] == 5 and s_all["window"].startswith("whole run")
    cs.out = ""
    assert cs.summary(t0, t0 + 1)["samples"] == 0
