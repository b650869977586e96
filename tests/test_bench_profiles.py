"""bench.py's link to the committed ncu summaries (CPU only).

The bench reports a kernel's measured DRAM traffic per launch from `profiles/<name>.md` when the
summary was taken on the current kernel sources.  These tests check the naming of the summaries
for the bench's flag combinations, that every summary carries a parsable traffic figure and
sources digest, and that the digest ignores comments but not code.
"""
import argparse
import os
import re

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def args(**kw):
    base = dict(config="8b", kv_dtype=None, qtok=1, prefix=False, wide_kernel="mma")
    base.update(kw)
    return argparse.Namespace(**base)


def test_profile_names():
    assert bench.profile_name(args()) == "pa_decode_partition_8b"
    assert bench.profile_name(args(qtok=5)) == "pa_decode_partition_8b_T5"
    assert bench.profile_name(args(kv_dtype="e4m3")) == "pa_decode_partition_8b_e4m3"
    assert bench.profile_name(args(config="70b", prefix=True)) == "pa_decode_partition_70b_prefix"
    assert bench.profile_name(args(qtok=4, wide_kernel="tcgen05")) == "pa_decode_partition_8b_T4_tcgen05"
    assert bench.profile_name(args(qtok=16), "tcgen05") == "pa_decode_partition_8b_T16_tcgen05"
    # a resized workload never takes the full-size summary's traffic
    assert bench.profile_name(args(num_seqs=4096, uniform_lens="0,40")) == "pa_decode_partition_8b_n4096_u0-40"
    assert bench.profile_name(args(block_size=32)) == "pa_decode_partition_8b_bs32"


def test_every_summary_has_traffic_and_digest():
    names = [f for f in os.listdir(os.path.join(ROOT, "profiles")) if f.endswith(".md")]
    assert names
    for f in names:
        text = open(os.path.join(ROOT, "profiles", f), encoding="utf-8").read()
        traffic = re.search(r"^traffic_bytes_per_launch: (\d+)$", text, re.M)
        digest = re.search(r"^kernel_sources_sha256_16: ([0-9a-f]{16})$", text, re.M)
        assert traffic and digest, f
        assert int(traffic.group(1)) > 0
        assert "--clock-control none" in text, f"{f}: every ncu command leaves the clocks alone"


def test_traffic_is_reported_only_for_the_sources_it_was_taken_on(tmp_path, monkeypatch):
    # a summary in a scratch root: reported while its digest matches, None once it does not
    (tmp_path / "profiles").mkdir()
    good = bench.sources_digest()
    (tmp_path / "profiles" / "x.md").write_text(f"traffic_bytes_per_launch: 123\nkernel_sources_sha256_16: {good}\n")
    (tmp_path / "profiles" / "y.md").write_text("traffic_bytes_per_launch: 123\nkernel_sources_sha256_16: 0000000000000000\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "sources_digest", lambda: good)
    assert bench.recorded_traffic("x") == 123
    assert bench.recorded_traffic("y") is None
    assert bench.recorded_traffic("missing") is None


def test_digest_ignores_comments_not_code(tmp_path, monkeypatch):
    src = tmp_path / "k.cuh"
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.setattr(bench, "KERNEL_SOURCES", ["k.cuh"])
    src.write_text("int a = 1;  // one\n\n")
    d0 = bench.sources_digest()
    src.write_text("int a = 1;  // another comment\n// a new comment line\n")
    assert bench.sources_digest() == d0
    src.write_text("int a = 2;\n")
    assert bench.sources_digest() != d0
