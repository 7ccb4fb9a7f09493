"""Host-side rules of bench.py (not gpu): the algorithmic bytes a decode call must move, and the
ncu traffic figure, which is reported only while the profiled sources are unchanged."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench      # noqa: E402
import workloads  # noqa: E402


def test_algorithmic_decode_bytes_of_the_headline_workload():
    """32 x 4 units x 1,147 entries: every entry's key and value (2 x 128 bf16) and its fp32
    (alpha, beta) once, the 896 query rows in and out (bf16), one fp32 lse per row."""
    w = workloads.WORKLOADS["gqa7_32k_decode_3p5pct"]
    ent = w.B * w.Hkv * (workloads.N_SINK + w.N + workloads.N_RECENT)
    alg, e = bench.algorithmic_decode_bytes(w, [ent])
    assert e == ent == 146816
    rows = w.B * w.R * w.Hq
    assert alg == ent * (2 * 128 * 2 + 8) + rows * 128 * 2 * 2 + rows * 4 == 76_806_656
    diag, _ = bench.algorithmic_decode_bytes(w, [ent], closure="diagonal")
    assert diag - alg == ent * 128 * 2           # one more d-vector of bf16 variances per entry
    assert round(diag / 1e6, 2) == 114.39


def test_profile_traffic_follows_the_source_hash(tmp_path, monkeypatch):
    """A summary whose recorded hash matches its sources gives its DRAM bytes; once any covered
    source changes by one byte the figure is withheld (the bench then reports traffic null)."""
    tree = tmp_path / "tree"
    os.makedirs(tree / "profiles")
    os.makedirs(tree / "src")
    sources = ["src/kernel.cu", "src/common.cuh"]
    for f, text in zip(sources, (b"__global__ void k() {}\n", b"// shared\n")):
        (tree / f).write_bytes(text)
    monkeypatch.setattr(bench, "ROOT", str(tree))
    sha = bench._source_sha(sources)
    (tree / "profiles" / "k_summary.md").write_text(
        f"# k\n\nsource_sha256_16: {sha}\ndram_bytes_per_launch: 79030528\n")
    assert bench._profile_traffic("k_summary.md", sources) == 79030528.0
    assert bench._profile_traffic("k_summary.md", sources[:1]) is None     # other file set
    with open(tree / sources[1], "ab") as fh:
        fh.write(b" ")
    assert bench._profile_traffic("k_summary.md", sources) is None
    assert bench._profile_traffic("no_such_summary.md", sources) is None
