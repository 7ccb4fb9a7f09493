"""Host-side rules of bench.py (not gpu): the algorithmic bytes a decode call must move, and the
ncu traffic figure, which is reported only while the profiled sources are unchanged."""
import os
import shutil
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
    """A summary whose source hash matches gives its DRAM bytes; once any covered source changes
    (here: a copy of the tree with one byte appended to a kernel file) the figure is withheld."""
    for name, sources in (("decode_gqa7_32k_summary.md", bench.DECODE_SOURCES),
                          ("coarsen_131k_summary.md", bench.COARSEN_SOURCES)):
        assert bench._profile_traffic(name, sources) is not None, f"{name}: hash does not match the sources"
        tree = tmp_path / name
        os.makedirs(tree / "profiles")
        shutil.copy(os.path.join(ROOT, "profiles", name), tree / "profiles" / name)
        for f in sources:
            os.makedirs(os.path.dirname(tree / f), exist_ok=True)
            shutil.copy(os.path.join(ROOT, f), tree / f)
        monkeypatch.setattr(bench, "ROOT", str(tree))
        assert bench._profile_traffic(name, sources) is not None
        with open(tree / sources[0], "ab") as fh:
            fh.write(b"\n")
        assert bench._profile_traffic(name, sources) is None
        monkeypatch.setattr(bench, "ROOT", ROOT)
    assert bench._profile_traffic("no_such_summary.md", bench.DECODE_SOURCES) is None
