"""Host logic of bench.py's roofline `traffic` key (CPU): the DRAM bytes recorded
from an ncu capture are reported only for the workload they were captured on and
only while every hashed kernel source is unchanged; otherwise the key is null."""
import hashlib
import os

import bench
from gated_delta_rule_130_b200 import inputs as I


def _tree(tmp_path, workload, sources, edit=None):
    """A copy of the layout bench.measured_traffic reads: profiles/ plus the hashed
    sources, the recorded file naming `workload` and the sources' digests."""
    (tmp_path / "profiles").mkdir()
    lines = ["# test capture", f"workload: {workload}", "dram_bytes_per_call: 123456"]
    for rel, text in sources.items():
        f = tmp_path / rel
        f.parent.mkdir(parents=True, exist_ok=True)
        f.write_text(text)
        lines.append(f"sha256 {rel}: {hashlib.sha256(text.encode()).hexdigest()}")
    (tmp_path / "profiles" / "traffic_gdn_chunk_fwd_tc.txt").write_text("\n".join(lines) + "\n")
    if edit:
        (tmp_path / edit).write_text("changed")


SOURCES = {"src/a.cu": "kernel a", "src/b.cuh": "header b"}


def test_traffic_reported_for_its_workload(tmp_path, monkeypatch):
    _tree(tmp_path, "headline_T4k", SOURCES)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("tcgen05", I.workload("headline_T4k")) == 123456.0


def test_traffic_null_for_other_workloads_and_paths(tmp_path, monkeypatch):
    _tree(tmp_path, "headline_T4k", SOURCES)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("tcgen05", I.workload("long_T32k")) is None
    # same name, other sizes: not the captured workload
    assert bench.measured_traffic("tcgen05", I.workload("headline_T4k", B=1)) is None
    assert bench.measured_traffic("simt", I.workload("headline_T4k")) is None


def test_traffic_null_once_a_source_changed(tmp_path, monkeypatch):
    _tree(tmp_path, "headline_T4k", SOURCES, edit="src/b.cuh")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("tcgen05", I.workload("headline_T4k")) is None


def test_committed_capture_names_a_workload_and_its_sources():
    f = os.path.join(bench.ROOT, "profiles", "traffic_gdn_chunk_fwd_tc.txt")
    text = open(f).read()
    names = [ln.split(":", 1)[1].strip() for ln in text.splitlines() if ln.startswith("workload:")]
    assert names == ["headline_T4k"]
    hashed = [ln for ln in text.splitlines() if ln.startswith("sha256 ")]
    assert any("chunk_tc.cu" in ln for ln in hashed)
