"""bench.py's roofline traffic record, on CPU: the DRAM bytes per launch taken from an
ncu capture are reported only while the sources of the captured kernel (its .cu and
the headers holding its device code) hash to what the record says."""
import json
import os
import shutil

import bench


def test_every_listed_kernel_source_exists():
    csrc = os.path.join(bench.ROOT, "weight_only_additive_b200", "csrc")
    for kernel, files in bench.KERNEL_SOURCES.items():
        assert files and files[0].endswith(".cu"), kernel
        for name in files:
            assert os.path.exists(os.path.join(csrc, name)), (kernel, name)


def test_committed_record_names_a_known_kernel_and_its_sources():
    with open(os.path.join(bench.ROOT, "profiles", "roofline_traffic.json")) as fh:
        records = json.load(fh)
    for key, rec in records.items():
        workload, kernel = key.split("/", 1)
        assert rec["kernel"] == kernel and kernel in bench.KERNEL_SOURCES
        assert rec["sources"] == ["weight_only_additive_b200/csrc/" + f for f in bench.KERNEL_SOURCES[kernel]]
        assert len(rec["source_sha256"]) == 64 and rec["dram_bytes_per_launch"] > 0
        assert rec["command"].startswith("ncu ") and "--clock-control none" in rec["command"]


def _fake_root(tmp_path, sha, kernel="lut_group_kernel", nbytes=123456):
    """A copy of the kernel's sources and a record with the given hash under tmp_path."""
    csrc = tmp_path / "weight_only_additive_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in bench.KERNEL_SOURCES[kernel]:
        shutil.copy(os.path.join(bench.ROOT, "weight_only_additive_b200", "csrc", name), csrc / name)
    (tmp_path / "profiles").mkdir()
    rec = {f"wl/{kernel}": {"kernel": kernel, "source_sha256": sha, "dram_bytes_per_launch": nbytes}}
    (tmp_path / "profiles" / "roofline_traffic.json").write_text(json.dumps(rec))
    return csrc


def test_traffic_reported_only_while_the_sources_match(tmp_path, monkeypatch):
    sha = bench.kernel_source_sha256("lut_group_kernel")
    csrc = _fake_root(tmp_path, sha)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.kernel_source_sha256("lut_group_kernel") == sha
    assert bench.measured_traffic("wl", "lut_group_kernel") == 123456
    assert bench.measured_traffic("other_workload", "lut_group_kernel") is None
    assert bench.measured_traffic("wl", "no_such_kernel") is None
    # a change to any of the kernel's files (a header included) voids the record
    hdr = csrc / bench.KERNEL_SOURCES["lut_group_kernel"][1]
    hdr.write_text(hdr.read_text() + "\n// changed\n")
    assert bench.measured_traffic("wl", "lut_group_kernel") is None


def test_record_for_another_kernel_is_not_used(tmp_path, monkeypatch):
    sha = bench.kernel_source_sha256("gemv_lut_kernel")
    _fake_root(tmp_path, sha, kernel="gemv_lut_kernel")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.measured_traffic("wl", "gemv_lut_kernel") == 123456
    assert bench.measured_traffic("wl", "lut_group_kernel") is None
