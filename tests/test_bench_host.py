"""Host-side pieces of bench.py and the committed profile summaries (CPU only):
the DRAM-traffic record is used only while its kernel source is unchanged, and
every ncu summary states the command that made it, with unlocked clocks."""
import hashlib
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402


def _fake_tree(tmp_path, src_text, record_sha):
    csrc = tmp_path / "hierarchical_latent_key_gemm_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(src_text)
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.txt").write_text(
        "# kernel | workload | source | sha256[:16] | dram bytes per launch | how\n"
        f"kern<1> | wl | k.cu | {record_sha} | 12345 | test record\n")


def test_traffic_record_holds_only_for_the_captured_source(tmp_path, monkeypatch):
    src = "__global__ void k() {}\n"
    sha = hashlib.sha256(src.encode()).hexdigest()[:16]
    _fake_tree(tmp_path, src, sha)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("kern<1>", "wl", "k.cu") == 12345
    assert bench.recorded_traffic("kern<1>", "other", "k.cu") is None
    assert bench.recorded_traffic("other<1>", "wl", "k.cu") is None
    # the source changed since the capture: no traffic figure
    (tmp_path / "hierarchical_latent_key_gemm_b200" / "csrc" / "k.cu").write_text(src + "// edited\n")
    assert bench.recorded_traffic("kern<1>", "wl", "k.cu") is None


def test_traffic_record_over_several_source_files(tmp_path, monkeypatch):
    a, b = "__global__ void k() {}\n", "// helper header\n"
    sha = hashlib.sha256((a + b).encode()).hexdigest()[:16]
    csrc = tmp_path / "hierarchical_latent_key_gemm_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "k.cu").write_text(a)
    (csrc / "h.cuh").write_text(b)
    prof = tmp_path / "profiles"
    prof.mkdir()
    (prof / "traffic.txt").write_text(f"kern<1> | wl | k.cu+h.cuh | {sha} | 777 | test record\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("kern<1>", "wl", "k.cu+h.cuh") == 777
    (csrc / "h.cuh").write_text(b + "// edited\n")      # a change in any of the files voids it
    assert bench.recorded_traffic("kern<1>", "wl", "k.cu+h.cuh") is None


def test_traffic_record_absent(tmp_path, monkeypatch):
    (tmp_path / "hierarchical_latent_key_gemm_b200" / "csrc").mkdir(parents=True)
    (tmp_path / "hierarchical_latent_key_gemm_b200" / "csrc" / "k.cu").write_text("x")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.recorded_traffic("kern<1>", "wl", "k.cu") is None


def test_profiles_are_text_summaries_with_their_commands():
    prof = os.path.join(ROOT, "profiles")
    names = sorted(os.listdir(prof))
    assert names, "no profile summaries"
    for n in names:
        assert n.endswith((".md", ".txt")), f"{n}: profiles/ holds text summaries only"
        if n.endswith(".md"):
            text = open(os.path.join(prof, n)).read()
            assert "ncu " in text, f"{n}: no ncu command"
            assert "--clock-control none" in text, f"{n}: ncu without --clock-control none"
            assert "bench.py" in text, f"{n}: the profiled command runs committed files"
