"""Host-side helpers of bench.py on CPU: the GEMM source hash that keys the
recorded ncu traffic (comments do not count, code does), the traffic lookup,
and the config description of a projection subset."""
import os
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
import workloads  # noqa: E402


def _tree(tmp_path, gemm_text, common_text="int x;\n"):
    d = tmp_path / "fp8_tensor_scaled_b200" / "csrc"
    d.mkdir(parents=True)
    (d / "gemm_sm100.cu").write_text(gemm_text)
    (d / "common.cuh").write_text(common_text)
    return str(tmp_path)


def test_source_hash_ignores_comments_and_blank_lines(tmp_path, monkeypatch):
    a = _tree(tmp_path / "a", "int f() { return 1; }  // one\n\n// note\n")
    b = _tree(tmp_path / "b", "// another note\nint f() { return 1; }\n")
    c = _tree(tmp_path / "c", "int f() { return 2; }\n")
    hashes = []
    for root in (a, b, c):
        monkeypatch.setattr(bench, "ROOT", root)
        hashes.append(bench.gemm_source_hash())
    assert hashes[0] == hashes[1] != hashes[2]


def test_traffic_lookup_of_the_committed_profile():
    # the profile records a per-launch byte count between the algorithmic
    # minimum (0.62 GB) and a few times it; when the GEMM code changed since
    # the capture the lookup is None (bench.py then reports traffic null)
    t = bench.gemm_traffic_per_launch()
    if t is None:
        pytest.skip("GEMM code changed since the recorded capture")
    assert 0.6e9 < t < 2.5e9


def test_traffic_is_null_when_the_code_changed(tmp_path, monkeypatch):
    root = _tree(tmp_path / "x", "int changed;\n")
    os.makedirs(os.path.join(root, "profiles"))
    with open(os.path.join(ROOT, "profiles", "fp8_gemm_llama2_70b_traffic.md")) as f:
        text = f.read()
    with open(os.path.join(root, "profiles", "fp8_gemm_llama2_70b_traffic.md"), "w") as f:
        f.write(text)
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.gemm_traffic_per_launch() is None


def test_config_of_a_projection_subset():
    full = bench.config_dict(workloads.C3, 1)
    sub = bench.config_dict(workloads.C3, 1, [3])
    assert full["workload"] == workloads.C3.name and len(full["linears"]) == 4
    assert sub["workload"] == workloads.C3.name + "-projections-3"
    assert sub["linears"] == ["down 28672->8192"]
