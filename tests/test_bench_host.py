"""bench.py host helpers (CPU only): the DRAM traffic of a launch taken from a committed capture --
directly, or scaled from a smaller case of the same kernel by algorithmic bytes, and dropped once the
kernel source has changed -- and the size of the CPU oracle's sample."""
import hashlib
import json
import os

import bench
from grouped_sparse_gemm_b200 import inputs


def _fake_root(tmp_path, entries, src=b"kernel source v1"):
    (tmp_path / "profiles").mkdir()
    csrc = tmp_path / "grouped_sparse_gemm_b200" / "csrc"
    csrc.mkdir(parents=True)
    (csrc / "gsg_gemm.cu").write_bytes(src)
    sha = hashlib.sha256(src).hexdigest()[:16]
    for e in entries.values():
        e.setdefault("gemm_src_sha", sha)
    (tmp_path / "profiles" / "gemm_traffic.json").write_text(json.dumps(entries))
    return str(tmp_path)


def test_traffic_direct_and_scaled(tmp_path, monkeypatch):
    root = _fake_root(tmp_path, {
        "small": {"dram_bytes_per_launch": 1000},
        "big": {"scaled_from": "small", "dram_bytes_per_launch_captured": 990, "algorithmic_bytes_captured": 1000}})
    monkeypatch.setattr(bench, "ROOT", root)
    assert bench.traffic_from_profiles("small", 1000)[0] == 1000
    b, how = bench.traffic_from_profiles("big", 6000)
    assert b == 5940 and "scaled" in how                 # 0.99 of the algorithmic bytes, at any size
    assert bench.traffic_from_profiles("other", 10)[0] is None


def test_traffic_dropped_when_the_kernel_changed(tmp_path, monkeypatch):
    root = _fake_root(tmp_path, {"small": {"dram_bytes_per_launch": 1000, "gemm_src_sha": "0" * 16}})
    monkeypatch.setattr(bench, "ROOT", root)
    b, how = bench.traffic_from_profiles("small", 1000)
    assert b is None and "changed" in how


def test_committed_traffic_record_is_consistent():
    """The committed record scales a capture whose DRAM bytes are close to its algorithmic bytes."""
    with open(os.path.join(bench.ROOT, "profiles", "gemm_traffic.json")) as f:
        d = json.load(f)
    for name, e in d.items():
        if e.get("scaled_from"):
            assert e["scaled_from"] in inputs.CONFIGS and name in inputs.CONFIGS
            r = e["dram_bytes_per_launch_captured"] / e["algorithmic_bytes_captured"]
            assert 0.9 < r < 1.2


def test_cpu_sample_size():
    assert bench.cpu_sample_experts(inputs.CONFIGS["30b_up_prefill"], None) == 24
    assert bench.cpu_sample_experts(inputs.CONFIGS["1t_up_prefill"], None) == 4
    assert bench.cpu_sample_experts(inputs.CONFIGS["1t_up_prefill"], 7) == 7


def test_binding_roof_of_the_workloads():
    """HBM binds every expert-projection workload; the tensor pipe binds the 65,536-token extra
    (the roofs: measured bf16 burst x 8 and the measured HBM copy, or the fallback figures)."""
    peaks, _ = bench.measured_peaks()
    tensor, hbm = float(peaks["bf16_tflops"]) * 8.0, float(peaks["hbm_gbs"])
    for name, cfg in inputs.CONFIGS.items():
        touched = min(cfg.E, cfg.R)
        nbytes = touched * cfg.N * cfg.K * 11 // 32 + cfg.R * cfg.K // 2 + cfg.R * cfg.K // 32 + cfg.R * cfg.N * 2
        flops = 2.0 * cfg.R * cfg.N * cfg.K
        assert bench.tensor_roof_binds(flops, nbytes, tensor, hbm) == name.startswith("1t_up_prefill_65k"), name
    # the ridge point: flop/B = tensor / hbm
    ridge = tensor * 1e12 / (hbm * 1e9)
    assert bench.tensor_roof_binds(1.01 * ridge, 1.0, tensor, hbm)
    assert not bench.tensor_roof_binds(0.99 * ridge, 1.0, tensor, hbm)

