"""Host-side logic of bench.py that needs no GPU: the roofline arithmetic, the
ncu traffic lookup (valid only for the kernel source it was captured on) and
the workload bookkeeping."""
import json
import os
import shutil

import pytest

import bench


def test_gemm_algorithmic_bytes_counts_weights_once_per_layer():
    from dynamic_layer_wise_b200 import inputs as I
    shape = I.LLADA_8B
    rows = [65] * shape.n_layers
    total, launches = bench.gemm_algorithmic_bytes(shape, rows)
    assert launches == 4 * shape.n_layers
    w_layer = sum(o * i for o, i in shape.weight_shapes().values()) * 2
    # weights dominate: 436 MB per layer; the 65-row activations and outputs add ~2 %
    act = sum(65 * (n_out + K) * 2 for n_out, K in [(12288, 4096), (4096, 4096), (24576, 4096), (4096, 12288)])
    assert total == pytest.approx(shape.n_layers * (w_layer + act))
    assert total < 1.03 * w_layer * shape.n_layers


def test_step_bytes_include_lm_head_and_kv_stream():
    from dynamic_layer_wise_b200 import inputs as I
    shape = I.LLADA_8B
    rows = [65] * shape.n_layers
    b = bench.step_algorithmic_bytes(shape, rows, 1024, 1, 256)
    w = shape.n_layers * sum(o * i for o, i in shape.weight_shapes().values()) * 2
    lm = shape.vocab * shape.d_model * 2
    kv = shape.n_layers * 2 * shape.n_kv_heads * 1024 * shape.head_dim * 2
    assert b > w + lm + kv
    assert abs(b / 1e9 - 15.57) < 0.05          # the 15.5 GB quoted for this workload


def test_traffic_lookup_requires_matching_source(tmp_path, monkeypatch):
    root = tmp_path / "repo"
    (root / "profiles").mkdir(parents=True)
    csrc = root / "dynamic_layer_wise_b200" / "csrc"
    csrc.mkdir(parents=True)
    for f in bench.GEMM_SOURCES:
        shutil.copy(os.path.join(bench.ROOT, "dynamic_layer_wise_b200", "csrc", f), csrc / f)
    monkeypatch.setattr(bench, "ROOT", str(root))
    sha = bench.kernel_source_sha(bench.GEMM_SOURCES)
    entry = {"k_gemm_tc": {"source_sha": sha, "dram_bytes": 110e6, "algorithmic_bytes": 100e6}}
    (root / "profiles" / "traffic.json").write_text(json.dumps(entry))
    # scaled from the captured launch to the average launch by algorithmic bytes
    assert bench.traffic_for("k_gemm_tc", bench.GEMM_SOURCES, 50e6) == pytest.approx(55e6)
    # any change of the kernel's sources invalidates the stored figure
    (csrc / "gemm_tc.h").write_text((csrc / "gemm_tc.h").read_text() + "\n// edited\n")
    assert bench.traffic_for("k_gemm_tc", bench.GEMM_SOURCES, 50e6) is None
    assert bench.traffic_for("absent", bench.GEMM_SOURCES, 50e6) is None


def test_committed_traffic_entry_is_well_formed():
    p = os.path.join(bench.ROOT, "profiles", "traffic.json")
    with open(p) as fh:
        t = json.load(fh)
    e = t["k_gemm_tc"]
    assert e["dram_bytes"] > 0 and e["algorithmic_bytes"] > 0
    assert 0.9 < e["dram_bytes"] / e["algorithmic_bytes"] < 1.5   # weights read once, no re-reads
