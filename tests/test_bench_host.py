"""Host-side logic of bench.py (no GPU): the algorithmic work the roofline divides by, the
choice of bound, the measured-traffic lookup and its invalidation, and the replica batches.

The expected numbers are written out from the layer's definition (bytes of the touched
experts' weights, 6 d F FLOPs per processed row), not from bench.py itself.
"""
import hashlib
import json
import os

import numpy as np
import pytest

import bench
from workloads import WORKLOADS


def test_algorithmic_work_decode_bf16():
    wl = WORKLOADS["decode"]
    counts = np.zeros(wl.E, np.int64)
    counts[:97] = 1                       # 97 touched routed experts
    w = bench.algorithmic_work(wl, counts)
    per_expert = 3 * 2048 * 6144 * 2      # gate, up, down in bf16
    assert w["touched_experts"] == 97
    assert w["gate_up_bytes"] == 98 * 2 * 2048 * 6144 * 2
    assert w["down_bytes"] == 98 * 2048 * 6144 * 2
    assert w["layer_bytes"] == 98 * per_expert + 256 * 6144 * 4 + 2 * 16 * 6144 * 2
    rows = 16 * 8 + 16
    assert w["expert_flops"] == 6 * 6144 * 2048 * rows
    assert w["gate_up_flops"] + w["down_flops"] == w["expert_flops"]
    assert w["router_flops"] == 2 * 16 * 6144 * 256


def test_algorithmic_work_fp8_counts_codes_and_scales():
    wl = WORKLOADS["decode_fp8"]
    counts = np.ones(wl.E, np.int64)
    w = bench.algorithmic_work(wl, counts)
    # one byte per code plus one scale byte per 32 codes
    assert w["gate_up_bytes"] == int(257 * 2 * 2048 * 6144 * (1 + 1 / 32))
    assert w["down_bytes"] == int(257 * 2048 * 6144 * (1 + 1 / 32))


def test_bound_follows_the_machine_balance():
    peaks = {"hbm_gbs": 6546.9, "bf16_tflops": 1676.5}
    for name, bound_hbm in (("decode", True), ("batched_decode", True), ("decode_fp8", True)):
        wl = WORKLOADS[name]
        w = bench.algorithmic_work(wl, np.ones(wl.E, np.int64))
        assert bench.hbm_bound(wl, w, peaks) is bound_hbm, name
    # prefill: 4 d F FLOPs per processed row over 4 F d bytes of gate+up weights per expert,
    # i.e. rows / (E + 1) = (8192 * 8 + 8192) / 257 = 286.9 FLOP/B, above the balance point
    # 1676.5e12 / 6546.9e9 = 256.1 FLOP/B: tensor bound
    wl = WORKLOADS["prefill"]
    counts = np.full(wl.E, 256, np.int64)
    w = bench.algorithmic_work(wl, counts)
    intensity = w["gate_up_flops"] / w["gate_up_bytes"]
    assert abs(intensity - (wl.T * wl.k + wl.T) / (wl.E + 1)) < 1e-9
    assert bench.hbm_bound(wl, w, peaks) is False


def test_measured_traffic_lookup_and_invalidation(tmp_path, monkeypatch):
    src_dir = tmp_path / "mixture_experts_layer_47_b200" / "csrc"
    src_dir.mkdir(parents=True)
    (tmp_path / "profiles").mkdir()
    kernel = src_dir / "k.cu"
    kernel.write_text("// kernel v1\n")
    sha = hashlib.sha256(kernel.read_bytes()).hexdigest()
    table = {
        "gate_up_gemm/hbm": {"bound": "hbm", "bytes_per_touched_expert": 1000,
                             "kernel_source": "k.cu", "kernel_source_sha256": sha,
                             "d_model": 6144, "d_ff": 2048},
        "gate_up_gemm/hbm/fp8": {"bound": "hbm", "bytes_per_touched_expert": 520,
                                 "kernel_source": "k.cu", "kernel_source_sha256": sha},
        "gate_up_gemm/hbm/fp8_mma": {"bound": "hbm", "bytes_per_touched_expert": 530,
                                     "kernel_source": "k.cu", "kernel_source_sha256": sha},
    }
    (tmp_path / "profiles" / "traffic.json").write_text(json.dumps(table))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    monkeypatch.delenv("MOE_GEMM_TILES", raising=False)
    assert bench.measured_traffic("gate_up_gemm", "hbm", 10) == 10000
    # FP8: the warp-MMA form's capture up to 16 tokens, the tcgen05 kernel's above or when a
    # tiling is picked
    assert bench.measured_traffic("gate_up_gemm", "hbm", 10, "fp8", T=16) == 5300
    assert bench.measured_traffic("gate_up_gemm", "hbm", 10, "fp8", T=256) == 5200
    monkeypatch.setenv("MOE_GEMM_TILES", "swap")
    assert bench.measured_traffic("gate_up_gemm", "hbm", 10, "fp8", T=16) == 5200
    monkeypatch.delenv("MOE_GEMM_TILES")
    # the dense layer has entries of its own (one expert of its width per launch)
    assert bench.measured_traffic("gate_up_gemm", "hbm", 1, "bf16", 6144, 2048,
                                  layer="dense") is None
    assert bench.measured_traffic("gate_up_gemm", "tensor", 10) is None   # no entry
    assert bench.measured_traffic("down_gemm", "hbm", 10) is None
    assert bench.measured_traffic("gate_up_gemm", "hbm", 1, "bf16", 6144, 18432) is None
    kernel.write_text("// kernel v2\n")                                     # source changed
    assert bench.measured_traffic("gate_up_gemm", "hbm", 10) is None


def test_committed_traffic_table_names_existing_sources():
    path = os.path.join(os.path.dirname(os.path.dirname(__file__)), "profiles", "traffic.json")
    with open(path) as f:
        table = json.load(f)
    assert table, "profiles/traffic.json is empty"
    for key, entry in table.items():
        kernel, bound = key.split("/")[:2]
        assert kernel in ("gate_up_gemm", "down_gemm") and bound in ("hbm", "tensor")
        assert entry["bound"] == bound and entry["bytes_per_touched_expert"] > 0
        src = os.path.join(bench.ROOT, "mixture_experts_layer_47_b200", "csrc",
                           entry["kernel_source"])
        assert os.path.exists(src), src


@pytest.mark.parametrize("name", ["decode", "prefill"])
def test_replica_batches_differ_per_rank_and_are_reproducible(name):
    wl = WORKLOADS[name]
    a1, a2, b1 = bench.rank_batch(wl, 1), bench.rank_batch(wl, 1), bench.rank_batch(wl, 2)
    assert a1.shape == (wl.T, wl.d)
    assert a1.equal(a2) and not a1.equal(b1)


def test_algorithmic_work_dense_layer():
    """The dense first layer: all of its weights, x and y; no router."""
    wl = WORKLOADS["dense_decode"]
    w = bench.algorithmic_work(wl, np.array([wl.T]))
    assert w["touched_experts"] == 1
    assert w["layer_bytes"] == 3 * 18432 * 6144 * 2 + 2 * 16 * 6144 * 2
    assert w["router_flops"] == 0
    assert w["expert_flops"] == 6 * 6144 * 18432 * 16
    peaks = {"hbm_gbs": 6546.9, "bf16_tflops": 1676.5}
    assert bench.hbm_bound(wl, w, peaks)
    pre = WORKLOADS["dense_prefill"]
    assert not bench.hbm_bound(pre, bench.algorithmic_work(pre, np.array([pre.T])), peaks)
