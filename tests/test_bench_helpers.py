"""bench.py host helpers (CPU): the traffic record is used only while the
kernel sources it names are unchanged, and the algorithmic byte counts follow
the workloads' shapes."""
import os
import shutil

import bench


def test_traffic_record_follows_its_sources(tmp_path, monkeypatch):
    csrc = tmp_path / "moe_expert_routing_token_b200" / "csrc"
    (tmp_path / "profiles").mkdir()
    csrc.mkdir(parents=True)
    (csrc / "a.cuh").write_text("kernel A v1\n")
    (csrc / "b.cu").write_text("host code\n")
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    sha = bench.kernel_source_hash(["a.cuh"])
    (tmp_path / "profiles" / "traffic_sigmoid_M64.txt").write_text(
        f"kernel_sources: a.cuh\nkernel_source_sha: {sha}\ndram_bytes_per_launch: 12345\n")
    assert bench.profiled_traffic("sigmoid", 64) == 12345.0
    (csrc / "b.cu").write_text("host code, changed\n")      # not a listed source: still valid
    assert bench.profiled_traffic("sigmoid", 64) == 12345.0
    (csrc / "a.cuh").write_text("kernel A v2\n")             # the kernel changed: no number
    assert bench.profiled_traffic("sigmoid", 64) is None
    assert bench.profiled_traffic("sigmoid", 128) is None    # no record for that size


def test_algorithmic_bytes():
    # bf16 E=256, k=8: 512 B of logits + 64 B of outputs per token + the 1 KiB bias
    assert bench.algorithmic_bytes("sigmoid", 16384) == 16384 * (512 + 64) + 1024
    # fp32 E=160, k=6, no bias
    assert bench.algorithmic_bytes("grouped", 16384) == 16384 * (640 + 48)
    # fused: hidden + weight + outputs + bias
    assert bench.algorithmic_bytes("fused", 8192) == 8192 * 7168 * 2 + 7168 * 256 * 2 + 8192 * 64 + 1024
    assert bench.perm_bytes(16384) == 16384 * 8 * 20 + (2 * 256 + 1) * 4


def test_top1_workload():
    from moe_expert_routing_token_b200 import inputs
    # hidden + the (E, K) weight + one (weight, id) pair per token; no bias
    assert bench.algorithmic_bytes("top1", 8192) == 8192 * 7168 * 2 + 8 * 7168 * 2 + 8192 * 8
    d = bench.workload_desc("top1", 64)
    assert d["K"] == 7168 and d["softcap"] == 30.0 and d["E"] == 8 and d["topk"] == 1
    x = inputs.make("top1", 6)
    assert tuple(x["hidden"].shape) == (6, 7168) and tuple(x["weight"].shape) == (8, 7168)
    assert x["bias"] is None and "logits" not in x
    r, _ = bench.oracle_call("top1", x, slice(0, 6))
    assert r.ids.shape == (6, 1) and (r.weights > 0).all() and (r.weights <= 1).all()
    # the new workload leaves the other workloads' seeds (and so their draws) as they were
    assert [inputs.default_seed(n, 16384) for n in ("softmax", "sigmoid", "biased", "grouped", "fused")] == \
        [1015, 2015, 3015, 4015, 5015]


def test_metric_labels():
    # the default workload keeps the headline metric's exact text
    assert bench.metric_for("sigmoid") == bench.METRIC == \
        "routed tokens/s & µs/call (E=256,k=8 biased grouped top-k); % of HBM roofline"
    assert bench.metric_for("biased") == bench.METRIC
    assert "E=8" in bench.metric_for("top1") and "tensor" in bench.metric_for("fused")
