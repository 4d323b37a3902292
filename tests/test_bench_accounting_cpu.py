"""bench.py's algorithmic accounting (the numerator of every roofline fraction) against
the definitions it states, on a small layer computed by hand:

- weights: the pages' storage of 4-bit codes plus one fp16 scale and one fp16 zero
  point per group of 128 («Kimi 2.7 Moe 从 4 bit 存储到 INT8 拆解», section 2.3):
  0.5 B per weight + 4 B per group, only for the experts some token is routed to;
- ops: 2 multiply-adds' worth per weight and routed row (up: 2F x H, down: H x F);
- the up GEMM also reads the routed INT8 rows and writes h in bf16, the down GEMM
  reads the INT8 h rows and writes fp32 y2."""

import hashlib
import json
import os

import numpy as np

import bench
from w4a8_quantized_moe_token_b200 import synth


def test_moe_accounting_by_hand():
    W = synth.Workload("hand", "moe", E=8, topk=2, T=5, H=300, F=200, routing="uniform")
    ids = np.array([[0, 3], [3, 5], [5, 0], [0, 3], [7, 3]], dtype=np.int32)  # experts 0, 3, 5, 7 touched
    acc = bench.moe_accounting(W, ids)
    touched, slots = 4, 10
    Hp, Fp = 384, 256  # H and F padded to whole groups of 128
    up_w = touched * (2 * 200 * Hp * 0.5 + 2 * 200 * (Hp // 128) * 4)
    dn_w = touched * (300 * Fp * 0.5 + 300 * (Fp // 128) * 4)
    assert acc["touched_experts"] == touched
    assert acc["weight_bytes"] == up_w + dn_w
    assert acc["kernel_ops"]["gemm_up"] == 2 * slots * (2 * 200) * 300
    assert acc["kernel_ops"]["gemm_down"] == 2 * slots * 300 * 200
    kb = acc["kernel_bytes"]
    assert kb["gemm_up"] == up_w + slots * Hp + slots * 200 * 2
    assert kb["gemm_down"] == dn_w + slots * Fp + slots * 300 * 4
    assert kb["requant"] == slots * 200 * 2 + slots * Fp
    assert kb["combine"] == slots * 300 * 4 + 5 * 300 * 2 + slots * 8


def test_weight_bytes_per_weight_at_group_128():
    # 0.5 B + 4 B / 128 = 0.53125 B per weight when K is a multiple of the group
    assert bench.packed_matrix_bytes(4096, 7168) == 4096 * 7168 * 0.53125


def test_traffic_is_dropped_when_a_source_changes(tmp_path, monkeypatch):
    src = tmp_path / "k.cu"
    src.write_text("kernel v1\n")
    prof = tmp_path / "profiles"
    prof.mkdir()
    entry = {"kernel": "gemm_up", "dram_bytes_per_launch": 1234,
             "sources": {"k.cu": hashlib.sha256(b"kernel v1\n").hexdigest()}}
    (prof / "dram_traffic.json").write_text(json.dumps({"wl": entry}))
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.load_traffic("wl", "gemm_up") == 1234.0
    assert bench.load_traffic("wl", "gemm_down") is None
    assert bench.load_traffic("other", "gemm_up") is None
    src.write_text("kernel v2\n")
    assert bench.load_traffic("wl", "gemm_up") is None


def test_committed_traffic_entries_are_well_formed():
    """Each committed traffic figure names its kernel, a positive byte count, the
    capture command and the existing source files it was taken on (the bench drops it
    by itself once one of them changes)."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    with open(os.path.join(root, "profiles", "dram_traffic.json")) as f:
        d = json.load(f)
    entries = {k: v for k, v in d.items() if not k.startswith("_")}
    assert entries
    for wl, e in entries.items():
        assert e["kernel"] and e["dram_bytes_per_launch"] > 0 and e["capture"].startswith("ncu "), wl
        assert "--clock-control none" in e["capture"], wl
        assert e["sources"], wl
        for rel, digest in e["sources"].items():
            assert os.path.exists(os.path.join(root, rel)) and len(digest) == 64, (wl, rel)
