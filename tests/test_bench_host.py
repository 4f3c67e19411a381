"""Host logic of bench.py (no GPU): the DRAM-traffic record it reports for
the heads call must belong to the committed kernel sources, and its
algorithmic byte counts must follow the workload's shapes."""
import hashlib
import json
import os

import bench
from speculative_decoding_medusa_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_heads_traffic_record_matches_the_sources():
    """The ncu record is taken on the sources it names; a kernel change
    without a new capture would make the bench report no traffic."""
    with open(os.path.join(ROOT, "profiles", "heads_topk_traffic.json")) as f:
        rec = json.load(f)
    h = hashlib.sha256()
    for name in rec["source_files"]:
        with open(os.path.join(ROOT, name), "rb") as f:
            h.update(f.read())
    assert h.hexdigest() == rec["source_sha256"], "re-capture the heads DRAM traffic"
    per = rec["per_kernel"].values()
    assert rec["dram_bytes_per_call"] == sum(k["dram_read"] + k["dram_write"] for k in per)
    assert abs(rec["traffic_ratio"] - rec["dram_bytes_per_call"]
               / rec["algorithmic_bytes_per_call"]) < 1e-4
    traffic, src = bench.heads_traffic(1e9)
    assert traffic is not None and abs(traffic / 1e9 - rec["traffic_ratio"]) < 1e-9, src


def test_algorithmic_bytes_of_the_bench_workload():
    """Llama-3-8B shape: 4 heads of (d^2 + d + V d) bf16 weights plus h; the
    KV prefix, tree Q/K/V/O and logits as the roofline counts them."""
    w = W.WORKLOADS["llama3_8b"]
    prefix = [6000] * w.B
    ab = bench.algorithmic_bytes(w, prefix, w.N)
    assert ab["heads"] == w.K * (w.d * w.d + w.d + w.V * w.d) * 2 + w.B * w.d * 2
    assert ab["verify"] == w.B * w.N * w.V * 2
    kv = sum(prefix) * w.Hkv * w.dh * 2 * 2
    tree = w.B * w.N * (w.Hq + 2 * w.Hkv + w.Hq + 2 * w.Hkv) * w.dh * 2
    assert ab["attention"] == kv + tree
    assert ab["total"] == ab["heads"] + ab["attention"] + ab["verify"]
