"""Host-side pieces of bench.py that need no GPU: the ncu DRAM traffic record
it reports beside the roofline, and the byte accounting that record shares
with the bench's own numbers."""
import json
import os

import bench
from scatter_gemm_b200 import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _record():
    with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
        return json.load(f)


def test_traffic_is_reported_only_for_the_sources_it_was_taken_on():
    d = bench.load_traffic()
    assert d is None or d["csrc_hash"] == bench.csrc_hash()
    # the hash covers every file the record names, and nothing else
    assert tuple(_record()["hashed_sources"]) == bench.EXPAND_SOURCES


def test_traffic_record_matches_the_sweep_byte_accounting():
    d = _record()
    assert d["op"] == "expand"
    # the mean algorithmic bytes of one expand over the bench's qkv sweep
    alg = [W.bytes_expand(W.make_problem("qkv", seed=0, tok=t)) for t in W.QKV_TOK_SWEEP]
    assert d["algorithmic_bytes_per_launch"] == round(sum(alg) / len(alg))
    # DRAM traffic above the algorithmic bytes would mean re-reads; below them
    # (dirty base rows still in the L2 when the kernel ends, and the L2-resident
    # inputs of the small sizes) is expected under the flush-then-run method
    assert 0 < d["dram_bytes_per_launch"] <= 1.1 * d["algorithmic_bytes_per_launch"]
    assert 0 < d["shrink_dram_bytes_per_launch"]
