"""The benchmark's roofline numerators, pinned against literal enumeration (CPU).

bench.py reports achieved bandwidth as algorithmic bytes over time and prefill
throughput as useful FLOPs over time.  Here the closed forms it uses are checked
against counts built element by element on small workloads: every K/V row a
decode must read, every distinct (block, row) a shared-prefix decode must read,
and every (query head, visible key) pair of a causal chunk.
"""

import numpy as np

import bench
from paged_kv_cache_413_b200 import workloads as W


def test_decode_bytes_enumerated():
    for name, over in [("tiny", {}), ("llama2_70b_gqa", {"num_seqs": 5})]:
        wl = W.make_workload(name, **over)
        cfg = wl.cfg
        elt = W.ELT_BYTES
        total = 0
        for L in wl.seq_lens.numpy():
            for _kvh in range(cfg.num_kv_heads):
                for _tok in range(int(L)):
                    total += 2 * cfg.head_dim * elt[cfg.cache_dtype]      # K row + V row
            total += cfg.num_heads * cfg.head_dim * (elt[cfg.q_dtype] + elt[cfg.out_dtype])
            total += 4 * (-(-int(L) // cfg.block_size)) + 4                 # table + length
        assert bench.decode_bytes(wl, cfg.out_dtype) == total


def test_unique_kv_bytes_counts_each_shared_row_once():
    wl = W.make_workload("beam_cow_fp8", num_seqs=3)
    cfg = wl.cfg
    bt, lens = wl.block_tables.numpy(), wl.seq_lens.numpy()
    rows = set()
    for i, L in enumerate(lens):
        for pos in range(int(L)):
            rows.add((int(bt[i, pos // cfg.block_size]), pos % cfg.block_size))
    per_row = cfg.num_kv_heads * cfg.head_dim * 2 * W.ELT_BYTES[cfg.cache_dtype]
    assert bench.unique_kv_bytes(wl) == len(rows) * per_row
    # and sharing saves: the per-sequence count is larger
    assert bench.unique_kv_bytes(wl) < int(lens.sum()) * per_row


def test_prefill_flops_enumerated():
    wl = W.make_prefill_workload(3, (5, 40), (1, 12), num_heads=8, num_kv_heads=2,
                                 head_dim=128, dtype="bf16", seed=1)
    cfg = wl.cfg
    L, qs = wl.seq_lens.numpy(), wl.query_start.numpy()
    pairs = 0
    for i in range(len(L)):
        q = int(qs[i + 1] - qs[i])
        for j in range(q):
            pos = int(L[i]) - q + j
            for _key in range(pos + 1):
                pairs += 1
    assert bench.prefill_flops(wl) == pairs * cfg.num_heads * cfg.head_dim * 4


def test_recorded_traffic_only_while_the_profiled_sources_hash_the_same(monkeypatch, tmp_path):
    """A recorded ncu figure is reported only for the sources it was taken on."""
    import json

    sha = bench.source_sha(bench.DECODE_SOURCES)
    rec = {"workloads": {
        "fresh": {"sources": list(bench.DECODE_SOURCES), "sources_sha256_16": sha,
                  "dram_bytes_per_launch": 1234},
        "stale": {"sources": list(bench.DECODE_SOURCES), "sources_sha256_16": "0" * 16,
                  "dram_bytes_per_launch": 99}}}
    path = tmp_path / "traffic.json"
    path.write_text(json.dumps(rec))
    monkeypatch.setattr(bench, "TRAFFIC_JSON", str(path))
    assert bench.recorded_traffic("fresh") == 1234
    assert bench.recorded_traffic("stale") is None
    assert bench.recorded_traffic("no_such_workload") is None
    # any change to a listed source retires the figure
    monkeypatch.setattr(bench, "source_sha", lambda names=None: "f" * 16)
    assert bench.recorded_traffic("fresh") is None
    monkeypatch.setattr(bench, "TRAFFIC_JSON", str(tmp_path / "missing.json"))
    assert bench.recorded_traffic("fresh") is None


def test_committed_traffic_records_are_complete():
    """Every committed record names existing sources, a summary under profiles/
    and the capture command, and carries a positive byte count."""
    import json
    import os

    with open(bench.TRAFFIC_JSON) as f:
        rec = json.load(f)["workloads"]
    for name, r in rec.items():
        for src in r["sources"]:
            assert os.path.exists(os.path.join(bench.ROOT, "paged_kv_cache_413_b200", "csrc", src))
        assert len(r["sources_sha256_16"]) == 16
        assert int(r["dram_bytes_per_launch"]) > 0
        assert os.path.exists(os.path.join(bench.ROOT, "profiles", r["summary"])), name
        assert "ncu" in r["command"] and "--clock-control none" in r["command"]


def test_committed_traffic_records_match_the_sources():
    """No committed record is stale: the sources of every workload's captured kernel
    still hash to the value recorded with its ncu capture, so bench.py reports each
    traffic figure (a kernel edit without a new capture fails here)."""
    import json

    with open(bench.TRAFFIC_JSON) as f:
        names = list(json.load(f)["workloads"])
    assert names
    for name in names:
        assert bench.recorded_traffic(name) is not None, f"{name}: sources changed since the capture"
