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


def _profile_record(path, key):
    import re
    text = open(path).read()
    sha = re.search(key + r":\s*([0-9a-f]{16})", text)
    dram = re.search(r"dram_bytes_per_launch:\s*([0-9]+)", text)
    return sha.group(1), int(dram.group(1))


def test_recorded_traffic_only_while_the_profiled_sources_hash_the_same(monkeypatch):
    """A committed ncu figure is reported only for the sources it was taken on."""
    import glob
    import os
    decode = sorted(glob.glob(os.path.join(bench.ROOT, "profiles",
                                           "paged_attention_decode_*.md")))
    prefill = sorted(glob.glob(os.path.join(bench.ROOT, "profiles", "prefill_tc_*.md")))
    assert decode and prefill
    now_d = bench.source_sha(bench.DECODE_SOURCES)
    now_p = bench.source_sha(bench.PREFILL_SOURCES)
    for path in decode:
        cfg = os.path.basename(path)[len("paged_attention_decode_"):-3]
        sha, dram = _profile_record(path, "decode_source_sha256_16")
        assert bench.recorded_traffic(cfg) == (dram if sha == now_d else None)
    for path in prefill:
        cfg = os.path.basename(path)[len("prefill_tc_"):-3]
        sha, dram = _profile_record(path, "prefill_source_sha256_16")
        assert bench.recorded_prefill_traffic(cfg) == (dram if sha == now_p else None)
    # both branches, whatever the committed sources hash to: the figure while the
    # hash matches, none after any change
    for path in decode:
        cfg = os.path.basename(path)[len("paged_attention_decode_"):-3]
        sha, dram = _profile_record(path, "decode_source_sha256_16")
        monkeypatch.setattr(bench, "source_sha", lambda names=None, s=sha: s)
        assert bench.recorded_traffic(cfg) == dram
        monkeypatch.setattr(bench, "source_sha", lambda names=None: "0" * 16)
        assert bench.recorded_traffic(cfg) is None
    for path in prefill:
        cfg = os.path.basename(path)[len("prefill_tc_"):-3]
        sha, dram = _profile_record(path, "prefill_source_sha256_16")
        monkeypatch.setattr(bench, "source_sha", lambda names=None, s=sha: s)
        assert bench.recorded_prefill_traffic(cfg) == dram
        monkeypatch.setattr(bench, "source_sha", lambda names=None: "0" * 16)
        assert bench.recorded_prefill_traffic(cfg) is None
    # and a workload without a profile has none
    monkeypatch.undo()
    assert bench.recorded_traffic("no_such_workload") is None
