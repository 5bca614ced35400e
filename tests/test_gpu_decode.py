"""GPU parity of paged decode attention against the oracle, through the C ABI.

Tolerance (max-abs over every output element): 8e-3 for fp16/bf16 outputs,
1e-3 for fp32 outputs.  Cases:
  * each workload scaled down so the oracle checks every output, several
    partition sizes (so the log-sum-exp reduce runs), every output type;
  * each workload at full size in the launch configuration the benchmark times,
    checked on sampled sequences;
  * GQA group sizes 1, 2, 3, 4, 8, 16 and head_dim 64 / 128, FP8 with fp16 and
    bf16 queries;
  * edge cases: empty context, one token, block and partition boundaries,
    lengths past the launch bound, block ids outside the pool, workspace errors;
  * invariants that must hold exactly on the GPU too: the output does not depend
    on where the blocks sit in the pool, and runs are bitwise repeatable.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_413_b200 as pa
from paged_kv_cache_413_b200 import workloads as W

import flow

pytestmark = pytest.mark.gpu


def _check(wl, out_dtype="f16", partition=0, seqs=None, prompts=None):
    d = flow.to_device(wl)
    flow.gpu_prepare(wl, d)
    out = flow.gpu_step(wl, d, out_dtype, partition)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    kc, vc = flow.oracle_caches(wl, prompts=prompts)
    ref = flow.oracle_decode(wl, kc, vc, seqs)
    got = out if seqs is None else out[torch.as_tensor(seqs, device=out.device)]
    err = flow.max_abs_err(got, ref)
    assert err <= flow.TOL[out_dtype], f"max abs error {err:.3e} > {flow.TOL[out_dtype]}"
    return out, err


@pytest.mark.parametrize("out_dtype", ["f16", "f32"])
@pytest.mark.parametrize("partition", [0, 16, 32, 48, 64])
def test_tiny(out_dtype, partition):
    wl = W.make_workload("tiny")
    _check(wl, out_dtype, partition)


@pytest.mark.parametrize("name,over,part", [
    ("llama2_7b", dict(num_seqs=6), 0),
    ("llama2_7b", dict(num_seqs=6), 256),
    ("llama2_70b_gqa", dict(num_seqs=10), 0),
    ("llama2_70b_gqa", dict(num_seqs=10), 128),
    ("long_splitk", dict(num_seqs=2, seq_lens=(4100, 2999)), 512),
    ("beam_cow_fp8", dict(num_seqs=3, shared_len=72), 0),
    ("beam_cow_fp8", dict(num_seqs=3, shared_len=1032), 256),
])
@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_scaled_workloads(name, over, part, out_dtype):
    wl = W.make_workload(name, **over)
    if out_dtype == "bf16" and wl.cfg.q_dtype == "f16":
        out_dtype = "f16"
    _check(wl, out_dtype, part)


@pytest.mark.parametrize("h,hkv,d,dt", [
    (8, 4, 128, "f16"), (6, 2, 128, "bf16"), (16, 4, 64, "bf16"), (64, 8, 64, "f16"),
    (32, 2, 128, "bf16"), (4, 4, 64, "bf16"), (24, 8, 128, "f16")])
def test_group_sizes(h, hkv, d, dt):
    cfg = W.DecodeConfig("gqa", num_seqs=5, seq_len_range=(1, 300), num_heads=h,
                         num_kv_heads=hkv, head_dim=d, q_dtype=dt, cache_dtype=dt, out_dtype=dt,
                         seed=h * 100 + hkv + d)
    for part in (0, 64):
        _check(W.make_workload(cfg), dt, part)


@pytest.mark.parametrize("qdt", ["f16", "bf16"])
@pytest.mark.parametrize("d,h,hkv", [(128, 32, 8), (64, 8, 8), (128, 8, 1)])
def test_fp8_cache(qdt, d, h, hkv):
    wl = W.make_workload("beam_cow_fp8", num_seqs=2, shared_len=40, head_dim=d, num_heads=h,
                         num_kv_heads=hkv, q_dtype=qdt, seed=d + h)
    _check(wl, qdt, 0)
    _check(wl, "f32", 16)


def test_edge_lengths():
    """Empty context (zero output), one token (returns V0), 16 = one full block,
    17, and partition boundaries 511/512/513/1024 with 512-token partitions."""
    lens = (0, 1, 16, 17, 511, 512, 513, 1024, 1025)
    cfg = W.DecodeConfig("edges", num_seqs=len(lens), seq_lens=lens, num_heads=8,
                         num_kv_heads=2, head_dim=128, q_dtype="bf16", cache_dtype="bf16",
                         out_dtype="bf16", seed=9)
    wl = W.make_workload(cfg)
    for part in (0, 512, 16):
        out, _ = _check(wl, "f32", part)
        assert torch.count_nonzero(out[0]).item() == 0


def test_one_token_returns_v_exactly():
    cfg = W.DecodeConfig("one", num_seqs=3, seq_lens=(1, 1, 1), num_heads=4, num_kv_heads=2,
                         head_dim=64, q_dtype="f16", cache_dtype="f16", out_dtype="f16", seed=3)
    wl = W.make_workload(cfg)
    d = flow.to_device(wl)
    out = flow.gpu_step(wl, d, "f16")
    v = wl.new_value.to(torch.float16).repeat_interleave(2, dim=1)
    assert torch.equal(out.cpu(), v)


def test_block_permutation_invariance_and_repeatability():
    """Same logical K/V in two physical layouts: bitwise-equal outputs; a second
    run is bitwise equal too (no order-dependent accumulation)."""
    wl = W.make_workload("llama2_70b_gqa", num_seqs=8)
    d = flow.to_device(wl)
    a = flow.gpu_step(wl, d, "bf16", 128)
    a2 = flow.gpu_step(wl, d, "bf16", 128)
    assert torch.equal(a, a2)
    nb = wl.num_blocks
    perm = torch.from_numpy(np.random.default_rng(0).permutation(nb)).cuda()
    kc2 = torch.empty_like(d.key_cache)
    vc2 = torch.empty_like(d.value_cache)
    kc2[perm] = d.key_cache
    vc2[perm] = d.value_cache
    bt = d.block_tables.long()
    bt2 = torch.where(bt >= 0, perm[bt.clamp(min=0)], bt).int()
    out = torch.empty_like(a)
    ws = flow.workspace_for(wl, 128)
    pa.pa_paged_attention_decode(out, d.query, kc2, vc2, bt2.contiguous(), d.seq_lens,
                                 max_seq_len=flow.max_seq_len(wl), scale=wl.scale,
                                 partition_size=128, workspace=ws)
    assert torch.equal(out, a)


def test_bad_device_data_sets_error_bits_without_fault():
    wl = W.make_workload("tiny")
    d = flow.to_device(wl)
    flow.gpu_step(wl, d, "f16")
    pa.pa_get_device_error()
    bt = d.block_tables.clone()
    bt[3, 2] = 10_000                      # outside the 64-block pool
    out = torch.empty(d.query.shape, dtype=torch.float16, device="cuda")
    pa.pa_paged_attention_decode(out, d.query, d.key_cache, d.value_cache, bt, d.seq_lens,
                                 max_seq_len=100, scale=wl.scale)
    assert pa.pa_get_device_error() & 0x2
    sl = d.seq_lens.clone()
    sl[1] = 500                            # past max_seq_len
    pa.pa_paged_attention_decode(out, d.query, d.key_cache, d.value_cache, d.block_tables, sl,
                                 max_seq_len=100, scale=wl.scale)
    assert pa.pa_get_device_error() & 0x4
    assert pa.pa_get_device_error() == 0


def test_workspace_errors():
    wl = W.make_workload("tiny")
    d = flow.to_device(wl)
    out = torch.empty(d.query.shape, dtype=torch.float16, device="cuda")
    need = pa.pa_paged_attention_workspace_size(4, 4, 4, 64, 100, 16)
    assert need > 0
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(pa.PaError, match="WORKSPACE"):
        pa.pa_paged_attention_decode(out, d.query, d.key_cache, d.value_cache, d.block_tables,
                                     d.seq_lens, max_seq_len=100, scale=wl.scale,
                                     partition_size=16, workspace=small)
    with pytest.raises(pa.PaError, match="WORKSPACE"):
        pa.pa_paged_attention_decode(out, d.query, d.key_cache, d.value_cache, d.block_tables,
                                     d.seq_lens, max_seq_len=100, scale=wl.scale,
                                     partition_size=16)


# ---- longest-first work order (units of >= 1024 tokens, <= 256 sequences) ----

@pytest.mark.parametrize("h,hkv,dt,part", [(8, 8, "f16", 2048), (32, 8, "bf16", 1024),
                                           (16, 2, "bf16", 1024)])
def test_longest_first_order_covers_every_sequence(h, hkv, dt, part):
    # ties, an empty context, one-token and multi-partition sequences; every output
    # of every sequence is compared
    rng = np.random.default_rng(h + hkv)
    lens = list(rng.integers(1, 3000, size=37)) + [0, 1, 700, 700, 700, 2999, 2999, 16, 17]
    cfg = W.DecodeConfig("lpt", num_seqs=len(lens), seq_lens=tuple(int(x) for x in lens),
                         num_heads=h, num_kv_heads=hkv, head_dim=128, q_dtype=dt,
                         cache_dtype=dt, out_dtype=dt, seed=h * hkv)
    _check(W.make_workload(cfg), dt, part)


# ---- full-size workloads, launch configuration of the benchmark, every output ----

def test_full_llama2_7b():
    # every sequence: this launch hands out sequences longest first, so a wrong
    # rank-to-sequence mapping would leave some outputs unwritten
    wl = W.make_workload("llama2_7b")
    _check(wl, "f16", wl.cfg.partition_size)


def test_full_llama2_70b_gqa():
    # every output of all 256 sequences, in the benchmark's launch configuration
    wl = W.make_workload("llama2_70b_gqa")
    _check(wl, "bf16", wl.cfg.partition_size)


def test_full_long_splitk():
    # every output of all 8 sequences (64 partitions each, merged by the reduce)
    wl = W.make_workload("long_splitk")
    _check(wl, "bf16", wl.cfg.partition_size)


def test_full_beam_cow_fp8():
    # the per-sequence decode of the copy-on-write step: every output of all 256 beams
    wl = W.make_workload("beam_cow_fp8")
    _check(wl, "bf16", wl.cfg.partition_size)


@pytest.mark.parametrize("bs", [32, 64, 128])
@pytest.mark.parametrize("name,over,part,out_dtype", [
    ("llama2_7b", dict(num_seqs=5), 0, "f32"),
    ("llama2_70b_gqa", dict(num_seqs=6), 48, "bf16"),
    ("tiny", {}, 16, "f32"),
])
def test_block_sizes(bs, name, over, part, out_dtype):
    """Blocks of 32, 64 and 128 tokens (read as 16-token tiles), partitions that
    cut blocks in the middle included."""
    wl = W.make_workload(name, block_size=bs, num_blocks=None, **over)
    _check(wl, out_dtype, part)


@pytest.mark.parametrize("bs", [32, 64])
def test_block_sizes_fp8_beam(bs):
    wl = W.make_workload("beam_cow_fp8", num_seqs=2, shared_len=bs * 3 + 5, block_size=bs,
                         seed=bs)
    _check(wl, "f32", 0)
