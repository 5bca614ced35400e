"""GPU parity of the multi-query (chunked prefill) attention against the oracle.

Each sequence's chunk (its last q tokens) is written by reshape_and_cache, then
every chunk token attends causally over its context.  Cases: GQA group sizes 1..8,
chunks from 1 token (equal to decode) to whole prompts, chunks spanning several
row blocks, block sizes 16..128, fp16/bf16, every output type.  Chunks with fewer
than 128 (token, head) rows per kv head run on the 64-row mma.sync kernel, larger
ones on the 128-row tcgen05 kernel: both sides of that edge are covered.
"""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_413_b200 as pa
from paged_kv_cache_413_b200 import workloads as W

import flow

pytestmark = pytest.mark.gpu


def _run(wl, out_dtype, scale=None, max_q=None):
    d = flow.to_device(wl)
    qs = wl.query_start.cuda()
    pa.pa_reshape_and_cache(d.new_key, d.new_value, d.key_cache, d.value_cache, d.slot_mapping)
    out = torch.full(d.query.shape, float("nan"), dtype=flow.TORCH_DT[out_dtype], device="cuda")
    if max_q is None:
        max_q = int((wl.query_start[1:] - wl.query_start[:-1]).max())
    pa.pa_paged_attention_prefill(out, d.query, d.key_cache, d.value_cache, d.block_tables,
                                  d.seq_lens, qs, max_query_len=max_q,
                                  max_seq_len=flow.max_seq_len(wl),
                                  scale=wl.scale if scale is None else scale)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    return d, out


def _check(wl, out_dtype, scale=None, max_q=None):
    scale = wl.scale if scale is None else scale
    d, out = _run(wl, out_dtype, scale, max_q)
    kc, vc = oracle.reshape_and_cache(wl.new_key, wl.new_value, wl.key_cache, wl.value_cache,
                                      wl.slot_mapping, src_dtype=wl.src_dtype,
                                      cache_dtype=wl.cfg.cache_dtype)
    ref = oracle.paged_attention_prefill(wl.query, kc, vc, wl.block_tables, wl.seq_lens,
                                         wl.query_start, scale=scale, q_dtype=wl.cfg.q_dtype,
                                         cache_dtype=wl.cfg.cache_dtype)
    err = flow.max_abs_err(out, ref)
    assert err <= flow.TOL[out_dtype], f"max abs error {err:.3e}"
    return d, out


@pytest.mark.parametrize("h,hkv", [(8, 8), (16, 4), (64, 8), (12, 4)])
@pytest.mark.parametrize("dt,out_dtype", [("bf16", "f32"), ("f16", "f16"), ("bf16", "bf16")])
def test_prefill_groups(h, hkv, dt, out_dtype):
    wl = W.make_prefill_workload(4, (20, 300), (1, 60), num_heads=h, num_kv_heads=hkv, dtype=dt,
                                 seed=h + hkv)
    _check(wl, out_dtype)


@pytest.mark.parametrize("bs", [16, 64, 128])
def test_prefill_whole_prompts_and_block_sizes(bs):
    # chunk = the whole context: the first query sees one token
    wl = W.make_prefill_workload(3, (1, 130), (130, 130), num_heads=16, num_kv_heads=4,
                                 dtype="bf16", seed=bs, block_size=bs)
    _check(wl, "f32")


def test_prefill_long_chunk_over_long_context():
    wl = W.make_prefill_workload(2, (1500, 2100), (300, 520), num_heads=64, num_kv_heads=8,
                                 dtype="bf16", seed=7)
    _check(wl, "bf16")


def test_prefill_single_token_equals_decode():
    wl = W.make_prefill_workload(5, (1, 400), (1, 1), num_heads=32, num_kv_heads=8,
                                 dtype="bf16", seed=3)
    d, out = _run(wl, "f32")
    dec = torch.empty_like(out)
    pa.pa_paged_attention_decode(dec, d.query, d.key_cache, d.value_cache, d.block_tables,
                                 d.seq_lens, max_seq_len=flow.max_seq_len(wl), scale=wl.scale,
                                 partition_size=1024)
    assert (out - dec).abs().max().item() <= 1e-3


@pytest.mark.parametrize("chunk", [15, 16, 17, 33])
def test_prefill_row_block_edges(chunk):
    # GQA-8: 120, 128, 136 and 264 rows per kv head around the 128-row tile
    wl = W.make_prefill_workload(3, (chunk, 300), (chunk, chunk), num_heads=64, num_kv_heads=8,
                                 dtype="bf16", seed=chunk)
    _check(wl, "f32")


@pytest.mark.parametrize("dt", ["f16", "bf16"])
def test_prefill_ragged_chunks_both_kernels(dt):
    # chunks of 1..8 tokens (at most 32 rows per kv head): the 64-row kernel
    wl = W.make_prefill_workload(6, (200, 900), (1, 8), num_heads=32, num_kv_heads=8,
                                 dtype=dt, seed=11)
    _check(wl, dt)
    # chunks of 1..190 tokens (up to 6 row blocks of 128): CTAs past a short
    # sequence's rows have nothing to do and leave before any barrier
    wl2 = W.make_prefill_workload(6, (700, 900), (1, 190), num_heads=32, num_kv_heads=8,
                                  dtype=dt, seed=12)
    _check(wl2, dt)


@pytest.mark.parametrize("scale", [0.0, -0.06])
@pytest.mark.parametrize("chunk", [(1, 12), (40, 90)])
def test_prefill_zero_and_negative_scale(scale, chunk):
    # a zero scale gives the mean of the visible V rows; a negative one reverses the order
    wl = W.make_prefill_workload(3, (100, 400), chunk, num_heads=32, num_kv_heads=8,
                                 dtype="bf16", seed=21)
    _check(wl, "f32", scale=scale)


def test_full_chunked_prefill_70b():
    # the workload and launch the benchmark times (16 sequences, 512-token chunks over
    # 2048..4096-token contexts, GQA-8, bf16 out: the persistent tcgen05 kernel),
    # checked on the shortest and the longest sequence and one in between
    import bench

    spec = dict(bench.PREFILL["chunked_prefill_70b"])
    wl = W.make_prefill_workload(spec.pop("num_seqs"), spec.pop("context"), spec.pop("chunk"),
                                 **spec)
    d, out = _run(wl, "bf16")
    L = wl.seq_lens.numpy()
    seqs = sorted({int(L.argmin()), int(L.argmax()), 7})
    qs = wl.query_start.numpy().astype(np.int64)
    rows = np.concatenate([np.arange(qs[s], qs[s + 1]) for s in seqs])
    nt = torch.as_tensor(rows)
    kc, vc = oracle.reshape_and_cache(wl.new_key[nt], wl.new_value[nt], wl.key_cache,
                                      wl.value_cache, wl.slot_mapping.numpy()[rows],
                                      src_dtype=wl.src_dtype, cache_dtype=wl.cfg.cache_dtype)
    sub_qs = np.concatenate([[0], np.cumsum([qs[s + 1] - qs[s] for s in seqs])])
    ref = oracle.paged_attention_prefill(wl.query[nt], kc, vc, wl.block_tables.numpy()[seqs],
                                         L[seqs], sub_qs, scale=wl.scale, q_dtype="bf16",
                                         cache_dtype="bf16")
    err = flow.max_abs_err(out[torch.as_tensor(rows, device=out.device)], ref)
    assert err <= flow.TOL["bf16"], f"max abs error {err:.3e}"
    assert torch.isfinite(out.float()).all()


@pytest.mark.parametrize("seed,chunk,dt", [(16, (0, 60), "bf16"), (0, (0, 8), "f16")])
def test_prefill_empty_chunks_and_loose_bound(seed, chunk, dt):
    # some sequences have no query rows this step (q_i = 0); the first case runs the
    # tcgen05 kernel (up to 60 x 4 rows), the second the mma.sync one
    wl = W.make_prefill_workload(6, (60, 400), chunk, num_heads=32, num_kv_heads=8, dtype=dt,
                                 seed=seed)
    q = (wl.query_start[1:] - wl.query_start[:-1]).numpy()
    assert (q == 0).any()
    _check(wl, dt)
    # a host bound above the real longest chunk only adds tiles with no rows
    _check(wl, dt, max_q=int(q.max()) * 3 + 5)
