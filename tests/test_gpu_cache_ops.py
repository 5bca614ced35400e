"""GPU parity of reshape_and_cache and copy_blocks against the oracle: bit-exact,
whole pools compared (untouched bytes included)."""

import numpy as np
import pytest
import torch

import oracle
import paged_kv_cache_413_b200 as pa
from paged_kv_cache_413_b200 import workloads as W

import flow

pytestmark = pytest.mark.gpu


def _pool(nb, hkv, d, dtype, fill_seed=0):
    g = torch.Generator().manual_seed(fill_seed)
    if dtype == "e4m3":
        return torch.randint(0, 256, (nb, hkv, 16, d), generator=g, dtype=torch.uint8).view(
            torch.float8_e4m3fn)
    return torch.randn(nb, hkv, 16, d, generator=g).to(flow.TORCH_DT[dtype])


@pytest.mark.parametrize("src,cache", [("f16", "f16"), ("bf16", "bf16"), ("f16", "e4m3"),
                                       ("bf16", "e4m3")])
# rows of 8-element chunks: 32, 128, 15 (one CTA a token); 512 (4 CTAs, the 7B row);
# 2048 (8 CTAs of two chunks a thread); 225 (2 CTAs, the second partly idle)
@pytest.mark.parametrize("hkv,d", [(4, 64), (8, 128), (3, 40), (32, 128), (128, 128), (9, 200)])
def test_reshape_and_cache_bit_exact(src, cache, hkv, d):
    nb, t = 37, 300
    rng = np.random.default_rng(hkv * 1000 + d)
    key = torch.from_numpy(rng.standard_normal((t, hkv, d), dtype=np.float32) * 3).to(
        flow.TORCH_DT[src])
    val = torch.from_numpy(rng.standard_normal((t, hkv, d), dtype=np.float32)).to(
        flow.TORCH_DT[src])
    slots = torch.from_numpy(rng.permutation(nb * 16)[:t].astype(np.int64))
    slots[::17] = -1  # padding tokens are skipped
    kc, vc = _pool(nb, hkv, d, cache, 1), _pool(nb, hkv, d, cache, 2)
    ks, vs = (0.0137, 0.00291) if cache == "e4m3" else (1.0, 1.0)
    ref_k, ref_v = oracle.reshape_and_cache(key, val, kc, vc, slots, src_dtype=src,
                                            cache_dtype=cache, k_scale=ks, v_scale=vs)
    dk, dv = kc.cuda(), vc.cuda()
    pa.pa_reshape_and_cache(key.cuda(), val.cuda(), dk, dv, slots.cuda(), k_scale=ks,
                            v_scale=vs)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    assert np.array_equal(flow.storage_bytes(dk).reshape(-1), ref_k.view(np.uint8).reshape(-1))
    assert np.array_equal(flow.storage_bytes(dv).reshape(-1), ref_v.view(np.uint8).reshape(-1))


@pytest.mark.parametrize("src", ["f16", "bf16"])
@pytest.mark.parametrize("scale", [1.0, 0.75, 3.0e-3, 1.7e2])
def test_fp8_quantisation_every_source_value(src, scale):
    """Every finite 16-bit source pattern through the cache write: E4M3 rounding,
    ties, subnormals and saturation all decided exactly as the oracle decides."""
    bits = np.arange(1 << 16, dtype=np.uint16)
    vals = torch.from_numpy(bits.view(np.int16)).view(flow.TORCH_DT[src])
    vals = vals[torch.isfinite(vals.float())]
    d, hkv = 128, 1
    t = vals.numel() // d
    key = vals[:t * d].reshape(t, hkv, d).contiguous()
    val = torch.flip(key, dims=[0]).contiguous()
    nb = -(-t // 16)
    kc = _pool(nb, hkv, d, "e4m3", 3)
    vc = _pool(nb, hkv, d, "e4m3", 4)
    slots = torch.arange(t, dtype=torch.int64)
    ref_k, ref_v = oracle.reshape_and_cache(key, val, kc, vc, slots, src_dtype=src,
                                            cache_dtype="e4m3", k_scale=scale, v_scale=scale)
    dk, dv = kc.cuda(), vc.cuda()
    pa.pa_reshape_and_cache(key.cuda(), val.cuda(), dk, dv, slots.cuda(), k_scale=scale,
                            v_scale=scale)
    assert np.array_equal(flow.storage_bytes(dk).reshape(-1), ref_k.reshape(-1))
    assert np.array_equal(flow.storage_bytes(dv).reshape(-1), ref_v.reshape(-1))


def test_reshape_slot_out_of_range_sets_error_and_skips():
    kc = torch.zeros(4, 2, 16, 64, dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    key = torch.ones(2, 2, 64, dtype=torch.float16, device="cuda")
    pa.pa_get_device_error()
    pa.pa_reshape_and_cache(key, key, kc, vc,
                            torch.tensor([3, 64], dtype=torch.int64, device="cuda"))
    err = pa.pa_get_device_error()
    assert err & 0x1
    assert kc.view(-1, 64).ne(0).any(dim=1).sum().item() == 2  # slot 3 for both heads
    assert pa.pa_get_device_error() == 0  # cleared


@pytest.mark.parametrize("dtype,layers", [("f16", 1), ("e4m3", 3), ("bf16", 70)])
def test_copy_blocks_bit_exact(dtype, layers):
    nb, hkv, d = 40, 8, 128 if dtype != "bf16" else 64
    rng = np.random.default_rng(5)
    kcs = [_pool(nb, hkv, d, dtype, 10 + i) for i in range(layers)]
    vcs = [_pool(nb, hkv, d, dtype, 100 + i) for i in range(layers)]
    perm = rng.permutation(nb)
    pairs = torch.from_numpy(np.stack([perm[:12], perm[12:24]], axis=1).astype(np.int64))
    ref_k, ref_v = oracle.copy_blocks(kcs, vcs, pairs, dtype=dtype)
    dk = [x.cuda() for x in kcs]
    dv = [x.cuda() for x in vcs]
    pa.pa_copy_blocks(dk, dv, pairs.cuda())
    for g, r in list(zip(dk, ref_k)) + list(zip(dv, ref_v)):
        assert np.array_equal(flow.storage_bytes(g).reshape(-1), r.view(np.uint8).reshape(-1))
    assert pa.pa_get_device_error() == 0


def test_copy_blocks_bad_id_sets_error():
    kc = torch.zeros(4, 1, 16, 64, dtype=torch.float16, device="cuda")
    vc = torch.zeros_like(kc)
    pa.pa_get_device_error()
    pa.pa_copy_blocks([kc], [vc], torch.tensor([[0, 9]], dtype=torch.int64, device="cuda"))
    assert pa.pa_get_device_error() & 0x10


def test_beam_workload_cache_writes_bit_exact():
    """The copy-on-write recipe (prefix fill in FP8, copies, new tokens), scaled down."""
    wl = W.make_workload("beam_cow_fp8", num_seqs=6, shared_len=72)
    d = flow.to_device(wl)
    flow.gpu_prepare(wl, d)
    pa.pa_reshape_and_cache(d.new_key, d.new_value, d.key_cache, d.value_cache, d.slot_mapping,
                            k_scale=wl.k_scale, v_scale=wl.v_scale)
    ref_k, ref_v = flow.oracle_caches(wl)
    assert np.array_equal(flow.storage_bytes(d.key_cache).reshape(-1), ref_k.reshape(-1))
    assert np.array_equal(flow.storage_bytes(d.value_cache).reshape(-1), ref_v.reshape(-1))
    assert pa.pa_get_device_error() == 0


@pytest.mark.parametrize("dtype,layers", [("bf16", 2), ("e4m3", 1)])
def test_swap_blocks_device_host_round_trip(dtype, layers):
    nb_gpu, nb_cpu, hkv, d = 48, 20, 8, 128
    rng = np.random.default_rng(11)
    gk = [_pool(nb_gpu, hkv, d, dtype, 200 + i) for i in range(layers)]
    gv = [_pool(nb_gpu, hkv, d, dtype, 300 + i) for i in range(layers)]
    ck = [_pool(nb_cpu, hkv, d, dtype, 400 + i) for i in range(layers)]
    cv = [_pool(nb_cpu, hkv, d, dtype, 500 + i) for i in range(layers)]
    out_pairs = np.stack([rng.permutation(nb_gpu)[:15], rng.permutation(nb_cpu)[:15]], 1)
    ref_ck, ref_cv = oracle.swap_blocks(ck, cv, gk, gv, out_pairs, dtype=dtype)
    dgk = [x.cuda() for x in gk]
    dgv = [x.cuda() for x in gv]
    hck = [x.pin_memory() for x in ck]
    hcv = [x.pin_memory() for x in cv]
    # swap out: device -> pinned host, mapping itself in pinned host memory
    pa.pa_swap_blocks(hck, hcv, dgk, dgv, torch.from_numpy(out_pairs.astype(np.int64)).pin_memory())
    torch.cuda.synchronize()
    for g, r in list(zip(hck, ref_ck)) + list(zip(hcv, ref_cv)):
        assert np.array_equal(flow.storage_bytes(g).reshape(-1), r.view(np.uint8).reshape(-1))
    # swap in: pinned host -> other device blocks, mapping on the device
    in_pairs = np.stack([out_pairs[:, 1], rng.permutation(nb_gpu)[:15]], 1)
    ref_gk, ref_gv = oracle.swap_blocks(gk, gv, ref_ck, ref_cv, in_pairs, dtype=dtype)
    pa.pa_swap_blocks(dgk, dgv, hck, hcv, torch.from_numpy(in_pairs.astype(np.int64)).cuda())
    for g, r in list(zip(dgk, ref_gk)) + list(zip(dgv, ref_gv)):
        assert np.array_equal(flow.storage_bytes(g).reshape(-1), r.view(np.uint8).reshape(-1))
    assert pa.pa_get_device_error() == 0


def test_swap_rejects_pageable_host_memory():
    kc = torch.zeros(4, 1, 16, 64, dtype=torch.float16, device="cuda")
    host = torch.zeros(4, 1, 16, 64, dtype=torch.float16)  # not pinned
    with pytest.raises(ValueError):
        pa.pa_swap_blocks([host], [host], [kc], [kc], torch.tensor([[0, 1]]).cuda())


def test_preempt_swap_out_and_resume_gives_identical_decode():
    """Swap a sequence's blocks out to host memory, let the pool reuse them, swap
    them back into different blocks: decode is bitwise the same as before."""
    wl = W.make_workload("llama2_70b_gqa", num_seqs=6, pool_factor=3.0)
    d = flow.to_device(wl)
    before = flow.gpu_step(wl, d, "bf16", 128)
    seq = 2
    blocks = d.block_tables[seq][d.block_tables[seq] >= 0].long()
    n = blocks.numel()
    hk = torch.empty((n,) + tuple(d.key_cache.shape[1:]), dtype=d.key_cache.dtype).pin_memory()
    hv = torch.empty_like(hk).pin_memory()
    out_map = torch.stack([blocks.cpu(), torch.arange(n)], 1).contiguous()
    pa.pa_swap_blocks([hk], [hv], [d.key_cache], [d.value_cache], out_map.cuda())
    # the freed blocks are overwritten by someone else; the sequence comes back elsewhere
    d.key_cache[blocks] = float("nan")
    d.value_cache[blocks] = float("nan")
    free = torch.tensor(sorted(set(range(wl.num_blocks)) - set(d.block_tables.flatten().tolist())))
    new_blocks = free[:n]
    in_map = torch.stack([torch.arange(n), new_blocks], 1).contiguous()
    pa.pa_swap_blocks([d.key_cache], [d.value_cache], [hk], [hv], in_map.pin_memory())
    bt = d.block_tables.clone()
    bt[seq, :n] = new_blocks.to(torch.int32).cuda()
    out = torch.empty_like(before)
    pa.pa_paged_attention_decode(out, d.query, d.key_cache, d.value_cache, bt, d.seq_lens,
                                 max_seq_len=flow.max_seq_len(wl), scale=wl.scale,
                                 partition_size=128, workspace=flow.workspace_for(wl, 128))
    assert torch.equal(out, before)
    assert pa.pa_get_device_error() == 0


@pytest.mark.parametrize("bs,cache", [(64, "bf16"), (32, "e4m3")])
def test_reshape_and_cache_block_sizes(bs, cache):
    nb, hkv, d, t = 9, 8, 128, 200
    rng = np.random.default_rng(bs)
    key = torch.from_numpy(rng.standard_normal((t, hkv, d), dtype=np.float32)).to(torch.bfloat16)
    val = torch.from_numpy(rng.standard_normal((t, hkv, d), dtype=np.float32)).to(torch.bfloat16)
    slots = torch.from_numpy(rng.permutation(nb * bs)[:t].astype(np.int64))
    g = torch.Generator().manual_seed(1)
    if cache == "e4m3":
        kc = torch.randint(0, 256, (nb, hkv, bs, d), generator=g, dtype=torch.uint8).view(
            torch.float8_e4m3fn)
    else:
        kc = torch.randn(nb, hkv, bs, d, generator=g).to(torch.bfloat16)
    vc = kc.clone()
    ks, vs = (0.02, 0.03) if cache == "e4m3" else (1.0, 1.0)
    ref_k, ref_v = oracle.reshape_and_cache(key, val, kc, vc, slots, src_dtype="bf16",
                                            cache_dtype=cache, k_scale=ks, v_scale=vs)
    dk, dv = kc.cuda(), vc.cuda()
    pa.pa_reshape_and_cache(key.cuda(), val.cuda(), dk, dv, slots.cuda(), k_scale=ks, v_scale=vs)
    assert np.array_equal(flow.storage_bytes(dk).reshape(-1), ref_k.view(np.uint8).reshape(-1))
    assert np.array_equal(flow.storage_bytes(dv).reshape(-1), ref_v.view(np.uint8).reshape(-1))
