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
@pytest.mark.parametrize("hkv,d", [(4, 64), (8, 128), (3, 40)])
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
