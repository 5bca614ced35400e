"""Pins for the oracle's cache writes and block copies (CPU only).

reshape_and_cache is pinned against the special case where the block table is
the identity, so the pool of one head is a contiguous token array and a slot is
simply a token index into it; the FP8 path against torch's own fp32 -> E4M3
conversion; and the new-token slot of every generated workload against the
mapping golden file through a one-hot attention read.  copy_blocks is pinned
by byte comparison and by the in-order semantics of chained pairs.
"""

import os

import numpy as np
import torch

import oracle
from paged_kv_cache_413_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _contiguous_view(cache: np.ndarray) -> np.ndarray:
    """[NB, Hkv, BS, D] -> [Hkv, NB*BS, D]: valid when tables are the identity."""
    nb, hkv, bs, d = cache.shape
    return cache.transpose(1, 0, 2, 3).reshape(hkv, nb * bs, d)


def test_reshape_identity_table_is_contiguous_write():
    rng = np.random.default_rng(0)
    nb, hkv, bs, d, t = 6, 3, 16, 8, 20
    key = rng.standard_normal((t, hkv, d)).astype(np.float16)
    val = rng.standard_normal((t, hkv, d)).astype(np.float16)
    kc0 = np.full((nb, hkv, bs, d), np.nan, dtype=np.float16)
    vc0 = kc0.copy()
    slots = rng.permutation(nb * bs)[:t].astype(np.int64)
    slots[3] = -1  # padding token
    kc, vc = oracle.reshape_and_cache(key.view(np.uint16), val.view(np.uint16),
                                      kc0.view(np.uint16), vc0.view(np.uint16), slots,
                                      src_dtype="f16", cache_dtype="f16")
    kcv = _contiguous_view(kc.view(np.float16))
    vcv = _contiguous_view(vc.view(np.float16))
    written = np.zeros(nb * bs, dtype=bool)
    for i, s in enumerate(slots):
        if s < 0:
            continue
        written[s] = True
        assert np.array_equal(kcv[:, s, :].view(np.uint16), key[i].view(np.uint16))
        assert np.array_equal(vcv[:, s, :].view(np.uint16), val[i].view(np.uint16))
    assert np.isnan(kcv[:, ~written, :].astype(np.float32)).all()
    assert np.isnan(vcv[:, ~written, :].astype(np.float32)).all()


def test_reshape_bf16_bit_copy_keeps_nan_payloads():
    bits = np.array([[[0x7FC1, 0xFF80, 0x0001, 0x8000]]], dtype=np.uint16)  # NaN, -inf, tiny, -0
    kc0 = np.zeros((1, 1, 16, 4), dtype=np.uint16)
    kc, _ = oracle.reshape_and_cache(bits, bits, kc0, kc0, np.array([5]), src_dtype="bf16",
                                     cache_dtype="bf16")
    assert np.array_equal(kc[0, 0, 5], bits[0, 0])
    assert not kc[0, 0, :5].any() and not kc[0, 0, 6:].any()


def test_reshape_fp8_matches_torch_quantisation():
    rng = np.random.default_rng(1)
    nb, hkv, bs, d, t = 4, 2, 16, 32, 10
    x32 = rng.standard_normal((t, hkv, d)).astype(np.float32)
    key = torch.from_numpy(x32).to(torch.bfloat16)
    val = torch.from_numpy(x32[::-1].copy()).to(torch.bfloat16)
    k_scale = float(np.float32(np.abs(x32).max() / 448.0))
    v_scale = 0.0123
    kc0 = np.full((nb, hkv, bs, d), 0x7F, dtype=np.uint8)
    slots = np.arange(t, dtype=np.int64) * 5
    kc, vc = oracle.reshape_and_cache(key, val, kc0, kc0, slots, src_dtype="bf16",
                                      cache_dtype="e4m3", k_scale=k_scale, v_scale=v_scale)
    # IEEE fp32 division by the scale, then torch's RNE conversion (all in range here)
    ref_k = (key.float() / torch.tensor(k_scale, dtype=torch.float32))
    ref_v = (val.float() / torch.tensor(v_scale, dtype=torch.float32))
    assert ref_k.abs().max() < 448 and ref_v.abs().max() < 448
    ref_k = ref_k.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    ref_v = ref_v.to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    kv = _contiguous_view(kc)
    vv = _contiguous_view(vc)
    for i, s in enumerate(slots):
        assert np.array_equal(kv[:, s, :], ref_k[i])
        assert np.array_equal(vv[:, s, :], ref_v[i])
    untouched = np.ones(nb * bs, dtype=bool)
    untouched[slots] = False
    assert (kv[:, untouched, :] == 0x7F).all()


def test_reshape_rejects_out_of_range_slot():
    kc0 = np.zeros((2, 1, 16, 4), dtype=np.uint16)
    x = np.zeros((1, 1, 4), dtype=np.uint16)
    try:
        oracle.reshape_and_cache(x, x, kc0, kc0, np.array([32]), src_dtype="f16",
                                 cache_dtype="f16")
    except ValueError:
        return
    raise AssertionError("slot past the pool was accepted")


def test_copy_blocks_bytes_and_order():
    rng = np.random.default_rng(2)
    layers = [rng.integers(0, 255, (8, 2, 16, 16), dtype=np.uint8) for _ in range(3)]
    vlayers = [rng.integers(0, 255, (8, 2, 16, 16), dtype=np.uint8) for _ in range(3)]
    pairs = np.array([[1, 4], [4, 6], [0, 2]], dtype=np.int64)  # chain: 1 -> 4 -> 6
    kcs, vcs = oracle.copy_blocks(layers, vlayers, pairs, dtype="e4m3")
    for src_l, got in list(zip(layers, kcs)) + list(zip(vlayers, vcs)):
        exp = src_l.copy()
        exp[4] = src_l[1]
        exp[6] = src_l[1]    # in order: the second pair sees the first's result
        exp[2] = src_l[0]
        assert np.array_equal(got, exp)


def _golden_mapping():
    rows = []
    with open(os.path.join(GOLDEN, "page_mapping.txt")) as f:
        for line in f:
            line = line.split("#")[0].strip()
            if not line:
                continue
            tbl, pos, blk, off = [x.strip() for x in line.split("|")]
            rows.append(([int(x) for x in tbl.split(",")], int(pos), int(blk), int(off)))
    return rows


def test_decode_gather_follows_page_mapping():
    """A one-hot read: V rows carry their own physical (block, offset); the key of
    the selected logical position alone matches q, with a huge scale, so the
    output is the V row the gather fetched for that logical position."""
    d, bs, hkv = 4, 16, 1
    for table, pos, blk, off in _golden_mapping():
        nb = max(table) + 1
        kc = np.zeros((nb, hkv, bs, d), dtype=np.float32)
        vc = np.zeros((nb, hkv, bs, d), dtype=np.float32)
        for b in range(nb):
            for o in range(bs):
                vc[b, 0, o] = [b, o, 0, 1]
        L = pos + 1
        # logical position pos gets key e0; every other used position key 0
        kc[blk, 0, off, 0] = 1.0
        q = np.array([[[1.0, 0, 0, 0]]], dtype=np.float32)
        out = oracle.paged_attention_decode(q, kc, vc, np.array([table], dtype=np.int32),
                                            np.array([L], dtype=np.int32), scale=200.0,
                                            q_dtype="f32", cache_dtype="f32")
        assert np.allclose(out[0, 0], [blk, off, 0, 1], atol=1e-40 + 1e-60), (table, pos, out)


def test_generated_new_token_slot_is_last_position():
    """The workload's slot mapping writes the new token at logical position L-1:
    after the oracle's cache write, a one-hot read of position L-1 returns it."""
    wl = W.make_workload("tiny")
    kc, vc = oracle.reshape_and_cache(wl.new_key, wl.new_value, wl.key_cache, wl.value_cache,
                                      wl.slot_mapping, src_dtype="f16", cache_dtype="f16")
    kc64 = oracle.to_f64(kc, "f16")
    vc64 = oracle.to_f64(vc, "f16")
    bt = wl.block_tables.numpy()
    for i, L in enumerate(wl.seq_lens.numpy()):
        pos = int(L) - 1
        blk, off = bt[i, pos // 16], pos % 16
        assert np.array_equal(kc64[blk, :, off, :], wl.new_key[i].double().numpy())
        assert np.array_equal(vc64[blk, :, off, :], wl.new_value[i].double().numpy())
    # nothing else in the context is NaN any more; everything outside stays NaN
    used = np.zeros(kc64.shape[:1] + kc64.shape[2:3], dtype=bool)
    for i, L in enumerate(wl.seq_lens.numpy()):
        for pos in range(int(L)):
            used[bt[i, pos // 16], pos % 16] = True
    assert not np.isnan(kc64.transpose(0, 2, 1, 3)[used]).any()
    assert np.isnan(kc64.transpose(0, 2, 1, 3)[~used]).all()


def test_swap_blocks_moves_bytes_between_pools():
    rng = np.random.default_rng(4)
    gpu_k = [rng.integers(0, 255, (10, 2, 16, 8), dtype=np.uint8) for _ in range(2)]
    gpu_v = [rng.integers(0, 255, (10, 2, 16, 8), dtype=np.uint8) for _ in range(2)]
    cpu_k = [np.zeros((6, 2, 16, 8), dtype=np.uint8) for _ in range(2)]
    cpu_v = [np.zeros((6, 2, 16, 8), dtype=np.uint8) for _ in range(2)]
    pairs = np.array([[9, 0], [3, 5], [4, 1]], dtype=np.int64)  # gpu block -> cpu block
    out_k, out_v = oracle.swap_blocks(cpu_k, cpu_v, gpu_k, gpu_v, pairs, dtype="e4m3")
    for dst, src in list(zip(out_k, gpu_k)) + list(zip(out_v, gpu_v)):
        assert np.array_equal(dst[0], src[9]) and np.array_equal(dst[5], src[3])
        assert np.array_equal(dst[1], src[4])
        assert not dst[[2, 3, 4]].any()
    # and back into other gpu blocks
    back_k, back_v = oracle.swap_blocks(gpu_k, gpu_v, out_k, out_v, [[0, 2], [5, 7]],
                                        dtype="e4m3")
    assert np.array_equal(back_k[1][2], gpu_k[1][9]) and np.array_equal(back_v[0][7], gpu_v[0][3])
    try:
        oracle.swap_blocks(cpu_k, cpu_v, gpu_k, gpu_v, [[10, 0]], dtype="e4m3")
    except ValueError:
        pass
    else:
        raise AssertionError("out-of-range source block accepted")
