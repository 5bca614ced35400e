"""Pins for the oracle's decode attention and split statistics (CPU only).

* brute force against torch's fp64 scaled_dot_product_attention on a pool whose
  block tables are the identity, so no gather is needed on the reference side;
* permutation invariance: the same logical K/V under another block permutation
  gives a bitwise-equal output (the pages: paging changes storage, not results);
* closed forms: identical keys or scale 0 give the mean of V; one token gives V0;
  a hand-computed two-token case; GQA head-to-kv-head mapping;
* shared-prefix beams with equal queries are bitwise identical, and differ once
  their last tokens differ;
* FP8 pools are read as decode(code) * scale;
* the split statistics merged by log-sum-exp equal the unsplit result.
"""

import math

import numpy as np
import pytest
import torch

import oracle


def _sdpa_contiguous(q, k, v, scale, group):
    """q [H, D], k/v [Hkv, L, D] fp64 -> [H, D] via torch SDPA (library routine)."""
    qt = torch.from_numpy(q)[None, :, None, :]                     # [1, H, 1, D]
    kt = torch.from_numpy(k).repeat_interleave(group, dim=0)[None]  # [1, H, L, D]
    vt = torch.from_numpy(v).repeat_interleave(group, dim=0)[None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, scale=scale)
    return o[0, :, 0, :].numpy()


def _identity_layout(rng, lens, hkv, d, bs=16, dtype=np.float32):
    """Each sequence owns consecutive physical blocks (identity tables)."""
    nblk = [-(-L // bs) for L in lens]
    nb = sum(nblk) + 2
    kc = rng.standard_normal((nb, hkv, bs, d)).astype(dtype)
    vc = rng.standard_normal((nb, hkv, bs, d)).astype(dtype)
    width = max(nblk)
    bt = np.full((len(lens), width), -1, dtype=np.int32)
    start = 0
    for i, n in enumerate(nblk):
        bt[i, :n] = np.arange(start, start + n)
        start += n
    return kc, vc, bt


@pytest.mark.parametrize("group", [1, 4])
def test_decode_matches_sdpa_on_identity_layout(group):
    rng = np.random.default_rng(3)
    lens = [1, 5, 16, 17, 40]
    hkv, d, bs = 2, 16, 16
    h = hkv * group
    kc, vc, bt = _identity_layout(rng, lens, hkv, d)
    q = rng.standard_normal((len(lens), h, d)).astype(np.float32)
    scale = 0.3
    out = oracle.paged_attention_decode(q, kc, vc, bt, np.array(lens, np.int32), scale=scale,
                                        q_dtype="f32", cache_dtype="f32")
    for i, L in enumerate(lens):
        first = bt[i, 0]
        # identity tables: a sequence is a contiguous run of tokens in the pool
        k = kc[first:first + bt.shape[1]].transpose(1, 0, 2, 3).reshape(hkv, -1, d)[:, :L]
        v = vc[first:first + bt.shape[1]].transpose(1, 0, 2, 3).reshape(hkv, -1, d)[:, :L]
        ref = _sdpa_contiguous(q[i].astype(np.float64), k.astype(np.float64),
                               v.astype(np.float64), scale, group)
        np.testing.assert_allclose(out[i], ref, rtol=0, atol=1e-12)


def test_decode_permutation_invariance_bitwise():
    rng = np.random.default_rng(4)
    lens = [3, 16, 31, 64]
    hkv, d, bs = 2, 8, 16
    kc, vc, bt = _identity_layout(rng, lens, hkv, d)
    q = rng.standard_normal((len(lens), 4, d)).astype(np.float32)
    a = oracle.paged_attention_decode(q, kc, vc, bt, np.array(lens, np.int32), scale=0.5,
                                      q_dtype="f32", cache_dtype="f32")
    perm = rng.permutation(kc.shape[0])          # physical block b moves to perm[b]
    kc2 = np.empty_like(kc)
    vc2 = np.empty_like(vc)
    kc2[perm] = kc
    vc2[perm] = vc
    bt2 = np.where(bt >= 0, perm[np.maximum(bt, 0)], -1).astype(np.int32)
    b = oracle.paged_attention_decode(q, kc2, vc2, bt2, np.array(lens, np.int32), scale=0.5,
                                      q_dtype="f32", cache_dtype="f32")
    assert np.array_equal(a, b)


def test_identical_keys_give_mean_of_v_and_scale_zero_too():
    rng = np.random.default_rng(5)
    L, d = 37, 8
    kc, vc, bt = _identity_layout(rng, [L], 1, d)
    q = rng.standard_normal((1, 1, d)).astype(np.float32)
    vmean = vc.transpose(1, 0, 2, 3).reshape(1, -1, d)[0, :L].astype(np.float64).mean(axis=0)
    kc_same = np.broadcast_to(kc[0, :, 0:1, :], kc.shape).copy()
    out = oracle.paged_attention_decode(q, kc_same, vc, bt, np.array([L], np.int32), scale=0.7,
                                        q_dtype="f32", cache_dtype="f32")
    np.testing.assert_allclose(out[0, 0], vmean, rtol=0, atol=1e-14)
    out0 = oracle.paged_attention_decode(q, kc, vc, bt, np.array([L], np.int32), scale=0.0,
                                         q_dtype="f32", cache_dtype="f32")
    np.testing.assert_allclose(out0[0, 0], vmean, rtol=0, atol=1e-14)


def test_one_token_returns_v0_exactly():
    rng = np.random.default_rng(6)
    kc, vc, bt = _identity_layout(rng, [1, 1], 2, 8)
    q = (rng.standard_normal((2, 2, 8)) * 30).astype(np.float32)
    out = oracle.paged_attention_decode(q, kc, vc, bt, np.array([1, 1], np.int32), scale=9.0,
                                        q_dtype="f32", cache_dtype="f32")
    for i in range(2):
        assert np.array_equal(out[i], vc[bt[i, 0], :, 0, :].astype(np.float64))


def test_hand_computed_two_tokens():
    # scores 0 and ln 3 -> weights 1/4, 3/4
    kc = np.zeros((1, 1, 16, 2), dtype=np.float64)
    vc = np.zeros((1, 1, 16, 2), dtype=np.float64)
    kc[0, 0, 1] = [math.log(3.0), 0.0]
    vc[0, 0, 0] = [4.0, -8.0]
    vc[0, 0, 1] = [0.0, 8.0]
    q = np.array([[[1.0, 5.0]]], dtype=np.float32)
    out = oracle.paged_attention_decode(q, kc.astype(np.float32), vc.astype(np.float32),
                                        np.array([[0]], np.int32), np.array([2], np.int32),
                                        scale=1.0, q_dtype="f32", cache_dtype="f32")
    # ln 3 rounded to fp32 in the cache: weights follow that value
    l3 = float(np.float32(math.log(3.0)))
    w1 = math.exp(l3) / (1 + math.exp(l3))
    np.testing.assert_allclose(out[0, 0], [4.0 * (1 - w1), -8.0 * (1 - w1) + 8.0 * w1],
                               rtol=0, atol=1e-14)
    assert abs(w1 - 0.75) < 1e-7


def test_gqa_head_to_kv_head_mapping():
    """Query head h reads kv head h // (H / Hkv): V is constant per kv head."""
    hkv, group, d, L = 4, 3, 8, 20
    rng = np.random.default_rng(7)
    kc, vc, bt = _identity_layout(rng, [L], hkv, d)
    for j in range(hkv):
        vc[:, j] = float(j + 1)
    q = rng.standard_normal((1, hkv * group, d)).astype(np.float32)
    out = oracle.paged_attention_decode(q, kc, vc, bt, np.array([L], np.int32), scale=0.1,
                                        q_dtype="f32", cache_dtype="f32")
    for h in range(hkv * group):
        np.testing.assert_allclose(out[0, h], h // group + 1, rtol=0, atol=1e-13)


def test_large_logits_stay_finite():
    rng = np.random.default_rng(8)
    kc, vc, bt = _identity_layout(rng, [50], 1, 8)
    q = (rng.standard_normal((1, 1, 8)) * 100).astype(np.float32)
    out = oracle.paged_attention_decode(q, kc, vc, bt, np.array([50], np.int32), scale=100.0,
                                        q_dtype="f32", cache_dtype="f32")
    assert np.isfinite(out).all()


def test_shared_prefix_beams_identical_until_divergence():
    rng = np.random.default_rng(9)
    d, bs, hkv = 8, 16, 2
    nb = 8
    kc = rng.standard_normal((nb, hkv, bs, d)).astype(np.float32)
    vc = rng.standard_normal((nb, hkv, bs, d)).astype(np.float32)
    # two beams share blocks 3, 5 (32 tokens) and then own blocks 1 and 6
    bt = np.array([[3, 5, 1], [3, 5, 6]], dtype=np.int32)
    q1 = rng.standard_normal((1, 4, d)).astype(np.float32)
    q = np.concatenate([q1, q1])
    same = oracle.paged_attention_decode(q, kc, vc, bt, np.array([32, 32], np.int32), scale=0.4,
                                         q_dtype="f32", cache_dtype="f32")
    assert np.array_equal(same[0], same[1])
    # copy-on-write copy of the own blocks keeps them identical ...
    kc[6], vc[6] = kc[1], vc[1]
    cow = oracle.paged_attention_decode(q, kc, vc, bt, np.array([40, 40], np.int32), scale=0.4,
                                        q_dtype="f32", cache_dtype="f32")
    assert np.array_equal(cow[0], cow[1])
    # ... until one beam writes a different token
    kc[6, :, 7] += 1.0
    div = oracle.paged_attention_decode(q, kc, vc, bt, np.array([40, 40], np.int32), scale=0.4,
                                        q_dtype="f32", cache_dtype="f32")
    assert not np.array_equal(div[0], div[1])
    assert np.array_equal(div[0], cow[0])


def test_fp8_pool_reads_decode_times_scale():
    rng = np.random.default_rng(10)
    d, hkv, L = 16, 2, 45
    kc, vc, bt = _identity_layout(rng, [L], hkv, d)
    codes_k = rng.integers(0, 256, kc.shape, dtype=np.uint8)
    codes_v = rng.integers(0, 256, vc.shape, dtype=np.uint8)
    codes_k[(codes_k & 0x7F) == 0x7F] = 0x10       # no NaN codes
    codes_v[(codes_v & 0x7F) == 0x7F] = 0x21
    ks, vs = 0.05, 0.002
    q = torch.randn(1, 2 * hkv, d, generator=torch.Generator().manual_seed(0)).to(torch.bfloat16)
    out = oracle.paged_attention_decode(q, codes_k, codes_v, bt, np.array([L], np.int32),
                                        scale=0.25, q_dtype="bf16", cache_dtype="e4m3",
                                        k_scale=ks, v_scale=vs)
    kf = torch.from_numpy(codes_k).view(torch.float8_e4m3fn).double().numpy() * ks
    vf = torch.from_numpy(codes_v).view(torch.float8_e4m3fn).double().numpy() * vs
    k = kf.transpose(1, 0, 2, 3).reshape(hkv, -1, d)[:, :L]
    v = vf.transpose(1, 0, 2, 3).reshape(hkv, -1, d)[:, :L]
    ref = _sdpa_contiguous(q[0].double().numpy(), k, v, 0.25, 2)
    np.testing.assert_allclose(out[0], ref, rtol=0, atol=1e-12)


@pytest.mark.parametrize("part", [16, 32, 48, 512])
def test_partition_stats_merge_to_unsplit(part):
    rng = np.random.default_rng(12)
    lens = [1, 16, 17, 100, 130]
    hkv, d = 2, 8
    kc, vc, bt = _identity_layout(rng, lens, hkv, d)
    q = rng.standard_normal((len(lens), 4, d)).astype(np.float32)
    sl = np.array(lens, np.int32)
    full = oracle.paged_attention_decode(q, kc, vc, bt, sl, scale=0.3, q_dtype="f32",
                                         cache_dtype="f32")
    maxp = -(-max(lens) // part)
    m, l, o = oracle.decode_partition_stats(q, kc, vc, bt, sl, partition_size=part,
                                            max_parts=maxp, scale=0.3, q_dtype="f32",
                                            cache_dtype="f32")
    np.testing.assert_allclose(oracle.lse_merge(m, l, o), full, rtol=0, atol=1e-12)
    # a range's own statistics: brute force on the first sequence with > 1 range
    i = 3
    k = kc[bt[i, 0]:].transpose(1, 0, 2, 3).reshape(hkv, -1, d)[:, :lens[i]].astype(np.float64)
    s = (k[0] @ q[i, 0].astype(np.float64)) * 0.3
    lo = 0
    hi = min(part, lens[i])
    assert m[i, 0, 0] == s[lo:hi].max()
    np.testing.assert_allclose(l[i, 0, 0], np.exp(s[lo:hi] - s[lo:hi].max()).sum(), rtol=1e-14)
    if maxp > -(-lens[i] // part):
        assert l[i, 0, -1] == 0.0 and m[i, 0, -1] == -np.inf


def test_lse_merge_closed_form():
    # two ranges: (m=0, l=1, o=2) and (m=ln 3, l=1, o=6) -> weights 1 : 3 -> 5
    m = np.array([[0.0, math.log(3.0), 0.0]])
    l = np.array([[1.0, 1.0, 0.0]])
    o = np.array([[[2.0], [6.0], [1e300]]])
    np.testing.assert_allclose(oracle.lse_merge(m, l, o), [[5.0]], rtol=1e-15)


def test_prefill_one_query_equals_decode():
    rng = np.random.default_rng(13)
    lens = [1, 9, 16, 33]
    kc, vc, bt = _identity_layout(rng, lens, 2, 8)
    q = rng.standard_normal((len(lens), 4, 8)).astype(np.float32)
    dec = oracle.paged_attention_decode(q, kc, vc, bt, np.array(lens, np.int32), scale=0.4,
                                        q_dtype="f32", cache_dtype="f32")
    pre = oracle.paged_attention_prefill(q, kc, vc, bt, np.array(lens, np.int32),
                                         np.arange(len(lens) + 1, dtype=np.int32), scale=0.4,
                                         q_dtype="f32", cache_dtype="f32")
    assert np.array_equal(pre, dec)


@pytest.mark.parametrize("group", [1, 4])
def test_prefill_matches_causal_sdpa(group):
    rng = np.random.default_rng(14)
    lens, nq = [20, 37, 5], [7, 37, 1]
    hkv, d = 2, 16
    kc, vc, bt = _identity_layout(rng, lens, hkv, d)
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    q = rng.standard_normal((int(qs[-1]), hkv * group, d)).astype(np.float32)
    out = oracle.paged_attention_prefill(q, kc, vc, bt, np.array(lens, np.int32), qs, scale=0.3,
                                         q_dtype="f32", cache_dtype="f32")
    for i, (L, n) in enumerate(zip(lens, nq)):
        first = bt[i, 0]
        k = kc[first:first + bt.shape[1]].transpose(1, 0, 2, 3).reshape(hkv, -1, d)[:, :L]
        v = vc[first:first + bt.shape[1]].transpose(1, 0, 2, 3).reshape(hkv, -1, d)[:, :L]
        qt = torch.from_numpy(q[qs[i]:qs[i + 1]].astype(np.float64)).permute(1, 0, 2)[None]
        kt = torch.from_numpy(k.astype(np.float64)).repeat_interleave(group, 0)[None]
        vt = torch.from_numpy(v.astype(np.float64)).repeat_interleave(group, 0)[None]
        # query j sits at position L - n + j: it may see keys 0 .. L - n + j
        mask = torch.arange(L)[None, :] <= (L - n + torch.arange(n))[:, None]
        ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask,
                                                               scale=0.3)[0].permute(1, 0, 2)
        np.testing.assert_allclose(out[qs[i]:qs[i + 1]], ref.numpy(), rtol=0, atol=1e-12)


def test_prefill_first_query_of_a_full_prompt_sees_one_token():
    # a whole 3-token prompt as queries: query 0 sees only token 0 -> exactly V0
    kc = np.zeros((1, 1, 16, 2), dtype=np.float32)
    vc = np.zeros((1, 1, 16, 2), dtype=np.float32)
    kc[0, 0, :3] = [[1, 0], [0, 1], [1, 1]]
    vc[0, 0, :3] = [[3, -1], [5, 2], [-7, 4]]
    q = np.array([[[1.0, 0.0]], [[0.0, 2.0]], [[1.0, 1.0]]], dtype=np.float32)
    out = oracle.paged_attention_prefill(q, kc, vc, np.array([[0]], np.int32),
                                         np.array([3], np.int32), np.array([0, 3], np.int32),
                                         scale=1.0, q_dtype="f32", cache_dtype="f32")
    assert np.array_equal(out[0, 0], [3.0, -1.0])
    # query 1 (position 1): scores 0 and 2 over tokens 0, 1
    w = np.exp([0.0, 2.0]) / np.exp([0.0, 2.0]).sum()
    np.testing.assert_allclose(out[1, 0], w[0] * vc[0, 0, 0] + w[1] * vc[0, 0, 1], atol=1e-15)


def _layout(rng, seqs_kv, bs, hkv, d):
    """Scatter each sequence's logical [Hkv, L, D] K/V into bs-token blocks of a
    shuffled pool; unused rows hold NaN.  Returns (kc, vc, tables)."""
    nblk = [-(-kv[0].shape[1] // bs) for kv in seqs_kv]
    nb = sum(nblk) + 3
    phys = rng.permutation(nb)
    kc = np.full((nb, hkv, bs, d), np.nan, dtype=np.float32)
    vc = np.full((nb, hkv, bs, d), np.nan, dtype=np.float32)
    bt = np.full((len(seqs_kv), max(nblk)), -1, dtype=np.int32)
    nxt = 0
    for i, (k, v) in enumerate(seqs_kv):
        L = k.shape[1]
        for j in range(nblk[i]):
            b = phys[nxt]
            nxt += 1
            bt[i, j] = b
            n = min(bs, L - j * bs)
            kc[b, :, :n] = k[:, j * bs:j * bs + n]
            vc[b, :, :n] = v[:, j * bs:j * bs + n]
    return kc, vc, bt


def test_block_size_relayout_is_bitwise_invariant():
    # the same logical K/V, stored in 16-, 32-, 64- or 128-token blocks of a shuffled
    # pool, gives bit-identical decode and chunked-prefill outputs
    rng = np.random.default_rng(12)
    hkv, d, h = 2, 16, 8
    lens = [1, 15, 16, 17, 63, 64, 65, 130]
    f32 = lambda *shape: rng.standard_normal(shape).astype(np.float32)
    seqs = [(f32(hkv, L, d), f32(hkv, L, d)) for L in lens]
    q = f32(len(lens), h, d)
    nq = [min(L, 3) for L in lens]
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    qp = f32(int(qs[-1]), h, d)
    sl = np.array(lens, np.int32)
    dec, pre = [], []
    for bs in (16, 32, 64, 128):
        kc, vc, bt = _layout(np.random.default_rng(bs), seqs, bs, hkv, d)
        dec.append(oracle.paged_attention_decode(q, kc, vc, bt, sl, scale=0.4, q_dtype="f32",
                                                 cache_dtype="f32"))
        pre.append(oracle.paged_attention_prefill(qp, kc, vc, bt, sl, qs, scale=0.4,
                                                  q_dtype="f32", cache_dtype="f32"))
    for a in dec[1:]:
        assert np.array_equal(a, dec[0])
    for a in pre[1:]:
        assert np.array_equal(a, pre[0])
    assert np.isfinite(dec[0]).all() and np.isfinite(pre[0]).all()
