"""GPU parity of the shared-prefix decode (copy-on-write groups) against the oracle.

The oracle is the ordinary per-sequence decode: sharing blocks changes where the
bytes come from, never the result.  Cases: beam-search workloads with an FP8
cache (the copy-on-write recipe), random groups of sequences forked from a common
prefix with GQA group sizes 1..16 (groups larger than one CTA's share included),
broken promises (they set PA_DEVERR_PREFIX and fault nothing), E4M3 caches of
every group shape (the tensor-core kernel), and the full-size beam workload, every
output.
"""

import numpy as np
import pytest
import torch

import paged_kv_cache_413_b200 as pa
from paged_kv_cache_413_b200 import workloads as W

import flow

pytestmark = pytest.mark.gpu


def _run_shared(wl, d, out_dtype, group_starts=None, prefix_lens=None, max_group_size=None):
    gs = (wl.group_starts if group_starts is None else group_starts).cuda()
    pl = (wl.prefix_lens if prefix_lens is None else prefix_lens).cuda()
    if max_group_size is None:
        max_group_size = int((gs[1:] - gs[:-1]).max())
    out = torch.full(d.query.shape, float("nan"), dtype=flow.TORCH_DT[out_dtype], device="cuda")
    pa.pa_paged_attention_decode_shared_prefix(
        out, d.query, d.key_cache, d.value_cache, d.block_tables, d.seq_lens, gs, pl,
        max_seq_len=flow.max_seq_len(wl), max_group_size=max_group_size, scale=wl.scale,
        k_scale=wl.k_scale, v_scale=wl.v_scale)
    return out


def _check(wl, out_dtype, seqs=None, prompts=None):
    d = flow.to_device(wl)
    flow.gpu_prepare(wl, d)
    pa.pa_reshape_and_cache(d.new_key, d.new_value, d.key_cache, d.value_cache, d.slot_mapping,
                            k_scale=wl.k_scale, v_scale=wl.v_scale)
    out = _run_shared(wl, d, out_dtype)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    kc, vc = flow.oracle_caches(wl, prompts=prompts)
    ref = flow.oracle_decode(wl, kc, vc, seqs)
    got = out if seqs is None else out[torch.as_tensor(seqs, device="cuda")]
    err = flow.max_abs_err(got, ref)
    assert err <= flow.TOL[out_dtype], f"max abs error {err:.3e}"
    return d, out


@pytest.mark.parametrize("qdt", ["bf16", "f16"])
@pytest.mark.parametrize("shared_len,out_dtype", [(72, "f32"), (1032, "bf16"), (40, "f32")])
def test_beam_fp8(qdt, shared_len, out_dtype):
    wl = W.make_workload("beam_cow_fp8", num_seqs=3, shared_len=shared_len, q_dtype=qdt,
                         seed=shared_len)
    if out_dtype == "bf16" and qdt == "f16":
        out_dtype = "f16"
    _check(wl, out_dtype)


@pytest.mark.parametrize("h,hkv", [(16, 4), (64, 8), (8, 8), (32, 2), (12, 4), (16, 8)])
@pytest.mark.parametrize("dt", ["bf16", "f16"])
def test_groups(h, hkv, dt):
    wl = W.make_group_workload(6, (1, 7), (0, 4), (1, 50), num_heads=h, num_kv_heads=hkv,
                               dtype=dt, seed=h * 10 + hkv)
    d, out = _check(wl, "f32")
    # and the same inputs through the ordinary decode agree with it closely
    ref = torch.empty_like(out)
    pa.pa_paged_attention_decode(ref, d.query, d.key_cache, d.value_cache, d.block_tables,
                                 d.seq_lens, max_seq_len=flow.max_seq_len(wl), scale=wl.scale,
                                 partition_size=1024)
    assert (out - ref).abs().max().item() <= 2e-3


def test_long_suffixes_and_group_of_one():
    wl = W.make_group_workload(4, (1, 3), (0, 2), (100, 700), num_heads=32, num_kv_heads=8,
                               dtype="bf16", seed=77)
    _check(wl, "bf16")


def test_broken_promises_set_error_bits_without_fault():
    # G = 4: one CTA serves 4 sequences, so groups of 6 need two CTAs each
    wl = W.make_group_workload(3, (6, 6), (2, 2), (5, 20), num_heads=16, num_kv_heads=4,
                               dtype="bf16", seed=5)
    d = flow.to_device(wl)
    pa.pa_reshape_and_cache(d.new_key, d.new_value, d.key_cache, d.value_cache, d.slot_mapping)
    torch.cuda.synchronize()
    pa.pa_get_device_error()
    # a member's table differs inside the prefix
    bt = d.block_tables.clone()
    bt[1, 0] = bt[7, 0]
    d2 = flow.Dev(**{**d.__dict__, "block_tables": bt})
    _run_shared(wl, d2, "f32")
    assert pa.pa_get_device_error() & 0x20
    # prefix not a multiple of the block size
    _run_shared(wl, d, "f32", prefix_lens=wl.prefix_lens + 3)
    assert pa.pa_get_device_error() & 0x20
    # a group larger than the launch covers (max_group_size 4 -> one CTA per group)
    _run_shared(wl, d, "f32", max_group_size=4)
    assert pa.pa_get_device_error() & 0x20
    # and the promise kept: no bits
    _run_shared(wl, d, "f32")
    assert pa.pa_get_device_error() == 0


def test_full_beam_cow_fp8_shared():
    # every output of the full-size workload, in the benchmark's launch configuration
    wl = W.make_workload("beam_cow_fp8")
    _check(wl, "bf16")


@pytest.mark.parametrize("h,hkv,qdt", [(32, 8, "bf16"), (16, 16, "f16"), (32, 16, "bf16"),
                                       (64, 8, "f16"), (64, 4, "bf16"), (24, 8, "bf16")])
def test_groups_fp8(h, hkv, qdt):
    """E4M3 caches: GQA groups of 1 to 16 heads, members whose own tiles span several
    128-token stages, prefixes of 0 to 5 blocks, groups of 1 to 7 members."""
    wl = W.make_group_workload(5, (1, 7), (0, 5), (1, 300), num_heads=h, num_kv_heads=hkv,
                               dtype=qdt, seed=h * 3 + hkv, cache_dtype="e4m3")
    d, out = _check(wl, "f32")
    ref = torch.empty_like(out)
    pa.pa_paged_attention_decode(ref, d.query, d.key_cache, d.value_cache, d.block_tables,
                                 d.seq_lens, max_seq_len=flow.max_seq_len(wl), scale=wl.scale,
                                 k_scale=wl.k_scale, v_scale=wl.v_scale, partition_size=1024)
    assert (out - ref).abs().max().item() <= 2e-3


@pytest.mark.parametrize("bs", [32, 64, 128])
def test_groups_fp8_block_sizes(bs):
    wl = W.make_group_workload(4, (2, 6), (0, 4), (1, 200), num_heads=32, num_kv_heads=8,
                               dtype="bf16", seed=bs + 1, block_size=bs, cache_dtype="e4m3")
    _check(wl, "bf16")


def test_fp8_long_prefix_and_one_token_members():
    """A 4000-token prefix (32 stages) shared by 6 members, next to groups whose
    members own every token (prefix 0) and one-token members."""
    wl = W.make_group_workload(3, (6, 6), (250, 250), (1, 40), num_heads=32, num_kv_heads=8,
                               dtype="bf16", seed=11, cache_dtype="e4m3")
    _check(wl, "f32")
    wl = W.make_group_workload(6, (1, 4), (0, 0), (1, 1), num_heads=16, num_kv_heads=4,
                               dtype="f16", seed=12, cache_dtype="e4m3")
    _check(wl, "f16")


@pytest.mark.parametrize("bs", [32, 64])
def test_groups_block_sizes(bs):
    wl = W.make_group_workload(5, (1, 6), (0, 3), (1, 90), num_heads=32, num_kv_heads=8,
                               dtype="bf16", seed=bs, block_size=bs)
    _check(wl, "f32")


@pytest.mark.parametrize("qdt", ["bf16", "f16"])
def test_fp8_persistent_walk_many_units_and_empty_contexts(qdt):
    """E4M3 caches, far more units than resident CTAs (1440 here: each CTA walks
    several, their stages through one ring), units past a small group's members
    (no sequence: nothing written), and whole groups whose contexts are empty
    (prefix 0, length 0: zero outputs) among them."""
    wl = W.make_group_workload(90, (1, 7), (0, 3), (1, 60), num_heads=32, num_kv_heads=8,
                               dtype=qdt, seed=31, cache_dtype="e4m3")
    d = flow.to_device(wl)
    pa.pa_reshape_and_cache(d.new_key, d.new_value, d.key_cache, d.value_cache, d.slot_mapping,
                            k_scale=wl.k_scale, v_scale=wl.v_scale)
    gs = wl.group_starts.tolist()
    sl, pl = wl.seq_lens.clone(), wl.prefix_lens.clone()
    empty = []
    for g in (3, 40, 89):
        empty += list(range(gs[g], gs[g + 1]))
        pl[g] = 0
    sl[empty] = 0
    d2 = flow.Dev(**{**d.__dict__, "seq_lens": sl.cuda()})
    out = _run_shared(wl, d2, "f32", prefix_lens=pl)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    assert torch.equal(out[empty], torch.zeros_like(out[empty]))
    rest = [i for i in range(len(sl)) if i not in set(empty)]
    kc, vc = flow.oracle_caches(wl)
    ref = flow.oracle_decode(wl, kc, vc, rest)
    err = flow.max_abs_err(out[torch.as_tensor(rest, device="cuda")], ref)
    assert err <= flow.TOL["f32"], f"max abs error {err:.3e}"


@pytest.mark.parametrize("out_dtype", ["bf16", "f32"])
def test_fp8_unaligned_output_is_rejected(out_dtype):
    """The tensor-core kernel writes its outputs in 16-byte pieces; the entry point
    takes only 16-byte aligned data pointers and refuses an output that starts one
    element past a boundary before anything is launched (the output stays as it
    was), then decodes the same batch into an aligned output."""
    wl = W.make_group_workload(12, (1, 5), (1, 4), (1, 40), num_heads=32, num_kv_heads=8,
                               dtype="bf16", seed=37, cache_dtype="e4m3")
    d = flow.to_device(wl)
    pa.pa_reshape_and_cache(d.new_key, d.new_value, d.key_cache, d.value_cache, d.slot_mapping,
                            k_scale=wl.k_scale, v_scale=wl.v_scale)
    dt = flow.TORCH_DT[out_dtype]
    flat = torch.full((d.query.numel() + 1,), 7.0, dtype=dt, device="cuda")
    out = flat[1:].view(d.query.shape)
    assert out.data_ptr() % 16 != 0
    gs, pl = wl.group_starts.cuda(), wl.prefix_lens.cuda()
    with pytest.raises(pa.PaError, match="INVALID_ARG"):
        pa.pa_paged_attention_decode_shared_prefix(
            out, d.query, d.key_cache, d.value_cache, d.block_tables, d.seq_lens, gs, pl,
            max_seq_len=flow.max_seq_len(wl), max_group_size=int((gs[1:] - gs[:-1]).max()),
            scale=wl.scale, k_scale=wl.k_scale, v_scale=wl.v_scale)
    torch.cuda.synchronize()
    assert torch.all(flat == 7.0)
    got = _run_shared(wl, d, out_dtype)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    kc, vc = flow.oracle_caches(wl)
    err = flow.max_abs_err(got, flow.oracle_decode(wl, kc, vc, None))
    assert err <= flow.TOL[out_dtype], f"max abs error {err:.3e}"
