"""The allocation-free decode entry point (GPU).

pa_paged_attention_decode_static_workspace is for callers that cannot allocate
device memory -- a plugin whose host process owns every allocation, or an engine
that has already handed nearly all HBM to its KV block pool.  Its split-partition
scratch is the library's fixed per-GPU array instead of a caller workspace.

This file is collected last on purpose, and must pass both alone in a fresh
process and after every other test.  Through the C ABI it checks that two calls
in a row (the second finds the first call's leftovers in the shared scratch)
give outputs bit for bit equal to the workspace entry point's -- the same
kernels on the same partitions, so any stale scratch read would show -- and
within the tests' tolerance of the oracle; that the second call changes no free
device memory; that a call with no sequences is the set-up call and nothing else;
and that sizes beyond the fixed maximum are rejected.
"""

import pytest
import torch

import paged_kv_cache_413_b200 as pa
from paged_kv_cache_413_b200 import workloads as W

import flow

pytestmark = pytest.mark.gpu


def _static(out, d, wl, max_len, part):
    pa.pa_paged_attention_decode_static_workspace(
        out, d.query, d.key_cache, d.value_cache, d.block_tables, d.seq_lens,
        max_seq_len=max_len, scale=wl.scale, k_scale=wl.k_scale, v_scale=wl.v_scale,
        partition_size=part)


@pytest.mark.parametrize("name,over,part,out_dtype", [
    ("long_splitk", dict(num_seqs=3, seq_lens=(4100, 2999, 513)), 512, "bf16"),
    ("llama2_70b_gqa", dict(num_seqs=12), 128, "f32"),
    ("llama2_7b", dict(num_seqs=8), 0, "f16"),
])
def test_static_workspace_matches_workspace_entry_point(name, over, part, out_dtype):
    wl = W.make_workload(name, **over)
    d = flow.to_device(wl)
    ref = flow.gpu_step(wl, d, out_dtype, part)        # existing entry point, own workspace
    torch.cuda.synchronize()
    max_len = flow.max_seq_len(wl)
    need = pa.pa_paged_attention_workspace_size(d.query.shape[0], wl.cfg.num_heads,
                                                wl.cfg.num_kv_heads, wl.cfg.head_dim, max_len,
                                                part)
    assert 0 < need <= pa.binding.PA_STATIC_WORKSPACE_BYTES
    outs = []
    for call in range(2):
        out = torch.full_like(ref, float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        _static(out, d, wl, max_len, part)
        torch.cuda.synchronize()
        if call == 1:  # the first call may set up the array; the second allocates nothing
            assert torch.cuda.mem_get_info()[0] == free_before
        outs.append(out)
    assert pa.pa_get_device_error() == 0
    kc, vc = flow.oracle_caches(wl)
    oracle_out = flow.oracle_decode(wl, kc, vc)
    for out in outs:
        assert torch.equal(out, ref)
        err = flow.max_abs_err(out, oracle_out)
        assert err <= flow.TOL[out_dtype], err


def test_static_workspace_call_without_sequences_is_only_the_set_up():
    wl = W.make_workload("tiny")
    d = flow.to_device(wl)
    out = torch.full(d.query.shape, float("nan"), dtype=torch.float16, device="cuda")
    empty_q = d.query[:0]
    pa.pa_paged_attention_decode_static_workspace(
        out[:0], empty_q, d.key_cache, d.value_cache, d.block_tables[:0], d.seq_lens[:0],
        max_seq_len=0, scale=wl.scale)
    torch.cuda.synchronize()
    free_before = torch.cuda.mem_get_info()[0]
    pa.pa_paged_attention_decode_static_workspace(
        out[:0], empty_q, d.key_cache, d.value_cache, d.block_tables[:0], d.seq_lens[:0],
        max_seq_len=0, scale=wl.scale)
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free_before
    assert torch.isnan(out).all()  # nothing was written


def test_static_workspace_rejects_sizes_beyond_the_maximum():
    wl = W.make_workload("tiny")
    d = flow.to_device(wl)
    out = torch.empty(d.query.shape, dtype=torch.float16, device="cuda")
    # 4 seqs x 4 heads x 8192 partitions of 16 tokens x (64 + 2) floats: ~34.6 MB of scratch
    max_len = 16 * 8192
    bt = torch.zeros(4, 8192, dtype=torch.int32, device="cuda")
    assert pa.pa_paged_attention_workspace_size(4, 4, 4, 64, max_len, 16) > \
        pa.binding.PA_STATIC_WORKSPACE_BYTES
    with pytest.raises(pa.PaError, match="static scratch"):
        pa.pa_paged_attention_decode_static_workspace(
            out, d.query, d.key_cache, d.value_cache, bt, d.seq_lens, max_seq_len=max_len,
            scale=wl.scale, partition_size=16)
