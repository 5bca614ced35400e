"""Stream order of a decode step through the C ABI, checked against the oracle.

The decode kernels are launched as programmatic dependents of the cache write
before them: their CTAs may be scheduled while the write is still running, and
each waits for it before touching global memory.  The split-K merge is in turn
a dependent of the decode.  These tests run several steps on one stream with no
host synchronisation.  Each step does these things:
  1. sets the new tokens' slots to NaN again (a plain torch kernel);
  2. (copy-on-write workloads) copies the diverging beams' blocks again;
  3. writes that step's new K/V (different values every step);
  4. decodes that step's queries into an output of its own.
Consecutive decodes share one split-K workspace.  Two kinds of mistake would show:
  * a decode that read the pool before its step's write finished gives NaN or
    the wrong token;
  * a write that ran before the copies finished is overwritten by them, which
    also leaves the wrong token;
  * a decode whose partials overwrote a workspace the previous merge was still
    reading gives wrong outputs.
Every step is checked against the oracle.  The same chain, captured in a CUDA
graph and replayed, must give the same bytes.
"""

import dataclasses

import numpy as np
import pytest
import torch

import paged_kv_cache_413_b200 as pa
from paged_kv_cache_413_b200 import workloads as W

import flow

pytestmark = pytest.mark.gpu

STEPS = 4


def _step_inputs(wl, n, seed):
    """n copies of the workload, each with its own new tokens and queries."""
    rng = np.random.default_rng(seed)
    draw = lambda t: torch.from_numpy(rng.standard_normal(tuple(t.shape), dtype=np.float32)).to(
        t.dtype)
    return [dataclasses.replace(wl, new_key=draw(wl.new_key), new_value=draw(wl.new_value),
                                query=draw(wl.query)) for _ in range(n)]


def _poisoner(wl, d):
    """A closure that sets every new-token slot of the device pools to NaN."""
    sm = d.slot_mapping[d.slot_mapping >= 0]
    bs = wl.cfg.block_size
    blk, off = sm // bs, sm % bs
    fp8 = wl.cfg.cache_dtype == "e4m3"
    # device scalars, so that the closure copies nothing from the host (graph capture)
    dev = d.key_cache.device
    val = torch.full((), 0x7F, dtype=torch.uint8, device=dev) if fp8 else \
        torch.full((), float("nan"), dtype=d.key_cache.dtype, device=dev)

    def poison():
        for pool in (d.key_cache, d.value_cache):
            if fp8:
                pool.view(torch.uint8)[blk, :, off, :] = val  # E4M3 NaN
            else:
                pool[blk, :, off, :] = val

    return poison


def _chain(wl, d, steps, outs, launch_decode):
    poison = _poisoner(wl, d)
    dev = [(s.new_key.cuda(), s.new_value.cuda(), s.query.cuda()) for s in steps]
    copies = d.block_mapping if d.block_mapping is not None and d.block_mapping.numel() else None

    def run():
        for (nk, nv, q), out in zip(dev, outs):
            poison()
            if copies is not None:
                pa.pa_copy_blocks([d.key_cache], [d.value_cache], copies)
            pa.pa_reshape_and_cache(nk, nv, d.key_cache, d.value_cache, d.slot_mapping,
                                    k_scale=wl.k_scale, v_scale=wl.v_scale)
            launch_decode(q, out)

    return run


def _check_steps(steps, outs, out_dtype):
    for k, (s, out) in enumerate(zip(steps, outs)):
        kc, vc = flow.oracle_caches(s)
        ref = flow.oracle_decode(s, kc, vc)
        err = flow.max_abs_err(out, ref)
        assert err <= flow.TOL[out_dtype], f"step {k}: max abs error {err:.3e}"


def _decode_launcher(wl, d, partition, ws):
    def launch(q, out):
        pa.pa_paged_attention_decode(out, q, d.key_cache, d.value_cache, d.block_tables,
                                     d.seq_lens, max_seq_len=flow.max_seq_len(wl), scale=wl.scale,
                                     k_scale=wl.k_scale, v_scale=wl.v_scale,
                                     partition_size=partition, workspace=ws)
    return launch


def _shared_launcher(wl, d):
    gs, pl = wl.group_starts.cuda(), wl.prefix_lens.cuda()
    mg = int((wl.group_starts[1:] - wl.group_starts[:-1]).max())

    def launch(q, out):
        pa.pa_paged_attention_decode_shared_prefix(
            out, q, d.key_cache, d.value_cache, d.block_tables, d.seq_lens, gs, pl,
            max_seq_len=flow.max_seq_len(wl), max_group_size=mg, scale=wl.scale,
            k_scale=wl.k_scale, v_scale=wl.v_scale)
    return launch


def _outputs(wl, out_dtype, n):
    return [torch.full(tuple(wl.query.shape), float("nan"), dtype=flow.TORCH_DT[out_dtype],
                       device="cuda") for _ in range(n)]


@pytest.mark.parametrize("name,over,part,out_dtype", [
    ("llama2_7b", dict(num_seqs=6), 0, "f16"),       # SIMT consumer, one partition
    ("llama2_7b", dict(num_seqs=6), 256, "f32"),     # SIMT consumer + merge
    ("llama2_70b_gqa", dict(num_seqs=10), 0, "bf16"),  # tensor-core consumer
    ("llama2_70b_gqa", dict(num_seqs=10), 128, "f32"),  # tensor-core consumer + merge
    ("long_splitk", dict(num_seqs=2, seq_lens=(2100, 1500)), 512, "bf16"),
])
def test_steps_on_one_stream(name, over, part, out_dtype):
    wl = W.make_workload(name, **over)
    d = flow.to_device(wl)
    flow.gpu_prepare(wl, d)
    steps = _step_inputs(wl, STEPS, seed=1000 * len(name) + part)
    outs = _outputs(wl, out_dtype, STEPS)
    ws = flow.workspace_for(wl, part)
    _chain(wl, d, steps, outs, _decode_launcher(wl, d, part, ws))()
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    _check_steps(steps, outs, out_dtype)


@pytest.mark.parametrize("qdt,shared_len,out_dtype", [("bf16", 72, "f32"), ("f16", 1032, "f16")])
def test_shared_prefix_steps_on_one_stream(qdt, shared_len, out_dtype):
    wl = W.make_workload("beam_cow_fp8", num_seqs=3, shared_len=shared_len, q_dtype=qdt,
                         seed=shared_len + 7)
    d = flow.to_device(wl)
    flow.gpu_prepare(wl, d)
    steps = _step_inputs(wl, STEPS, seed=shared_len)
    outs = _outputs(wl, out_dtype, STEPS)
    _chain(wl, d, steps, outs, _shared_launcher(wl, d))()
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    _check_steps(steps, outs, out_dtype)


@pytest.mark.parametrize("shared", [False, True])
def test_chain_in_a_cuda_graph(shared):
    if shared:
        wl = W.make_workload("beam_cow_fp8", num_seqs=3, shared_len=264, seed=11)
        out_dtype = "bf16"
    else:
        wl = W.make_workload("llama2_70b_gqa", num_seqs=10)
        out_dtype = "f32"
    part = 0 if shared else 128
    d = flow.to_device(wl)
    flow.gpu_prepare(wl, d)
    steps = _step_inputs(wl, STEPS, seed=5)
    launch = _shared_launcher(wl, d) if shared else \
        _decode_launcher(wl, d, part, flow.workspace_for(wl, part))
    eager = _outputs(wl, out_dtype, STEPS)
    _chain(wl, d, steps, eager, launch)()
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    _check_steps(steps, eager, out_dtype)

    replayed = _outputs(wl, out_dtype, STEPS)
    run = _chain(wl, d, steps, replayed, launch)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=side):
        run()
    torch.cuda.current_stream().wait_stream(side)
    for _ in range(2):
        for o in replayed:
            o.fill_(float("nan"))
        g.replay()
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    for k, (a, b) in enumerate(zip(eager, replayed)):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8)), f"step {k} differs"
    del g


@pytest.mark.parametrize("name,over,part,shared", [
    ("llama2_7b", dict(num_seqs=6), 256, False),
    ("llama2_70b_gqa", dict(num_seqs=10), 0, False),
    ("beam_cow_fp8", dict(num_seqs=3, shared_len=72), 0, True),
])
def test_query_written_by_the_kernel_just_before(name, over, part, shared):
    """One query buffer for every step, filled by a torch elementwise kernel right
    before each decode: a decode that read it early would see the previous step's
    queries."""
    wl = W.make_workload(name, **over)
    d = flow.to_device(wl)
    flow.gpu_prepare(wl, d)
    pa.pa_reshape_and_cache(d.new_key, d.new_value, d.key_cache, d.value_cache, d.slot_mapping,
                            k_scale=wl.k_scale, v_scale=wl.v_scale)
    steps = _step_inputs(wl, STEPS, seed=77)
    out_dtype = "f32"
    outs = _outputs(wl, out_dtype, STEPS)
    launch = _shared_launcher(wl, d) if shared else \
        _decode_launcher(wl, d, part, flow.workspace_for(wl, part))
    qs = [s.query.cuda() for s in steps]
    qbuf = torch.empty_like(qs[0])
    torch.cuda.synchronize()
    for q, out in zip(qs, outs):
        torch.mul(q, 1, out=qbuf)  # an elementwise kernel, not a copy
        launch(qbuf, out)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    # the pool holds the workload's own new tokens; only the queries change
    kc, vc = flow.oracle_caches(wl)
    for k, (s, out) in enumerate(zip(steps, outs)):
        ref = flow.oracle_decode(dataclasses.replace(wl, query=s.query), kc, vc)
        err = flow.max_abs_err(out, ref)
        assert err <= flow.TOL[out_dtype], f"step {k}: max abs error {err:.3e}"
