"""Failure detection on the GPU without a fault: a pipeline wait that runs out.

The library is built once more (build.TIMEOUT_TEST_FLAGS) with pipeline waits that
give up after 2 ms instead of about a second, and with a decode producer that
never announces or copies the 4th 16-token tile (index 3) of any CTA: that
stage's phase never completes, like a flag that nothing sets.  A decode through
that build must return, raise PA_DEVERR_PIPE_TIMEOUT in the build's device error
word, and leave the context usable: the same build then decodes a batch whose
CTAs have at most 3 tiles without any error bit and matches the oracle, and the
normal library decodes the first batch correctly.  Nothing faults, traps or hangs.
"""

import ctypes
import time

import pytest
import torch

import paged_kv_cache_413_b200 as pa
from paged_kv_cache_413_b200 import binding
from paged_kv_cache_413_b200 import build as pa_build
from paged_kv_cache_413_b200 import workloads as W

import flow

pytestmark = pytest.mark.gpu

PIPE_TIMEOUT = 0x8


@pytest.fixture(scope="module")
def timeout_lib():
    return binding.declare(ctypes.CDLL(pa_build.build_timeout_test()))


def _decode(lib, wl, d, out, nseq):
    """pa_paged_attention_decode of the first nseq sequences, through `lib`."""
    cfg = wl.cfg
    rc = lib.pa_paged_attention_decode(
        out.data_ptr(), d.query.data_ptr(), d.key_cache.data_ptr(), d.value_cache.data_ptr(),
        d.block_tables.data_ptr(), d.block_tables.shape[1], d.seq_lens.data_ptr(), nseq,
        int(wl.seq_lens[:nseq].max()), cfg.num_heads, cfg.num_kv_heads, cfg.head_dim,
        cfg.block_size, wl.num_blocks, wl.scale, binding.PA_F16, binding.PA_F16, binding.PA_F32,
        1.0, 1.0, 0, None, 0, torch.cuda.current_stream().cuda_stream)
    assert rc == 0, binding.STATUS.get(rc, rc)


def _device_error(lib):
    flag = ctypes.c_int(0)
    assert lib.pa_get_device_error(ctypes.byref(flag), torch.cuda.current_stream().cuda_stream) == 0
    return flag.value


def test_starved_pipeline_wait_reports_timeout_and_context_stays_usable(timeout_lib):
    wl = W.make_workload("tiny")            # lengths 1, 17, 33, 100: 1, 2, 3 and 7 tiles
    d = flow.to_device(wl)
    pa.pa_reshape_and_cache(d.new_key, d.new_value, d.key_cache, d.value_cache, d.slot_mapping)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    kc, vc = flow.oracle_caches(wl)
    ref = flow.oracle_decode(wl, kc, vc)

    # the 100-token sequence's CTAs reach tile 3: their waits on it run out
    _device_error(timeout_lib)
    out = torch.empty(d.query.shape, dtype=torch.float32, device="cuda")
    t0 = time.perf_counter()
    _decode(timeout_lib, wl, d, out, 4)
    bits = _device_error(timeout_lib)       # synchronises: the launch has returned
    assert time.perf_counter() - t0 < 10.0
    assert bits & PIPE_TIMEOUT
    # the sequences whose CTAs stop short of tile 3 were not disturbed
    assert flow.max_abs_err(out[:3], ref[:3]) <= flow.TOL["f32"]

    # the same build again, on CTAs of at most 3 tiles: no error, oracle-correct
    out3 = torch.full(d.query.shape, float("nan"), dtype=torch.float32, device="cuda")
    _decode(timeout_lib, wl, d, out3, 3)
    assert _device_error(timeout_lib) == 0
    assert flow.max_abs_err(out3[:3], ref[:3]) <= flow.TOL["f32"]

    # and the normal library on the full batch
    good = torch.empty(d.query.shape, dtype=torch.float32, device="cuda")
    pa.pa_paged_attention_decode(good, d.query, d.key_cache, d.value_cache, d.block_tables,
                                 d.seq_lens, max_seq_len=100, scale=wl.scale)
    torch.cuda.synchronize()
    assert pa.pa_get_device_error() == 0
    assert flow.max_abs_err(good, ref) <= flow.TOL["f32"]
