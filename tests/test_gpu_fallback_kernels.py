"""The kernels the launchers fall back to (GPU).

The E4M3 shared-prefix decode and the two-tile chunked prefill check once that
their build has the register count their setmaxnreg split assumes and otherwise
take a slower kernel with the same result: the shared-prefix decode on mma.sync,
the prefill one 128-row tile per CTA.  PA_FALLBACK_KERNELS=1 selects those kernels,
so that this file can check them against the oracle like the others.
"""

import pytest
import torch

import paged_kv_cache_413_b200 as pa
from paged_kv_cache_413_b200 import workloads as W

import flow
import test_gpu_prefill as prefill_tests
import test_gpu_shared_prefix as shared_tests

pytestmark = pytest.mark.gpu


@pytest.fixture
def fallback(monkeypatch):
    monkeypatch.setenv("PA_FALLBACK_KERNELS", "1")


@pytest.mark.parametrize("qdt", ["bf16", "f16"])
def test_shared_prefix_e4m3_on_mma_sync(fallback, qdt):
    wl = W.make_workload("beam_cow_fp8", num_seqs=3, shared_len=520, q_dtype=qdt, seed=9)
    shared_tests._check(wl, "f32")
    wl = W.make_group_workload(5, (1, 7), (0, 5), (1, 300), num_heads=32, num_kv_heads=8,
                               dtype=qdt, seed=19, cache_dtype="e4m3")
    shared_tests._check(wl, "f32")


@pytest.mark.parametrize("dt,out_dtype", [("bf16", "bf16"), ("f16", "f16"), ("bf16", "f32")])
def test_prefill_one_tile_per_cta(fallback, dt, out_dtype):
    # 64 query heads on 8 kv heads and chunks of up to 60 tokens: up to 4 row blocks
    # per (sequence, kv head), which the two-tile kernel would take
    wl = W.make_prefill_workload(4, (100, 500), (20, 60), num_heads=64, num_kv_heads=8,
                                 dtype=dt, seed=23)
    prefill_tests._check(wl, out_dtype)
