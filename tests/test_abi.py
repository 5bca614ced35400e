"""The C ABI library loads and exports what include/pa.h declares (CPU only).

Calls here only exercise host-side validation, which returns before any CUDA
call, and the pure host workspace-size function.
"""

import ctypes
import os
import re

import pytest

import paged_kv_cache_413_b200 as pa
from paged_kv_cache_413_b200 import build as pa_build
from paged_kv_cache_413_b200.binding import EXPORTS

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    pa_build.build()
    return pa.library()


def _declared():
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(pa_[a-z_]+)\s*\(", src)))


def test_header_declares_the_entry_points():
    assert sorted(EXPORTS) == _declared()


def test_every_declared_symbol_is_exported(lib):
    for name in _declared():
        assert hasattr(lib, name), name
        assert ctypes.cast(getattr(lib, name), ctypes.c_void_p).value


# the entry points that compute something the pages define; the rest are host
# helpers (sizes, status strings, the device error word)
COMPUTE_ENTRY_POINTS = ["pa_reshape_and_cache", "pa_paged_attention_decode",
                        "pa_paged_attention_decode_shared_prefix", "pa_paged_attention_prefill",
                        "pa_copy_blocks", "pa_swap_blocks",
                        "pa_paged_attention_decode_static_workspace"]
PAGES = ("vLLM 推理优化技术深度调研报告", "vLLM推理引擎PagedAttention原理与性能优化实战",
         "vLLM 是什么")


def test_every_compute_entry_point_cites_the_pages():
    """The comment block before each compute entry point names the page (by its
    title) and the section that defines the operation."""
    src = open(os.path.join(ROOT, "include", "pa.h")).read()
    for name in COMPUTE_ENTRY_POINTS:
        m = re.search(r"/\*((?:(?!\*/).)*)\*/\s*int\s+" + name + r"\s*\(", src, re.S)
        assert m, f"{name}: no comment block before its declaration"
        com = m.group(1)
        joined = re.sub(r"\s*\n\s*\*\s*", "", com)  # a title may wrap over lines
        assert any(p in joined or p.replace(" ", "") in joined for p in PAGES), \
            f"{name}: cites no page"
        assert re.search(r"\bsec\b|§", com), f"{name}: cites no section"


def test_status_strings(lib):
    assert pa.pa_status_string(0) == "PA_OK"
    assert pa.pa_status_string(-3) == "PA_ERR_WORKSPACE"
    assert pa.pa_status_string(7) == "PA_UNKNOWN_STATUS"


def test_workspace_size_host_function(lib):
    ws = pa.pa_paged_attention_workspace_size
    up = lambda x: (x + 255) // 256 * 256
    # explicit partitions: one partition needs no workspace
    assert ws(64, 32, 32, 128, 512, 512) == 0
    # 8 seqs x 32 heads x 64 partitions of 512: m, l (256-byte aligned) and o
    rows = 8 * 32 * 64
    assert ws(8, 32, 8, 128, 32768, 512) == up(rows * 4) * 2 + up(rows * 128 * 4)
    # default: >= 2048 (sequence, head group) units keep sequences whole
    assert ws(64, 32, 32, 128, 2048, 0) == 0          # MHA: 64 x 32 units
    assert ws(256, 64, 8, 128, 768, 0) == 0           # GQA-8: 256 x 8 units
    # default: 8 x 32 / 4 = 64 units -> 32 partitions of 1024 tokens
    rows = 8 * 32 * 32
    assert ws(8, 32, 8, 128, 32768, 0) == up(rows * 4) * 2 + up(rows * 128 * 4)
    # default never goes below 256-token partitions
    rows = 4 * 4 * 4
    assert ws(4, 4, 4, 64, 1000, 0) == up(rows * 4) * 2 + up(rows * 64 * 4)
    assert ws(4, 4, 4, 64, 100, 0) == 0
    assert ws(8, 32, 8, 128, 1000, 24) == 0           # not a multiple of 16
    assert ws(8, 30, 8, 128, 1000, 0) == 0            # heads not a multiple of kv heads
    part = pa.pa_paged_attention_partition_size
    assert part(64, 32, 32, 2048, 0) == 2048
    assert part(256, 64, 8, 768, 0) == 768
    assert part(256, 32, 8, 1036, 0) == 1040            # whole, rounded up to a block
    assert part(8, 32, 8, 32768, 0) == 1024
    assert part(8, 32, 8, 32768, 512) == 512
    assert part(4, 4, 4, 1000, 0) == 256
    assert part(4, 4, 4, 100, 0) == 112
    assert part(4, 4, 4, 100, 8) == 0


def test_host_validation_without_gpu(lib):
    P, nullp = ctypes.c_void_p, None
    # reshape: bad sizes / unsupported block size / scale
    assert lib.pa_reshape_and_cache(nullp, nullp, nullp, nullp, nullp, 4, 0, 64, 16, 8, 0, 0,
                                    1.0, 1.0, nullp) == -1
    assert lib.pa_reshape_and_cache(nullp, nullp, nullp, nullp, nullp, 4, 2, 64, 24, 8, 0, 0,
                                    1.0, 1.0, nullp) == -2          # block size 24
    assert lib.pa_reshape_and_cache(nullp, nullp, nullp, nullp, nullp, 4, 2, 64, 16, 8, 1, 3,
                                    0.0, 1.0, nullp) == -1
    assert lib.pa_reshape_and_cache(nullp, nullp, nullp, nullp, nullp, 4, 2, 64, 16, 8, 0, 1,
                                    1.0, 1.0, nullp) == -2          # f16 -> bf16 cache
    assert lib.pa_reshape_and_cache(nullp, nullp, nullp, nullp, nullp, 0, 2, 64, 16, 8, 0, 0,
                                    1.0, 1.0, nullp) == 0           # no tokens: no-op
    assert lib.pa_reshape_and_cache(nullp, nullp, nullp, nullp, nullp, 3, 2, 64, 16, 8, 0, 0,
                                    1.0, 1.0, nullp) == -1          # null pointers
    a = P(0x1000)
    mis = P(0x1008)
    assert lib.pa_reshape_and_cache(a, a, mis, a, a, 3, 2, 64, 16, 8, 0, 0, 1.0, 1.0,
                                    nullp) == -1                     # misaligned cache

    def dec(**kw):
        args = dict(out=a, q=a, kc=a, vc=a, bt=a, mb=8, sl=a, b=2, maxl=128, h=8, hkv=2, d=128,
                    bs=16, nb=64, scale=0.1, qd=0, cd=0, od=0, ks=1.0, vs=1.0, part=0, ws=nullp,
                    wsb=0)
        args.update(kw)
        return lib.pa_paged_attention_decode(*args.values(), nullp)

    assert dec(h=6, hkv=4) == -1                 # heads not a multiple of kv heads
    assert dec(d=96) == -2                       # head_dim
    assert dec(bs=24) == -2                      # block size (16, 32, 64, 128 only)
    assert dec(qd=0, cd=1) == -2                 # f16 q with bf16 cache
    assert dec(od=3) == -2                       # fp8 output
    assert dec(part=24) == -1                    # partition not a multiple of 16
    assert dec(mb=4) == -1                       # table too narrow for max_seq_len
    assert dec(maxl=4096, mb=256) == -3          # needs a workspace, none given
    assert dec(cd=3, ks=0.0) == -1               # fp8 without a scale
    assert dec(out=mis) == -1                    # misaligned output
    assert dec(b=0) == 0                         # empty batch: no-op
    # copy_blocks
    assert lib.pa_copy_blocks(nullp, nullp, 0, nullp, 5, 4096, 8, nullp) == 0
    assert lib.pa_copy_blocks(nullp, nullp, 2, nullp, 5, 4096, 8, nullp) == -1
    assert lib.pa_copy_blocks(nullp, nullp, 2, nullp, 5, 4096, 0, nullp) == -1
    assert lib.pa_get_device_error(nullp, nullp) == -1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import paged_kv_cache_413_b200.binding as b
    monkeypatch.setattr(b, "_LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(b, "_lib", None)
    with pytest.raises(RuntimeError, match="no fallback"):
        b.library()
