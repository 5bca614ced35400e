"""CPU oracle for paged-KV decode -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path never does: the CUDA
library in ``paged_kv_cache_413_b200`` fails loudly when it is missing instead of
falling back to anything here.

The arithmetic lives in ``pa_oracle.c`` (plain C, fp64, OpenMP over
(sequence, kv head)); this module only builds it with gcc, loads it with ctypes
and marshals numpy arrays.  It imports nothing from the CUDA path.

What each function computes, and the passage it follows:

* ``reshape_and_cache`` -- new K/V rows into the slots of the slot mapping
  ("vLLM 推理优化技术深度调研报告" sec 2, memory flow; "vLLM 是什么…" sec 2).
* ``copy_blocks`` -- whole-block copies, the copy step of copy-on-write
  ("vLLM推理引擎PagedAttention原理与性能优化实战" sec 3.2).
* ``swap_blocks`` -- whole-block moves between two pools (swapping to CPU memory,
  "vLLM 是什么…" sec 5 misconception 3).
* ``paged_attention_decode`` -- explicit gather through the block table, then
  textbook softmax(scale * q K^T) V ("vLLM 推理优化技术深度调研报告" sec 3
  formulas 3 and 4; dim. 1 sec 1 misconception 2).
* ``paged_attention_prefill`` -- several query tokens per sequence, each attending
  causally over the gathered context ("vLLM推理引擎PagedAttention原理与性能优化实战"
  sec 6, chunked prefill).
* ``decode_partition_stats`` / ``lse_merge`` -- the same definition applied to
  token ranges, and the log-sum-exp merge of those ranges.
* ``e4m3_encode`` / ``e4m3_decode`` / ``f16_decode`` / ``bf16_decode`` -- the
  number formats from their definitions (OCP OFP8 E4M3, IEEE binary16, bfloat16).

Every function is pinned by ``tests/test_oracle_*.py`` against closed forms,
library routines on special cases, brute force and the invariants the pages
state.  No function here is "parity unpinned".
"""

from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
# The oracle's own mutation test points this at a deliberately broken build.
_LIB_OVERRIDE = os.environ.get("PA_ORACLE_LIB_OVERRIDE")
_lock = threading.Lock()
_lib = None

# dtype codes of pa_oracle.c
DTYPES = {"f16": 0, "bf16": 1, "f32": 2, "e4m3": 3}
_ELT = {"f16": 2, "bf16": 2, "f32": 4, "e4m3": 1}
_NP_STORAGE = {"f16": np.uint16, "bf16": np.uint16, "f32": np.float32, "e4m3": np.uint8}


def build(force: bool = False) -> str:
    """Compile pa_oracle.c into liboracle.so next to it (gcc, -O2, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + ".tmp.%d" % os.getpid()
        cmd = ["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            if _LIB_OVERRIDE:
                lib = ctypes.CDLL(_LIB_OVERRIDE)
            else:
                build()
                lib = ctypes.CDLL(_LIB)
            P, I, L, F, D = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64,
                             ctypes.c_float, ctypes.c_double)
            lib.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, L, I, I, I, L, I, I, F, F]
            lib.oracle_reshape_and_cache.restype = I
            lib.oracle_copy_blocks.argtypes = [P, P, I, P, L, L]
            lib.oracle_copy_blocks.restype = I
            lib.oracle_swap_blocks.argtypes = [P, P, P, P, I, P, L, L, L, L]
            lib.oracle_swap_blocks.restype = I
            lib.oracle_paged_attention_decode.argtypes = [
                P, P, P, P, P, I, P, I, I, I, I, I, L, D, I, I, D, D]
            lib.oracle_paged_attention_decode.restype = I
            lib.oracle_paged_attention_prefill.argtypes = [
                P, P, P, P, P, I, P, P, I, I, I, I, I, L, D, I, I, D, D]
            lib.oracle_paged_attention_prefill.restype = I
            lib.oracle_decode_partition_stats.argtypes = [
                P, P, P, I, I, P, P, P, P, I, P, I, I, I, I, I, L, D, I, I, D, D]
            lib.oracle_decode_partition_stats.restype = I
            lib.oracle_lse_merge.argtypes = [P, P, P, P, L, I, I]
            lib.oracle_lse_merge.restype = None
            lib.oracle_f32_to_e4m3.argtypes = [P, P, L]
            lib.oracle_f32_to_e4m3.restype = None
            lib.oracle_to_f64.argtypes = [P, P, L, I]
            lib.oracle_to_f64.restype = I
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = I
            lib.oracle_set_num_threads.argtypes = [I]
            lib.oracle_set_num_threads.restype = I
            _lib = lib
    return _lib


def _raw(a, dtype: str | None = None) -> np.ndarray:
    """A C-contiguous numpy view of the storage bits of ``a`` (numpy or torch CPU)."""
    if not isinstance(a, np.ndarray):
        import torch  # plain CPU tensors only

        t = a.detach()
        if t.device.type != "cpu":
            raise ValueError("oracle inputs must live in host memory")
        t = t.contiguous()
        if t.dtype in (torch.float16, torch.bfloat16):
            t = t.view(torch.int16)
        elif t.dtype == getattr(torch, "float8_e4m3fn", None):
            t = t.view(torch.uint8)
        a = t.numpy()
    a = np.ascontiguousarray(a)
    if dtype is not None:
        want = _NP_STORAGE[dtype]
        if a.dtype.itemsize != np.dtype(want).itemsize:
            raise ValueError(f"array of {a.dtype} does not hold {dtype} elements")
        a = a.view(want)
    return a


def _ptr(a: np.ndarray) -> int:
    return a.ctypes.data


def num_threads() -> int:
    """OpenMP threads the oracle's decode loop uses."""
    return _load().oracle_num_threads()


def set_num_threads(n: int) -> int:
    """Use n OpenMP threads in later calls (the bench's single-thread timing);
    returns the count now in force."""
    return _load().oracle_set_num_threads(int(n))


def to_f64(a, dtype: str) -> np.ndarray:
    """Decode an array of ``dtype`` storage (f16/bf16/f32/e4m3) to fp64."""
    r = _raw(a, dtype)
    out = np.empty(r.shape, dtype=np.float64)
    if _load().oracle_to_f64(_ptr(out), _ptr(r), r.size, DTYPES[dtype]) != 0:
        raise ValueError("bad dtype")
    return out


def f16_decode(bits) -> np.ndarray:
    return to_f64(np.asarray(bits, dtype=np.uint16), "f16")


def bf16_decode(bits) -> np.ndarray:
    return to_f64(np.asarray(bits, dtype=np.uint16), "bf16")


def e4m3_decode(codes) -> np.ndarray:
    return to_f64(np.asarray(codes, dtype=np.uint8), "e4m3")


def e4m3_encode(x) -> np.ndarray:
    """Round fp32 values to E4M3 codes (RNE, saturating to +-448, NaN -> 0x7F)."""
    x = np.ascontiguousarray(np.asarray(x, dtype=np.float32))
    out = np.empty(x.shape, dtype=np.uint8)
    _load().oracle_f32_to_e4m3(_ptr(out), _ptr(x), x.size)
    return out


def reshape_and_cache(key, value, key_cache, value_cache, slot_mapping, *, src_dtype: str,
                      cache_dtype: str, k_scale: float = 1.0, v_scale: float = 1.0,
                      inplace: bool = False):
    """Return (key_cache, value_cache) numpy storage arrays with the tokens written.

    key, value: [T, H_kv, D] of ``src_dtype``; caches: [NB, H_kv, BS, D] of
    ``cache_dtype``; slot_mapping: [T] int64 (negative = skip).  The caches are
    copied first unless ``inplace`` (then contiguous host caches are written).
    """
    k = _raw(key, src_dtype)
    v = _raw(value, src_dtype)
    kc = _raw(key_cache, cache_dtype)
    vc = _raw(value_cache, cache_dtype)
    if not inplace:
        kc, vc = kc.copy(), vc.copy()
    elif not (kc.flags.writeable and vc.flags.writeable):
        raise ValueError("in-place cache write needs writeable host caches")
    sm = np.ascontiguousarray(np.asarray(slot_mapping, dtype=np.int64))
    nb, hkv, bs, d = kc.shape
    t = sm.shape[0]
    if k.shape != (t, hkv, d) or v.shape != (t, hkv, d) or vc.shape != kc.shape:
        raise ValueError("shape mismatch")
    rc = _load().oracle_reshape_and_cache(_ptr(k), _ptr(v), _ptr(kc), _ptr(vc), _ptr(sm), t, hkv,
                                          d, bs, nb, DTYPES[src_dtype], DTYPES[cache_dtype],
                                          float(k_scale), float(v_scale))
    if rc != 0:
        raise ValueError("oracle_reshape_and_cache rejected its arguments")
    return kc, vc


def copy_blocks(key_caches, value_caches, block_mapping, *, dtype: str):
    """Return copies of the per-layer caches with every (src, dst) block copied."""
    kcs = [_raw(x, dtype).copy() for x in key_caches]
    vcs = [_raw(x, dtype).copy() for x in value_caches]
    bm = np.ascontiguousarray(np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2))
    if not kcs:
        return kcs, vcs
    nb = kcs[0].shape[0]
    block_bytes = kcs[0].nbytes // nb
    for x in kcs + vcs:
        if x.shape != kcs[0].shape:
            raise ValueError("all layers must share one shape")
    if bm.size and (bm.min() < 0 or bm.max() >= nb):
        raise ValueError("block id out of range")
    kp = (ctypes.c_void_p * len(kcs))(*[_ptr(x) for x in kcs])
    vp = (ctypes.c_void_p * len(vcs))(*[_ptr(x) for x in vcs])
    rc = _load().oracle_copy_blocks(ctypes.cast(kp, ctypes.c_void_p),
                                    ctypes.cast(vp, ctypes.c_void_p), len(kcs), _ptr(bm),
                                    bm.shape[0], block_bytes)
    if rc != 0:
        raise ValueError("oracle_copy_blocks rejected its arguments")
    return kcs, vcs


def swap_blocks(dst_key_caches, dst_value_caches, src_key_caches, src_value_caches,
                block_mapping, *, dtype: str):
    """Return copies of the destination pools with every (src, dst) block moved in."""
    dk = [_raw(x, dtype).copy() for x in dst_key_caches]
    dv = [_raw(x, dtype).copy() for x in dst_value_caches]
    sk = [_raw(x, dtype) for x in src_key_caches]
    sv = [_raw(x, dtype) for x in src_value_caches]
    bm = np.ascontiguousarray(np.asarray(block_mapping, dtype=np.int64).reshape(-1, 2))
    if not dk:
        return dk, dv
    block_bytes = dk[0].nbytes // dk[0].shape[0]
    if sk[0].nbytes // sk[0].shape[0] != block_bytes:
        raise ValueError("source and destination blocks differ in size")
    arr = lambda xs: ctypes.cast((ctypes.c_void_p * len(xs))(*[_ptr(x) for x in xs]),
                                 ctypes.c_void_p)
    rc = _load().oracle_swap_blocks(arr(dk), arr(dv), arr(sk), arr(sv), len(dk), _ptr(bm),
                                    bm.shape[0], block_bytes, sk[0].shape[0], dk[0].shape[0])
    if rc != 0:
        raise ValueError("oracle_swap_blocks rejected its arguments")
    return dk, dv


def _decode_args(query, key_cache, value_cache, block_tables, seq_lens, q_dtype, cache_dtype):
    q = _raw(query, q_dtype)
    kc = _raw(key_cache, cache_dtype)
    vc = _raw(value_cache, cache_dtype)
    bt = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
    sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    b, h, d = q.shape
    nb, hkv, bs, d2 = kc.shape
    if d2 != d or vc.shape != kc.shape or bt.ndim != 2 or bt.shape[0] != b or sl.shape != (b,):
        raise ValueError("shape mismatch")
    return q, kc, vc, bt, sl, b, h, d, nb, hkv, bs


def paged_attention_decode(query, key_cache, value_cache, block_tables, seq_lens, *,
                           scale: float, q_dtype: str, cache_dtype: str, k_scale: float = 1.0,
                           v_scale: float = 1.0) -> np.ndarray:
    """fp64 [B, H, D] attention output of one query token per sequence."""
    q, kc, vc, bt, sl, b, h, d, nb, hkv, bs = _decode_args(query, key_cache, value_cache,
                                                           block_tables, seq_lens, q_dtype,
                                                           cache_dtype)
    out = np.zeros((b, h, d), dtype=np.float64)
    rc = _load().oracle_paged_attention_decode(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(bt),
                                               bt.shape[1], _ptr(sl), b, h, hkv, d, bs, nb,
                                               float(scale), DTYPES[q_dtype],
                                               DTYPES[cache_dtype], float(k_scale),
                                               float(v_scale))
    if rc != 0:
        raise ValueError("oracle_paged_attention_decode rejected its arguments")
    return out


def paged_attention_prefill(query, key_cache, value_cache, block_tables, seq_lens,
                            query_start, *, scale: float, q_dtype: str, cache_dtype: str,
                            k_scale: float = 1.0, v_scale: float = 1.0) -> np.ndarray:
    """fp64 [total_queries, H, D]: causal multi-query attention over the paged cache."""
    q = _raw(query, q_dtype)
    kc = _raw(key_cache, cache_dtype)
    vc = _raw(value_cache, cache_dtype)
    bt = np.ascontiguousarray(np.asarray(block_tables, dtype=np.int32))
    sl = np.ascontiguousarray(np.asarray(seq_lens, dtype=np.int32))
    qs = np.ascontiguousarray(np.asarray(query_start, dtype=np.int32))
    tq, h, d = q.shape
    nb, hkv, bs, d2 = kc.shape
    b = sl.shape[0]
    if d2 != d or vc.shape != kc.shape or bt.shape[0] != b or qs.shape != (b + 1,) or \
            qs[-1] != tq:
        raise ValueError("shape mismatch")
    out = np.zeros((tq, h, d), dtype=np.float64)
    rc = _load().oracle_paged_attention_prefill(_ptr(out), _ptr(q), _ptr(kc), _ptr(vc), _ptr(bt),
                                                bt.shape[1], _ptr(sl), _ptr(qs), b, h, hkv, d,
                                                bs, nb, float(scale), DTYPES[q_dtype],
                                                DTYPES[cache_dtype], float(k_scale),
                                                float(v_scale))
    if rc != 0:
        raise ValueError("oracle_paged_attention_prefill rejected its arguments")
    return out


def decode_partition_stats(query, key_cache, value_cache, block_tables, seq_lens, *,
                           partition_size: int, max_parts: int, scale: float, q_dtype: str,
                           cache_dtype: str, k_scale: float = 1.0, v_scale: float = 1.0):
    """(m, l, o): per token range of ``partition_size`` tokens, fp64.

    m, l: [B, H, max_parts]; o: [B, H, max_parts, D].
    """
    q, kc, vc, bt, sl, b, h, d, nb, hkv, bs = _decode_args(query, key_cache, value_cache,
                                                           block_tables, seq_lens, q_dtype,
                                                           cache_dtype)
    m = np.zeros((b, h, max_parts), dtype=np.float64)
    l = np.zeros((b, h, max_parts), dtype=np.float64)
    o = np.zeros((b, h, max_parts, d), dtype=np.float64)
    rc = _load().oracle_decode_partition_stats(_ptr(m), _ptr(l), _ptr(o), max_parts,
                                               partition_size, _ptr(q), _ptr(kc), _ptr(vc),
                                               _ptr(bt), bt.shape[1], _ptr(sl), b, h, hkv, d, bs,
                                               nb, float(scale), DTYPES[q_dtype],
                                               DTYPES[cache_dtype], float(k_scale),
                                               float(v_scale))
    if rc != 0:
        raise ValueError("oracle_decode_partition_stats rejected its arguments")
    return m, l, o


def lse_merge(m, l, o) -> np.ndarray:
    """Merge per-range statistics ([..., P], [..., P], [..., P, D]) into [..., D]."""
    m = np.ascontiguousarray(np.asarray(m, dtype=np.float64))
    l = np.ascontiguousarray(np.asarray(l, dtype=np.float64))
    o = np.ascontiguousarray(np.asarray(o, dtype=np.float64))
    parts, d = o.shape[-2], o.shape[-1]
    rows = int(np.prod(m.shape[:-1]))
    out = np.zeros(m.shape[:-1] + (d,), dtype=np.float64)
    _load().oracle_lse_merge(_ptr(out), _ptr(m), _ptr(l), _ptr(o), rows, parts, d)
    return out
