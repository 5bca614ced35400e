"""Thin Python binding of libpa.so (ctypes): argument marshalling only.

Every function has the name of the C entry point it calls (see include/pa.h) and
takes torch CUDA tensors, which supply device memory and streams; every step of
the computation runs in the library's kernels.  There is no fallback: if
libpa.so is missing or cannot be loaded, the first call raises.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

_LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libpa.so")
_lock = threading.Lock()
_lib = None

PA_F16, PA_BF16, PA_F32, PA_FP8_E4M3 = 0, 1, 2, 3
STATUS = {0: "PA_OK", -1: "PA_ERR_INVALID_ARG", -2: "PA_ERR_UNSUPPORTED",
          -3: "PA_ERR_WORKSPACE", -4: "PA_ERR_CUDA"}
DEVERR = {0x1: "SLOT_RANGE", 0x2: "BLOCK_RANGE", 0x4: "SEQ_LEN", 0x8: "PIPE_TIMEOUT",
          0x10: "COPY_RANGE", 0x20: "PREFIX"}
EXPORTS = ("pa_reshape_and_cache", "pa_paged_attention_workspace_size",
           "pa_paged_attention_partition_size",
           "pa_paged_attention_decode", "pa_copy_blocks", "pa_status_string",
           "pa_get_device_error", "pa_paged_attention_decode_static_workspace",
           "pa_paged_attention_decode_shared_prefix", "pa_swap_blocks",
           "pa_paged_attention_prefill")
PA_STATIC_WORKSPACE_BYTES = 16 * 1024 * 1024

_DTYPE = {torch.float16: PA_F16, torch.bfloat16: PA_BF16, torch.float32: PA_F32,
          torch.float8_e4m3fn: PA_FP8_E4M3}


class PaError(RuntimeError):
    """A libpa entry point returned a status other than PA_OK."""

    def __init__(self, fn: str, status: int):
        super().__init__(f"{fn} returned {STATUS.get(status, status)}")
        self.status = status


def library_path() -> str:
    return _LIB_PATH


def declare(lib: ctypes.CDLL) -> ctypes.CDLL:
    """Set the ctypes signatures of every entry point of a loaded libpa build."""
    P, I, L, F, S = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_float,
                     ctypes.c_size_t)
    lib.pa_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I, L, I, I, F, F, P]
    lib.pa_reshape_and_cache.restype = I
    lib.pa_paged_attention_workspace_size.argtypes = [I, I, I, I, I, I]
    lib.pa_paged_attention_workspace_size.restype = S
    lib.pa_paged_attention_partition_size.argtypes = [I, I, I, I, I]
    lib.pa_paged_attention_partition_size.restype = I
    lib.pa_paged_attention_decode.argtypes = [P, P, P, P, P, I, P, I, I, I, I, I, I, L, F,
                                              I, I, I, F, F, I, P, S, P]
    lib.pa_paged_attention_decode.restype = I
    lib.pa_paged_attention_decode_static_workspace.argtypes = [
        P, P, P, P, P, I, P, I, I, I, I, I, I, L, F, I, I, I, F, F, I, P]
    lib.pa_paged_attention_decode_static_workspace.restype = I
    lib.pa_paged_attention_decode_shared_prefix.argtypes = [
        P, P, P, P, P, I, P, I, I, P, P, I, I, I, I, I, I, L, F, I, I, I, F, F, P]
    lib.pa_paged_attention_decode_shared_prefix.restype = I
    lib.pa_copy_blocks.argtypes = [P, P, I, P, I, S, L, P]
    lib.pa_copy_blocks.restype = I
    lib.pa_paged_attention_prefill.argtypes = [P, P, P, P, P, I, P, P, I, I, I, I, I,
                                               I, I, L, F, I, I, I, P]
    lib.pa_paged_attention_prefill.restype = I
    lib.pa_swap_blocks.argtypes = [P, P, P, P, I, P, I, S, L, L, P]
    lib.pa_swap_blocks.restype = I
    lib.pa_status_string.argtypes = [I]
    lib.pa_status_string.restype = ctypes.c_char_p
    lib.pa_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_int), P]
    lib.pa_get_device_error.restype = I
    return lib


def library() -> ctypes.CDLL:
    """Load libpa.so (once); raise if it has not been built."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(_LIB_PATH):
                raise RuntimeError(
                    f"libpa.so not found at {_LIB_PATH}: build it with "
                    "`python -m paged_kv_cache_413_b200.build` (there is no fallback path)")
            _lib = declare(ctypes.CDLL(_LIB_PATH))
    return _lib


def _check(fn: str, status: int) -> None:
    if status != 0:
        raise PaError(fn, status)


def _stream(stream) -> int:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, torch.cuda.Stream):
        return stream.cuda_stream
    return int(stream)


class _Current:
    """No-op context: the call's device is already the current one."""

    def __enter__(self):
        return self

    def __exit__(self, *exc):
        return False


_CURRENT = _Current()


def _device_of(*tensors):
    """A context that makes current the device every CUDA tensor of a call lives on
    (so the library launches there, on that device's current stream); a no-op when
    it is current already.  Tensors on two different devices are rejected."""
    idx = None
    for t in tensors:
        if isinstance(t, torch.Tensor) and t.is_cuda:
            i = t.get_device()
            if idx is None:
                idx = i
            elif i != idx:
                raise ValueError("all CUDA tensors of a call must be on the same device")
    if idx is None:
        raise ValueError("the call has no CUDA tensor")
    return _CURRENT if idx == torch.cuda.current_device() else torch.cuda.device(idx)


def _dev(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr()


def _dt(t: torch.Tensor, name: str) -> int:
    if t.dtype not in _DTYPE:
        raise ValueError(f"{name}: unsupported dtype {t.dtype}")
    return _DTYPE[t.dtype]


def pa_reshape_and_cache(key: torch.Tensor, value: torch.Tensor, key_cache: torch.Tensor,
                         value_cache: torch.Tensor, slot_mapping: torch.Tensor, *,
                         k_scale: float = 1.0, v_scale: float = 1.0, stream=None) -> None:
    """key/value [T, H_kv, D]; caches [NB, H_kv, BS, D]; slot_mapping [T] int64."""
    if slot_mapping.dtype != torch.int64:
        raise ValueError("slot_mapping must be int64")
    nb, hkv, bs, d = key_cache.shape
    t = slot_mapping.shape[0]
    if key.shape != (t, hkv, d) or value.shape != key.shape or value_cache.shape != key_cache.shape:
        raise ValueError("shape mismatch between key/value and the caches")
    with _device_of(key, value, key_cache, value_cache, slot_mapping):
        _check("pa_reshape_and_cache", library().pa_reshape_and_cache(
            _dev(key, "key"), _dev(value, "value"), _dev(key_cache, "key_cache"),
            _dev(value_cache, "value_cache"), _dev(slot_mapping, "slot_mapping"), t, hkv, d, bs, nb,
            _dt(key, "key"), _dt(key_cache, "key_cache"), float(k_scale), float(v_scale),
            _stream(stream)))


def pa_paged_attention_workspace_size(num_seqs: int, num_heads: int, num_kv_heads: int,
                                      head_dim: int, max_seq_len: int,
                                      partition_size: int = 0) -> int:
    return int(library().pa_paged_attention_workspace_size(num_seqs, num_heads, num_kv_heads,
                                                            head_dim, max_seq_len,
                                                            partition_size))


def pa_paged_attention_partition_size(num_seqs: int, num_heads: int, num_kv_heads: int,
                                      max_seq_len: int, partition_size: int = 0) -> int:
    return int(library().pa_paged_attention_partition_size(num_seqs, num_heads, num_kv_heads,
                                                            max_seq_len, partition_size))


def pa_paged_attention_decode(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                              value_cache: torch.Tensor, block_tables: torch.Tensor,
                              seq_lens: torch.Tensor, *, max_seq_len: int, scale: float,
                              k_scale: float = 1.0, v_scale: float = 1.0,
                              partition_size: int = 0, workspace: torch.Tensor | None = None,
                              stream=None) -> None:
    """out/query [B, H, D]; caches [NB, H_kv, BS, D]; block_tables [B, W] int32; seq_lens [B] int32."""
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_tables and seq_lens must be int32")
    b, h, d = query.shape
    nb, hkv, bs, d2 = key_cache.shape
    if out.shape != query.shape or d2 != d or value_cache.shape != key_cache.shape or \
            block_tables.dim() != 2 or block_tables.shape[0] != b or seq_lens.shape != (b,):
        raise ValueError("shape mismatch")
    ws_ptr, ws_bytes = 0, 0
    if workspace is not None:
        ws_ptr, ws_bytes = _dev(workspace, "workspace"), workspace.numel() * workspace.element_size()
    with _device_of(out, query, key_cache, value_cache, block_tables, seq_lens, workspace):
        _check("pa_paged_attention_decode", library().pa_paged_attention_decode(
            _dev(out, "out"), _dev(query, "query"), _dev(key_cache, "key_cache"),
            _dev(value_cache, "value_cache"), _dev(block_tables, "block_tables"),
            block_tables.shape[1], _dev(seq_lens, "seq_lens"), b, int(max_seq_len), h, hkv, d, bs,
            nb, float(scale), _dt(query, "query"), _dt(key_cache, "key_cache"), _dt(out, "out"),
            float(k_scale), float(v_scale), int(partition_size), ws_ptr, ws_bytes, _stream(stream)))


def pa_paged_attention_decode_static_workspace(out: torch.Tensor, query: torch.Tensor,
                                               key_cache: torch.Tensor, value_cache: torch.Tensor,
                                               block_tables: torch.Tensor, seq_lens: torch.Tensor,
                                               *, max_seq_len: int, scale: float,
                                               k_scale: float = 1.0, v_scale: float = 1.0,
                                               partition_size: int = 0, stream=None) -> None:
    """Decode without a caller workspace, for callers that cannot allocate device memory
    (plugins whose host owns all allocations; engines that gave nearly all HBM to the KV
    pool).  The scratch is the library's fixed 16 MiB per-GPU array: sizes that need more
    raise PaError(PA_ERR_WORKSPACE); calls that overlap on the GPU race on it."""
    if block_tables.dtype != torch.int32 or seq_lens.dtype != torch.int32:
        raise ValueError("block_tables and seq_lens must be int32")
    b, h, d = query.shape
    nb, hkv, bs, d2 = key_cache.shape
    if out.shape != query.shape or d2 != d or value_cache.shape != key_cache.shape or \
            block_tables.dim() != 2 or block_tables.shape[0] != b or seq_lens.shape != (b,):
        raise ValueError("shape mismatch")
    with _device_of(out, query, key_cache, value_cache, block_tables, seq_lens):
        status = library().pa_paged_attention_decode_static_workspace(
        _dev(out, "out"), _dev(query, "query"), _dev(key_cache, "key_cache"),
        _dev(value_cache, "value_cache"), _dev(block_tables, "block_tables"),
        block_tables.shape[1], _dev(seq_lens, "seq_lens"), b, int(max_seq_len), h, hkv, d, bs,
        nb, float(scale), _dt(query, "query"), _dt(key_cache, "key_cache"), _dt(out, "out"),
        float(k_scale), float(v_scale), int(partition_size), _stream(stream))
    if status == -3:
        raise PaError("pa_paged_attention_decode_static_workspace (needs more than the "
                      f"{PA_STATIC_WORKSPACE_BYTES} bytes of static scratch)", status)
    _check("pa_paged_attention_decode_static_workspace", status)


def pa_paged_attention_decode_shared_prefix(out: torch.Tensor, query: torch.Tensor,
                                            key_cache: torch.Tensor, value_cache: torch.Tensor,
                                            block_tables: torch.Tensor, seq_lens: torch.Tensor,
                                            group_starts: torch.Tensor,
                                            prefix_lens: torch.Tensor, *, max_seq_len: int,
                                            max_group_size: int, scale: float,
                                            k_scale: float = 1.0, v_scale: float = 1.0,
                                            stream=None) -> None:
    """Decode for groups sharing the blocks of a prefix (beams, parallel samples).
    group_starts [G + 1] int32, prefix_lens [G] int32 (tokens, block multiples)."""
    for t, name in ((block_tables, "block_tables"), (seq_lens, "seq_lens"),
                    (group_starts, "group_starts"), (prefix_lens, "prefix_lens")):
        if t.dtype != torch.int32:
            raise ValueError(f"{name} must be int32")
    b, h, d = query.shape
    nb, hkv, bs, d2 = key_cache.shape
    ng = prefix_lens.shape[0]
    if out.shape != query.shape or d2 != d or value_cache.shape != key_cache.shape or \
            block_tables.dim() != 2 or block_tables.shape[0] != b or seq_lens.shape != (b,) or \
            group_starts.shape != (ng + 1,):
        raise ValueError("shape mismatch")
    with _device_of(out, query, key_cache, value_cache, block_tables, seq_lens,
                    group_starts, prefix_lens):
        _check("pa_paged_attention_decode_shared_prefix",
               library().pa_paged_attention_decode_shared_prefix(
                   _dev(out, "out"), _dev(query, "query"), _dev(key_cache, "key_cache"),
                   _dev(value_cache, "value_cache"), _dev(block_tables, "block_tables"),
                   block_tables.shape[1], _dev(seq_lens, "seq_lens"), b, int(max_seq_len),
                   _dev(group_starts, "group_starts"), _dev(prefix_lens, "prefix_lens"), ng,
                   int(max_group_size), h, hkv, d, bs, nb, float(scale), _dt(query, "query"),
                   _dt(key_cache, "key_cache"), _dt(out, "out"), float(k_scale), float(v_scale),
                   _stream(stream)))


def pa_paged_attention_prefill(out: torch.Tensor, query: torch.Tensor, key_cache: torch.Tensor,
                               value_cache: torch.Tensor, block_tables: torch.Tensor,
                               seq_lens: torch.Tensor, query_start: torch.Tensor, *,
                               max_query_len: int, max_seq_len: int, scale: float,
                               stream=None) -> None:
    """Causal multi-query attention (chunked prefill); query/out [total_q, H, D],
    query_start [B + 1] int32."""
    for t, name in ((block_tables, "block_tables"), (seq_lens, "seq_lens"),
                    (query_start, "query_start")):
        if t.dtype != torch.int32:
            raise ValueError(f"{name} must be int32")
    tq, h, d = query.shape
    nb, hkv, bs, d2 = key_cache.shape
    b = seq_lens.shape[0]
    if out.shape != query.shape or d2 != d or value_cache.shape != key_cache.shape or \
            block_tables.dim() != 2 or block_tables.shape[0] != b or \
            query_start.shape != (b + 1,):
        raise ValueError("shape mismatch")
    with _device_of(out, query, key_cache, value_cache, block_tables, seq_lens,
                    query_start):
        _check("pa_paged_attention_prefill", library().pa_paged_attention_prefill(
            _dev(out, "out"), _dev(query, "query"), _dev(key_cache, "key_cache"),
            _dev(value_cache, "value_cache"), _dev(block_tables, "block_tables"),
            block_tables.shape[1], _dev(seq_lens, "seq_lens"), _dev(query_start, "query_start"), b,
            int(max_query_len), int(max_seq_len), h, hkv, d, bs, nb, float(scale),
            _dt(query, "query"), _dt(key_cache, "key_cache"), _dt(out, "out"), _stream(stream)))


def pa_copy_blocks(key_caches: list, value_caches: list, block_mapping: torch.Tensor, *,
                   stream=None) -> None:
    """Per-layer caches (lists of [NB, ...] tensors); block_mapping [NP, 2] int64 (src, dst)."""
    if block_mapping.dtype != torch.int64:
        raise ValueError("block_mapping must be int64")
    n = len(key_caches)
    if n == 0 or block_mapping.numel() == 0:
        return
    if len(value_caches) != n:
        raise ValueError("key_caches and value_caches differ in length")
    nb = key_caches[0].shape[0]
    block_bytes = key_caches[0].numel() * key_caches[0].element_size() // nb
    for c in list(key_caches) + list(value_caches):
        if c.shape != key_caches[0].shape or c.dtype != key_caches[0].dtype:
            raise ValueError("all layers must share one shape and dtype")
    kp = (ctypes.c_void_p * n)(*[_dev(c, "key_caches[i]") for c in key_caches])
    vp = (ctypes.c_void_p * n)(*[_dev(c, "value_caches[i]") for c in value_caches])
    with _device_of(*key_caches, *value_caches, block_mapping):
        _check("pa_copy_blocks", library().pa_copy_blocks(
            ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p), n,
            _dev(block_mapping, "block_mapping"), block_mapping.shape[0], block_bytes, nb,
            _stream(stream)))


def _dev_or_pinned(t: torch.Tensor, name: str) -> int:
    if not isinstance(t, torch.Tensor) or not t.is_contiguous():
        raise ValueError(f"{name} must be a contiguous tensor")
    if t.device.type == "cuda" or (t.device.type == "cpu" and t.is_pinned()):
        return t.data_ptr()
    raise ValueError(f"{name} must be a CUDA tensor or pinned host memory")


def pa_swap_blocks(dst_key_caches: list, dst_value_caches: list, src_key_caches: list,
                   src_value_caches: list, block_mapping: torch.Tensor, *, stream=None) -> None:
    """Move blocks between pools (device <-> pinned host); block_mapping [NP, 2] int64."""
    if block_mapping.dtype != torch.int64:
        raise ValueError("block_mapping must be int64")
    n = len(dst_key_caches)
    if n == 0 or block_mapping.numel() == 0:
        return
    if not (len(dst_value_caches) == len(src_key_caches) == len(src_value_caches) == n):
        raise ValueError("all four pool lists need one entry per layer")
    d0, s0 = dst_key_caches[0], src_key_caches[0]
    block_bytes = d0.numel() * d0.element_size() // d0.shape[0]
    if s0.numel() * s0.element_size() // s0.shape[0] != block_bytes:
        raise ValueError("source and destination blocks differ in size")
    for c in list(dst_key_caches) + list(dst_value_caches):
        if c.shape != d0.shape or c.dtype != d0.dtype:
            raise ValueError("destination layers must share one shape and dtype")
    for c in list(src_key_caches) + list(src_value_caches):
        if c.shape != s0.shape or c.dtype != s0.dtype:
            raise ValueError("source layers must share one shape and dtype")
    arr = lambda xs, nm: ctypes.cast((ctypes.c_void_p * n)(*[_dev_or_pinned(c, nm) for c in xs]),
                                     ctypes.c_void_p)
    with _device_of(*dst_key_caches, *dst_value_caches, *src_key_caches,
                    *src_value_caches, block_mapping):
        _check("pa_swap_blocks", library().pa_swap_blocks(
            arr(dst_key_caches, "dst_key_caches[i]"), arr(dst_value_caches, "dst_value_caches[i]"),
            arr(src_key_caches, "src_key_caches[i]"), arr(src_value_caches, "src_value_caches[i]"),
            n, _dev_or_pinned(block_mapping, "block_mapping"), block_mapping.shape[0], block_bytes,
            s0.shape[0], d0.shape[0], _stream(stream)))


def pa_status_string(status: int) -> str:
    return library().pa_status_string(status).decode()


def pa_get_device_error(stream=None) -> int:
    """Synchronise the stream, return and clear the device error bits."""
    flag = ctypes.c_int(0)
    _check("pa_get_device_error", library().pa_get_device_error(ctypes.byref(flag),
                                                                _stream(stream)))
    return flag.value
