"""One decode step of a workload, on the GPU through the C ABI and on the CPU oracle.

A step is: (copy-on-write workloads only, once before the step) fill the shared
prefix with reshape_and_cache and copy the diverging beams' last blocks with
copy_blocks; then reshape_and_cache of the new tokens; then decode.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np
import torch

import oracle
import paged_kv_cache_413_b200 as pa
from paged_kv_cache_413_b200 import workloads as W

TOL = {"f16": 8e-3, "bf16": 8e-3, "f32": 1e-3}
TORCH_DT = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32}


@dataclass
class Dev:
    query: torch.Tensor
    key_cache: torch.Tensor
    value_cache: torch.Tensor
    block_tables: torch.Tensor
    seq_lens: torch.Tensor
    new_key: torch.Tensor
    new_value: torch.Tensor
    slot_mapping: torch.Tensor
    prefix_key: torch.Tensor | None = None
    prefix_value: torch.Tensor | None = None
    prefix_slot_mapping: torch.Tensor | None = None
    block_mapping: torch.Tensor | None = None


def to_device(wl: W.Workload, dev: str = "cuda") -> Dev:
    f = lambda t: None if t is None else t.to(dev)
    return Dev(f(wl.query), f(wl.key_cache), f(wl.value_cache), f(wl.block_tables),
               f(wl.seq_lens), f(wl.new_key), f(wl.new_value), f(wl.slot_mapping),
               f(wl.prefix_key), f(wl.prefix_value), f(wl.prefix_slot_mapping),
               f(wl.block_mapping))


def max_seq_len(wl: W.Workload) -> int:
    return int(wl.seq_lens.max()) if wl.seq_lens.numel() else 0


def gpu_prepare(wl: W.Workload, d: Dev) -> None:
    """Copy-on-write workloads: fill the shared prefix, then copy diverging blocks."""
    if d.prefix_key is not None:
        pa.pa_reshape_and_cache(d.prefix_key, d.prefix_value, d.key_cache, d.value_cache,
                                d.prefix_slot_mapping, k_scale=wl.k_scale, v_scale=wl.v_scale)
    if d.block_mapping is not None and d.block_mapping.numel():
        pa.pa_copy_blocks([d.key_cache], [d.value_cache], d.block_mapping)


def workspace_for(wl: W.Workload, partition_size: int, dev: str = "cuda"):
    n = pa.pa_paged_attention_workspace_size(wl.cfg.num_seqs * max(1, wl.cfg.beam_width),
                                             wl.cfg.num_heads, wl.cfg.num_kv_heads,
                                             wl.cfg.head_dim, max_seq_len(wl), partition_size)
    return torch.empty(n, dtype=torch.uint8, device=dev) if n else None


def gpu_step(wl: W.Workload, d: Dev, out_dtype: str, partition_size: int = 0,
             workspace=None) -> torch.Tensor:
    pa.pa_reshape_and_cache(d.new_key, d.new_value, d.key_cache, d.value_cache, d.slot_mapping,
                            k_scale=wl.k_scale, v_scale=wl.v_scale)
    out = torch.empty(d.query.shape, dtype=TORCH_DT[out_dtype], device=d.query.device)
    if workspace is None:
        workspace = workspace_for(wl, partition_size, str(d.query.device))
    pa.pa_paged_attention_decode(out, d.query, d.key_cache, d.value_cache, d.block_tables,
                                 d.seq_lens, max_seq_len=max_seq_len(wl), scale=wl.scale,
                                 k_scale=wl.k_scale, v_scale=wl.v_scale,
                                 partition_size=partition_size, workspace=workspace)
    return out


def oracle_caches(wl: W.Workload, prompts=None):
    """The caches after the whole step's writes, computed by the oracle.

    prompts: for copy-on-write workloads, restrict the prefix fill, the copies and
    the new tokens to these prompts (a sample of a full-size workload).
    """
    cd, sd = wl.cfg.cache_dtype, wl.src_dtype
    kc, vc = wl.key_cache, wl.value_cache
    slots = wl.slot_mapping.numpy()
    nk, nv = wl.new_key, wl.new_value
    if wl.prefix_key is not None:
        pk, pv, ps = wl.prefix_key, wl.prefix_value, wl.prefix_slot_mapping.numpy()
        bm = wl.block_mapping.numpy()
        if prompts is not None:
            S, Wd, T = wl.cfg.shared_len, wl.cfg.beam_width, wl.cfg.new_tokens_per_seq
            tok = np.concatenate([np.arange(p * S, (p + 1) * S) for p in prompts])
            pk, pv, ps = pk[tok], pv[tok], ps[tok]
            bm = np.concatenate([bm[p * (Wd - 1):(p + 1) * (Wd - 1)] for p in prompts])
            seqs = [p * Wd + w for p in prompts for w in range(Wd)]
            new = np.concatenate([np.arange(s * T, (s + 1) * T) for s in seqs])
            nk, nv, slots = nk[new], nv[new], slots[new]
        kc, vc = oracle.reshape_and_cache(pk, pv, kc, vc, ps, src_dtype=sd, cache_dtype=cd,
                                          k_scale=wl.k_scale, v_scale=wl.v_scale)
        (kc,), (vc,) = oracle.copy_blocks([kc], [vc], bm, dtype=cd)
    kc, vc = oracle.reshape_and_cache(nk, nv, kc, vc, slots, src_dtype=sd, cache_dtype=cd,
                                      k_scale=wl.k_scale, v_scale=wl.v_scale)
    return kc, vc


def oracle_decode(wl: W.Workload, kc, vc, seqs=None) -> np.ndarray:
    """fp64 outputs of the sequences `seqs` (all when None)."""
    q, bt, sl = wl.query, wl.block_tables.numpy(), wl.seq_lens.numpy()
    if seqs is not None:
        idx = torch.as_tensor(np.asarray(seqs, dtype=np.int64))
        q, bt, sl = q[idx], bt[np.asarray(seqs)], sl[np.asarray(seqs)]
    return oracle.paged_attention_decode(q, kc, vc, bt, sl, scale=wl.scale,
                                         q_dtype=wl.cfg.q_dtype, cache_dtype=wl.cfg.cache_dtype,
                                         k_scale=wl.k_scale, v_scale=wl.v_scale)


def storage_bytes(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    return t.view(torch.uint8).numpy() if t.dtype != torch.uint8 else t.numpy()


def max_abs_err(gpu_out: torch.Tensor, ref: np.ndarray) -> float:
    g = gpu_out.detach().cpu().double().numpy()
    assert np.isfinite(g).all(), "non-finite output"
    return float(np.abs(g - ref).max()) if ref.size else 0.0
