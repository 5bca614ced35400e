"""Seeded synthetic workloads for paged-KV decode.

This module builds inputs only.  It holds none of the attention arithmetic and
serves both the CUDA path (tests, ``bench.py``) and the CPU oracle's tests.

What it builds, per named configuration:

* per-sequence lengths, drawn in a fixed order from ``numpy.random.default_rng(seed)``;
* a shuffled physical block pool and per-sequence block tables, through
  :class:`BlockPool`, a host-side block manager fixture (allocation from a free
  list, reference counts, copy-on-write forks) in the manner the pages describe
  for the Block Manager ("vLLM推理引擎PagedAttention原理与性能优化实战" sec 2.2 and
  sec 3.2);
* the cache contents of every context position, the query of the new token and
  the new token's K/V with the slot it must be written to.  A sequence length
  counts the new token, so the new token's slot is the position ``L - 1``.

Every slot that no sequence owns, and the slot each new token will be written to,
is filled with NaN (0x7F for E4M3), so that any read of a slot outside a
sequence, or a missing cache write, poisons the attention output.

Draw order: sequence lengths, block permutation, Q, K pool, V pool, new-token K,
new-token V.  Value distributions: uniform in [-1, 1] (tiny case) or N(0, 1),
drawn in fp32 and rounded to the storage type.
"""

from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np
import torch

BLOCK_SIZE = 16

_TORCH = {"f16": torch.float16, "bf16": torch.bfloat16, "f32": torch.float32,
          "e4m3": torch.float8_e4m3fn}
ELT_BYTES = {"f16": 2, "bf16": 2, "f32": 4, "e4m3": 1}


@dataclass(frozen=True)
class DecodeConfig:
    """Shape and data recipe of one decode workload (one attention layer)."""

    name: str
    num_seqs: int
    num_heads: int
    num_kv_heads: int
    head_dim: int
    seq_lens: tuple | None = None            # fixed lengths, or None to draw
    seq_len_range: tuple | None = None       # inclusive (lo, hi) for uniform draws
    num_blocks: int | None = None            # fixed pool size, else pool_factor * needed
    pool_factor: float = 1.1
    dist: str = "normal"                     # "normal" or "uniform"
    q_dtype: str = "f16"
    cache_dtype: str = "f16"
    out_dtype: str = "f16"
    partition_size: int = 0                  # 0 = library's choice
    block_size: int = BLOCK_SIZE
    seed: int = 0
    # beam-search copy-on-write workloads
    beam_width: int = 1
    shared_len: int = 0                      # tokens shared by all beams of a prompt
    new_tokens_per_seq: int = 1

    def scaled(self, **kw) -> "DecodeConfig":
        d = dict(self.__dict__)
        d.update(kw)
        return DecodeConfig(**d)


CONFIGS: dict[str, DecodeConfig] = {
    # correctness case: MHA, head_dim 64, pool of 64 blocks
    "tiny": DecodeConfig("tiny", num_seqs=4, seq_lens=(1, 17, 33, 100), num_heads=4,
                         num_kv_heads=4, head_dim=64, num_blocks=64, dist="uniform",
                         q_dtype="f16", cache_dtype="f16", out_dtype="f16", seed=1),
    # Llama-2-7B-shaped layer: MHA 32 heads, lengths U[128, 2048], fp16
    "llama2_7b": DecodeConfig("llama2_7b", num_seqs=64, seq_len_range=(128, 2048), num_heads=32,
                              num_kv_heads=32, head_dim=128, q_dtype="f16", cache_dtype="f16",
                              out_dtype="f16", seed=2),
    # Llama-2-70B-shaped GQA layer: 64 query heads / 8 KV heads, 512-in + up to 256-out, bf16
    "llama2_70b_gqa": DecodeConfig("llama2_70b_gqa", num_seqs=256, seq_len_range=(512, 768),
                                   num_heads=64, num_kv_heads=8, head_dim=128, q_dtype="bf16",
                                   cache_dtype="bf16", out_dtype="bf16", seed=3),
    # long context: 8 x 32768 tokens, 512-token partitions merged by log-sum-exp
    "long_splitk": DecodeConfig("long_splitk", num_seqs=8, seq_lens=(32768,) * 8, num_heads=32,
                                num_kv_heads=8, head_dim=128, q_dtype="bf16", cache_dtype="bf16",
                                out_dtype="bf16", partition_size=512, seed=4),
    # beam search with a shared prefix and an FP8 E4M3 cache
    "beam_cow_fp8": DecodeConfig("beam_cow_fp8", num_seqs=64, beam_width=4, shared_len=1032,
                                 new_tokens_per_seq=4, num_heads=32, num_kv_heads=8,
                                 head_dim=128, q_dtype="bf16", cache_dtype="e4m3",
                                 out_dtype="bf16", seed=5),
}


class BlockPool:
    """Host-side block manager fixture: a shuffled free list with reference counts.

    ``allocate`` pops the next free physical block, ``fork`` shares a table's
    blocks with a new owner (reference count + 1), ``cow_last`` gives a table a
    private copy of its last block when that block is shared, returning the
    (src, dst) pair the device copy must perform.
    """

    def __init__(self, order: np.ndarray):
        self.free = [int(b) for b in order]
        self.free.reverse()
        self.refs: dict[int, int] = {}

    def allocate(self) -> int:
        if not self.free:
            raise RuntimeError("block pool exhausted")
        b = self.free.pop()
        self.refs[b] = 1
        return b

    def allocate_for(self, num_tokens: int, block_size: int) -> list[int]:
        return [self.allocate() for _ in range(-(-num_tokens // block_size))]

    def fork(self, table: list[int]) -> list[int]:
        for b in table:
            self.refs[b] += 1
        return list(table)

    def cow_last(self, table: list[int]) -> tuple[int, int] | None:
        last = table[-1]
        if self.refs[last] == 1:
            return None
        self.refs[last] -= 1
        new = self.allocate()
        table[-1] = new
        return last, new


@dataclass
class Workload:
    """All host (CPU) tensors of one decode step; see module docstring."""

    cfg: DecodeConfig
    query: torch.Tensor              # [B, H, D] q_dtype
    key_cache: torch.Tensor          # [NB, H_kv, BS, D] cache_dtype
    value_cache: torch.Tensor
    block_tables: torch.Tensor       # [B, max_blocks] int32, -1 past a sequence's blocks
    seq_lens: torch.Tensor           # [B] int32 (includes the new token)
    new_key: torch.Tensor            # [T, H_kv, D] src dtype
    new_value: torch.Tensor
    slot_mapping: torch.Tensor       # [T] int64
    scale: float
    k_scale: float = 1.0
    v_scale: float = 1.0
    src_dtype: str = "f16"
    # copy-on-write workloads: prefix fill and block copies done before the step
    prefix_key: torch.Tensor | None = None
    prefix_value: torch.Tensor | None = None
    prefix_slot_mapping: torch.Tensor | None = None
    block_mapping: torch.Tensor | None = None   # [NP, 2] int64 (src, dst)
    refs: dict = field(default_factory=dict)
    # sequences sharing the physical blocks of a prefix (copy-on-write groups)
    group_starts: torch.Tensor | None = None    # [num_groups + 1] int32
    prefix_lens: torch.Tensor | None = None     # [num_groups] int32, tokens
    # several query tokens per sequence (chunked prefill): query is then
    # [total_queries, H, D] and sequence i's rows are query_start[i] .. query_start[i+1]-1
    query_start: torch.Tensor | None = None     # [num_seqs + 1] int32

    @property
    def num_blocks(self) -> int:
        return self.key_cache.shape[0]

    @property
    def max_blocks_per_seq(self) -> int:
        return self.block_tables.shape[1]


def _draw(rng: np.random.Generator, shape, dist: str) -> np.ndarray:
    n = int(np.prod(shape))
    if dist == "uniform":
        a = rng.uniform(-1.0, 1.0, size=n).astype(np.float32)
    else:
        a = rng.standard_normal(size=n, dtype=np.float32)
    return a.reshape(shape)


def _to_storage(a: np.ndarray, dtype: str) -> torch.Tensor:
    return torch.from_numpy(a).to(_TORCH[dtype])


def _fill_nan(shape, dtype: str) -> torch.Tensor:
    if dtype == "e4m3":
        return torch.full(shape, 0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn)
    return torch.full(shape, float("nan"), dtype=_TORCH[dtype])


def _scale(head_dim: int) -> float:
    return float(np.float32(1.0) / np.sqrt(np.float32(head_dim)))


def _table_tensor(tables: list[list[int]], width: int) -> torch.Tensor:
    bt = np.full((len(tables), width), -1, dtype=np.int32)
    for i, t in enumerate(tables):
        bt[i, :len(t)] = t
    return torch.from_numpy(bt)


def _slot(table: list[int], pos: int, bs: int) -> int:
    return table[pos // bs] * bs + pos % bs


def make_workload(cfg: DecodeConfig | str, **overrides) -> Workload:
    """Build the seeded workload of a configuration (optionally scaled down)."""
    if isinstance(cfg, str):
        cfg = CONFIGS[cfg]
    if overrides:
        cfg = cfg.scaled(**overrides)
    if cfg.beam_width > 1:
        return _make_beam_workload(cfg)
    rng = np.random.default_rng(cfg.seed)
    B, H, Hkv, D, bs = cfg.num_seqs, cfg.num_heads, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    # 1. sequence lengths
    if cfg.seq_lens is not None:
        lens = np.asarray(cfg.seq_lens[:B], dtype=np.int64)
        if lens.shape[0] != B:
            lens = np.resize(lens, B)
        max_len = int(lens.max()) if B else 0
    else:
        lo, hi = cfg.seq_len_range
        lens = rng.integers(lo, hi + 1, size=B).astype(np.int64)
        max_len = hi
    need = int(sum(-(-int(L) // bs) for L in lens))
    nb = cfg.num_blocks if cfg.num_blocks is not None else max(1, math.ceil(cfg.pool_factor * need))
    # 2. block permutation -> tables
    pool = BlockPool(rng.permutation(nb))
    tables = [pool.allocate_for(int(L), bs) for L in lens]
    width = max(1, -(-max_len // bs))
    # 3. query, 4./5. pools, 6./7. new-token K and V
    src = cfg.cache_dtype if cfg.cache_dtype != "e4m3" else cfg.q_dtype
    q = _to_storage(_draw(rng, (B, H, D), cfg.dist), cfg.q_dtype)
    kpool = _draw(rng, (nb, Hkv, bs, D), cfg.dist)
    vpool = _draw(rng, (nb, Hkv, bs, D), cfg.dist)
    nk = _draw(rng, (B, Hkv, D), cfg.dist)
    nv = _draw(rng, (B, Hkv, D), cfg.dist)
    # poison every slot outside a sequence's context, and each new token's slot
    owned = np.zeros((nb, bs), dtype=bool)
    slots = np.empty(B, dtype=np.int64)
    for i, L in enumerate(lens):
        L = int(L)
        for j, b in enumerate(tables[i]):
            n_in = min(bs, L - j * bs)
            owned[b, :n_in] = True
        if L > 0:
            s = _slot(tables[i], L - 1, bs)
            slots[i] = s
            owned[s // bs, s % bs] = False
        else:
            slots[i] = -1
    for b in np.nonzero(~owned.all(axis=1))[0]:
        kpool[b][:, ~owned[b], :] = np.nan
        vpool[b][:, ~owned[b], :] = np.nan
    k_scale = v_scale = 1.0
    if cfg.cache_dtype == "e4m3":
        raise ValueError("E4M3 caches are built through the copy-on-write recipe")
    return Workload(cfg=cfg, query=q, key_cache=_to_storage(kpool, cfg.cache_dtype),
                    value_cache=_to_storage(vpool, cfg.cache_dtype),
                    block_tables=_table_tensor(tables, width),
                    seq_lens=torch.from_numpy(lens.astype(np.int32)),
                    new_key=_to_storage(nk, src), new_value=_to_storage(nv, src),
                    slot_mapping=torch.from_numpy(slots), scale=_scale(D), k_scale=k_scale,
                    v_scale=v_scale, src_dtype=src, refs=dict(pool.refs))


def _make_beam_workload(cfg: DecodeConfig) -> Workload:
    """Beam search over shared prompts with copy-on-write of the last shared block.

    Each of ``num_seqs`` prompts has ``shared_len`` tokens common to its
    ``beam_width`` beams; the beams' block tables point at the same physical
    blocks (reference count = beam width).  On divergence every beam but the
    first gets a private copy of the partially filled last shared block (one
    (src, dst) pair each); the first beam keeps the original.  Then each beam
    appends ``new_tokens_per_seq`` tokens into its own last block and decodes.
    """
    rng = np.random.default_rng(cfg.seed)
    P, W, S, T = cfg.num_seqs, cfg.beam_width, cfg.shared_len, cfg.new_tokens_per_seq
    H, Hkv, D, bs = cfg.num_heads, cfg.num_kv_heads, cfg.head_dim, cfg.block_size
    B = P * W
    L = S + T
    n_shared = -(-S // bs)
    if -(-L // bs) != n_shared:
        raise ValueError("the new tokens must fit in the last shared block")
    need = P * (n_shared + (W - 1 if S % bs else 0))
    nb = cfg.num_blocks if cfg.num_blocks is not None else max(1, math.ceil(cfg.pool_factor * need))
    pool = BlockPool(rng.permutation(nb))
    shared = [pool.allocate_for(S, bs) for _ in range(P)]
    tables, pairs = [], []
    for p in range(P):
        beams = [pool.fork(shared[p]) for _ in range(W)]
        for b in shared[p]:          # the prompt's own handle is released after forking
            pool.refs[b] -= 1
        for w in range(1, W):        # beam 0 keeps the original last block
            pair = pool.cow_last(beams[w]) if S % bs else None
            if pair is not None:
                pairs.append(pair)
        tables.extend(beams)
    src = cfg.q_dtype
    q = _to_storage(_draw(rng, (B, H, D), cfg.dist), cfg.q_dtype)
    pk = _draw(rng, (P, S, Hkv, D), cfg.dist)
    pv = _draw(rng, (P, S, Hkv, D), cfg.dist)
    nk = _draw(rng, (B, T, Hkv, D), cfg.dist)
    nv = _draw(rng, (B, T, Hkv, D), cfg.dist)
    prefix_slots = np.array([_slot(shared[p], pos, bs) for p in range(P) for pos in range(S)],
                            dtype=np.int64)
    new_slots = np.array([_slot(tables[i], S + t, bs) for i in range(B) for t in range(T)],
                         dtype=np.int64)
    if cfg.cache_dtype == "e4m3":
        k_scale = float(np.float32(max(np.abs(pk).max(), np.abs(nk).max()) / np.float32(448.0)))
        v_scale = float(np.float32(max(np.abs(pv).max(), np.abs(nv).max()) / np.float32(448.0)))
    else:
        k_scale = v_scale = 1.0
    kc = _fill_nan((nb, Hkv, bs, D), cfg.cache_dtype)
    vc = _fill_nan((nb, Hkv, bs, D), cfg.cache_dtype)
    starts, prefixes = _shared_prefixes(tables, [W] * P, [L] * B, bs)
    return Workload(cfg=cfg, query=q, key_cache=kc, value_cache=vc,
                    block_tables=_table_tensor(tables, -(-L // bs)),
                    seq_lens=torch.full((B,), L, dtype=torch.int32),
                    new_key=_to_storage(nk.reshape(B * T, Hkv, D), src),
                    new_value=_to_storage(nv.reshape(B * T, Hkv, D), src),
                    slot_mapping=torch.from_numpy(new_slots), scale=_scale(D), k_scale=k_scale,
                    v_scale=v_scale, src_dtype=src,
                    prefix_key=_to_storage(pk.reshape(P * S, Hkv, D), src),
                    prefix_value=_to_storage(pv.reshape(P * S, Hkv, D), src),
                    prefix_slot_mapping=torch.from_numpy(prefix_slots),
                    block_mapping=torch.tensor(pairs, dtype=torch.int64).reshape(-1, 2),
                    refs=dict(pool.refs), group_starts=starts, prefix_lens=prefixes)


def _shared_prefixes(tables, group_sizes, lens, bs):
    """group_starts and, per group, the tokens of the leading full blocks whose
    block-table entries every member shares (what the block manager knows from
    its forks)."""
    starts, prefixes, s = [0], [], 0
    for n in group_sizes:
        members = tables[s:s + n]
        full = min(int(L) for L in lens[s:s + n]) // bs
        k = 0
        while k < full and len({t[k] for t in members}) == 1:
            k += 1
        prefixes.append(k * bs)
        s += n
        starts.append(s)
    return (torch.tensor(starts, dtype=torch.int32), torch.tensor(prefixes, dtype=torch.int32))


def make_group_workload(num_groups: int, group_size: tuple, prefix_blocks: tuple,
                        own_len: tuple, *, num_heads: int, num_kv_heads: int,
                        head_dim: int = 128, dtype: str = "bf16", seed: int = 0,
                        pool_factor: float = 1.3, block_size: int = BLOCK_SIZE,
                        cache_dtype: str | None = None) -> Workload:
    """Groups of sequences forked from a shared prompt prefix.

    Each group draws a size in ``group_size`` and a number of shared full blocks
    in ``prefix_blocks`` (inclusive ranges); every member then owns
    ``own_len`` tokens (at least 1: its last token is the new one) in blocks of
    its own.  Draw order: group sizes, prefix blocks, own lengths, block
    permutation, Q, K pool, V pool, new-token K, new-token V.

    The cache is ``dtype`` (16-bit, a bit copy of the draws rounded to it) unless
    ``cache_dtype`` is "e4m3": the pool then holds the draws divided by one fp32
    scale per pool (amax / 448 over the pool's and the new tokens' draws) and
    rounded to E4M3, and the new tokens (``dtype``) are quantised by the step's
    cache write with the same scales.
    """
    bs = block_size
    rng = np.random.default_rng(seed)
    sizes = rng.integers(group_size[0], group_size[1] + 1, size=num_groups)
    pblks = rng.integers(prefix_blocks[0], prefix_blocks[1] + 1, size=num_groups)
    B = int(sizes.sum())
    own = rng.integers(max(1, own_len[0]), own_len[1] + 1, size=B)
    lens = np.concatenate([[pblks[g] * bs] * sizes[g] for g in range(num_groups)]).astype(np.int64) + own
    need = int(pblks.sum()) + int(sum(-(-int(o) // bs) for o in own))
    nb = max(1, math.ceil(pool_factor * need))
    pool = BlockPool(rng.permutation(nb))
    tables, i = [], 0
    for g in range(num_groups):
        shared = [pool.allocate() for _ in range(int(pblks[g]))]
        for _ in range(int(sizes[g])):
            tables.append(pool.fork(shared) + pool.allocate_for(int(own[i]), bs))
            i += 1
        for b in shared:
            pool.refs[b] -= 1
    Hkv, D = num_kv_heads, head_dim
    q = _to_storage(_draw(rng, (B, num_heads, D), "normal"), dtype)
    kpool = _draw(rng, (nb, Hkv, bs, D), "normal")
    vpool = _draw(rng, (nb, Hkv, bs, D), "normal")
    nk = _draw(rng, (B, Hkv, D), "normal")
    nv = _draw(rng, (B, Hkv, D), "normal")
    owned = np.zeros((nb, bs), dtype=bool)
    slots = np.empty(B, dtype=np.int64)
    for i, L in enumerate(lens):
        L = int(L)
        for j, b in enumerate(tables[i]):
            owned[b, :min(bs, L - j * bs)] = True
        s = _slot(tables[i], L - 1, bs)
        slots[i] = s
    for i, L in enumerate(lens):  # the new tokens' slots stay poisoned until written
        s = int(slots[i])
        owned[s // bs, s % bs] = False
    cdt = cache_dtype or dtype
    k_scale = v_scale = 1.0
    if cdt == "e4m3":
        amax = lambda a, b: np.float32(max(np.nanmax(np.abs(a)), np.abs(b).max()))
        k_scale = float(amax(kpool, nk) / np.float32(448.0))
        v_scale = float(amax(vpool, nv) / np.float32(448.0))
        kpool = kpool / np.float32(k_scale)
        vpool = vpool / np.float32(v_scale)
    for b in np.nonzero(~owned.all(axis=1))[0]:
        kpool[b][:, ~owned[b], :] = np.nan
        vpool[b][:, ~owned[b], :] = np.nan
    cfg = DecodeConfig("groups", num_seqs=B, num_heads=num_heads, num_kv_heads=Hkv, head_dim=D,
                       seq_lens=tuple(int(x) for x in lens), num_blocks=nb, q_dtype=dtype,
                       cache_dtype=cdt, out_dtype=dtype, seed=seed, block_size=bs)
    starts, prefixes = _shared_prefixes(tables, [int(x) for x in sizes], lens, bs)
    width = max(len(t) for t in tables)
    return Workload(cfg=cfg, query=q, key_cache=_to_storage(kpool, cdt),
                    value_cache=_to_storage(vpool, cdt), block_tables=_table_tensor(tables, width),
                    seq_lens=torch.from_numpy(lens.astype(np.int32)),
                    new_key=_to_storage(nk, dtype), new_value=_to_storage(nv, dtype),
                    slot_mapping=torch.from_numpy(slots), scale=_scale(D), k_scale=k_scale,
                    v_scale=v_scale, src_dtype=dtype, refs=dict(pool.refs), group_starts=starts,
                    prefix_lens=prefixes)


def make_prefill_workload(num_seqs: int, context: tuple, chunk: tuple, *, num_heads: int,
                          num_kv_heads: int, head_dim: int = 128, dtype: str = "bf16",
                          seed: int = 0, block_size: int = BLOCK_SIZE,
                          pool_factor: float = 1.1) -> Workload:
    """Chunked prefill: sequence i has L_i tokens (``context`` range, inclusive),
    the last q_i of which (``chunk`` range, q_i <= L_i) are the chunk being
    processed: their K/V are written by the step's cache write and their queries
    attend causally.  Draw order: lengths, chunk sizes, block permutation, Q,
    K pool, V pool, chunk K, chunk V.
    """
    bs = block_size
    rng = np.random.default_rng(seed)
    lens = rng.integers(context[0], context[1] + 1, size=num_seqs).astype(np.int64)
    nq = np.minimum(rng.integers(chunk[0], chunk[1] + 1, size=num_seqs), lens).astype(np.int64)
    need = int(sum(-(-int(L) // bs) for L in lens))
    nb = max(1, math.ceil(pool_factor * need))
    pool = BlockPool(rng.permutation(nb))
    tables = [pool.allocate_for(int(L), bs) for L in lens]
    Hkv, D = num_kv_heads, head_dim
    qs = np.concatenate([[0], np.cumsum(nq)]).astype(np.int32)
    T = int(qs[-1])
    q = _to_storage(_draw(rng, (T, num_heads, D), "normal"), dtype)
    kpool = _draw(rng, (nb, Hkv, bs, D), "normal")
    vpool = _draw(rng, (nb, Hkv, bs, D), "normal")
    nk = _draw(rng, (T, Hkv, D), "normal")
    nv = _draw(rng, (T, Hkv, D), "normal")
    owned = np.zeros((nb, bs), dtype=bool)
    slots = np.empty(T, dtype=np.int64)
    for i, L in enumerate(lens):
        L = int(L)
        for j, b in enumerate(tables[i]):
            owned[b, :min(bs, L - j * bs)] = True
        for t in range(int(nq[i])):
            slots[qs[i] + t] = _slot(tables[i], L - int(nq[i]) + t, bs)
    for sl in slots:  # the chunk's slots stay poisoned until the cache write
        owned[int(sl) // bs, int(sl) % bs] = False
    for b in np.nonzero(~owned.all(axis=1))[0]:
        kpool[b][:, ~owned[b], :] = np.nan
        vpool[b][:, ~owned[b], :] = np.nan
    cfg = DecodeConfig("prefill", num_seqs=num_seqs, num_heads=num_heads, num_kv_heads=Hkv,
                       head_dim=D, seq_lens=tuple(int(x) for x in lens), num_blocks=nb,
                       q_dtype=dtype, cache_dtype=dtype, out_dtype=dtype, seed=seed,
                       block_size=bs, new_tokens_per_seq=0)
    width = max(1, max(len(t) for t in tables))
    return Workload(cfg=cfg, query=q, key_cache=_to_storage(kpool, dtype),
                    value_cache=_to_storage(vpool, dtype), block_tables=_table_tensor(tables, width),
                    seq_lens=torch.from_numpy(lens.astype(np.int32)),
                    new_key=_to_storage(nk, dtype), new_value=_to_storage(nv, dtype),
                    slot_mapping=torch.from_numpy(slots), scale=_scale(D), src_dtype=dtype,
                    refs=dict(pool.refs), query_start=torch.from_numpy(qs))
