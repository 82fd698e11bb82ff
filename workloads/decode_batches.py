"""Seeded synthetic decode batches for paged decode attention.

Each batch is the state of one decode step of a paged KV cache, as the pages on
PagedAttention describe it ("vLLM Fundamentals: Paged Attention and Batching",
sections "Paged Attention" and "Just a python process"; "Deep Dive into vLLM",
section 2.1): one preallocated pool of fixed-size physical blocks, laid out
[num_blocks][block_size][num_kv_heads][head_dim] in bf16, and a per-sequence
block table that maps logical block b of a sequence to a physical block.

Recipe (the same for every consumer: oracle tests, CUDA tests, benchmark):

1. ``rng = numpy.random.default_rng(seed)``; context lengths are drawn first
   (integer uniform, both ends inclusive), then the pool permutation
   ``rng.permutation(num_blocks)``.  Physical blocks are handed out in
   permutation order, sequence after sequence, each sequence taking
   ceil(L / block_size) blocks.  Unused table entries hold -1.
2. Values come from a ``torch.Generator`` seeded with ``seed`` on the device the
   batch is built on, in this order: q, K pool, V pool, new k, new v.  All are
   N(0, 1) in fp32, rounded to bf16 (round to nearest even).
3. The step appends one token per sequence at logical position L - 1
   (``slot_mapping``); attention then runs over all L tokens, that one
   included.  Before the append, the slot at L - 1, every slot past L - 1 in a
   sequence's last block and every unused block hold NaN when ``poison`` is on,
   so that a stray read or a missed append shows up as NaN.

FP8 cache (``kv_dtype="fp8"``): the pools hold e4m3 codes drawn directly,
not quantized from anything -- sign uniform, exponent field uniform in
[4, 11], mantissa field uniform in [0, 7] (values 2^-3 .. 30 in magnitude) --
and one fp32 scale per kv head for K, 2^-4 (1 + h / Hkv), and for V,
2^-4 (1 + h / (2 Hkv)). The step's new k / v stay bf16 (the append quantizes
them). Poisoned slots hold the NaN code 0x7f.

This module holds no attention arithmetic and no quantization.
"""
from __future__ import annotations

import dataclasses
import math
from typing import Callable, Dict, List, Optional, Sequence

import numpy as np
import torch

BF16_NAN_BITS = 0x7FC0

_CHUNK = 1 << 26  # values generated per randn call when building large pools


@dataclasses.dataclass(frozen=True)
class Config:
    """One synthetic decode workload (head geometry, block size, length mix)."""

    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    scale: float
    lengths: Callable[[np.random.Generator], np.ndarray]
    max_context: int               # engine's maximum context: sets max_blocks_per_seq
    pool: str = "factor"           # "factor" | "fixed" | "shared_prefix"
    pool_factor: float = 1.0
    pool_blocks: int = 0           # for pool == "fixed"
    prefix_tokens: int = 0         # for pool == "shared_prefix"
    description: str = ""


def _fixed(values: List[int]) -> Callable[[np.random.Generator], np.ndarray]:
    return lambda rng: np.asarray(values, dtype=np.int64)


def _uniform(n: int, lo: int, hi: int) -> Callable[[np.random.Generator], np.ndarray]:
    return lambda rng: rng.integers(lo, hi + 1, size=n, dtype=np.int64)


def _prefix_plus_suffix(n: int, prefix: int, lo: int, hi: int):
    return lambda rng: prefix + rng.integers(lo, hi + 1, size=n, dtype=np.int64)


def _skewed(rng: np.random.Generator) -> np.ndarray:
    long = [65536, 32768, 16384, 8192, 8192, 4096, 4096, 4096]
    short = rng.integers(16, 256 + 1, size=120, dtype=np.int64)
    return np.concatenate([np.asarray(long, dtype=np.int64), short])


CONFIGS: Dict[str, Config] = {
    c.name: c
    for c in [
        Config(
            "tiny", 0, 4, 2, 1, 64, 16, 1.0 / 8.0, _fixed([1, 7, 16, 33]), 33,
            pool="fixed", pool_blocks=16,
            description="4 seqs, lens {1,7,16,33}, 2 q / 1 kv head, D64, bs16, 16-block pool",
        ),
        Config(
            "opt125m", 1, 32, 12, 12, 64, 16, 1.0 / math.sqrt(64), _uniform(32, 1, 2048), 2048,
            pool_factor=1.25,
            description="OPT-125m heads: 32 seqs, 12/12 heads, D64, bs16, lens U[1,2048], pool 1.25x",
        ),
        Config(
            "llama3_8b", 2, 256, 32, 8, 128, 16, 1.0 / math.sqrt(128), _uniform(256, 128, 4096), 4096,
            pool_factor=1.2,
            description="Llama-3-8B GQA heads: 256 seqs, 32/8 heads, D128, bs16, lens U[128,4096], pool 1.2x",
        ),
        Config(
            "qwen25_7b_prefix", 3, 64, 28, 4, 128, 16, 1.0 / math.sqrt(128),
            _prefix_plus_suffix(64, 1024, 1, 512), 1024 + 512,
            pool="shared_prefix", prefix_tokens=1024,
            description="Qwen2.5-7B heads: 64 seqs, 28/4 heads, D128, bs16, shared 1024-token "
                        "prefix (64 blocks) + private suffix U[1,512]",
        ),
        Config(
            "skewed_long", 4, 128, 32, 8, 128, 32, 1.0 / math.sqrt(128), _skewed, 65536,
            pool_factor=1.0,
            description="Llama-3-8B GQA heads, bs32: 8 long seqs 64K..4K + 120 seqs U[16,256]",
        ),
    ]
}
CONFIG_ORDER = ["tiny", "opt125m", "llama3_8b", "qwen25_7b_prefix", "skewed_long"]

# An extra bench workload (not one of the five parity configs above): a long
# shared prompt whose K/V does not fit in L2, the case prefix groups are for.
CONFIGS["shared_long_prefix"] = Config(
    "shared_long_prefix", 5, 32, 32, 8, 128, 16, 1.0 / math.sqrt(128),
    _prefix_plus_suffix(32, 32768, 1, 512), 32768 + 512,
    pool="shared_prefix", prefix_tokens=32768,
    description="Llama-3-8B GQA heads: 32 seqs sharing a 32768-token prompt (2048 blocks, 134 MB of K/V) "
                "+ private suffix U[1,512], D128, bs16",
)


@dataclasses.dataclass
class DecodeBatch:
    """Inputs of one decode step (pre-append pool state plus the step's tokens)."""

    name: str
    seed: int
    num_seqs: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    scale: float
    max_blocks_per_seq: int
    num_blocks: int
    context_lens: torch.Tensor      # int32 [S] (host)
    block_tables: torch.Tensor      # int32 [S][MB] (host), -1 padded
    slot_mapping: torch.Tensor      # int64 [S] (host), -1 = no append
    q: torch.Tensor                 # bf16 [S][Hq][D]
    k_cache: torch.Tensor           # bf16 [NB][bs][Hkv][D]
    v_cache: torch.Tensor           # bf16 [NB][bs][Hkv][D]
    k_new: torch.Tensor             # bf16 [S][Hkv][D]
    v_new: torch.Tensor             # bf16 [S][Hkv][D]
    kv_dtype: str = "bf16"          # "bf16", or "fp8": pools of e4m3 codes (uint8) with per-head scales
    k_scale: Optional[torch.Tensor] = None   # fp32 [Hkv] (fp8 only)
    v_scale: Optional[torch.Tensor] = None

    @property
    def device(self) -> torch.device:
        return self.q.device

    def clone(self) -> "DecodeBatch":
        return dataclasses.replace(
            self,
            **{f.name: getattr(self, f.name).clone()
               for f in dataclasses.fields(self)
               if isinstance(getattr(self, f.name), torch.Tensor)},
        )

    def to(self, device) -> "DecodeBatch":
        """Value tensors moved to ``device``; the index tensors follow them."""
        return dataclasses.replace(
            self,
            **{f.name: getattr(self, f.name).to(device)
               for f in dataclasses.fields(self)
               if isinstance(getattr(self, f.name), torch.Tensor)},
        )


def _randn_bf16(shape, gen: torch.Generator, device) -> torch.Tensor:
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.bfloat16, device=device)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        out[lo:hi] = torch.randn(hi - lo, generator=gen, device=device, dtype=torch.float32).to(torch.bfloat16)
    return out.view(*shape)


def _random_e4m3(shape, gen: torch.Generator, device) -> torch.Tensor:
    """e4m3 codes drawn field by field (see the module docstring)."""
    n = int(np.prod(shape))
    out = torch.empty(n, dtype=torch.uint8, device=device)
    for lo in range(0, n, _CHUNK):
        hi = min(n, lo + _CHUNK)
        sign = torch.randint(0, 2, (hi - lo,), generator=gen, device=device, dtype=torch.int32)
        expo = torch.randint(4, 12, (hi - lo,), generator=gen, device=device, dtype=torch.int32)
        mant = torch.randint(0, 8, (hi - lo,), generator=gen, device=device, dtype=torch.int32)
        out[lo:hi] = (sign * 128 + expo * 8 + mant).to(torch.uint8)
    return out.view(*shape)


E4M3_NAN_CODE = 0x7F


def fp8_scales(num_kv_heads: int):
    """The recipe's per-head scales (fp32 [Hkv]) for K and V."""
    h = torch.arange(num_kv_heads, dtype=torch.float64)
    k = (2.0 ** -4) * (1 + h / num_kv_heads)
    v = (2.0 ** -4) * (1 + h / (2 * num_kv_heads))
    return k.to(torch.float32), v.to(torch.float32)


def _assign_tables(cfg: Config, lens: np.ndarray, rng: np.random.Generator):
    bs = cfg.block_size
    nblk = (lens + bs - 1) // bs
    mb = (cfg.max_context + bs - 1) // bs
    if cfg.pool == "shared_prefix":
        pre = cfg.prefix_tokens // bs
        assert cfg.prefix_tokens % bs == 0
        private = nblk - pre
        num_blocks = int(pre + private.sum())
    else:
        needed = int(nblk.sum())
        if cfg.pool == "fixed":
            num_blocks = cfg.pool_blocks
        else:
            num_blocks = int(math.ceil(cfg.pool_factor * needed))
        assert num_blocks >= needed
    perm = rng.permutation(num_blocks).astype(np.int64)
    tables = np.full((len(lens), mb), -1, dtype=np.int32)
    cursor = 0
    if cfg.pool == "shared_prefix":
        shared = perm[:pre]
        cursor = pre
        for s in range(len(lens)):
            tables[s, :pre] = shared
            k = int(private[s])
            tables[s, pre:pre + k] = perm[cursor:cursor + k]
            cursor += k
    else:
        for s in range(len(lens)):
            k = int(nblk[s])
            tables[s, :k] = perm[cursor:cursor + k]
            cursor += k
    return tables, num_blocks, mb


def _slot_mapping(tables: np.ndarray, lens: np.ndarray, bs: int) -> np.ndarray:
    """Physical slot of logical position L-1 of each sequence (-1 when L == 0)."""
    slots = np.full(len(lens), -1, dtype=np.int64)
    for s, L in enumerate(lens):
        if L > 0:
            pos = int(L) - 1
            slots[s] = int(tables[s, pos // bs]) * bs + pos % bs
    return slots


def _valid_slot_mask(tables: np.ndarray, present: np.ndarray, bs: int, num_blocks: int) -> np.ndarray:
    """True for pool slots that hold a token before the step (positions < present[s])."""
    mask = np.zeros(num_blocks * bs, dtype=bool)
    for s, n in enumerate(present):
        n_before = max(int(n), 0)
        for b in range((n_before + bs - 1) // bs):
            p = int(tables[s, b])
            k = min(bs, n_before - b * bs)
            mask[p * bs:p * bs + k] = True
    return mask


def _poison(cache: torch.Tensor, mask: np.ndarray) -> None:
    nb, bs, hkv, d = cache.shape
    bad = torch.from_numpy(~mask).to(cache.device)
    if cache.dtype == torch.uint8:
        cache.view(nb * bs, hkv * d)[bad] = E4M3_NAN_CODE
        return
    flat = cache.view(nb * bs, hkv * d).view(torch.int16)
    flat[bad] = np.int16(BF16_NAN_BITS)


def _build(cfg: Config, lens: np.ndarray, rng: np.random.Generator, seed: int, device,
           poison: bool, with_append: bool, kv_dtype: str = "bf16") -> DecodeBatch:
    assert kv_dtype in ("bf16", "fp8")
    tables, num_blocks, mb = _assign_tables(cfg, lens, rng)
    bs = cfg.block_size
    if with_append:
        slots = _slot_mapping(tables, lens, bs)
    else:
        slots = np.full(len(lens), -1, dtype=np.int64)

    gen = torch.Generator(device=device)
    gen.manual_seed(seed)
    Hq, Hkv, D = cfg.num_q_heads, cfg.num_kv_heads, cfg.head_dim
    S = len(lens)
    q = _randn_bf16((S, Hq, D), gen, device)
    if kv_dtype == "fp8":
        k_cache = _random_e4m3((num_blocks, bs, Hkv, D), gen, device)
        v_cache = _random_e4m3((num_blocks, bs, Hkv, D), gen, device)
        k_scale, v_scale = fp8_scales(Hkv)
        k_scale, v_scale = k_scale.to(device), v_scale.to(device)
    else:
        k_cache = _randn_bf16((num_blocks, bs, Hkv, D), gen, device)
        v_cache = _randn_bf16((num_blocks, bs, Hkv, D), gen, device)
        k_scale = v_scale = None
    k_new = _randn_bf16((S, Hkv, D), gen, device)
    v_new = _randn_bf16((S, Hkv, D), gen, device)
    if poison:
        # tokens present before the step: positions < L-1 (with an append) or < L
        present = lens - 1 if with_append else lens
        mask = _valid_slot_mask(tables, np.maximum(present, 0), bs, num_blocks)
        _poison(k_cache, mask)
        _poison(v_cache, mask)
    return DecodeBatch(
        name=cfg.name, seed=seed, num_seqs=S, num_q_heads=Hq, num_kv_heads=Hkv, head_dim=D,
        block_size=bs, scale=cfg.scale, max_blocks_per_seq=mb, num_blocks=num_blocks,
        context_lens=torch.from_numpy(lens.astype(np.int32)),
        block_tables=torch.from_numpy(tables),
        slot_mapping=torch.from_numpy(slots),
        q=q, k_cache=k_cache, v_cache=v_cache, k_new=k_new, v_new=v_new,
        kv_dtype=kv_dtype, k_scale=k_scale, v_scale=v_scale,
    )


def make_batch(name: str, seed: Optional[int] = None, device="cpu", poison: bool = True,
               lens_override: Optional[List[int]] = None, kv_dtype: str = "bf16") -> DecodeBatch:
    """Build the decode batch ``name`` with its values on ``device``."""
    cfg = CONFIGS[name]
    seed = cfg.seed if seed is None else seed
    rng = np.random.default_rng(seed)
    lens = cfg.lengths(rng)
    if lens_override is not None:
        lens = np.asarray(lens_override, dtype=np.int64)
        cfg = dataclasses.replace(cfg, max_context=max(cfg.max_context, int(lens.max(initial=1))))
    return _build(cfg, lens, rng, seed, device, poison, with_append=True, kv_dtype=kv_dtype)


def make_custom(seed: int, lens: Sequence[int], num_q_heads: int, num_kv_heads: int, head_dim: int,
                block_size: int, scale: Optional[float] = None, pool_factor: float = 1.5,
                max_context: Optional[int] = None, device="cpu", poison: bool = True,
                with_append: bool = True, shared_prefix_tokens: int = 0, kv_dtype: str = "bf16") -> DecodeBatch:
    """A batch of any geometry, built by the same recipe as the named configs.

    ``with_append=False`` gives a pool that already holds all L tokens of every
    sequence and a slot mapping of -1 (no append in the step).
    """
    lens = np.asarray(lens, dtype=np.int64)
    mc = int(max_context if max_context is not None else max(int(lens.max(initial=1)), 1))
    cfg = Config(
        name="custom", seed=seed, num_seqs=len(lens), num_q_heads=num_q_heads,
        num_kv_heads=num_kv_heads, head_dim=head_dim, block_size=block_size,
        scale=(1.0 / math.sqrt(head_dim)) if scale is None else scale,
        lengths=_fixed(list(lens)), max_context=mc,
        pool="shared_prefix" if shared_prefix_tokens else "factor",
        pool_factor=pool_factor, prefix_tokens=shared_prefix_tokens,
    )
    rng = np.random.default_rng(seed)
    return _build(cfg, lens, rng, seed, device, poison, with_append, kv_dtype=kv_dtype)


def permute_pool(batch: DecodeBatch, seed: int) -> DecodeBatch:
    """Move every physical block to a new place in the pool and rewrite the tables.

    The logical content of every sequence is unchanged: only where its blocks
    live changes ("Deep Dive into vLLM", section 2.1: the block table maps
    logical to physical blocks).
    """
    nb = batch.num_blocks
    new_of_old = np.random.default_rng(seed).permutation(nb).astype(np.int64)
    old_of_new = np.empty_like(new_of_old)
    old_of_new[new_of_old] = np.arange(nb)
    idx = torch.from_numpy(old_of_new).to(batch.k_cache.device)
    tables = batch.block_tables.numpy()
    new_tables = np.where(tables >= 0, new_of_old[np.clip(tables, 0, None)], -1).astype(np.int32)
    slots = batch.slot_mapping.numpy()
    bs = batch.block_size
    new_slots = np.where(slots >= 0, new_of_old[np.clip(slots // bs, 0, None)] * bs + slots % bs, -1)
    return dataclasses.replace(
        batch,
        k_cache=batch.k_cache.index_select(0, idx),
        v_cache=batch.v_cache.index_select(0, idx),
        block_tables=torch.from_numpy(new_tables),
        slot_mapping=torch.from_numpy(new_slots.astype(np.int64)),
    )


def unshare_prefix(batch: DecodeBatch) -> DecodeBatch:
    """Give every sequence its own copy of every physical block it shares.

    Sharing a physical block and owning a private copy of it must give the same
    attention output ("Deep Dive into vLLM", section 2.2, Flexible Sharing).
    """
    tables = batch.block_tables.numpy().copy()
    lens = batch.context_lens.numpy()
    bs = batch.block_size
    owner: Dict[int, int] = {}
    extra: List[int] = []
    nb = batch.num_blocks
    for s in range(batch.num_seqs):
        for b in range((int(lens[s]) + bs - 1) // bs):
            p = int(tables[s, b])
            if p in owner and owner[p] != s:
                tables[s, b] = nb + len(extra)
                extra.append(p)
            else:
                owner[p] = s
    if not extra:
        return batch
    idx = torch.as_tensor(extra, dtype=torch.int64, device=batch.k_cache.device)
    k = torch.cat([batch.k_cache, batch.k_cache.index_select(0, idx)])
    v = torch.cat([batch.v_cache, batch.v_cache.index_select(0, idx)])
    slots = _slot_mapping(tables, lens, bs)
    return dataclasses.replace(
        batch, k_cache=k, v_cache=v, num_blocks=nb + len(extra),
        block_tables=torch.from_numpy(tables), slot_mapping=torch.from_numpy(slots),
    )


def kv_element_bytes(batch: DecodeBatch) -> int:
    return 1 if batch.kv_dtype == "fp8" else 2


def kv_bytes(batch: DecodeBatch) -> int:
    """Algorithmic K+V bytes one decode step reads: every attended token once per kv head."""
    total_tokens = int(batch.context_lens.to(torch.int64).sum())
    return total_tokens * 2 * batch.num_kv_heads * batch.head_dim * kv_element_bytes(batch)


def unique_kv_bytes(batch: DecodeBatch) -> int:
    """K+V bytes of the distinct physical slots a step reads (shared blocks counted once)."""
    tables = batch.block_tables.numpy()
    lens = batch.context_lens.numpy()
    bs = batch.block_size
    used: Dict[int, int] = {}
    for s in range(batch.num_seqs):
        L = int(lens[s])
        for b in range((L + bs - 1) // bs):
            p = int(tables[s, b])
            used[p] = max(used.get(p, 0), min(bs, L - b * bs))
    return sum(used.values()) * 2 * batch.num_kv_heads * batch.head_dim * kv_element_bytes(batch)


@dataclasses.dataclass
class PrefillBatch(DecodeBatch):
    """A mixed batch of query chunks: q is [T][Hq][D], the queries of sequence s
    are rows query_start[s] .. query_start[s + 1] - 1, the last n_s of its L_s
    tokens (already in the pool). k_new / v_new / slot_mapping are unused."""

    query_start: Optional[torch.Tensor] = None   # int32 [S + 1] (host)


def make_prefill(seed: int, chunk_lens: Sequence[int], context_lens: Sequence[int], num_q_heads: int,
                 num_kv_heads: int, head_dim: int, block_size: int, scale: Optional[float] = None,
                 pool_factor: float = 1.25, device="cpu", poison: bool = True) -> PrefillBatch:
    """A chunked-prefill / mixed batch by the decode recipe (pool of all L tokens,
    poisoned elsewhere), then the T = sum(chunk_lens) query rows, N(0, 1) in bf16
    from the same generator stream, drawn after the pool."""
    n = np.asarray(chunk_lens, dtype=np.int64)
    lens = np.asarray(context_lens, dtype=np.int64)
    assert len(n) == len(lens) and (n <= lens).all() and (n >= 0).all()
    b = make_custom(seed, lens, num_q_heads, num_kv_heads, head_dim, block_size, scale=scale,
                    pool_factor=pool_factor, device=device, poison=poison, with_append=False)
    gen = torch.Generator(device=device)
    gen.manual_seed(seed + 1_000_003)
    T = int(n.sum())
    q = _randn_bf16((max(T, 0), num_q_heads, head_dim), gen, device) if T else torch.empty(
        0, num_q_heads, head_dim, dtype=torch.bfloat16, device=device)
    qs = np.zeros(len(n) + 1, dtype=np.int32)
    qs[1:] = np.cumsum(n)
    fields = {f.name: getattr(b, f.name) for f in dataclasses.fields(DecodeBatch)}
    fields["q"] = q
    return PrefillBatch(**fields, query_start=torch.from_numpy(qs))


def prefill_flops(batch: PrefillBatch) -> int:
    """Multiply-adds x 2 of q.K and P.V: every query token attends to p + 1 positions."""
    qs = batch.query_start.numpy()
    lens = batch.context_lens.numpy()
    total = 0
    for s in range(len(lens)):
        n = int(qs[s + 1] - qs[s])
        L = int(lens[s])
        total += n * (L - n) + n * (n + 1) // 2  # sum over queries of (p + 1)
    return total * batch.num_q_heads * batch.head_dim * 4
