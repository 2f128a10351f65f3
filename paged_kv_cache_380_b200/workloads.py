"""Seeded synthetic inputs for the paged-KV-cache attention workloads.

This module only draws random numbers and lays them out (numpy only).  It
holds none of the attention arithmetic, imports neither the CUDA binding nor
the oracle, and serves both: the GPU path and the fp64 oracle are fed the same
arrays from here.

Layouts (the plainest reading of a page as ``(page_size, d_model)`` in
"Flash Attention与Paged KV Cache优化大模型计算效率" §3.2 "分页式缓存设计"):

* pools ``k_pages``/``v_pages``: ``[num_pages, page_size, num_kv_heads, head_dim]``;
  slot ``s = page * page_size + offset`` is row ``s`` of the pool viewed as
  ``[num_pages * page_size, num_kv_heads * head_dim]``;
* ``block_tables``: ``int32 [batch, max_pages_per_seq]``, logical page -> physical
  page; entries past a sequence's last page are -1 (never read);
* ``context_lens``: ``int32 [batch]``;
* decode ``q``: ``[batch, num_q_heads, head_dim]``; prefill ``q``: packed
  ``[total_q, num_q_heads, head_dim]`` with ``q_start int32 [batch + 1]``;
* new tokens for the cache append: ``k_new``/``v_new`` ``[T, num_kv_heads, head_dim]``
  and ``slot_mapping int64 [T]``.

bf16 data is carried as uint16 bit patterns (numpy has no bf16): values are
drawn as float32 from ``standard_normal`` and rounded to bf16 to nearest even,
so the same bits reach the GPU and the oracle.

Random streams: ``numpy.random.SeedSequence(380 + config_index)`` spawned into
six children used, in this order, for context lengths, the physical page
permutation, Q, K, V and the slot mapping.

Pages of the pool that no sequence owns, and the rows of a sequence's last
page past its context length, hold a NaN canary, so a kernel that reads one
produces NaN instead of a plausible wrong answer.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np

CANARY_BITS = {"bf16": 0x7FC0, "f16": 0x7E00}   # quiet NaNs
STORAGE = {"f32": np.float32, "bf16": np.uint16, "f16": np.uint16}


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + (((u >> 16) & 1) + 0x7FFF)) >> 16).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _normal(rng: np.random.Generator, shape, dtype: str) -> np.ndarray:
    x = rng.standard_normal(shape, dtype=np.float32)
    if dtype == "f32":
        return x
    if dtype == "bf16":
        return to_bf16_bits(x)
    if dtype == "f16":
        return x.astype(np.float16).view(np.uint16)
    raise ValueError(dtype)


def _canary_fill(a: np.ndarray, dtype: str) -> None:
    if dtype == "f32":
        a.fill(np.nan)
    else:
        a.fill(CANARY_BITS[dtype])


def _streams(config_index: int):
    kids = np.random.SeedSequence(380 + config_index).spawn(6)
    names = ("ctx", "perm", "q", "k", "v", "slot")
    return {n: np.random.default_rng(k) for n, k in zip(names, kids)}


@dataclass
class Case:
    """One seeded input set (numpy, host).  ``kind`` is 'decode' or 'prefill'."""
    name: str
    kind: str
    dtype: str                      # storage dtype of q, K and V ('f32' | 'bf16' | 'f16')
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    page_size: int
    q: np.ndarray
    k_pages: np.ndarray
    v_pages: np.ndarray
    block_tables: np.ndarray
    context_lens: np.ndarray
    scale: float
    q_start: Optional[np.ndarray] = None
    k_new: Optional[np.ndarray] = None
    v_new: Optional[np.ndarray] = None
    slot_mapping: Optional[np.ndarray] = None
    meta: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def num_pages(self) -> int:
        return int(self.k_pages.shape[0])

    @property
    def max_pages_per_seq(self) -> int:
        return int(self.block_tables.shape[1])


def _deal_pages(rng_perm, num_pages: int, pages_per_seq, max_pages: int):
    """Deal a seeded permutation of the pool out to the sequences' logical pages."""
    perm = rng_perm.permutation(num_pages).astype(np.int32)
    bt = np.full((len(pages_per_seq), max(max_pages, 1)), -1, dtype=np.int32)
    pos = 0
    for b, n in enumerate(pages_per_seq):
        bt[b, :n] = perm[pos:pos + n]
        pos += n
    return bt, perm, pos


def _fill_sequence(pool_flat: np.ndarray, bt_row: np.ndarray, ps: int, values: np.ndarray,
                   start: int = 0) -> None:
    """Place logical tokens start..start+len(values)-1 of one sequence into the pool."""
    n = values.shape[0]
    if n == 0:
        return
    i = np.arange(start, start + n)
    slots = bt_row[i // ps].astype(np.int64) * ps + i % ps
    pool_flat[slots] = values


def decode_case(*, name: str, config_index: int, batch: int, num_q_heads: int, num_kv_heads: int,
                head_dim: int, page_size: int, dtype: str, context_lens,
                num_pages: Optional[int] = None, pool_factor: float = 1.25,
                new_tokens: Optional[str] = None, num_new: int = 0) -> Case:
    """Decode inputs: one query per sequence over a shuffled paged pool.

    ``context_lens`` is an int array or a callable ``rng -> int array``.
    ``new_tokens``: None; 'random' (``num_new`` rows scattered to distinct
    random slots of the whole pool, drawn without replacement); or 'append'
    (each sequence's token at position ctx-1 is left out of the pool and
    delivered as a new row with its slot).
    """
    r = _streams(config_index)
    cl = np.asarray(context_lens(r["ctx"]) if callable(context_lens) else context_lens,
                    dtype=np.int32)
    assert cl.shape == (batch,) and (cl >= 0).all()
    ps, Hkv, D = page_size, num_kv_heads, head_dim
    pages_per_seq = [int(math.ceil(c / ps)) for c in cl]
    needed = sum(pages_per_seq)
    P = num_pages if num_pages is not None else max(1, int(math.ceil(pool_factor * needed)))
    assert P >= needed
    max_pages = max(pages_per_seq) if pages_per_seq else 1
    bt, _, _ = _deal_pages(r["perm"], P, pages_per_seq, max_pages)

    q = _normal(r["q"], (batch, num_q_heads, D), dtype)
    store = STORAGE[dtype]
    k_pages = np.empty((P, ps, Hkv, D), dtype=store)
    v_pages = np.empty((P, ps, Hkv, D), dtype=store)
    _canary_fill(k_pages, dtype)
    _canary_fill(v_pages, dtype)
    kf = k_pages.reshape(P * ps, Hkv, D)
    vf = v_pages.reshape(P * ps, Hkv, D)
    append = new_tokens == "append"
    k_new = v_new = slots = None
    if append:
        k_new = np.empty((batch, Hkv, D), dtype=store)
        v_new = np.empty((batch, Hkv, D), dtype=store)
        slots = np.full(batch, -1, dtype=np.int64)
    for b in range(batch):
        c = int(cl[b])
        kb = _normal(r["k"], (c, Hkv, D), dtype)
        vb = _normal(r["v"], (c, Hkv, D), dtype)
        if append and c > 0:
            _fill_sequence(kf, bt[b], ps, kb[:c - 1])
            _fill_sequence(vf, bt[b], ps, vb[:c - 1])
            k_new[b], v_new[b] = kb[c - 1], vb[c - 1]
            slots[b] = int(bt[b, (c - 1) // ps]) * ps + (c - 1) % ps
        else:
            _fill_sequence(kf, bt[b], ps, kb)
            _fill_sequence(vf, bt[b], ps, vb)
    if new_tokens == "random":
        k_new = _normal(r["k"], (num_new, Hkv, D), dtype)
        v_new = _normal(r["v"], (num_new, Hkv, D), dtype)
        slots = r["slot"].choice(P * ps, size=num_new, replace=False).astype(np.int64)
    return Case(name=name, kind="decode", dtype=dtype, num_q_heads=num_q_heads,
                num_kv_heads=Hkv, head_dim=D, page_size=ps, q=q, k_pages=k_pages,
                v_pages=v_pages, block_tables=bt, context_lens=cl, scale=1.0 / math.sqrt(D),
                k_new=k_new, v_new=v_new, slot_mapping=slots,
                meta={"needed_pages": needed, "config_index": config_index})


def prefill_case(*, name: str, config_index: int, num_seqs: int, num_q_heads: int,
                 num_kv_heads: int, head_dim: int, page_size: int, dtype: str,
                 shared_prefix: int, chunk_lens, private_prefix: int = 0,
                 pool_factor: float = 1.25) -> Case:
    """Chunked-prefill inputs with a shared prefix.

    Every sequence starts with the same ``shared_prefix`` tokens (a whole
    number of pages, stored once: the block tables of all sequences point at
    the same physical pages, as a refcounted shared prompt would), then
    ``private_prefix`` tokens of its own already cached, then a chunk of
    ``chunk_lens[b]`` new tokens whose queries are packed into ``q``.  The
    chunk's K/V are not in the pool yet: they come as ``k_new``/``v_new``
    with their ``slot_mapping`` (cache append first, then attention).
    """
    assert shared_prefix % page_size == 0
    r = _streams(config_index)
    ps, Hkv, D = page_size, num_kv_heads, head_dim
    n = np.asarray(chunk_lens, dtype=np.int64)
    assert n.shape == (num_seqs,)
    cl = (shared_prefix + private_prefix + n).astype(np.int32)
    shared_pages = shared_prefix // ps
    own_pages = [int(math.ceil(int(c) / ps)) - shared_pages for c in cl]
    needed = shared_pages + sum(own_pages)
    P = max(1, int(math.ceil(pool_factor * needed)))
    perm = r["perm"].permutation(P).astype(np.int32)
    max_pages = shared_pages + max(own_pages)
    bt = np.full((num_seqs, max_pages), -1, dtype=np.int32)
    bt[:, :shared_pages] = perm[:shared_pages]
    pos = shared_pages
    for b in range(num_seqs):
        bt[b, shared_pages:shared_pages + own_pages[b]] = perm[pos:pos + own_pages[b]]
        pos += own_pages[b]

    q_start = np.zeros(num_seqs + 1, dtype=np.int32)
    q_start[1:] = np.cumsum(n)
    total_q = int(q_start[-1])
    q = _normal(r["q"], (total_q, num_q_heads, D), dtype)
    store = STORAGE[dtype]
    k_pages = np.empty((P, ps, Hkv, D), dtype=store)
    v_pages = np.empty((P, ps, Hkv, D), dtype=store)
    _canary_fill(k_pages, dtype)
    _canary_fill(v_pages, dtype)
    kf = k_pages.reshape(P * ps, Hkv, D)
    vf = v_pages.reshape(P * ps, Hkv, D)
    _fill_sequence(kf, bt[0], ps, _normal(r["k"], (shared_prefix, Hkv, D), dtype))
    _fill_sequence(vf, bt[0], ps, _normal(r["v"], (shared_prefix, Hkv, D), dtype))
    k_new = np.empty((total_q, Hkv, D), dtype=store)
    v_new = np.empty((total_q, Hkv, D), dtype=store)
    slots = np.empty(total_q, dtype=np.int64)
    for b in range(num_seqs):
        kb = _normal(r["k"], (private_prefix, Hkv, D), dtype)
        vb = _normal(r["v"], (private_prefix, Hkv, D), dtype)
        _fill_sequence(kf, bt[b], ps, kb, start=shared_prefix)
        _fill_sequence(vf, bt[b], ps, vb, start=shared_prefix)
        lo, hi = int(q_start[b]), int(q_start[b + 1])
        k_new[lo:hi] = _normal(r["k"], (hi - lo, Hkv, D), dtype)
        v_new[lo:hi] = _normal(r["v"], (hi - lo, Hkv, D), dtype)
        i = np.arange(shared_prefix + private_prefix, int(cl[b]))
        slots[lo:hi] = bt[b, i // ps].astype(np.int64) * ps + i % ps
    return Case(name=name, kind="prefill", dtype=dtype, num_q_heads=num_q_heads,
                num_kv_heads=Hkv, head_dim=D, page_size=ps, q=q, k_pages=k_pages,
                v_pages=v_pages, block_tables=bt, context_lens=cl, scale=1.0 / math.sqrt(D),
                q_start=q_start, k_new=k_new, v_new=v_new, slot_mapping=slots,
                meta={"needed_pages": needed, "shared_pages": shared_pages,
                      "config_index": config_index})


# ---- the five named workloads -----------------------------------------------

def tiny_decode_f32() -> Case:
    """Tiny paged decode: batch 2, 4 q heads, 2 KV heads, D 64, fp32, page 16,
    contexts {37, 100}, a 16-page pool dealt out by a seeded permutation."""
    return decode_case(name="tiny_decode_f32", config_index=0, batch=2, num_q_heads=4,
                       num_kv_heads=2, head_dim=64, page_size=16, dtype="f32",
                       context_lens=np.array([37, 100]), num_pages=16)


def llama2_7b_mha_decode(batch: int = 64, new_tokens: str = "random") -> Case:
    """Llama-2-7B-shaped MHA decode: 32/32 heads, D 128, bf16, page 16,
    contexts uniform in [512, 4096], pool 1.25x the pages needed, plus the
    cache append of 64 new K/V rows through a random slot mapping."""
    ctx = (lambda rng: rng.integers(512, 4097, size=batch))
    return decode_case(name="llama2_7b_mha_decode", config_index=1, batch=batch, num_q_heads=32,
                       num_kv_heads=32, head_dim=128, page_size=16, dtype="bf16",
                       context_lens=ctx, new_tokens=new_tokens, num_new=batch)


def _lognormal_ctx(batch):
    def draw(rng):
        x = np.rint(np.exp(rng.normal(math.log(2048.0), 0.7, size=batch)))
        return np.clip(x, 64, 8192).astype(np.int64)
    return draw


def llama2_70b_gqa_decode(batch: int = 128) -> Case:
    """Llama-2-70B-shaped GQA decode: 64 q heads, 8 KV heads (group 8), D 128,
    bf16, page 16, contexts log-normal (median 2048, sigma 0.7) clipped to
    [64, 8192], shuffled pool."""
    return decode_case(name="llama2_70b_gqa_decode", config_index=2, batch=batch,
                       num_q_heads=64, num_kv_heads=8, head_dim=128, page_size=16, dtype="bf16",
                       context_lens=_lognormal_ctx(batch))


def long_ctx_split_kv(context_len: int = 131072, batch: int = 4) -> Case:
    """Long-context split-KV decode: batch 4, 32 q heads, 8 KV heads, D 128,
    131072-token contexts, page 256, bf16 K/V (the INT8 variant quantises
    these same K/V rows, one fp16 scale per (token, KV head))."""
    return decode_case(name="long_ctx_split_kv", config_index=3, batch=batch, num_q_heads=32,
                       num_kv_heads=8, head_dim=128, page_size=256, dtype="bf16",
                       context_lens=np.full(batch, context_len))


def chunked_prefill_shared_prefix(num_seqs: int = 8, prefix: int = 1024, chunk: int = 512) -> Case:
    """Causal chunked prefill: 8 sequences share their first 1024 tokens (64
    refcounted pages of 16), each then has 512 new query tokens attending
    causally over prefix + own chunk; 32 q heads, 8 KV heads, D 128, bf16."""
    return prefill_case(name="chunked_prefill_shared_prefix", config_index=4, num_seqs=num_seqs,
                        num_q_heads=32, num_kv_heads=8, head_dim=128, page_size=16, dtype="bf16",
                        shared_prefix=prefix, chunk_lens=np.full(num_seqs, chunk))


def cached_token_slots(case: Case) -> np.ndarray:
    """Pool slot of every cached token of a decode case, sequence by sequence (int64)."""
    ps = case.page_size
    out = []
    for b in range(case.batch):
        n = int(case.context_lens[b])
        pos = np.arange(n, dtype=np.int64)
        pages = case.block_tables[b, :(n + ps - 1) // ps].astype(np.int64)
        out.append(pages[pos // ps] * ps + pos % ps)
    return np.concatenate(out) if out else np.zeros(0, np.int64)


def full_cache_scatter(case: Case):
    """The bandwidth case of the cache append: every cached token of ``case`` is
    written again, to a seeded random permutation of the pool's slots.

    Returns (src_slots, dst_slots): row t of the scatter is pool row src_slots[t]
    (its K and V values), written to slot dst_slots[t] (distinct slots).
    """
    src = cached_token_slots(case)
    num_slots = case.k_pages.shape[0] * case.page_size
    rng = np.random.default_rng(np.random.SeedSequence(380 + case.meta["config_index"]).spawn(7)[6])
    dst = rng.permutation(num_slots)[: src.shape[0]].astype(np.int64)
    return src, dst


WORKLOADS = {
    "tiny_decode_f32": tiny_decode_f32,
    "llama2_7b_mha_decode": llama2_7b_mha_decode,
    "llama2_70b_gqa_decode": llama2_70b_gqa_decode,
    "long_ctx_split_kv": long_ctx_split_kv,
    "chunked_prefill_shared_prefix": chunked_prefill_shared_prefix,
}
