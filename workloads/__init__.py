"""Seeded synthetic inputs for paged attention.

This module only draws random inputs: sequence lengths, a block table (a
seeded permutation of the physical page pool handed out to the sequences in
order), packed queries, the new tokens' keys/values and the cache pool's
contents.  It holds none of the method's arithmetic: it never computes a
slot, a causal bound or an attention value, so both the fp64 oracle and the
CUDA library can take their inputs from here.

Pages handed to a sequence are filled with random values in every row (rows
past the sequence's end included); pages no sequence owns hold ``fill``
(0 for timing, NaN to poison them in correctness runs).  The new tokens'
K/V are separate arrays that ``pa_scatter_kv`` writes into the cache.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import numpy as np


@dataclass
class Spec:
    """Shape of one synthetic continuous batch."""

    name: str
    q_lens: np.ndarray          # int64 [batch]
    past: np.ndarray            # int64 [batch]
    q_heads: int
    kv_heads: int
    head_size: int
    block_size: int
    num_blocks: int             # physical pages in the pool
    dist: str = "normal"        # "normal" -> N(0,1), "uniform" -> U[-1,1]
    seed: int = 0
    elem: str = "f16"           # "f16": float16 arrays; "bf16": bfloat16 bit patterns as uint16
    extra: dict = field(default_factory=dict)

    @property
    def batch(self) -> int:
        return int(self.q_lens.size)

    @property
    def seqlens_kv(self) -> np.ndarray:
        return (self.past + self.q_lens).astype(np.int64)

    @property
    def token_count(self) -> int:
        return int(self.q_lens.sum())

    @property
    def pages_per_seq(self) -> np.ndarray:
        return -(-self.seqlens_kv // self.block_size)


def _pool(pages: np.ndarray) -> int:
    return int(pages.sum())


def spec_tiny() -> Spec:
    """batch 2, q_heads 2, kv_heads 1, head_size 16, block_size 16, q_lens {1,4},
    past {7,20} (read as pairs (1,7) and (4,20)), U[-1,1], 16-block pool."""
    return Spec("tiny correctness", np.array([1, 4]), np.array([7, 20]), 2, 1, 16, 16, 16,
                dist="uniform", seed=1000)


def spec_decode_gqa(rng_seed: int = 1001) -> Spec:
    """64 sequences, q_len 1, past U[512,4096], 32/8 heads, d 128, bs 16, 20000-block pool."""
    rng = np.random.Generator(np.random.PCG64(rng_seed))
    past = rng.integers(512, 4096, size=64, endpoint=True)
    return Spec("decode-heavy GQA", np.ones(64, dtype=np.int64), past, 32, 8, 128, 16, 20000,
                seed=rng_seed)


def spec_prefill_mha(rng_seed: int = 1002) -> Spec:
    """8 sequences, q_len = total_kv = 2048 (past 0), 16/16 heads, d 128, bs 256."""
    q = np.full(8, 2048, dtype=np.int64)
    past = np.zeros(8, dtype=np.int64)
    s = Spec("causal prefill MHA", q, past, 16, 16, 128, 256, 0, seed=rng_seed)
    s.num_blocks = _pool(s.pages_per_seq)
    return s


def spec_mixed(rng_seed: int = 1003) -> Spec:
    """32 sequences: 16 decode (q_len 1, past U[1024,8192]) then 16 prefill chunks
    (q_len U[64,512], past U[0,2048]); 32/8 heads, d 128, bs 16; the pool is exactly
    the pages the batch needs."""
    rng = np.random.Generator(np.random.PCG64(rng_seed))
    dpast = rng.integers(1024, 8192, size=16, endpoint=True)
    pq = rng.integers(64, 512, size=16, endpoint=True)
    ppast = rng.integers(0, 2048, size=16, endpoint=True)
    q = np.concatenate([np.ones(16, dtype=np.int64), pq])
    past = np.concatenate([dpast, ppast])
    s = Spec("mixed continuous batch", q, past, 32, 8, 128, 16, 0, seed=rng_seed)
    s.num_blocks = _pool(s.pages_per_seq)
    return s


def spec_long_decode(rng_seed: int = 1004) -> Spec:
    """8 sequences, q_len U{1..4}, past U[32768,131072], 64/8 heads, d 128, bs 256;
    the pool is exactly the pages the batch needs, permuted as a whole."""
    rng = np.random.Generator(np.random.PCG64(rng_seed))
    q = rng.integers(1, 4, size=8, endpoint=True)
    past = rng.integers(32768, 131072, size=8, endpoint=True)
    s = Spec("long-context decode GQA 8", q, past, 64, 8, 128, 256, 0, seed=rng_seed)
    s.num_blocks = _pool(s.pages_per_seq)
    return s


def spec_prefill_mha_d256(rng_seed: int = 1005) -> Spec:
    """The causal prefill MHA shape at head size 256: 8 sequences, q_len =
    total_kv = 2048, 16/16 heads, bs 256 (a head size the pages' XQA kernels
    are built for; not one of the five benchmark configurations)."""
    q = np.full(8, 2048, dtype=np.int64)
    past = np.zeros(8, dtype=np.int64)
    s = Spec("causal prefill MHA, head size 256", q, past, 16, 16, 256, 256, 0, seed=rng_seed)
    s.num_blocks = _pool(s.pages_per_seq)
    return s


CONFIGS = {
    0: spec_tiny,
    1: spec_decode_gqa,
    2: spec_prefill_mha,
    3: spec_mixed,
    4: spec_long_decode,
}

CONFIG_KEYS = {
    "tiny": 0, "decode": 1, "prefill": 2, "mixed": 3, "long_decode": 4,
}


def custom(q_lens, past, q_heads, kv_heads, head_size, block_size, num_blocks=None,
           dist="normal", seed=7, name="custom", elem="f16") -> Spec:
    q = np.asarray(q_lens, dtype=np.int64)
    p = np.asarray(past, dtype=np.int64)
    s = Spec(name, q, p, q_heads, kv_heads, head_size, block_size, 0, dist=dist, seed=seed,
             elem=elem)
    need = _pool(s.pages_per_seq)
    s.num_blocks = max(need, 1) if num_blocks is None else int(num_blocks)
    assert s.num_blocks >= need
    return s


def _to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float32 -> bfloat16 bit patterns (uint16), rounded to nearest-even by torch."""
    import torch
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


BF16_NAN = np.uint16(0x7FC0)


def _draw(rng, n, dist, elem="f16", chunk=1 << 24):
    out = np.empty(n, dtype=np.uint16 if elem == "bf16" else np.float16)
    for lo in range(0, n, chunk):
        hi = min(n, lo + chunk)
        if dist == "uniform":
            v = rng.uniform(-1.0, 1.0, size=hi - lo)
        else:
            v = rng.standard_normal(size=hi - lo, dtype=np.float32)
        out[lo:hi] = _to_bf16_bits(v) if elem == "bf16" else v
    return out


def fill_value(elem: str, fill: float):
    """`fill` in the element type's storage (bf16: its bit pattern)."""
    if elem != "bf16":
        return fill
    if np.isnan(fill):
        return BF16_NAN
    return _to_bf16_bits(np.array([fill], dtype=np.float32))[0]


def generate(spec: Spec, fill: float = 0.0, seed: int | None = None, block_order=None) -> dict:
    """Draw one batch of inputs for ``spec``.

    Returns numpy arrays: query [T, q_heads, d], key/value [T, kv_heads, d]
    (the new tokens), key_cache/value_cache [num_blocks, block_size, kv_heads,
    d], block_table int32 [batch, max_blocks_per_seq] (-1 past a sequence's
    pages), cu_seqlens_q int32 [batch + 1], seqlens_kv int32 [batch], all
    float16 where floating point (bfloat16 bit patterns as uint16 when
    ``spec.elem`` is "bf16").  ``block_order`` overrides the seeded pool
    permutation (used by the page-permutation tests).
    """
    rng = np.random.Generator(np.random.PCG64(spec.seed if seed is None else seed))
    pages = spec.pages_per_seq
    maxb = max(1, int(pages.max()) if pages.size else 1)
    if block_order is None:
        order = rng.permutation(spec.num_blocks)
    else:
        order = np.asarray(block_order)
        assert order.size >= int(pages.sum())
    block_table = np.full((spec.batch, maxb), -1, dtype=np.int32)
    nxt = 0
    for b in range(spec.batch):
        n = int(pages[b])
        block_table[b, :n] = order[nxt:nxt + n]
        nxt += n
    T = spec.token_count
    qh, kvh, d, bs = spec.q_heads, spec.kv_heads, spec.head_size, spec.block_size
    el = spec.elem
    query = _draw(rng, T * qh * d, spec.dist, el).reshape(T, qh, d)
    key = _draw(rng, T * kvh * d, spec.dist, el).reshape(T, kvh, d)
    value = _draw(rng, T * kvh * d, spec.dist, el).reshape(T, kvh, d)
    cdt = np.uint16 if el == "bf16" else np.float16
    key_cache = np.full((spec.num_blocks, bs, kvh, d), fill_value(el, fill), dtype=cdt)
    value_cache = np.full((spec.num_blocks, bs, kvh, d), fill_value(el, fill), dtype=cdt)
    used = block_table[block_table >= 0]
    per_page = bs * kvh * d
    for cache in (key_cache, value_cache):
        flat = cache.reshape(spec.num_blocks, per_page)
        vals = _draw(rng, used.size * per_page, spec.dist, el).reshape(used.size, per_page)
        flat[used] = vals
    cu = np.zeros(spec.batch + 1, dtype=np.int32)
    cu[1:] = np.cumsum(spec.q_lens)
    return {
        "query": query, "key": key, "value": value,
        "key_cache": key_cache, "value_cache": value_cache,
        "block_table": block_table, "cu_seqlens_q": cu,
        "seqlens_kv": spec.seqlens_kv.astype(np.int32),
    }
