"""Seeded synthetic workloads for MLA decode: shapes, sizes and random draws only.

This module holds no step of the method's arithmetic.  It names the five workloads
(sizes, dtypes, length mixes, page order) and draws their inputs from seeded numpy
generators; both the CUDA path's callers and the tests' CPU checks consume what it
returns.  Distributions follow the workloads' statement: hidden states h ~ N(0, 1),
weights ~ N(0, 1/fan_in).  Where a decode-only input is drawn directly, it is drawn
from the distribution its projection produces (see ``draw_decode_inputs``).
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

PAGE_SIZE = 64


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    n_heads: int
    d_model: int
    d_c: int
    d_rope: int
    d_nope: int
    d_v: int
    s_q: int = 1
    causal: bool = False
    act_dtype: str = "bf16"      # "f32" or "bf16": q, o_lat, out, h and weights
    cache_dtype: str = "bf16"    # "f32", "bf16" or "fp8"
    lengths: tuple | None = None  # fixed lengths, or None for a uniform draw
    len_range: tuple | None = None
    shuffle_pages: bool = False
    n_split: int = 0             # 0: library picks; >0: fixed chunks per sequence
    seed: int = 0
    theta: float = 10000.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.d_nope + self.d_rope)

    @property
    def row_width(self) -> int:
        return self.d_c + self.d_rope


WORKLOADS = {
    # Tiny fp32 case: two sequences of 37 and 100 tokens, 4 heads, narrow dims.
    "tiny_fp32": Workload("tiny_fp32", batch=2, n_heads=4, d_model=64, d_c=64, d_rope=16,
                          d_nope=32, d_v=32, act_dtype="f32", cache_dtype="f32",
                          lengths=(37, 100), seed=0),
    # DeepSeek-V2-Lite-shaped: 32 sequences of 4096 tokens, 16 heads, pages in order.
    "v2lite_bf16": Workload("v2lite_bf16", batch=32, n_heads=16, d_model=2048, d_c=512,
                            d_rope=64, d_nope=128, d_v=128, lengths=(4096,) * 32, seed=1),
    # DeepSeek-V3-shaped: 64 sequences, lengths uniform in [1024, 8192], 128 heads,
    # shuffled block table.  The headline decode workload.
    "v3_bf16": Workload("v3_bf16", batch=64, n_heads=128, d_model=7168, d_c=512, d_rope=64,
                        d_nope=128, d_v=128, len_range=(1024, 8192), shuffle_pages=True,
                        seed=2),
    # Long context: 4 sequences of 131072 tokens, KV split into 32 chunks per sequence.
    "long_bf16": Workload("long_bf16", batch=4, n_heads=128, d_model=2048, d_c=512, d_rope=64,
                          d_nope=128, d_v=128, lengths=(131072,) * 4, n_split=32, seed=3),
    # FP8 latent cache (e4m3 + one fp32 scale per 128 values per token, bf16 k_rope) with
    # two MTP draft query tokens per sequence under a causal mask.
    "fp8_mtp2": Workload("fp8_mtp2", batch=128, n_heads=128, d_model=7168, d_c=512, d_rope=64,
                         d_nope=128, d_v=128, s_q=2, causal=True, cache_dtype="fp8",
                         len_range=(512, 4096), seed=4),
}


def rng_for(w: Workload, stream: int = 0) -> np.random.Generator:
    """Independent seeded generator per (workload seed, stream id)."""
    return np.random.Generator(np.random.PCG64([w.seed, stream]))


def draw_lengths(w: Workload) -> np.ndarray:
    if w.lengths is not None:
        return np.asarray(w.lengths, dtype=np.int32)
    lo, hi = w.len_range
    return rng_for(w, 1).integers(lo, hi + 1, size=w.batch).astype(np.int32)


def make_block_table(lengths, capacity_extra: int, shuffle: bool, rng: np.random.Generator | None,
                     page_size: int = PAGE_SIZE):
    """Assign pages to sequences.  Sequence b owns ceil((L_b + capacity_extra) / page) pages;
    the pool is numbered 0 .. num_pages-1, in order or shuffled.  Unused table entries
    hold 0 (a valid page id that no kernel reads)."""
    lengths = np.asarray(lengths)
    need = (lengths + capacity_extra + page_size - 1) // page_size
    need = np.maximum(need, 1)
    num_pages = int(need.sum())
    ids = np.arange(num_pages, dtype=np.int32)
    if shuffle:
        ids = rng.permutation(ids).astype(np.int32)
    max_pages = int(need.max())
    table = np.zeros((len(lengths), max_pages), dtype=np.int32)
    off = 0
    for b, n in enumerate(need):
        table[b, :n] = ids[off:off + n]
        off += n
    return table, num_pages


def draw_weights(w: Workload, dtype=np.float32):
    """W_DKV [d_c, d_model], W_KR [d_rope, d_model], W_UK [H, d_nope, d_c], W_UV [H, d_v, d_c],
    each N(0, 1/fan_in)."""
    r = rng_for(w, 2)
    w_dkv = r.standard_normal((w.d_c, w.d_model), dtype=np.float32) / math.sqrt(w.d_model)
    w_kr = r.standard_normal((w.d_rope, w.d_model), dtype=np.float32) / math.sqrt(w.d_model)
    w_uk = r.standard_normal((w.n_heads, w.d_nope, w.d_c), dtype=np.float32) / math.sqrt(w.d_c)
    w_uv = r.standard_normal((w.n_heads, w.d_v, w.d_c), dtype=np.float32) / math.sqrt(w.d_c)
    return (w_dkv.astype(dtype), w_kr.astype(dtype), w_uk.astype(dtype), w_uv.astype(dtype))


def draw_hidden(w: Workload, n_tokens: int, stream: int = 3) -> np.ndarray:
    """Hidden states h ~ N(0, 1), [n_tokens, d_model] float32."""
    return rng_for(w, stream).standard_normal((n_tokens, w.d_model), dtype=np.float32)


def draw_query_heads(w: Workload, n_tokens: int, stream: int = 4):
    """Per-head query parts before absorption: q_nope [T, H, d_nope], q_rope [T, H, d_rope].

    A query W_UQ h with h ~ N(0, 1) and W_UQ ~ N(0, 1/d_model) has entries ~ N(0, 1), so
    the parts are drawn from N(0, 1) directly."""
    r = rng_for(w, stream)
    q_nope = r.standard_normal((n_tokens, w.n_heads, w.d_nope), dtype=np.float32)
    q_rope = r.standard_normal((n_tokens, w.n_heads, w.d_rope), dtype=np.float32)
    return q_nope, q_rope


def draw_decode_inputs(w: Workload, lengths, stream: int = 5):
    """Inputs of the attention step alone, drawn from the distributions the projections
    produce: cached latent rows c ~ N(0, 1) and k_rope ~ N(0, 1) (W_DKV h and a rotation of
    W_KR h have unit-variance entries), packed query q_lat ~ N(0, d_nope/d_c) (W_UK^T q_nope
    with W_UK ~ N(0, 1/d_c)) and q_rope ~ N(0, 1).

    Returns (rows [sum(L), d_c + d_rope] float32 in sequence order, q [len(L)*S_q, H, d_c + d_rope])."""
    r = rng_for(w, stream)
    total = int(np.sum(lengths))
    rows = r.standard_normal((total, w.row_width), dtype=np.float32)
    n_tok = len(lengths) * w.s_q
    q = r.standard_normal((n_tok, w.n_heads, w.row_width), dtype=np.float32)
    q[..., : w.d_c] *= np.float32(math.sqrt(w.d_nope / w.d_c))
    return rows, q


def scatter_rows_to_pages(rows, lengths, block_table, num_pages, page_size: int = PAGE_SIZE,
                          fill=0.0):
    """Lay per-sequence rows [sum(L), width] out as pages [num_pages, page_size, width]
    (pure data movement; slots past each sequence's length hold ``fill``)."""
    rows = np.asarray(rows)
    width = rows.shape[1]
    pages = np.full((num_pages, page_size, width), fill, dtype=rows.dtype)
    off = 0
    for b, length in enumerate(lengths):
        length = int(length)
        for p in range((length + page_size - 1) // page_size):
            lo = p * page_size
            hi = min(length, lo + page_size)
            pages[block_table[b, p], : hi - lo] = rows[off + lo: off + hi]
        off += length
    return pages
