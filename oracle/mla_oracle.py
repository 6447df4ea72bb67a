"""Plain fp64 CPU oracle for Multi-head Latent Attention (MLA) decode over a latent KV cache.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only the test suite, ``__graft_entry__.smoke()``
and the CPU-baseline / reference legs of ``bench.py`` may import or call this module.
The library (``mla_latent_kv_27_b200``) never imports it and has no CPU fallback.
This module shares no code with the CUDA path: it is numpy in float64, written from
the pages listed below, slow on purpose, and meant to be checked against them by eye.

Pages followed (cited by page title and section):

* [DSV2]  "DeepSeek-V2 大模型论文原文 PDF" (hncyxsy.com/news/273095)
          section 1.1 (MHA cache 2*n_h*d_h per token and layer), 2.1 (joint low-rank
          compression c_KV = W_DKV h, k_C = W_UK c_KV, v_C = W_UV c_KV), 2.2 (matrix
          absorption: q^T W_UK is precomputed, W_UV moves to the output side),
          2.3 (decoupled RoPE: d_h = d_rope + d_nope; the cache holds the latent plus a
          small positional key), 4.1 (no re-expansion of K/V at inference).
* [HDU]   "8.1 DeepSeek 架构：MLA、DeepSeekMoE 与 FP8 训练" (hdu-wiki.cn), section 2
          (c_t = W^{DKV} h_t, k_t = W^{UK} c_t, v_t = W^{UV} c_t); section 5 and Q4
          (FP8 with one scale per tile/block, not one global scale).
* [DS25]  "从一份技术报告说起：DeepSeek 2025 到底在做什么" (m.nlpx.cn/news/79410),
          section 2.2 (RoPE on part of the dimensions; latent rank about 512),
          section 3.3 (worked example: 512 + 64 = 576 values per token vs
          2*32*128 = 8192 for MHA, about 14.2x), section 5.2 (precompute RoPE cos/sin).
* [IP]    "DeepSeek大模型核心技术解析：MOE架构与MLA注意力机制" (intelliparadigm.com),
          section 3.3 (A = softmax(q k^T / sqrt(d_h)), o = A v), section 4.1 (decode reads
          the whole history), section 6.1 (blocked KV storage), section 6.3 (FP8 KV cache
          with dynamic quantisation).
* [SHQ]   "从MLA到DeepSeekMoE：DeepSeek系列大模型架构演进与技术拆解" (sheratonhq.com),
          section 2.1 (MHA cache arithmetic: 2 x 5120 fp16 values, about 20 KB per token).

Readings taken where the pages are silent:

* RoPE pairs are interleaved, (x[2i], x[2i+1]) rotated by pos * theta^(-2i/d_rope).
* Query token j of S_q sits at position L - S_q + j; with the causal mask it attends key
  positions <= its own; without it, it attends all L cached tokens.
* The softmax scale is 1/sqrt(d_nope + d_rope).
* An empty attention set gives o = 0 and lse = -inf.
* FP8 (OCP E4M3): one fp32 scale per token per 128-element block of c_KV,
  s = amax / 448 (s = 1 when amax = 0); the code is the round-to-nearest-even,
  saturating E4M3 of fp32(x * fp32(448 / amax)).  The code is an integer decided by
  floating point, so that decision is made in fp32, the precision of the kernel.

Parity pins for every function live in tests/test_oracle.py; no function here is
"parity unpinned".
"""
from __future__ import annotations

import math

import numpy as np

# --------------------------------------------------------------------------------------
# Cache size arithmetic  ([DSV2] 1.1, [DS25] 3.3, [SHQ] 2.1)
# --------------------------------------------------------------------------------------


def mha_values_per_token(n_heads: int, head_dim: int) -> int:
    """Values a standard MHA layer caches per token: one key and one value per head
    ([DSV2] 1.1: 2 * n_h * d_h per token and layer)."""
    return 2 * n_heads * head_dim


def mla_values_per_token(d_c: int, d_rope: int) -> int:
    """Values an MLA layer caches per token: the latent c_KV plus the one shared
    decoupled-RoPE key ([DSV2] 2.3; [DS25] 3.3: 512 + 64 = 576)."""
    return d_c + d_rope


# --------------------------------------------------------------------------------------
# Decoupled RoPE  ([DSV2] 2.3, [DS25] 2.2 and 5.2)
# --------------------------------------------------------------------------------------


def rope_cos_sin(positions, d_rope: int, theta: float = 10000.0):
    """cos/sin of the rotation angles pos * theta^(-2i/d_rope), i = 0 .. d_rope/2 - 1.

    Returns two float64 arrays of shape positions.shape + (d_rope // 2,).  These are
    the tables [DS25] 5.2 recommends precomputing."""
    assert d_rope % 2 == 0
    pos = np.asarray(positions, dtype=np.float64)
    i = np.arange(d_rope // 2, dtype=np.float64)
    inv_freq = theta ** (-2.0 * i / d_rope)
    ang = pos[..., None] * inv_freq
    return np.cos(ang), np.sin(ang)


def rope_rotate(x, positions, theta: float = 10000.0):
    """Rotate the RoPE part x[..., d_rope] at the given positions.

    Pair (x[2i], x[2i+1]) is rotated by angle pos * theta^(-2i/d_rope):
        y[2i]   = x[2i] cos a - x[2i+1] sin a
        y[2i+1] = x[2i] sin a + x[2i+1] cos a
    ``positions`` broadcasts against x.shape[:-1]."""
    x = np.asarray(x, dtype=np.float64)
    d_rope = x.shape[-1]
    cos, sin = rope_cos_sin(np.broadcast_to(np.asarray(positions), x.shape[:-1]), d_rope, theta)
    x_even = x[..., 0::2]
    x_odd = x[..., 1::2]
    y = np.empty_like(x)
    y[..., 0::2] = x_even * cos - x_odd * sin
    y[..., 1::2] = x_even * sin + x_odd * cos
    return y


# --------------------------------------------------------------------------------------
# Step a1: compress the new tokens into the cache  ([DSV2] 2.1, 2.3; [HDU] 2)
# --------------------------------------------------------------------------------------


def compress_kv(h, w_dkv, w_kr, positions, theta: float = 10000.0):
    """c_KV = W_DKV h and k_rope = RoPE_pos(W_KR h) for each token.

    h: [T, d_model]; w_dkv: [d_c, d_model]; w_kr: [d_rope, d_model]; positions: [T].
    Returns (c [T, d_c], k_rope [T, d_rope]) in float64."""
    h = np.asarray(h, dtype=np.float64)
    c = h @ np.asarray(w_dkv, dtype=np.float64).T
    kr = h @ np.asarray(w_kr, dtype=np.float64).T
    return c, rope_rotate(kr, np.asarray(positions), theta)


# --------------------------------------------------------------------------------------
# Step a2: absorb W_UK into the query  ([DSV2] 2.2)
# --------------------------------------------------------------------------------------


def absorb_query(q_nope, q_rope, q_positions, w_uk, theta: float = 10000.0):
    """q_lat[t, h] = W_UK[h]^T q_nope[t, h];  q_rope[t, h] rotated at the query position.

    q_nope: [T, H, d_nope]; q_rope: [T, H, d_rope]; q_positions: [T];
    w_uk: [H, d_nope, d_c] (head h's block of the [n_h*d_nope, d_c] up-projection).
    Returns (q_lat [T, H, d_c], q_rope_rot [T, H, d_rope])."""
    q_nope = np.asarray(q_nope, dtype=np.float64)
    w_uk = np.asarray(w_uk, dtype=np.float64)
    q_lat = np.einsum("thn,hnc->thc", q_nope, w_uk)
    pos = np.asarray(q_positions)[:, None]
    return q_lat, rope_rotate(q_rope, pos, theta)


# --------------------------------------------------------------------------------------
# Paged cache: reading a sequence back through its block table  ([IP] 6.1)
# --------------------------------------------------------------------------------------


def gather_rows(paged, block_table_row, length: int, page_size: int):
    """Rows 0 .. length-1 of one sequence from a paged array [num_pages, page_size, ...]:
    token t lives in page block_table_row[t // page_size], slot t % page_size."""
    paged = np.asarray(paged)
    out = np.empty((length,) + paged.shape[2:], dtype=np.float64)
    for t in range(length):
        out[t] = paged[int(block_table_row[t // page_size]), t % page_size]
    return out


# --------------------------------------------------------------------------------------
# Step a3: attention over the latent cache, absorbed form  ([DSV2] 2.2, 2.3; [IP] 3.3)
# --------------------------------------------------------------------------------------


def key_mask(s_q: int, length: int, causal: bool):
    """Boolean [S_q, L]: query j (at position L - S_q + j) may attend key position p."""
    if not causal:
        return np.ones((s_q, length), dtype=bool)
    qpos = length - s_q + np.arange(s_q)
    return np.arange(length)[None, :] <= qpos[:, None]


def decode_attention(q_lat, q_rope, c, k_rope, scale: float, mask=None):
    """One sequence of MLA decode in the absorbed form.

    s[j, h, t] = (q_lat[j, h] . c[t] + q_rope[j, h] . k_rope[t]) * scale
    p = softmax_t(s) over the attended keys;  o_lat[j, h] = sum_t p[j, h, t] c[t];
    lse[j, h] = log sum_t exp(s[j, h, t]).

    q_lat: [S_q, H, d_c]; q_rope: [S_q, H, d_rope] (already rotated);
    c: [L, d_c]; k_rope: [L, d_rope] (already rotated); mask: [S_q, L] or None.
    Returns (o_lat [S_q, H, d_c], lse [S_q, H]).  A query with no attended key gets
    o_lat = 0 and lse = -inf."""
    q_lat = np.asarray(q_lat, dtype=np.float64)
    q_rope = np.asarray(q_rope, dtype=np.float64)
    c = np.asarray(c, dtype=np.float64)
    k_rope = np.asarray(k_rope, dtype=np.float64)
    s_q, n_heads, d_c = q_lat.shape
    length = c.shape[0]
    o = np.zeros((s_q, n_heads, d_c))
    lse = np.full((s_q, n_heads), -np.inf)
    if mask is None:
        mask = np.ones((s_q, length), dtype=bool)
    for j in range(s_q):
        keys = np.nonzero(mask[j])[0]
        if keys.size == 0:
            continue
        s = (q_lat[j] @ c[keys].T + q_rope[j] @ k_rope[keys].T) * scale  # [H, n_keys]
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        denom = e.sum(axis=1, keepdims=True)
        p = e / denom
        o[j] = p @ c[keys]
        lse[j] = (m + np.log(denom))[:, 0]
    return o, lse


def softmax_probs(q_lat, q_rope, c, k_rope, scale: float):
    """The probabilities p[h, t] of one query token (no mask); exposed for pins."""
    s = (np.asarray(q_lat, np.float64) @ np.asarray(c, np.float64).T
         + np.asarray(q_rope, np.float64) @ np.asarray(k_rope, np.float64).T) * scale
    e = np.exp(s - s.max(axis=-1, keepdims=True))
    return e / e.sum(axis=-1, keepdims=True)


def decode_paged(q_lat, q_rope, latent_rows, block_table, seq_lens, s_q: int, scale: float,
                 d_c: int, page_size: int, causal: bool = False, seqs=None):
    """Decode every sequence (or the listed ``seqs``) of a batch from a paged cache.

    q_lat: [B*S_q, H, d_c]; q_rope: [B*S_q, H, d_rope] (rotated);
    latent_rows: [num_pages, page_size, d_c + d_rope] float (c_KV || k_rope, as stored);
    block_table: [B, max_pages]; seq_lens: [B].
    Returns (o_lat [B*S_q, H, d_c], lse [B*S_q, H]); rows of skipped sequences are NaN."""
    q_lat = np.asarray(q_lat, dtype=np.float64)
    n_tok, n_heads, _ = q_lat.shape
    o = np.full((n_tok, n_heads, d_c), np.nan)
    lse = np.full((n_tok, n_heads), np.nan)
    batch = len(seq_lens)
    for b in (range(batch) if seqs is None else seqs):
        length = int(seq_lens[b])
        rows = gather_rows(latent_rows, block_table[b], length, page_size)
        sl = slice(b * s_q, (b + 1) * s_q)
        o[sl], lse[sl] = decode_attention(q_lat[sl], q_rope[sl], rows[:, :d_c], rows[:, d_c:],
                                          scale, key_mask(s_q, length, causal))
    return o, lse


# --------------------------------------------------------------------------------------
# Step a4: split-KV partials and their log-sum-exp combine (no page gives this step;
# it is the plain reading of splitting the softmax sum over disjoint key chunks)
# --------------------------------------------------------------------------------------


def split_partials(q_lat, q_rope, c, k_rope, scale: float, bounds, mask=None):
    """Partial (o_i, lse_i) of one sequence over key chunks [bounds[i], bounds[i+1]).

    Each partial is decode_attention restricted to its chunk (normalised within the
    chunk).  Returns (o_parts [n, S_q, H, d_c], lse_parts [n, S_q, H])."""
    c = np.asarray(c, dtype=np.float64)
    k_rope = np.asarray(k_rope, dtype=np.float64)
    s_q = np.asarray(q_lat).shape[0]
    if mask is None:
        mask = np.ones((s_q, c.shape[0]), dtype=bool)
    o_parts, lse_parts = [], []
    for lo, hi in zip(bounds[:-1], bounds[1:]):
        o_i, lse_i = decode_attention(q_lat, q_rope, c[lo:hi], k_rope[lo:hi], scale, mask[:, lo:hi])
        o_parts.append(o_i)
        lse_parts.append(lse_i)
    return np.stack(o_parts), np.stack(lse_parts)


def combine_partials(o_parts, lse_parts):
    """lse = log sum_i exp(lse_i);  o = sum_i exp(lse_i - lse) o_i.

    o_parts: [n, ..., d_c]; lse_parts: [n, ...].  All-empty inputs give o = 0, lse = -inf."""
    o_parts = np.asarray(o_parts, dtype=np.float64)
    lse_parts = np.asarray(lse_parts, dtype=np.float64)
    m = lse_parts.max(axis=0)
    finite = np.isfinite(m)
    m_safe = np.where(finite, m, 0.0)
    w = np.exp(lse_parts - m_safe)  # exp(-inf) = 0 for empty chunks
    total = w.sum(axis=0)
    lse = np.where(finite, m_safe + np.log(np.where(finite, total, 1.0)), -np.inf)
    wn = np.where(finite, w / np.where(finite, total, 1.0), 0.0)
    o = (wn[..., None] * o_parts).sum(axis=0)
    return o, lse


# --------------------------------------------------------------------------------------
# Step a5: W_UV applied on the output side  ([DSV2] 2.2)
# --------------------------------------------------------------------------------------


def output_up(o_lat, w_uv):
    """out[t, h] = W_UV[h] o_lat[t, h];  w_uv: [H, d_v, d_c]; o_lat: [T, H, d_c]."""
    return np.einsum("hvc,thc->thv", np.asarray(w_uv, np.float64), np.asarray(o_lat, np.float64))


# --------------------------------------------------------------------------------------
# Brute force, non-absorbed MLA: K and V materialised per head  ([DSV2] 2.1, 2.3; [IP] 3.3)
# --------------------------------------------------------------------------------------


def bruteforce_attention(q_nope, q_rope_rot, c, k_rope, w_uk, w_uv, scale: float, mask=None):
    """Standard multi-head attention with explicit per-head keys and values.

    k[t, h] = [W_UK[h] c_t ; k_rope_t],  v[t, h] = W_UV[h] c_t,  q[j, h] = [q_nope ; q_rope],
    out[j, h] = sum_t softmax_t(q . k * scale) v[t, h].
    q_nope: [S_q, H, d_nope]; q_rope_rot: [S_q, H, d_rope]; c: [L, d_c]; k_rope: [L, d_rope].
    Returns out [S_q, H, d_v]."""
    q_nope = np.asarray(q_nope, np.float64)
    q_rope_rot = np.asarray(q_rope_rot, np.float64)
    c = np.asarray(c, np.float64)
    k_rope = np.asarray(k_rope, np.float64)
    w_uk = np.asarray(w_uk, np.float64)
    w_uv = np.asarray(w_uv, np.float64)
    s_q, n_heads, _ = q_nope.shape
    length = c.shape[0]
    d_v = w_uv.shape[1]
    if mask is None:
        mask = np.ones((s_q, length), dtype=bool)
    out = np.zeros((s_q, n_heads, d_v))
    for h in range(n_heads):
        k_nope = c @ w_uk[h].T                                   # [L, d_nope]
        k_full = np.concatenate([k_nope, k_rope], axis=1)         # [L, d_nope + d_rope]
        v = c @ w_uv[h].T                                        # [L, d_v]
        for j in range(s_q):
            keys = np.nonzero(mask[j])[0]
            if keys.size == 0:
                continue
            q_full = np.concatenate([q_nope[j, h], q_rope_rot[j, h]])
            s = (k_full[keys] @ q_full) * scale
            p = np.exp(s - s.max())
            p /= p.sum()
            out[j, h] = p @ v[keys]
    return out


# --------------------------------------------------------------------------------------
# FP8 E4M3 cache encoding  ([IP] 6.3 FP8 KV cache; [HDU] 5 and Q4 per-block scales)
# --------------------------------------------------------------------------------------

E4M3_MAX = 448.0


def e4m3_decode(codes):
    """Value of each OCP FP8 E4M3 code: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa
    bits; exponent field 0 is subnormal (m/8 * 2^-6); S.1111.111 is NaN; no infinities."""
    codes = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(codes & 0x80, -1.0, 1.0)
    e = (codes >> 3) & 0xF
    m = codes & 0x7
    val = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * 2.0 ** (e - 7.0))
    val = np.where((e == 0xF) & (m == 0x7), np.nan, val)
    return sign * val


_E4M3_POS = e4m3_decode(np.arange(127, dtype=np.uint8))  # codes 0x00..0x7E, increasing


def e4m3_encode(x):
    """Round to the nearest E4M3 value, ties to the even code (even mantissa), saturating
    at +-448; NaN maps to 0x7F.  Plain definition: nearest entry of the value table."""
    x = np.asarray(x, dtype=np.float64)
    mag = np.minimum(np.abs(x), E4M3_MAX)
    hi = np.clip(np.searchsorted(_E4M3_POS, mag, side="left"), 0, 126)
    lo = np.clip(hi - 1, 0, 126)
    d_lo = np.abs(mag - _E4M3_POS[lo])
    d_hi = np.abs(_E4M3_POS[hi] - mag)
    pick_lo = (d_lo < d_hi) | ((d_lo == d_hi) & (lo % 2 == 0))
    code = np.where(pick_lo, lo, hi).astype(np.uint8)
    code = np.where(np.signbit(x) & (code != 0), code | 0x80, code).astype(np.uint8)
    return np.where(np.isnan(x), np.uint8(0x7F), code).astype(np.uint8)


def fp8_quantize_blocks(c, block: int = 128):
    """Per-token, per-block dynamic E4M3 quantisation of c_KV.

    c: [..., d_c] (d_c % block == 0).  For every block: amax = max |x| (in fp32),
    s = fp32(amax / 448) (1 when amax = 0), code = E4M3(fp32(x * fp32(448 / amax))).
    Returns (codes uint8 [..., d_c], scales float32 [..., d_c // block])."""
    c32 = np.asarray(c, dtype=np.float32)
    shp = c32.shape
    assert shp[-1] % block == 0
    blocks = c32.reshape(shp[:-1] + (shp[-1] // block, block))
    amax = np.abs(blocks).max(axis=-1)
    zero = amax == 0
    safe = np.where(zero, np.float32(1.0), amax).astype(np.float32)
    scale = np.where(zero, np.float32(1.0), (safe / np.float32(E4M3_MAX)).astype(np.float32)).astype(np.float32)
    inv = np.where(zero, np.float32(1.0), (np.float32(E4M3_MAX) / safe).astype(np.float32)).astype(np.float32)
    scaled = (blocks * inv[..., None]).astype(np.float32)
    codes = e4m3_encode(scaled.astype(np.float64)).reshape(shp)
    return codes, scale.astype(np.float32)


def fp8_dequantize_blocks(codes, scales, block: int = 128):
    """x = E4M3 value * block scale, in float64."""
    v = e4m3_decode(codes)
    shp = v.shape
    v = v.reshape(shp[:-1] + (shp[-1] // block, block))
    return (v * np.asarray(scales, dtype=np.float64)[..., None]).reshape(shp)


# --------------------------------------------------------------------------------------
# Whole decode step from hidden states (for the small end-to-end cases)
# --------------------------------------------------------------------------------------


def mla_step(h_cache, cache_positions, w_dkv, w_kr, q_nope, q_rope, q_positions, w_uk, w_uv,
             scale: float, causal: bool = False, theta: float = 10000.0):
    """One sequence end to end: build its cache from h, absorb the query, attend, and apply
    W_UV.  Returns (out [S_q, H, d_v], o_lat [S_q, H, d_c], lse [S_q, H])."""
    c, kr = compress_kv(h_cache, w_dkv, w_kr, cache_positions, theta)
    q_lat, q_rot = absorb_query(q_nope, q_rope, q_positions, w_uk, theta)
    s_q = q_lat.shape[0]
    o_lat, lse = decode_attention(q_lat, q_rot, c, kr, scale, key_mask(s_q, c.shape[0], causal))
    return output_up(o_lat, w_uv), o_lat, lse


def default_scale(d_nope: int, d_rope: int) -> float:
    """1/sqrt(d_nope + d_rope): the per-head query/key width of the decoupled split."""
    return 1.0 / math.sqrt(d_nope + d_rope)
