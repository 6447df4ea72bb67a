"""Shared glue for the parity tests: seeded numpy inputs -> device tensors -> libmla calls,
and the same inputs -> the fp64 oracle.  Inputs handed to both sides are identical (bf16
rounding is applied once, before either side sees the data)."""
from __future__ import annotations

import math

import numpy as np
import torch

from mla_latent_kv_27_b200 import workloads as wl
from oracle import mla_oracle as orc


def round_to(x: np.ndarray, dtype: str) -> np.ndarray:
    """Round to the act/cache dtype once; returns float64 for the oracle."""
    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def to_dev(x: np.ndarray, dtype: str):
    t = torch.from_numpy(np.ascontiguousarray(x))
    tdt = {"bf16": torch.bfloat16, "f32": torch.float32, "i32": torch.int32, "u8": torch.uint8}[dtype]
    return t.to(tdt).cuda().contiguous()


def dims_for(lib, w: wl.Workload):
    cache = {"f32": lib.MLA_F32, "bf16": lib.MLA_BF16, "fp8": lib.MLA_FP8_E4M3}[w.cache_dtype]
    act = {"f32": lib.MLA_F32, "bf16": lib.MLA_BF16}[w.act_dtype]
    return lib.mla_dims(w.d_model, w.d_c, w.d_rope, w.d_nope, w.d_v, w.n_heads, wl.PAGE_SIZE, act,
                        cache, w.scale)


class DeviceCache:
    """A paged cache on the device built from per-sequence rows (fp64 values already rounded
    to the cache dtype, or, for fp8, E4M3 codes + scales + bf16 rope rows)."""

    def __init__(self, lib, w, lengths, table, num_pages, rows=None, codes=None, scales=None, rope=None,
                 device_table=None):
        if w.cache_dtype == "fp8":
            pc = wl.scatter_rows_to_pages(codes, lengths, table, num_pages, fill=0).astype(np.uint8)
            ps = wl.scatter_rows_to_pages(scales, lengths, table, num_pages, fill=1.0).astype(np.float32)
            pr = wl.scatter_rows_to_pages(rope, lengths, table, num_pages, fill=0.0)
            self.rows, self.scales, self.rope = to_dev(pc, "u8"), to_dev(ps, "f32"), to_dev(pr, "bf16")
            ptrs = (self.rows.data_ptr(), self.scales.data_ptr(), self.rope.data_ptr())
        else:
            pr = wl.scatter_rows_to_pages(rows, lengths, table, num_pages, fill=0.0)
            self.rows = to_dev(pr, w.cache_dtype)
            self.scales = self.rope = None
            ptrs = (self.rows.data_ptr(), None, None)
        self.table = to_dev(table if device_table is None else device_table, "i32")
        self.desc = lib.mla_cache(ptrs[0], ptrs[1], ptrs[2], self.table.data_ptr(), table.shape[1],
                                  num_pages, table.shape[0])


def decode_case(lib, w: wl.Workload, lengths, n_split=0, check_seqs=None, stream_seed=5,
                table_extra=0, poison_table=None, device_lengths=None, q_scale=1.0):
    """Run GPU decode and the oracle on the same seeded inputs.

    q_scale multiplies the drawn query (before the one rounding to the act dtype): the scaled
    logits of the standard draw are about N(0, 1), so q_scale = k spreads them to about N(0, k^2)
    and sharpens the softmax.

    Returns dict with gpu/oracle o_lat and lse (oracle rows for unchecked sequences are NaN),
    plus the oracle result against the unquantised latents for the fp8 cache."""
    lengths = np.asarray(lengths, dtype=np.int32)
    batch = len(lengths)
    rows, q = wl.draw_decode_inputs(w, lengths, stream=stream_seed)
    if q_scale != 1.0:
        q = q * np.float32(q_scale)
    table, num_pages = wl.make_block_table(lengths, table_extra, w.shuffle_pages, wl.rng_for(w, 6))
    dev_table = None if poison_table is None else poison_table(table.copy(), num_pages)
    q64 = round_to(q, w.act_dtype)
    res = {}
    if w.cache_dtype == "fp8":
        codes, scales = orc.fp8_quantize_blocks(rows[:, : w.d_c])
        rope64 = round_to(rows[:, w.d_c:], "bf16")
        dc = DeviceCache(lib, w, lengths, table, num_pages, codes=codes, scales=scales, rope=rope64,
                         device_table=dev_table)
        rows_dec = np.concatenate([fp16_operands(codes, scales), rope64], axis=1)
        rows_raw = np.concatenate([rows[:, : w.d_c].astype(np.float64), rope64], axis=1)
    else:
        rows64 = round_to(rows, w.cache_dtype)
        dc = DeviceCache(lib, w, lengths, table, num_pages, rows=rows64, device_table=dev_table)
        rows_dec = rows64
        rows_raw = None
    q_dev = to_dev(q64, w.act_dtype)
    lens_dev = to_dev(lengths if device_lengths is None else np.asarray(device_lengths, np.int32), "i32")
    dims = dims_for(lib, w)
    ws_bytes = lib.mla_decode_workspace_size(dims, batch, w.s_q, n_split, table.shape[1])
    ws = torch.empty(max(1, ws_bytes), dtype=torch.uint8, device="cuda")
    act = torch.bfloat16 if w.act_dtype == "bf16" else torch.float32
    o_dev = torch.full((batch * w.s_q, w.n_heads, w.d_c), float("nan"), dtype=act, device="cuda")
    lse_dev = torch.full((batch * w.s_q, w.n_heads), float("nan"), dtype=torch.float32, device="cuda")
    causal = int(w.causal)
    lib.mla_decode_attention(dims, q_dev, dc.desc, lens_dev, batch, w.s_q, causal, n_split, ws,
                             ws_bytes, o_dev, lse_dev)
    torch.cuda.synchronize()
    st, detail = lib.mla_check_device_error()
    res["device_status"] = (st, detail)
    res["o_gpu"] = o_dev.double().cpu().numpy()
    res["lse_gpu"] = lse_dev.double().cpu().numpy()
    pages_dec = wl.scatter_rows_to_pages(rows_dec, lengths, table, num_pages)
    res["o_ref"], res["lse_ref"] = orc.decode_paged(q64[..., : w.d_c], q64[..., w.d_c:], pages_dec, table,
                                                    lengths, w.s_q, w.scale, w.d_c, wl.PAGE_SIZE,
                                                    bool(causal), seqs=check_seqs)
    if rows_raw is not None:
        pages_raw = wl.scatter_rows_to_pages(rows_raw, lengths, table, num_pages)
        res["o_raw"], res["lse_raw"] = orc.decode_paged(q64[..., : w.d_c], q64[..., w.d_c:], pages_raw,
                                                        table, lengths, w.s_q, w.scale, w.d_c,
                                                        wl.PAGE_SIZE, bool(causal), seqs=check_seqs)
    res["abs_score"] = abs_score_max(q64, rows_dec, lengths, w, check_seqs)
    res["rows_for"] = (batch, w.s_q)
    res["min_len"] = lambda seqs: int(min(lengths[list(range(batch)) if seqs is None else list(seqs)]))
    return res


def fp16_operands(codes, scales, block: int = 128):
    """The FP8 cache as the FP8 path's fp16 tensor-core operands hold it: each E4M3 value (exact in
    fp32) times its fp32 block scale, the product rounded to fp32 and then once to fp16 (round to
    nearest even at each step, numpy's rounding as well as the device's).  Returned in float64.
    Compared with the exactly decoded cache this moves a value by at most 2^-11 of itself; the
    tests feed the oracle these values so that a sharp softmax, whose winner can hinge on that
    difference, is judged on the kernel's own operands.  The unquantised comparison (6e-2) and the
    E4M3 encoding are unchanged."""
    v = orc.e4m3_decode(codes).astype(np.float32)
    shp = v.shape
    v = v.reshape(shp[:-1] + (shp[-1] // block, block))
    prod = (v * np.asarray(scales, dtype=np.float32)[..., None]).astype(np.float32)
    return prod.astype(np.float16).astype(np.float64).reshape(shp)


def checked_rows(res, seqs):
    batch, s_q = res["rows_for"]
    seqs = range(batch) if seqs is None else seqs
    return np.concatenate([np.arange(b * s_q, (b + 1) * s_q) for b in seqs]) if len(list(seqs)) else np.zeros(0, int)


def abs_score_max(q, rows, lengths, w, seqs=None):
    """Per query row and head, max over the sequence's tokens of sum_i |q_i| |k_i| (latent and
    rope dims): a bound on |S_0|, |S_1| and |S| for any split of the dims.  NaN for rows of
    unchecked sequences; 0 for empty sequences."""
    out = np.full((len(lengths) * w.s_q, w.n_heads), np.nan)
    off = np.concatenate([[0], np.cumsum(lengths)])
    for b in range(len(lengths)) if seqs is None else seqs:
        k = np.abs(rows[off[b]:off[b + 1]])
        for j in range(w.s_q):
            r = b * w.s_q + j
            out[r] = (np.abs(q[r]) @ k.T).max(axis=1) if len(k) else 0.0
    return out


def lse_bound(res, rows, scale):
    """Tolerance on lse (bf16 and fp8 workloads), per row.  The workloads fix fp32 accumulation:
    a score is an fp32 sum of 576 products of 16-bit inputs, whose rounding error is a small
    multiple of 2^-24 * A with A = sum_i |q_i k_i| (here bounded by 1e-5 * A, about 170 units
    of 2^-24), and the lse, a smooth maximum of the scores, moves by no more than its largest
    score does.  2e-3 covers the rest (ex2.approx, the fp32 log and the row sum)."""
    return 1e-5 * scale * res["abs_score"][rows] + 2e-3


def max_rel_elementwise(g, r, floor=0.25):
    """max |g - r| / |r| over the entries with |r| >= floor (0 when there are none)."""
    g = np.asarray(g)
    r = np.asarray(r)
    sel = np.abs(r) >= floor
    if not sel.any():
        return 0.0
    return float((np.abs(g[sel] - r[sel]) / np.abs(r[sel])).max())


def max_abs(a, b):
    d = np.abs(np.asarray(a) - np.asarray(b))
    return float(d.max()) if d.size else 0.0


def max_rel(a, b):
    """max |a - b| / max |b| over the tensor (the fp32 workload's error measure)."""
    den = float(np.abs(b).max()) if np.size(b) else 0.0
    return max_abs(a, b) / den if den > 0 else max_abs(a, b)


def lse_close(g, r, atol):
    """|g - r| <= atol where the oracle's lse is finite (atol a scalar or an array shaped like
    r); -inf exactly where the oracle's is."""
    g = np.asarray(g)
    r = np.asarray(r)
    both_inf = np.isneginf(g) & np.isneginf(r)
    fin = np.isfinite(r)
    assert (both_inf | fin).all(), "oracle lse must be finite or -inf"
    assert (np.isneginf(g) == np.isneginf(r)).all(), "empty rows must give lse = -inf"
    tol = np.broadcast_to(np.asarray(atol, dtype=np.float64), r.shape)
    return bool((np.abs(g[fin] - r[fin]) <= tol[fin]).all())


def default_scale(w):
    return 1.0 / math.sqrt(w.d_nope + w.d_rope)
