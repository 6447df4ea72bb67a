"""GPU parity of the projection steps and of a whole decode step against the fp64 oracle.

Cache rows written by mla_append_cache are compared after rounding: bf16 rows within
2^-7 relative (one bf16 rounding of an fp32 sum, plus accumulation order) and 1e-3 absolute;
fp32 rows within 1e-5 relative to the row maximum; E4M3 codes within one code step of the
oracle's (the fp32 sums of the two sides may straddle a rounding boundary) and scales within
the fp32 accumulation error of the block maximum (SCALE_RTOL).  absorb/output: max abs error
<= 2e-2 and relative to max <= 1e-2 (bf16),
max relative <= 1e-5 (fp32).
"""
import dataclasses

import numpy as np
import pytest
import torch

from mla_latent_kv_27_b200 import workloads as wl
from oracle import mla_oracle as orc
from tests.parity_helpers import dims_for, max_abs, max_rel, round_to, to_dev

pytestmark = pytest.mark.gpu
W = wl.WORKLOADS


def _rope_tables(lib, w, rows):
    half = w.d_rope // 2
    c = torch.empty((rows, half), dtype=torch.float32, device="cuda")
    s = torch.empty((rows, half), dtype=torch.float32, device="cuda")
    lib.mla_rope_table(w.d_rope, rows, w.theta, c, s)
    return c, s


def test_rope_table_matches_oracle(lib):
    w = W["v3_bf16"]
    c, s = _rope_tables(lib, w, 131072 + 64)
    pos = np.array([0, 1, 63, 4095, 8191, 131071, 131135])
    rc, rs = orc.rope_cos_sin(pos, w.d_rope, w.theta)
    np.testing.assert_allclose(c.cpu().numpy()[pos], rc, rtol=0, atol=2e-7)
    np.testing.assert_allclose(s.cpu().numpy()[pos], rs, rtol=0, atol=2e-7)


def _append_case(lib, w, lengths, shuffle=True):
    """Append every token of the sequences through the GPU; return GPU rows decoded to fp64
    and the oracle's rows, both in sequence order."""
    lengths = np.asarray(lengths, np.int32)
    T = int(lengths.sum())
    w_dkv, w_kr, _, _ = wl.draw_weights(w)
    h = wl.draw_hidden(w, T)
    h64 = round_to(h, w.act_dtype)
    wd64, wk64 = round_to(w_dkv, w.act_dtype), round_to(w_kr, w.act_dtype)
    table, num_pages = wl.make_block_table(lengths, 0, shuffle, wl.rng_for(w, 6))
    seq = np.repeat(np.arange(len(lengths), dtype=np.int32), lengths)
    pos = np.concatenate([np.arange(n, dtype=np.int32) for n in lengths])
    dims = dims_for(lib, w)
    rows = int(table.shape[1] * wl.PAGE_SIZE)
    rc, rs = _rope_tables(lib, w, rows)
    from tests.parity_helpers import DeviceCache
    if w.cache_dtype == "fp8":
        dc = DeviceCache(lib, w, lengths, table, num_pages, codes=np.zeros((T, w.d_c), np.uint8),
                         scales=np.ones((T, w.d_c // 128), np.float32), rope=np.zeros((T, w.d_rope)))
    else:
        dc = DeviceCache(lib, w, lengths, table, num_pages, rows=np.zeros((T, w.row_width)))
    ws_bytes = lib.mla_append_workspace_size(dims, T)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    lib.mla_append_cache(dims, to_dev(h64, w.act_dtype), T, to_dev(seq, "i32"), to_dev(pos, "i32"),
                         to_dev(wd64, w.act_dtype), to_dev(wk64, w.act_dtype), rc, rs, rows, dc.desc,
                         ws, ws_bytes)
    torch.cuda.synchronize()
    assert lib.mla_check_device_error()[0] == 0
    c_ref, kr_ref = orc.compress_kv(h64, wd64, wk64, pos, w.theta)
    ti = torch.as_tensor(table, dtype=torch.long)
    page_of = ti[torch.as_tensor(seq, dtype=torch.long), torch.as_tensor(pos // 64, dtype=torch.long)]
    slot = torch.as_tensor(pos % 64, dtype=torch.long)
    if w.cache_dtype == "fp8":
        codes = dc.rows.cpu()[page_of, slot].numpy()
        scales = dc.scales.cpu()[page_of, slot].numpy()
        rope = dc.rope.cpu()[page_of, slot].double().numpy()
        return dict(codes=codes, scales=scales, rope=rope, c_ref=c_ref, kr_ref=kr_ref)
    g = dc.rows.cpu()[page_of, slot].double().numpy()
    return dict(c=g[:, : w.d_c], kr=g[:, w.d_c:], c_ref=c_ref, kr_ref=kr_ref)


def test_append_fp32(lib):
    w = W["tiny_fp32"]
    r = _append_case(lib, w, [37, 100])
    assert max_rel(r["c"], r["c_ref"]) <= 1e-5
    assert max_rel(r["kr"], r["kr_ref"]) <= 1e-5


@pytest.mark.parametrize("name", ["v2lite_bf16", "v3_bf16"])
def test_append_bf16(lib, name):
    w = W[name]
    r = _append_case(lib, w, [1, 64, 130])
    for g, ref in ((r["c"], r["c_ref"]), (r["kr"], r["kr_ref"])):
        assert (np.abs(g - ref) <= 2 ** -7 * np.abs(ref) + 1e-3).all(), max_abs(g, ref)


# An E4M3 block scale is amax / 448 of fp32 GEMM outputs, so it carries their rounding error:
# a length-d_model fp32 dot product whose partial sums are of the order of |c| is off by about
# 2^-24 * sqrt(d_model) * |c| (about 5e-6 relative to the block maximum at d_model = 7168);
# the tolerance keeps a factor of four over that.
SCALE_RTOL = 4 * 2.0 ** -24 * np.sqrt(7168)


def test_append_fp8(lib):
    w = W["fp8_mtp2"]
    r = _append_case(lib, w, [1, 64, 130])
    codes_ref, scales_ref = orc.fp8_quantize_blocks(r["c_ref"])
    np.testing.assert_allclose(r["scales"], scales_ref, rtol=SCALE_RTOL)
    v_gpu = orc.e4m3_decode(r["codes"])
    v_ref = orc.e4m3_decode(codes_ref)
    # at most one E4M3 step apart (the step at the larger magnitude bounds it)
    step = np.maximum(np.abs(v_ref), 2 ** -6) * 2 ** -3
    assert (np.abs(v_gpu - v_ref) <= step + 1e-12).all()
    assert (r["codes"] == codes_ref).mean() > 0.99
    assert (np.abs(r["rope"] - r["kr_ref"]) <= 2 ** -7 * np.abs(r["kr_ref"]) + 1e-3).all()


# Token counts that reach each launch shape of the fused bf16 append: one 64-token tile with a
# 16-CTA K split (T <= 64), two tiles with 8, four with 4, no split (64-token tiles), and the
# 256-token tile used for bulk appends.
APPEND_SHAPES = [[1], [64], [30, 34, 64], [1, 64, 130], [700, 800, 742], [2000, 2000]]


@pytest.mark.parametrize("lengths", APPEND_SHAPES)
def test_append_bf16_launch_shapes(lib, lengths):
    w = W["v3_bf16"]
    r = _append_case(lib, w, lengths)
    for g, ref in ((r["c"], r["c_ref"]), (r["kr"], r["kr_ref"])):
        assert (np.abs(g - ref) <= 2 ** -7 * np.abs(ref) + 1e-3).all(), max_abs(g, ref)


def test_append_bf16_k_shorter_than_split(lib):
    """d_model = 128 gives two 64-wide K chunks against a 16-CTA split: fourteen CTAs of each
    cluster contribute empty partial sums."""
    w = dataclasses.replace(W["v3_bf16"], d_model=128)
    r = _append_case(lib, w, [3, 61])
    for g, ref in ((r["c"], r["c_ref"]), (r["kr"], r["kr_ref"])):
        assert (np.abs(g - ref) <= 2 ** -7 * np.abs(ref) + 1e-3).all(), max_abs(g, ref)


@pytest.mark.parametrize("lengths", [[64], [2000, 2000]])
def test_append_fp8_launch_shapes(lib, lengths):
    w = W["fp8_mtp2"]
    r = _append_case(lib, w, lengths)
    codes_ref, scales_ref = orc.fp8_quantize_blocks(r["c_ref"])
    np.testing.assert_allclose(r["scales"], scales_ref, rtol=SCALE_RTOL)
    step = np.maximum(np.abs(orc.e4m3_decode(codes_ref)), 2 ** -6) * 2 ** -3
    assert (np.abs(orc.e4m3_decode(r["codes"]) - orc.e4m3_decode(codes_ref)) <= step + 1e-12).all()
    assert (np.abs(r["rope"] - r["kr_ref"]) <= 2 ** -7 * np.abs(r["kr_ref"]) + 1e-3).all()


@pytest.mark.parametrize("kind", ["seq", "pos", "page"])
@pytest.mark.parametrize("T", [5, 300])
def test_append_bad_token_is_reported_and_skipped(lib, kind, T):
    """A token whose sequence, position or page id is out of range is not written and is
    reported in the error word (kinds 4, 2, 1); the other tokens are stored as usual."""
    w = W["v3_bf16"]
    w_dkv, w_kr, _, _ = wl.draw_weights(w)
    h = round_to(wl.draw_hidden(w, T), "bf16")
    wd, wk = round_to(w_dkv, "bf16"), round_to(w_kr, "bf16")
    lengths = np.array([T], np.int32)
    table, num_pages = wl.make_block_table(lengths, 0, False, None)
    seq = np.zeros(T, np.int32)
    pos = np.arange(T, dtype=np.int32)
    rows = int(table.shape[1] * wl.PAGE_SIZE)
    bad = T // 2
    if kind == "seq":
        seq[bad] = 7
    elif kind == "pos":
        pos[bad] = rows + 5
    else:
        table = np.concatenate([table, np.zeros((1, table.shape[1]), np.int32)])
        table[1, 0] = num_pages + 3
        seq[bad], pos[bad] = 1, 0
    dims = dims_for(lib, w)
    rc, rs = _rope_tables(lib, w, rows)
    from tests.parity_helpers import DeviceCache
    dc = DeviceCache(lib, w, [T] + [0] * (len(table) - 1), table, num_pages, rows=np.zeros((T, w.row_width)))
    lib.mla_check_device_error()
    ws_bytes = lib.mla_append_workspace_size(dims, T)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    lib.mla_append_cache(dims, to_dev(h, "bf16"), T, to_dev(seq, "i32"), to_dev(pos, "i32"), to_dev(wd, "bf16"),
                         to_dev(wk, "bf16"), rc, rs, rows, dc.desc, ws, ws_bytes)
    st, detail = lib.mla_check_device_error()
    assert st == 4 and (detail >> 24) == {"seq": 4, "pos": 2, "page": 1}[kind], (st, detail)
    good = np.arange(T) != bad
    c_ref, kr_ref = orc.compress_kv(h[good], wd, wk, pos[good], w.theta)
    g = dc.rows.cpu()[torch.as_tensor(table[0, pos[good] // 64], dtype=torch.long),
                      torch.as_tensor(pos[good] % 64, dtype=torch.long)].double().numpy()
    for x, ref in ((g[:, : w.d_c], c_ref), (g[:, w.d_c:], kr_ref)):
        assert (np.abs(x - ref) <= 2 ** -7 * np.abs(ref) + 1e-3).all(), max_abs(x, ref)


def _absorb_case(lib, w, T):
    _, _, w_uk, _ = wl.draw_weights(w)
    q_nope, q_rope = wl.draw_query_heads(w, T)
    qn, qr, wu = (round_to(x, w.act_dtype) for x in (q_nope, q_rope, w_uk))
    pos = (np.arange(T, dtype=np.int32) * 977) % 9000
    dims = dims_for(lib, w)
    rc, rs = _rope_tables(lib, w, 9000)
    out = torch.empty((T, w.n_heads, w.row_width), dtype=torch.bfloat16 if w.act_dtype == "bf16" else torch.float32,
                      device="cuda")
    lib.mla_absorb_query(dims, to_dev(qn, w.act_dtype), to_dev(qr, w.act_dtype), to_dev(pos, "i32"), T,
                         to_dev(wu, w.act_dtype), rc, rs, 9000, out)
    torch.cuda.synchronize()
    q_lat, q_rot = orc.absorb_query(qn, qr, pos, wu, w.theta)
    g = out.double().cpu().numpy()
    return g[..., : w.d_c], g[..., w.d_c:], q_lat, q_rot


def test_absorb_unaligned_rope_input(lib):
    """q_rope 2 bytes off a 16-byte boundary: the library takes its two-launch absorb path
    (tensor-core GEMM, then the query RoPE) and gives the same result."""
    w = W["v3_bf16"]
    T = 7
    _, _, w_uk, _ = wl.draw_weights(w)
    q_nope, q_rope = wl.draw_query_heads(w, T)
    qn, qr, wu = (round_to(x, "bf16") for x in (q_nope, q_rope, w_uk))
    pos = (np.arange(T, dtype=np.int32) * 977) % 9000
    dims = dims_for(lib, w)
    rc, rs = _rope_tables(lib, w, 9000)
    buf = torch.empty(T * w.n_heads * w.d_rope + 1, dtype=torch.bfloat16, device="cuda")
    qr_dev = buf[1:].view(T, w.n_heads, w.d_rope)
    qr_dev.copy_(to_dev(qr, "bf16"))
    assert qr_dev.data_ptr() % 16 != 0
    out = torch.empty((T, w.n_heads, w.row_width), dtype=torch.bfloat16, device="cuda")
    lib.mla_absorb_query(dims, to_dev(qn, "bf16"), qr_dev, to_dev(pos, "i32"), T, to_dev(wu, "bf16"), rc, rs,
                         9000, out)
    torch.cuda.synchronize()
    q_lat, q_rot = orc.absorb_query(qn, qr, pos, wu, w.theta)
    g = out.double().cpu().numpy()
    for x, r in ((g[..., : w.d_c], q_lat), (g[..., w.d_c:], q_rot)):
        assert max_abs(x, r) <= 2e-2 and max_rel(x, r) <= 1e-2


@pytest.mark.parametrize("aligned", [True, False])
def test_absorb_bad_position_is_reported(lib, aligned):
    """A query position outside the RoPE table is reported (error kind 2) and that token's
    q_rope is passed through unrotated; the other tokens are unaffected.  Both absorb paths
    (one fused launch; GEMM + RoPE kernel when q_rope is not 16-byte aligned)."""
    w = W["v3_bf16"]
    T, rows = 9, 600
    _, _, w_uk, _ = wl.draw_weights(w)
    q_nope, q_rope = wl.draw_query_heads(w, T)
    qn, qr, wu = (round_to(x, "bf16") for x in (q_nope, q_rope, w_uk))
    pos = (np.arange(T, dtype=np.int32) * 61) % rows
    pos[4] = rows + 7
    dims = dims_for(lib, w)
    rc, rs = _rope_tables(lib, w, rows)
    buf = torch.empty(T * w.n_heads * w.d_rope + 8, dtype=torch.bfloat16, device="cuda")
    qr_dev = buf[(0 if aligned else 1):][: T * w.n_heads * w.d_rope].view(T, w.n_heads, w.d_rope)
    qr_dev.copy_(to_dev(qr, "bf16"))
    out = torch.empty((T, w.n_heads, w.row_width), dtype=torch.bfloat16, device="cuda")
    lib.mla_check_device_error()
    lib.mla_absorb_query(dims, to_dev(qn, "bf16"), qr_dev, to_dev(pos, "i32"), T, to_dev(wu, "bf16"), rc, rs,
                         rows, out)
    st, detail = lib.mla_check_device_error()
    assert st == 4 and (detail >> 24) == 2, (st, detail)
    g = out.double().cpu().numpy()
    good = np.arange(T) != 4
    q_lat, q_rot = orc.absorb_query(qn[good], qr[good], pos[good], wu, w.theta)
    assert max_abs(g[good][..., : w.d_c], q_lat) <= 2e-2 and max_abs(g[good][..., w.d_c:], q_rot) <= 2e-2
    assert np.array_equal(g[4][..., w.d_c:], qr[4])  # bf16 values passed through exactly
    q_lat4, _ = orc.absorb_query(qn[4:5], qr[4:5], np.zeros(1, np.int32), wu, w.theta)
    assert max_abs(g[4][..., : w.d_c], q_lat4[0]) <= 2e-2


@pytest.mark.parametrize("name,T", [("tiny_fp32", 2), ("v2lite_bf16", 32), ("v3_bf16", 64), ("fp8_mtp2", 256),
                                    ("v3_bf16", 5), ("v3_bf16", 130)])
def test_absorb(lib, name, T):
    w = W[name]
    g_lat, g_rot, r_lat, r_rot = _absorb_case(lib, w, T)
    if w.act_dtype == "f32":
        assert max_rel(g_lat, r_lat) <= 1e-5 and max_rel(g_rot, r_rot) <= 1e-5
    else:
        for g, r in ((g_lat, r_lat), (g_rot, r_rot)):
            assert max_abs(g, r) <= 2e-2 and max_rel(g, r) <= 1e-2, (max_abs(g, r), max_rel(g, r))


@pytest.mark.parametrize("name,T", [("tiny_fp32", 2), ("v2lite_bf16", 32), ("v3_bf16", 64), ("fp8_mtp2", 256),
                                    ("v3_bf16", 3), ("v3_bf16", 100)])
def test_output_up(lib, name, T):
    w = W[name]
    _, _, _, w_uv = wl.draw_weights(w)
    o = wl.rng_for(w, 9).standard_normal((T, w.n_heads, w.d_c), dtype=np.float32)
    o64, wv = round_to(o, w.act_dtype), round_to(w_uv, w.act_dtype)
    dims = dims_for(lib, w)
    out = torch.empty((T, w.n_heads, w.d_v), dtype=torch.bfloat16 if w.act_dtype == "bf16" else torch.float32,
                      device="cuda")
    lib.mla_output_up(dims, to_dev(o64, w.act_dtype), T, to_dev(wv, w.act_dtype), out)
    torch.cuda.synchronize()
    g = out.double().cpu().numpy()
    r = orc.output_up(o64, wv)
    if w.act_dtype == "f32":
        assert max_rel(g, r) <= 1e-5
    else:
        assert max_abs(g, r) <= 2e-2 and max_rel(g, r) <= 1e-2


# ------------------------------------------------------------------ the whole step

def _step_case(lib, w, lengths, query_after_cache=False):
    """Cache built by mla_append_cache from h (the step's S_q new tokens included, at the
    sequence's last positions), then absorb, decode, output_up.  With query_after_cache the
    single query sits one position past the L cached tokens instead and attends all of them.
    Oracle: mla_step per sequence from the same h."""
    lengths = np.asarray(lengths, np.int32)
    batch, s_q = len(lengths), w.s_q
    T = int(lengths.sum())
    w_dkv, w_kr, w_uk, w_uv = (round_to(x, w.act_dtype) for x in wl.draw_weights(w))
    h = round_to(wl.draw_hidden(w, T), w.act_dtype)
    q_nope, q_rope = (round_to(x, w.act_dtype) for x in wl.draw_query_heads(w, batch * s_q))
    table, num_pages = wl.make_block_table(lengths, 0, w.shuffle_pages, wl.rng_for(w, 6))
    seq = np.repeat(np.arange(batch, dtype=np.int32), lengths)
    pos = np.concatenate([np.arange(n, dtype=np.int32) for n in lengths])
    q_pos = (np.repeat(lengths, s_q) - s_q + np.tile(np.arange(s_q), batch)).astype(np.int32)
    if query_after_cache:
        assert s_q == 1
        q_pos = lengths.copy()
    dims = dims_for(lib, w)
    rows = int(table.shape[1] * wl.PAGE_SIZE) + s_q
    rc, rs = _rope_tables(lib, w, rows)
    from tests.parity_helpers import DeviceCache
    if w.cache_dtype == "fp8":
        dc = DeviceCache(lib, w, lengths, table, num_pages, codes=np.zeros((T, w.d_c), np.uint8),
                         scales=np.ones((T, w.d_c // 128), np.float32), rope=np.zeros((T, w.d_rope)))
    else:
        dc = DeviceCache(lib, w, lengths, table, num_pages, rows=np.zeros((T, w.row_width)))
    act = w.act_dtype
    ws_bytes = lib.mla_append_workspace_size(dims, T)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device="cuda")
    # every token of every sequence goes through the append kernel (the step's new tokens too)
    lib.mla_append_cache(dims, to_dev(h, act), T, to_dev(seq, "i32"), to_dev(pos, "i32"), to_dev(w_dkv, act),
                         to_dev(w_kr, act), rc, rs, rows, dc.desc, ws, ws_bytes)
    tdt = torch.bfloat16 if act == "bf16" else torch.float32
    q_packed = torch.empty((batch * s_q, w.n_heads, w.row_width), dtype=tdt, device="cuda")
    lib.mla_absorb_query(dims, to_dev(q_nope, act), to_dev(q_rope, act), to_dev(q_pos, "i32"), batch * s_q,
                         to_dev(w_uk, act), rc, rs, rows, q_packed)
    dws_bytes = lib.mla_decode_workspace_size(dims, batch, s_q, 0, table.shape[1])
    dws = torch.empty(max(dws_bytes, 1), dtype=torch.uint8, device="cuda")
    o_lat = torch.empty((batch * s_q, w.n_heads, w.d_c), dtype=tdt, device="cuda")
    lse = torch.empty((batch * s_q, w.n_heads), dtype=torch.float32, device="cuda")
    lib.mla_decode_attention(dims, q_packed, dc.desc, to_dev(lengths, "i32"), batch, s_q, int(s_q > 1), 0,
                             dws, dws_bytes, o_lat, lse)
    out = torch.empty((batch * s_q, w.n_heads, w.d_v), dtype=tdt, device="cuda")
    lib.mla_output_up(dims, o_lat, batch * s_q, to_dev(w_uv, act), out)
    torch.cuda.synchronize()
    assert lib.mla_check_device_error()[0] == 0
    out_ref = np.zeros((batch * s_q, w.n_heads, w.d_v))
    out_q = np.zeros_like(out_ref)
    off = 0
    for b, n in enumerate(lengths):
        sl = slice(b * s_q, (b + 1) * s_q)
        out_ref[sl], _, _ = orc.mla_step(h[off:off + n], np.arange(n), w_dkv, w_kr, q_nope[sl], q_rope[sl],
                                         q_pos[sl], w_uk, w_uv, w.scale, causal=s_q > 1, theta=w.theta)
        if w.cache_dtype == "fp8":
            # the same step with the cache as stored: E4M3 latents (oracle's encoder), bf16 k_rope
            c, kr = orc.compress_kv(h[off:off + n], w_dkv, w_kr, np.arange(n), w.theta)
            c = orc.fp8_dequantize_blocks(*orc.fp8_quantize_blocks(c))
            kr = round_to(kr, "bf16")
            q_lat, q_rot = orc.absorb_query(q_nope[sl], q_rope[sl], q_pos[sl], w_uk, w.theta)
            o, _ = orc.decode_attention(q_lat, q_rot, c, kr, w.scale, orc.key_mask(s_q, n, s_q > 1))
            out_q[sl] = orc.output_up(o, w_uv)
        off += n
    g = out.double().cpu().numpy()
    if w.cache_dtype == "fp8":
        return g, out_ref, out_q
    return g, out_ref


def test_step_tiny_fp32(lib):
    # The tiny workload as stated: 2 sequences of 37 and 100 cached tokens at positions
    # 0..L-1, one query per sequence at position L attending all of them.
    w = W["tiny_fp32"]
    g, r = _step_case(lib, w, list(w.lengths), query_after_cache=True)
    assert max_rel(g, r) <= 1e-5, max_rel(g, r)


def test_step_tiny_fp32_query_in_cache(lib):
    w = W["tiny_fp32"]
    g, r = _step_case(lib, w, [1, 64, 65])
    assert max_rel(g, r) <= 1e-5, max_rel(g, r)


@pytest.mark.parametrize("name,lengths", [("v2lite_bf16", [300, 64, 1]), ("v3_bf16", [1, 65, 200])])
def test_step_bf16(lib, name, lengths):
    w = dataclasses.replace(W[name], batch=len(lengths))
    g, r = _step_case(lib, w, lengths)
    assert max_abs(g, r) <= 2e-2, max_abs(g, r)
    assert max_rel(g, r) <= 1e-2, max_rel(g, r)


@pytest.mark.parametrize("lengths", [[2, 3, 150], [512, 700, 1030]])
def test_step_fp8(lib, lengths):
    """Against the oracle fed the cache as stored (E4M3 latents, bf16 k_rope): 2e-2 abs.
    Against the unquantised oracle: 6e-2 abs at the workload's lengths (>= 512)."""
    w = dataclasses.replace(W["fp8_mtp2"], batch=len(lengths))
    g, r, rq = _step_case(lib, w, lengths)
    assert max_abs(g, rq) <= 2e-2, max_abs(g, rq)
    if min(lengths) >= 512:
        assert max_abs(g, r) <= 6e-2, max_abs(g, r)


def test_bad_page_id_is_reported_not_faulted(lib):
    """A page id outside the pool is skipped by the kernel and reported via the error word."""
    from tests.parity_helpers import decode_case
    w = dataclasses.replace(W["v3_bf16"], batch=2, shuffle_pages=False)

    def poison(table, num_pages):
        table[1, 0] = num_pages + 1000
        return table
    for n_split in (1, 0):  # one chunk per row; the balanced persistent partition
        res = decode_case(lib, w, [70, 70], n_split=n_split, check_seqs=[0], poison_table=poison)
        st, detail = res["device_status"]
        assert st == 4 and (detail >> 24) == 1, (n_split, st, detail)
        assert np.isfinite(res["o_gpu"][0]).all()
        assert max_abs(res["o_gpu"][0], res["o_ref"][0]) <= 2e-2


@pytest.mark.parametrize("n_split", [1, 0])
def test_length_beyond_block_table_is_reported_not_faulted(lib, n_split):
    """A sequence length past its block-table row is clamped to the row and reported (error
    kind 2); other sequences are unaffected."""
    from tests.parity_helpers import decode_case
    w = dataclasses.replace(W["v3_bf16"], batch=2, shuffle_pages=False)
    res = decode_case(lib, w, [70, 70], n_split=n_split, check_seqs=[0], device_lengths=[70, 100000])
    st, detail = res["device_status"]
    assert st == 4 and (detail >> 24) == 2, (st, detail)
    assert np.isfinite(res["o_gpu"][0]).all()
    assert max_abs(res["o_gpu"][0], res["o_ref"][0]) <= 2e-2
