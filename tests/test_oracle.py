"""Pins for the fp64 oracle against what the pages and the mathematics fix (CPU only).

Each test is chosen so a plausible slip in the oracle (a dropped term, a wrong sign or
index, a transposed operand, a wrong tie rule) fails at least one of them.
"""
import math

import numpy as np
import pytest

from oracle import mla_oracle as orc
from tests.golden import load_kv, load_rows

RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------- cache size (pages' numbers)

def test_cache_size_worked_example_ds25():
    g = load_kv("cache_size_examples.txt")
    mha = orc.mha_values_per_token(int(g["ds25_n_heads"]), int(g["ds25_head_dim"]))
    mla = orc.mla_values_per_token(int(g["ds25_latent_rank"]), int(g["ds25_rope_dim"]))
    assert mha == g["ds25_mha_values"]
    assert mla == g["ds25_mla_values"]
    assert round(mha / mla, 1) == g["ds25_ratio"]


def test_mha_cache_bytes_example_shq():
    g = load_kv("cache_size_examples.txt")
    per_tok = orc.mha_values_per_token(int(g["shq_n_heads"]), int(g["shq_head_dim"])) * g["shq_bytes_per_value"]
    # "2 x 5120 float16 values, about 20 KB": 20480 B is exactly 20 KiB.
    assert per_tok == 2 * 5120 * 2
    assert per_tok / 1024 == g["shq_kb_per_token"]
    per_req = per_tok * g["shq_tokens"]
    assert abs(per_req / 1e6 - g["shq_mb_per_request"]) / g["shq_mb_per_request"] < 0.05
    assert abs(per_req * g["shq_batch"] / 1e9 - g["shq_gb_per_batch"]) / g["shq_gb_per_batch"] < 0.05


def test_cache_ratio_for_the_decode_shapes():
    # 576 values/token against 2*n_h*d_h for the V3-shaped (128 heads) and V2-Lite-shaped
    # (16 heads) workloads, head_dim 128.
    assert orc.mla_values_per_token(512, 64) == 576
    assert orc.mha_values_per_token(128, 128) / 576 == pytest.approx(56.888, abs=1e-3)
    assert orc.mha_values_per_token(16, 128) / 576 == pytest.approx(7.111, abs=1e-3)


# ---------------------------------------------------------------- RoPE

def test_rope_identity_at_position_zero():
    x = RNG.standard_normal((5, 16))
    np.testing.assert_array_equal(orc.rope_rotate(x, np.zeros(5)), x)


def test_rope_matches_complex_multiplication():
    # Independent formulation: pair (x0, x1) as the complex number x0 + i x1 times
    # exp(i * pos * theta^(-2k/d)).
    d = 16
    x = RNG.standard_normal((7, d))
    pos = np.array([0, 1, 2, 17, 511, 4095, 131071])
    z = x[:, 0::2] + 1j * x[:, 1::2]
    k = np.arange(d // 2)
    rot = np.exp(1j * pos[:, None] * (10000.0 ** (-2.0 * k / d))[None, :])
    w = z * rot
    y = orc.rope_rotate(x, pos)
    np.testing.assert_allclose(y[:, 0::2], w.real, rtol=0, atol=1e-12)
    np.testing.assert_allclose(y[:, 1::2], w.imag, rtol=0, atol=1e-12)


def test_rope_spot_value():
    # d_rope = 4, theta = 10000: the second pair turns at 10000^(-1/2) = 0.01 rad per
    # position, so at position 100 it has turned exactly 1 rad; the first pair 100 rad.
    x = np.array([[1.0, 0.0, 1.0, 0.0]])
    y = orc.rope_rotate(x, np.array([100]))
    np.testing.assert_allclose(y[0], [math.cos(100.0), math.sin(100.0), math.cos(1.0), math.sin(1.0)],
                               atol=1e-12)


def test_rope_norm_and_relative_position():
    d = 64
    x = RNG.standard_normal(d)
    y = RNG.standard_normal(d)
    for m, n in [(5, 2), (1000, 997), (70000, 69997)]:
        rx = orc.rope_rotate(x[None], np.array([m]))[0]
        ry = orc.rope_rotate(y[None], np.array([n]))[0]
        assert np.linalg.norm(rx) == pytest.approx(np.linalg.norm(x), rel=1e-12)
        # <R_m x, R_n y> depends only on m - n (= 3 in every case).
        ref = np.dot(orc.rope_rotate(x[None], np.array([3]))[0], y)
        assert np.dot(rx, ry) == pytest.approx(ref, rel=1e-9, abs=1e-9)


# ---------------------------------------------------------------- projections

def test_compress_selects_columns():
    d_model, d_c, d_r, T = 12, 6, 4, 3
    h = RNG.standard_normal((T, d_model))
    sel_c = [3, 0, 11, 5, 7, 2]
    sel_r = [1, 4, 9, 10]
    w_dkv = np.zeros((d_c, d_model))
    w_dkv[np.arange(d_c), sel_c] = 1.0
    w_kr = np.zeros((d_r, d_model))
    w_kr[np.arange(d_r), sel_r] = 1.0
    c, kr = orc.compress_kv(h, w_dkv, w_kr, np.zeros(T, dtype=int))
    np.testing.assert_array_equal(c, h[:, sel_c])
    np.testing.assert_array_equal(kr, h[:, sel_r])
    # A nonzero position rotates only the RoPE part.
    c2, kr2 = orc.compress_kv(h, w_dkv, w_kr, np.array([0, 1, 2]))
    np.testing.assert_array_equal(c2, c)
    np.testing.assert_allclose(kr2, orc.rope_rotate(h[:, sel_r], np.array([0, 1, 2])), atol=0)


def test_absorb_unit_weight_transposes():
    T, H, d_n, d_c, d_r = 2, 3, 4, 6, 2
    q_nope = RNG.standard_normal((T, H, d_n))
    q_rope = RNG.standard_normal((T, H, d_r))
    w_uk = np.zeros((H, d_n, d_c))
    w_uk[1, 2, 5] = 1.0  # head 1: q_lat[5] = q_nope[2]
    q_lat, q_rot = orc.absorb_query(q_nope, q_rope, np.array([0, 9]), w_uk)
    expect = np.zeros((T, H, d_c))
    expect[:, 1, 5] = q_nope[:, 1, 2]
    np.testing.assert_array_equal(q_lat, expect)
    np.testing.assert_array_equal(q_rot[0], q_rope[0])          # position 0: unrotated
    np.testing.assert_allclose(q_rot[1], orc.rope_rotate(q_rope[1], np.full(H, 9)), atol=0)


def test_output_up_unit_weight():
    T, H, d_v, d_c = 2, 2, 3, 5
    o = RNG.standard_normal((T, H, d_c))
    w_uv = np.zeros((H, d_v, d_c))
    w_uv[0, 2, 4] = 1.0  # head 0: out[2] = o_lat[4]
    out = orc.output_up(o, w_uv)
    expect = np.zeros((T, H, d_v))
    expect[:, 0, 2] = o[:, 0, 4]
    np.testing.assert_array_equal(out, expect)


# ---------------------------------------------------------------- attention core

def _tiny(s_q=1, L=7, H=3, d_c=8, d_r=4, d_n=4, d_v=5, seed=0):
    r = np.random.default_rng(seed)
    return dict(
        q_nope=r.standard_normal((s_q, H, d_n)), q_rope=r.standard_normal((s_q, H, d_r)),
        c=r.standard_normal((L, d_c)), k_rope=r.standard_normal((L, d_r)),
        w_uk=r.standard_normal((H, d_n, d_c)) / math.sqrt(d_c),
        w_uv=r.standard_normal((H, d_v, d_c)) / math.sqrt(d_c), scale=1.0 / math.sqrt(d_n + d_r))


@pytest.mark.parametrize("s_q,causal,L", [(1, False, 7), (2, True, 7), (2, False, 5), (3, True, 3)])
def test_absorption_identity_matches_bruteforce(s_q, causal, L):
    t = _tiny(s_q=s_q, L=L, seed=s_q * 10 + L)
    pos = np.arange(s_q) + L - s_q
    q_lat, q_rot = orc.absorb_query(t["q_nope"], t["q_rope"], pos, t["w_uk"])
    mask = orc.key_mask(s_q, L, causal)
    o_lat, _ = orc.decode_attention(q_lat, q_rot, t["c"], t["k_rope"], t["scale"], mask)
    out_absorbed = orc.output_up(o_lat, t["w_uv"])
    out_brute = orc.bruteforce_attention(t["q_nope"], q_rot, t["c"], t["k_rope"], t["w_uk"], t["w_uv"],
                                         t["scale"], mask)
    err = np.abs(out_absorbed - out_brute).max() / np.abs(out_brute).max()
    assert err < 1e-12


def test_softmax_rows_sum_to_one_and_lse_consistent():
    t = _tiny(L=50, H=4)
    q_lat = RNG.standard_normal((1, 4, 8)) * 3
    q_r = RNG.standard_normal((1, 4, 4))
    p = orc.softmax_probs(q_lat[0], q_r[0], t["c"], t["k_rope"], t["scale"])
    assert (p >= 0).all()
    np.testing.assert_allclose(p.sum(axis=1), 1.0, rtol=0, atol=1e-15)
    o, lse = orc.decode_attention(q_lat, q_r, t["c"], t["k_rope"], t["scale"])
    np.testing.assert_allclose(o[0], p @ t["c"], rtol=1e-13, atol=1e-14)
    s = (q_lat[0] @ t["c"].T + q_r[0] @ t["k_rope"].T) * t["scale"]
    np.testing.assert_allclose(np.exp(s - lse[0][:, None]).sum(axis=1), 1.0, atol=1e-13)


def test_constant_cache_reproduces_latent():
    L, H, d_c, d_r = 33, 5, 16, 4
    c0 = RNG.standard_normal(d_c)
    c = np.tile(c0, (L, 1))
    k_rope = RNG.standard_normal((L, d_r)) * 5   # scores differ per token, the value does not
    q_lat = RNG.standard_normal((1, H, d_c)) * 4
    q_r = RNG.standard_normal((1, H, d_r))
    o, _ = orc.decode_attention(q_lat, q_r, c, k_rope, 0.3)
    np.testing.assert_allclose(o[0], np.tile(c0, (H, 1)), rtol=1e-14, atol=1e-14)


def test_single_token_returns_its_latent():
    c = RNG.standard_normal((1, 8))
    kr = RNG.standard_normal((1, 4))
    q_lat = RNG.standard_normal((1, 2, 8))
    q_r = RNG.standard_normal((1, 2, 4))
    o, lse = orc.decode_attention(q_lat, q_r, c, kr, 0.5)
    np.testing.assert_array_equal(o[0], np.tile(c[0], (2, 1)))
    np.testing.assert_allclose(lse[0], (q_lat[0] @ c[0] + q_r[0] @ kr[0]) * 0.5, rtol=1e-15)


def test_two_token_hand_derived_golden():
    g = load_kv("softmax_two_token.txt")
    q_lat = np.array([[[2 * math.log(3.0), 0.0]]])
    q_r = np.zeros((1, 1, 2))
    c = np.array([[0.0, 0.0], [1.0, 4.0]])
    kr = np.zeros((2, 2))
    o, lse = orc.decode_attention(q_lat, q_r, c, kr, 0.5)
    p = orc.softmax_probs(q_lat[0], q_r[0], c, kr, 0.5)
    np.testing.assert_allclose(p[0], [g["p0"], g["p1"]], rtol=1e-14)
    np.testing.assert_allclose(o[0, 0], [g["o_lat_0"], g["o_lat_1"]], rtol=1e-14)
    assert lse[0, 0] == pytest.approx(g["lse"], rel=1e-14)


def test_zero_query_is_the_mean_and_lse_is_log_length():
    L = 40
    c = RNG.standard_normal((L, 8))
    kr = RNG.standard_normal((L, 4))
    o, lse = orc.decode_attention(np.zeros((1, 3, 8)), np.zeros((1, 3, 4)), c, kr, 0.7)
    np.testing.assert_allclose(o[0], np.tile(c.mean(axis=0), (3, 1)), rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lse[0], math.log(L), rtol=1e-15)


def test_rope_part_of_score_is_used():
    # Two tokens with equal latents differ only in k_rope: the score difference must be
    # exactly (q_rope . (kr_1 - kr_0)) * scale.
    c = np.ones((2, 4))
    kr = np.array([[0.0, 0.0], [1.0, 2.0]])
    q_r = np.array([[[0.5, 0.25]]])
    p = orc.softmax_probs(np.zeros((1, 4)), q_r[0], c, kr, 2.0)
    assert math.log(p[0, 1] / p[0, 0]) == pytest.approx((0.5 + 0.5) * 2.0, rel=1e-14)


def test_causal_mask_mtp_positions():
    t = _tiny(s_q=2, L=9, H=2)
    q_lat = RNG.standard_normal((2, 2, 8))
    q_r = RNG.standard_normal((2, 2, 4))
    mask = orc.key_mask(2, 9, True)
    assert mask[0].sum() == 8 and mask[1].sum() == 9
    o, lse = orc.decode_attention(q_lat, q_r, t["c"], t["k_rope"], t["scale"], mask)
    o0, lse0 = orc.decode_attention(q_lat[:1], q_r[:1], t["c"][:8], t["k_rope"][:8], t["scale"])
    np.testing.assert_allclose(o[0], o0[0], rtol=1e-13)
    o1, _ = orc.decode_attention(q_lat[1:], q_r[1:], t["c"], t["k_rope"], t["scale"])
    np.testing.assert_allclose(o[1], o1[0], rtol=1e-13)


def test_empty_sequence_defined_output():
    o, lse = orc.decode_attention(np.ones((1, 2, 4)), np.ones((1, 2, 2)), np.zeros((0, 4)),
                                  np.zeros((0, 2)), 1.0)
    assert (o == 0).all() and np.isneginf(lse).all()


# ---------------------------------------------------------------- split-KV combine

@pytest.mark.parametrize("bounds", [[0, 50], [0, 10, 50], [0, 17, 17, 33, 50], [0, 1, 2, 3, 50], [0, 0, 50, 50]])
def test_split_invariance(bounds):
    L = 50
    c = RNG.standard_normal((L, 8))
    kr = RNG.standard_normal((L, 4))
    q_lat = RNG.standard_normal((2, 3, 8)) * 2
    q_r = RNG.standard_normal((2, 3, 4))
    mask = orc.key_mask(2, L, True)
    o_ref, lse_ref = orc.decode_attention(q_lat, q_r, c, kr, 0.4, mask)
    o_p, lse_p = orc.split_partials(q_lat, q_r, c, kr, 0.4, bounds, mask)
    o, lse = orc.combine_partials(o_p, lse_p)
    np.testing.assert_allclose(o, o_ref, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, lse_ref, rtol=1e-13)


def test_combine_all_empty():
    o, lse = orc.combine_partials(np.ones((3, 2, 4)), np.full((3, 2), -np.inf))
    assert (o == 0).all() and np.isneginf(lse).all()


# ---------------------------------------------------------------- paged storage

def test_gather_rows_follows_block_table():
    pages = np.arange(4 * 64 * 2, dtype=np.float64).reshape(4, 64, 2)
    rows = orc.gather_rows(pages, [2, 0, 3], 130, 64)
    np.testing.assert_array_equal(rows[0], pages[2, 0])
    np.testing.assert_array_equal(rows[63], pages[2, 63])
    np.testing.assert_array_equal(rows[64], pages[0, 0])
    np.testing.assert_array_equal(rows[129], pages[3, 1])


def test_block_table_permutation_invariance():
    from mla_latent_kv_27_b200 import workloads as wl
    lengths = np.array([70, 5, 128])
    rows = RNG.standard_normal((lengths.sum(), 12))
    q = RNG.standard_normal((3, 2, 12))
    res = []
    for shuffle in (False, True):
        table, n_pages = wl.make_block_table(lengths, 0, shuffle, np.random.default_rng(7))
        pages = wl.scatter_rows_to_pages(rows, lengths, table, n_pages)
        res.append(orc.decode_paged(q[..., :8], q[..., 8:], pages, table, lengths, 1, 0.5, 8, 64))
    np.testing.assert_array_equal(res[0][0], res[1][0])
    np.testing.assert_array_equal(res[0][1], res[1][1])


@pytest.mark.parametrize("causal", [True, False])
def test_decode_paged_two_query_rows_match_one_query_decodes(causal):
    # S_q = 2 (the MTP layout): row b*S_q + j of decode_paged must be a one-query decode of
    # sequence b's own rows, truncated to the positions query j may see (L - S_q + j + 1 of them
    # with the causal mask, all L without), computed here without decode_paged's row layout,
    # its block-table gather or key_mask.  A row with nothing to attend is o = 0, lse = -inf.
    from mla_latent_kv_27_b200 import workloads as wl
    s_q, H, d_c, d_r, page = 2, 3, 8, 4, 4
    lengths = np.array([1, 2, 5, 9, 0])
    per_seq = [RNG.standard_normal((L, d_c + d_r)) for L in lengths]
    rows = np.concatenate([r for r in per_seq if len(r)], axis=0)
    q = RNG.standard_normal((len(lengths) * s_q, H, d_c + d_r))
    table, n_pages = wl.make_block_table(lengths, 0, True, np.random.default_rng(3), page_size=page)
    pages = wl.scatter_rows_to_pages(rows, lengths, table, n_pages, page_size=page)
    o, lse = orc.decode_paged(q[..., :d_c], q[..., d_c:], pages, table, lengths, s_q, 0.3, d_c, page,
                              causal=causal)
    for b, L in enumerate(lengths):
        for j in range(s_q):
            r = b * s_q + j
            n = max(0, L - s_q + j + 1) if causal else L
            if n == 0:
                assert (o[r] == 0).all() and np.isneginf(lse[r]).all()
                continue
            seen = per_seq[b][:n]
            o1, lse1 = orc.decode_attention(q[r:r + 1, :, :d_c], q[r:r + 1, :, d_c:], seen[:, :d_c],
                                            seen[:, d_c:], 0.3)
            np.testing.assert_allclose(o[r], o1[0], rtol=0, atol=1e-12)
            np.testing.assert_allclose(lse[r], lse1[0], rtol=0, atol=1e-12)


# ---------------------------------------------------------------- FP8 E4M3

def test_e4m3_golden_codes():
    for row in load_rows("e4m3_codes.txt"):
        if row[0] == "decode":
            code, val = int(row[1], 16), float(row[2])
            assert orc.e4m3_decode(np.uint8(code)) == val, row
        else:
            val, code = float(row[1]), int(row[2], 16)
            assert int(orc.e4m3_encode(val)) == code, row
    assert np.isnan(orc.e4m3_decode(np.uint8(0x7F)))
    assert np.isnan(orc.e4m3_decode(np.uint8(0xFF)))
    assert int(orc.e4m3_encode(np.nan)) == 0x7F


def test_e4m3_roundtrip_all_finite_codes():
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF, 0x80)], dtype=np.uint8)
    np.testing.assert_array_equal(orc.e4m3_encode(orc.e4m3_decode(codes)), codes)


def test_e4m3_encode_against_arithmetic_rounding():
    # Independent formulation: quantum 2^(e-3) in binade e (2^-9 below 2^-6), numpy's
    # round-half-to-even on the quotient, then saturate at 448.
    x = np.concatenate([RNG.uniform(-500, 500, 20000), RNG.uniform(-0.05, 0.05, 20000),
                        RNG.uniform(-2 ** -5, 2 ** -5, 5000)])
    mag = np.abs(x)
    e = np.floor(np.log2(np.maximum(mag, 2 ** -6)))
    quantum = 2.0 ** (e - 3)
    q = np.minimum(np.round(mag / quantum) * quantum, 448.0)
    np.testing.assert_array_equal(np.abs(orc.e4m3_decode(orc.e4m3_encode(x))), q)
    nz = q != 0
    assert (np.sign(orc.e4m3_decode(orc.e4m3_encode(x)))[nz] == np.sign(x)[nz]).all()


def test_fp8_block_quantisation_properties():
    c = RNG.standard_normal((6, 512)) * np.array([1e-3, 1, 10, 100])[np.arange(512) // 128]
    c[5, 128:256] = 0.0
    codes, scales = orc.fp8_quantize_blocks(c)
    assert codes.dtype == np.uint8 and scales.shape == (6, 4)
    blocks = np.abs(c.astype(np.float32)).reshape(6, 4, 128)
    # The largest magnitude of each nonzero block encodes to +-448 exactly.
    amax_idx = blocks.argmax(axis=-1)
    for t in range(6):
        for k in range(4):
            code = codes[t, k * 128 + amax_idx[t, k]] & 0x7F
            assert code == (0x7E if blocks[t, k].max() > 0 else 0)
    assert scales[5, 1] == 1.0 and (codes[5, 128:256] == 0).all()
    x_hat = orc.fp8_dequantize_blocks(codes, scales)
    # Relative step of E4M3 is 2^-3 in the normal range, so the error is at most 2^-4 of
    # the value, plus half a subnormal quantum times the scale near zero.
    bound = np.abs(c) * 2 ** -4 + np.repeat(scales, 128, axis=1) * 2 ** -10 * 1.0001
    assert (np.abs(x_hat - c) <= bound + 1e-6 * np.abs(c)).all()


# ---------------------------------------------------------------- whole step

def test_step_from_hidden_matches_bruteforce():
    r = np.random.default_rng(5)
    d_model, d_c, d_r, d_n, d_v, H, L = 16, 8, 4, 4, 5, 3, 11
    h = r.standard_normal((L, d_model))
    w_dkv = r.standard_normal((d_c, d_model)) / 4
    w_kr = r.standard_normal((d_r, d_model)) / 4
    w_uk = r.standard_normal((H, d_n, d_c)) / math.sqrt(d_c)
    w_uv = r.standard_normal((H, d_v, d_c)) / math.sqrt(d_c)
    q_nope = r.standard_normal((1, H, d_n))
    q_rope = r.standard_normal((1, H, d_r))
    scale = orc.default_scale(d_n, d_r)
    out, _, _ = orc.mla_step(h, np.arange(L), w_dkv, w_kr, q_nope, q_rope, np.array([L]), w_uk, w_uv, scale)
    c, kr = orc.compress_kv(h, w_dkv, w_kr, np.arange(L))
    q_rot = orc.rope_rotate(q_rope, np.array([[L]]))
    brute = orc.bruteforce_attention(q_nope, q_rot, c, kr, w_uk, w_uv, scale)
    np.testing.assert_allclose(out, brute, rtol=1e-12, atol=1e-13)
