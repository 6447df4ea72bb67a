"""GPU parity of mla_decode_attention (+ split combine) against the fp64 oracle.

Tolerances (stated by the workloads):
  fp32 cache/act:  max relative error (max |g - o| / max |o|) <= 1e-5
  bf16:            max abs error <= 2e-2, and additionally max relative error <= 1e-2 and an
                   element-wise relative error <= 2e-2 on every entry with |o| >= 0.25 (the
                   entries a sharp softmax makes large)
  fp8 cache:       max abs error <= 2e-2 (and the element-wise check) against the oracle fed
                   the cache as the FP8 path's fp16 operands hold it (each E4M3 value times its
                   block scale, rounded once to fp16: parity_helpers.fp16_operands), and
                   <= 6e-2 against the oracle fed the unquantised latents wherever every
                   checked sequence has at least 512 tokens (the workload's shortest); for
                   shorter sequences the E4M3 rounding of a handful of latents (up to 1/28
                   of a 128-value block's maximum each) is not averaged down, so only the
                   decoded-cache comparison applies there
lse is compared where finite and must be -inf exactly where the oracle's is: 1e-5 relative for
fp32; for bf16/fp8, per row, 2e-3 + 1e-5 * scale * max_t sum_i |q_i k_t,i| (fp32 accumulation;
see parity_helpers.lse_bound).
"""
import dataclasses

import numpy as np
import pytest

from mla_latent_kv_27_b200 import workloads as wl
from tests.parity_helpers import (checked_rows, decode_case, lse_bound, lse_close, max_abs, max_rel,
                                  max_rel_elementwise)

pytestmark = pytest.mark.gpu

W = wl.WORKLOADS


def _check(res, w, seqs=None, tol_abs=2e-2, tol_rel=1e-2, quant_check=True):
    rows = checked_rows(res, seqs)
    g, r = res["o_gpu"][rows], res["o_ref"][rows]
    assert res["device_status"][0] == 0, res["device_status"]
    assert np.isfinite(g).all()
    if w.act_dtype == "f32":
        assert max_rel(g, r) <= 1e-5, max_rel(g, r)
        fin = np.isfinite(res["lse_ref"][rows])
        assert max_rel(res["lse_gpu"][rows][fin], res["lse_ref"][rows][fin]) <= 1e-5
    else:
        assert max_abs(g, r) <= tol_abs, max_abs(g, r)
        assert max_rel(g, r) <= tol_rel, max_rel(g, r)
        assert max_rel_elementwise(g, r) <= 2e-2, max_rel_elementwise(g, r)
        assert lse_close(res["lse_gpu"][rows], res["lse_ref"][rows], lse_bound(res, rows, w.scale))
    if quant_check and "o_raw" in res and res["min_len"](seqs) >= 512:
        assert max_abs(g, res["o_raw"][rows]) <= 6e-2, max_abs(g, res["o_raw"][rows])


# ------------------------------------------------------------------ small cases: several tiles, ragged tails

def test_tiny_fp32_decode(lib):
    w = W["tiny_fp32"]
    _check(decode_case(lib, w, w.lengths, n_split=1), w)


@pytest.mark.parametrize("n_split", [0, 1, 2, 5])
def test_tiny_fp32_decode_splits(lib, n_split):
    w = W["tiny_fp32"]
    _check(decode_case(lib, w, [37, 100, 1, 64, 65], n_split=n_split), w)


@pytest.mark.parametrize("n_split", [0, 1, 3, 40])
def test_v2lite_shape_ragged(lib, n_split):
    w = dataclasses.replace(W["v2lite_bf16"], batch=5)
    _check(decode_case(lib, w, [1, 63, 64, 65, 1000], n_split=n_split), w)


@pytest.mark.parametrize("n_split", [0, 1, 4, 64])
def test_v3_shape_ragged_shuffled(lib, n_split):
    w = dataclasses.replace(W["v3_bf16"], batch=6)
    _check(decode_case(lib, w, [1, 2, 63, 64, 129, 777], n_split=n_split), w)


@pytest.mark.parametrize("n_split", [0, 1, 3])
def test_fp8_mtp_causal_ragged(lib, n_split):
    w = dataclasses.replace(W["fp8_mtp2"], batch=6)
    _check(decode_case(lib, w, [1, 2, 3, 64, 65, 700], n_split=n_split), w)


@pytest.mark.parametrize("causal", [True, False])
def test_small_head_mtp_rows(lib, causal):
    # 16 heads, two query tokens per sequence: the small-head kernel walks the two rows of a
    # sequence on neighbouring workers; tiny and ragged lengths leave the causal first row empty
    # or a page short
    w = dataclasses.replace(W["v2lite_bf16"], batch=7, s_q=2, causal=causal)
    _check(decode_case(lib, w, [1, 2, 64, 65, 129, 700, 3000], n_split=0), w)


def test_long_split_ragged_chunks(lib):
    w = dataclasses.replace(W["long_bf16"], batch=2)
    _check(decode_case(lib, w, [5000, 4097], n_split=32), w)


@pytest.mark.parametrize("heads", [1, 12, 16, 17, 20, 100])
@pytest.mark.parametrize("cache", ["bf16", "fp8"])
@pytest.mark.parametrize("n_split", [0, 2])
def test_fewer_than_128_heads(lib, heads, cache, n_split):
    # bf16 with at most 16 heads runs the small-head kernel (16 head rows per MMA); otherwise the
    # tcgen05 kernel pads the heads to 128 query rows; both store only the real ones
    base = W["fp8_mtp2"] if cache == "fp8" else W["v3_bf16"]
    w = dataclasses.replace(base, batch=4, n_heads=heads)
    _check(decode_case(lib, w, [1, 64, 200, 517], n_split=n_split), w)


@pytest.mark.parametrize("name", ["v3_bf16", "fp8_mtp2"])
def test_balanced_partition_workers_cross_rows(lib, name):
    # n_split = 0 with more pages than partition ranges: each persistent worker walks several
    # row segments (barrier phases carried across segments, partial and whole rows mixed)
    rng = np.random.default_rng(7)
    lengths = rng.integers(1, 700, size=40).astype(np.int32)
    lengths[[3, 17]] = 0
    w = dataclasses.replace(W[name], batch=len(lengths), shuffle_pages=True)
    _check(decode_case(lib, w, lengths, n_split=0), w)


def test_balanced_partition_many_short_rows(lib):
    # n_split = 0: more partition ranges than pages, rows cut at range boundaries, empty rows
    w = dataclasses.replace(W["v3_bf16"], batch=12)
    _check(decode_case(lib, w, [0, 1, 64, 65, 3, 0, 129, 2, 700, 64, 1, 300], n_split=0), w)


@pytest.mark.parametrize("name,changes", [
    ("v3_bf16", dict(n_heads=8, d_c=256, d_rope=32)),
    ("v3_bf16", dict(n_heads=160)),
    ("fp8_mtp2", dict(n_heads=12, d_c=256, d_rope=32)),
])
def test_general_path_shapes(lib, name, changes):
    # shapes outside the tensor-core kernel's (d_c = 512, d_rope = 64, H <= 128) take the
    # general kernel
    w = dataclasses.replace(W[name], batch=3, **changes)
    _check(decode_case(lib, w, [5, 64, 333], n_split=0), w)


@pytest.mark.parametrize("n_split", [0, 2])
def test_empty_sequences(lib, n_split):
    # L = 0 gives o_lat = 0 and lse = -inf; neighbours are unaffected.
    w = dataclasses.replace(W["v3_bf16"], batch=4)
    res = decode_case(lib, w, [0, 70, 0, 5], n_split=n_split)
    _check(res, w)
    assert (res["o_gpu"][[0, 2]] == 0).all()
    assert np.isneginf(res["lse_gpu"][[0, 2]]).all()


def test_mtp_first_query_of_a_one_token_sequence_is_empty(lib):
    # S_q = 2, L = 1: the first draft query sits at position -1 and attends nothing.
    w = dataclasses.replace(W["fp8_mtp2"], batch=2)
    res = decode_case(lib, w, [1, 9], n_split=1)
    _check(res, w)
    assert (res["o_gpu"][0] == 0).all() and np.isneginf(res["lse_gpu"][0]).all()


def test_block_table_permutation_invariance_gpu(lib):
    w0 = dataclasses.replace(W["v3_bf16"], batch=3, shuffle_pages=False)
    w1 = dataclasses.replace(w0, shuffle_pages=True)
    r0 = decode_case(lib, w0, [300, 64, 129], n_split=1)
    r1 = decode_case(lib, w1, [300, 64, 129], n_split=1)
    np.testing.assert_array_equal(r0["o_gpu"], r1["o_gpu"])
    np.testing.assert_array_equal(r0["lse_gpu"], r1["lse_gpu"])


# ------------------------------------------------------------------ full sizes, as bench.py launches them

@pytest.mark.parametrize("name", ["v2lite_bf16", "v3_bf16", "long_bf16", "fp8_mtp2"])
def test_full_size_decode(lib, name):
    # every query row of the batch against the oracle, in the launch configuration bench.py
    # times (the balanced partition cuts rows at arbitrary page boundaries: no row is skipped)
    w = W[name]
    lengths = wl.draw_lengths(w)
    res = decode_case(lib, w, lengths, n_split=w.n_split)
    _check(res, w)


# ------------------------------------------------------------------ sharp softmax, large scores

@pytest.mark.parametrize("name", ["v3_bf16", "fp8_mtp2", "v2lite_bf16"])
@pytest.mark.parametrize("q_scale", [10.0, 30.0])
@pytest.mark.parametrize("n_split", [0, 3])
def test_peaked_softmax(lib, name, q_scale, n_split):
    # logits spread over about N(0, q_scale^2): the row maximum grows across pages and the
    # softmax concentrates on a few tokens, so o_lat entries approach unit size
    lengths = wl.draw_lengths(W[name])[:8]
    w = dataclasses.replace(W[name], batch=8)
    res = decode_case(lib, w, lengths, n_split=n_split, q_scale=q_scale)
    # a sharp softmax does not average E4M3 rounding down: only the decoded-cache check applies
    _check(res, w, quant_check=False)
    r = res["o_ref"]
    assert np.abs(r).max() > 0.5  # the case is really peaked


@pytest.mark.parametrize("name", ["v3_bf16", "fp8_mtp2", "v2lite_bf16"])
def test_large_raw_scores(lib, name):
    # raw (unscaled) partial scores of 10^3 - 10^4: q scaled by 400 puts |q . k| over the
    # 288 dims each CTA of the tensor-core pair sums (and each quarter of the small-head kernel's
    # k-steps) in that range
    lengths = np.array([64, 700, 1500, 3000], dtype=np.int32)
    w = dataclasses.replace(W[name], batch=4)
    res = decode_case(lib, w, lengths, n_split=0, q_scale=400.0)
    _check(res, w, quant_check=False)
    assert np.nanmax(res["abs_score"]) > 1e4
