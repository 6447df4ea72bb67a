"""mla_decode_attention_noalloc: the decode entry point for callers that cannot allocate.

Some callers (a host framework that owns every device allocation and gives plug-ins no
allocator, or a latency-critical path where cudaMalloc would synchronise the device) cannot
pass scratch memory.  This variant keeps its split-KV partials in the library's own static
device buffer.  The test calls it through the C ABI twice in a row and checks each result
against the ordinary entry point (caller workspace) on the same inputs: on the tensor-core
path, whose length-balanced partition (whatever n_split says) puts the partials of rows cut
across partition ranges and the per-row slot table at the buffer's head, and on the general
kernel (more than 128 heads) with fixed splits.  Both entry points run the same deterministic
kernels on the same inputs, so the results must be bit-identical.  It builds all of its inputs
itself, so it passes alone in a fresh process as well as after the other tests.
"""
import dataclasses

import numpy as np
import pytest
import torch

from mla_latent_kv_27_b200 import workloads as wl
from tests.parity_helpers import DeviceCache, dims_for, round_to, to_dev

pytestmark = pytest.mark.gpu


def _inputs(lib, w, lengths, stream):
    rows, q = wl.draw_decode_inputs(w, lengths, stream=stream)
    table, num_pages = wl.make_block_table(lengths, 0, w.shuffle_pages, wl.rng_for(w, 6))
    cache = DeviceCache(lib, w, lengths, table, num_pages, rows=round_to(rows, "bf16"))
    return cache, to_dev(round_to(q, "bf16"), "bf16"), table


def _outputs(batch, w):
    o = torch.full((batch * w.s_q, w.n_heads, w.d_c), float("nan"), dtype=torch.bfloat16, device="cuda")
    lse = torch.full((batch * w.s_q, w.n_heads), float("nan"), dtype=torch.float32, device="cuda")
    return o, lse


@pytest.mark.parametrize("heads,n_split", [(16, 0), (128, 0), (128, 4), (160, 4)])
def test_noalloc_matches_workspace_entry_point_twice(lib, heads, n_split):
    w = dataclasses.replace(wl.WORKLOADS["v3_bf16"], batch=6, n_heads=heads)
    # 49 pages over 74 partition ranges: on the tensor-core path the longer rows span many ranges
    lengths = np.array([1, 70, 640, 129, 2000, 64], dtype=np.int32)
    dims = dims_for(lib, w)
    lens = to_dev(lengths, "i32")
    for call, stream in enumerate((11, 12)):
        cache, q, table = _inputs(lib, w, lengths, stream)
        need = lib.mla_decode_workspace_size(dims, len(lengths), 1, n_split, table.shape[1])
        assert 0 < need <= lib.MLA_NOALLOC_SCRATCH_BYTES
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
        o_ref, lse_ref = _outputs(len(lengths), w)
        lib.mla_decode_attention(dims, q, cache.desc, lens, len(lengths), 1, 0, n_split, ws, need, o_ref, lse_ref)
        o_na, lse_na = _outputs(len(lengths), w)
        lib.mla_decode_attention_noalloc(dims, q, cache.desc, lens, len(lengths), 1, 0, n_split, o_na, lse_na)
        torch.cuda.synchronize()
        assert lib.mla_check_device_error()[0] == 0
        g, r = o_na.double().cpu().numpy(), o_ref.double().cpu().numpy()
        assert np.isfinite(g).all(), f"call {call}"
        np.testing.assert_array_equal(g, r)
        np.testing.assert_array_equal(lse_na.cpu().numpy(), lse_ref.cpu().numpy())


def test_noalloc_rejects_requests_beyond_its_buffer(lib):
    # the general kernel (160 heads) with 64 fixed splits of 64 rows: 1.3 GB of partials (the
    # tensor-core path's partials never pass 146 slots, 39 MB at 128 heads)
    w = dataclasses.replace(wl.WORKLOADS["v3_bf16"], n_heads=160)
    dims = dims_for(lib, w)
    lengths = np.full(64, 4096, dtype=np.int32)
    cache, q, table = _inputs(lib, dataclasses.replace(w, batch=64, shuffle_pages=False), lengths[:1], 13)
    need = lib.mla_decode_workspace_size(dims, 64, 1, 64, table.shape[1])
    assert need > lib.MLA_NOALLOC_SCRATCH_BYTES
    o, lse = _outputs(64, w)
    with pytest.raises(lib.MlaError) as err:
        lib.mla_decode_attention_noalloc(dims, q, cache.desc, to_dev(lengths, "i32"), 64, 1, 0, 64, o, lse)
    assert err.value.status == 2  # MLA_ERR_UNSUPPORTED, nothing enqueued
    torch.cuda.synchronize()
    assert torch.isnan(o.float()).all()
