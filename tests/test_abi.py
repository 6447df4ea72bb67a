"""CPU checks of the C ABI: the library builds, loads without a GPU, exports every symbol
include/mla.h declares, its structs match the header, and host-side argument validation
returns the documented status without enqueuing any work."""
import ctypes
import pathlib
import re
import subprocess

import pytest

ROOT = pathlib.Path(__file__).resolve().parents[1]
HEADER = ROOT / "include" / "mla.h"


@pytest.fixture(scope="module")
def built():
    from mla_latent_kv_27_b200 import build as b
    return b.build()


def declared_functions():
    text = HEADER.read_text()
    return sorted(set(re.findall(r"MLA_API\s+[\w\s\*]+?\b(mla_\w+)\s*\(", text)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for required in ("mla_append_cache", "mla_absorb_query", "mla_decode_attention", "mla_output_up"):
        assert required in names


def test_library_exports_every_declared_symbol(built):
    out = subprocess.run(["nm", "-D", "--defined-only", str(built)], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\sT\s+(mla_\w+)", out))
    missing = set(declared_functions()) - exported
    assert not missing, missing
    lib = ctypes.CDLL(str(built))
    for name in declared_functions():
        assert getattr(lib, name) is not None


def test_binding_names_match_header(built):
    import mla_latent_kv_27_b200 as mla
    assert set(mla.EXPORTED) == set(declared_functions())
    for name in declared_functions():
        assert callable(getattr(mla, name))


def test_struct_layouts(built):
    import mla_latent_kv_27_b200 as mla
    assert ctypes.sizeof(mla.mla_dims) == 10 * 4
    assert ctypes.sizeof(mla.mla_cache) == 4 * 8 + 3 * 4 + 4  # three int32 tail fields, padded to 8


def test_status_strings(built):
    import mla_latent_kv_27_b200 as mla
    assert mla.mla_status_string(0) == "ok"
    for s in range(1, 6):
        assert mla.mla_status_string(s) not in ("ok", "unknown status")
    assert mla.mla_version() >= 100


def _dims(mla, **kw):
    base = dict(d_model=64, d_c=64, d_rope=16, d_nope=32, d_v=32, n_heads=4, page_size=64,
                act_dtype=mla.MLA_F32, cache_dtype=mla.MLA_F32, scale=0.1)
    base.update(kw)
    return mla.mla_dims(**base)


def test_validation_without_a_gpu(built):
    import mla_latent_kv_27_b200 as mla
    lib = mla.lib_handle()
    d = _dims(mla)
    byref = ctypes.byref
    # null dims / bad dims -> INVALID_ARG, before any CUDA call
    assert lib.mla_output_up(None, 1, 1, 1, 1, None) == 1
    assert lib.mla_output_up(byref(_dims(mla, d_c=0)), 1, 1, 1, 1, None) == 1
    assert lib.mla_output_up(byref(_dims(mla, d_rope=3)), 1, 1, 1, 1, None) == 1
    # n_tok == 0 is a no-op
    assert lib.mla_output_up(byref(d), None, 0, None, None, None) == 0
    assert lib.mla_absorb_query(byref(d), None, None, None, 0, None, None, None, 0, None, None) == 0
    # negative sizes
    assert lib.mla_output_up(byref(d), 1, -1, 1, 1, None) == 1
    # unsupported combinations
    assert lib.mla_output_up(byref(_dims(mla, act_dtype=mla.MLA_FP8_E4M3)), 1, 1, 1, 1, None) == 2
    assert lib.mla_output_up(byref(_dims(mla, cache_dtype=mla.MLA_BF16)), 1, 1, 1, 1, None) == 2
    fp8_bad = _dims(mla, act_dtype=mla.MLA_BF16, cache_dtype=mla.MLA_FP8_E4M3, d_c=96)
    assert lib.mla_output_up(byref(fp8_bad), 1, 1, 1, 1, None) == 2
    # decode: bad causal flag, batch 0 no-op, missing cache
    assert lib.mla_decode_attention(byref(d), 1, None, 1, 1, 1, 2, 0, None, 0, 1, None, None) == 1
    assert lib.mla_decode_attention(byref(d), None, None, None, 0, 1, 0, 0, None, 0, None, None, None) == 0
    assert lib.mla_decode_attention(byref(d), 1, None, 1, 1, 1, 0, 0, None, 0, 1, None, None) == 1
    # rope table arguments
    assert lib.mla_rope_table(15, 10, 10000.0, 1, 1, None) == 1
    assert lib.mla_rope_table(16, 0, 10000.0, 1, 1, None) == 1
    assert lib.mla_rope_table(16, 10, -1.0, 1, 1, None) == 1


def test_workspace_sizes(built):
    import mla_latent_kv_27_b200 as mla
    d = _dims(mla)
    assert mla.mla_append_workspace_size(d, 10) == 10 * (64 + 16) * 4
    assert mla.mla_decode_workspace_size(d, 2, 1, 1, 4) == 0          # one chunk: no partials
    assert mla.mla_decode_workspace_size(d, 2, 1, 3, 4) == 2 * 3 * 4 * (64 + 1) * 4
    assert mla.mla_decode_workspace_size(d, 2, 1, 0, 4) > 0           # library-chosen split
    assert mla.mla_decode_workspace_size(_dims(mla, d_c=-1), 2, 1, 3, 4) == 0
    # tensor-core shapes, any n_split: the length-balanced partition over 74 ranges, whose rows
    # cut across ranges write at most 2 * 74 - 2 partial slots of H x (d_c + 1) fp32, then two
    # int32 per row
    tc = _dims(mla, d_c=512, d_rope=64, n_heads=128, act_dtype=mla.MLA_BF16, cache_dtype=mla.MLA_BF16)
    for n_split in (0, 1, 32):
        assert mla.mla_decode_workspace_size(tc, 64, 1, n_split, 128) == 146 * 128 * 513 * 4 + 64 * 8
    assert mla.mla_decode_workspace_size(tc, 3, 2, 0, 9) == 146 * 128 * 513 * 4 + 6 * 8
    # at most 16 heads (bf16): the small-head kernel's partition, two workers per SM, 590 slots
    sh = _dims(mla, d_c=512, d_rope=64, n_heads=16, act_dtype=mla.MLA_BF16, cache_dtype=mla.MLA_BF16)
    assert mla.mla_decode_workspace_size(sh, 32, 1, 0, 64) == 590 * 16 * 513 * 4 + 32 * 8
    assert mla.mla_decode_workspace_size(sh, 32, 1, 4, 64) == 590 * 16 * 513 * 4 + 32 * 8
    # the bf16 tensor-core append reduces its partial sums on chip: no workspace
    tc_app = _dims(mla, d_model=7168, d_c=512, d_rope=64, d_nope=128, d_v=128, n_heads=128,
                   act_dtype=mla.MLA_BF16, cache_dtype=mla.MLA_BF16)
    assert mla.mla_append_workspace_size(tc_app, 64) == 0
    assert mla.mla_append_workspace_size(_dims(mla, act_dtype=mla.MLA_BF16, cache_dtype=mla.MLA_BF16,
                                                   d_c=96), 10) == 10 * (96 + 16) * 4
