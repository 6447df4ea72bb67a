"""ctypes binding of libmla (include/mla.h): argument marshalling only.

Every function has the C name and argument order.  Tensor arguments may be torch CUDA
tensors (their data pointer is passed) or raw integer device addresses; ``stream`` is a
torch.cuda.Stream, a raw cudaStream_t integer, or None for torch's current stream.  A
non-OK status raises MlaError.  Nothing here computes any step of the method: with the
shared library missing, importing this module raises ImportError.
"""
from __future__ import annotations

import ctypes
import os
import pathlib

_LIB_PATH = pathlib.Path(__file__).resolve().parent / "libmla.so"

MLA_OK, MLA_ERR_INVALID_ARG, MLA_ERR_UNSUPPORTED, MLA_ERR_CUDA, MLA_ERR_DEVICE, MLA_ERR_TIMEOUT = range(6)
MLA_F32, MLA_BF16, MLA_FP8_E4M3 = 0, 1, 2

EXPORTED = (
    "mla_rope_table", "mla_append_workspace_size", "mla_append_cache", "mla_absorb_query",
    "mla_decode_workspace_size", "mla_decode_attention", "mla_output_up", "mla_status_string",
    "mla_check_device_error", "mla_version", "mla_launch_count", "mla_decode_attention_noalloc",
)

MLA_NOALLOC_SCRATCH_BYTES = 64 << 20


class MlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {mla_status_string(status)} (status {status})")


class mla_dims(ctypes.Structure):
    _fields_ = [("d_model", ctypes.c_int32), ("d_c", ctypes.c_int32), ("d_rope", ctypes.c_int32),
                ("d_nope", ctypes.c_int32), ("d_v", ctypes.c_int32), ("n_heads", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("act_dtype", ctypes.c_int32),
                ("cache_dtype", ctypes.c_int32), ("scale", ctypes.c_float)]


class mla_cache(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("rope", ctypes.c_void_p),
                ("block_table", ctypes.c_void_p), ("max_pages_per_seq", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("num_seqs", ctypes.c_int32)]


def _load():
    if not _LIB_PATH.exists():
        raise ImportError(f"{_LIB_PATH} is missing: build it with `python -m mla_latent_kv_27_b200.build` "
                          "(the library has no fallback)")
    lib = ctypes.CDLL(os.fspath(_LIB_PATH))
    P, I32, SZ, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    D, C = ctypes.POINTER(mla_dims), ctypes.POINTER(mla_cache)
    sig = {
        "mla_rope_table": (I32, [I32, I32, F32, P, P, P]),
        "mla_append_workspace_size": (SZ, [D, I32]),
        "mla_append_cache": (I32, [D, P, I32, P, P, P, P, P, P, I32, C, P, SZ, P]),
        "mla_absorb_query": (I32, [D, P, P, P, I32, P, P, P, I32, P, P]),
        "mla_decode_workspace_size": (SZ, [D, I32, I32, I32, I32]),
        "mla_decode_attention": (I32, [D, P, C, P, I32, I32, I32, I32, P, SZ, P, P, P]),
        "mla_output_up": (I32, [D, P, I32, P, P, P]),
        "mla_decode_attention_noalloc": (I32, [D, P, C, P, I32, I32, I32, I32, P, P, P]),
        "mla_status_string": (ctypes.c_char_p, [I32]),
        "mla_check_device_error": (I32, [P, ctypes.POINTER(I32)]),
        "mla_version": (I32, []),
        "mla_launch_count": (ctypes.c_uint64, []),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = _load()


def lib_handle():
    return _lib


def _p(x):
    """Device address of a tensor / int / None."""
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError("libmla takes device tensors (got a host tensor)")
    return x.data_ptr()


def _s(stream):
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, where: str):
    if status != MLA_OK:
        raise MlaError(status, where)


def mla_status_string(status: int) -> str:
    return _lib.mla_status_string(status).decode()


def mla_version() -> int:
    return _lib.mla_version()


def mla_launch_count() -> int:
    return _lib.mla_launch_count()


def mla_rope_table(d_rope, max_pos, theta, cos_out, sin_out, stream=None):
    _check(_lib.mla_rope_table(d_rope, max_pos, theta, _p(cos_out), _p(sin_out), _s(stream)),
           "mla_rope_table")


def mla_append_workspace_size(dims: mla_dims, n_tok: int) -> int:
    return _lib.mla_append_workspace_size(ctypes.byref(dims), n_tok)


def mla_append_cache(dims, h, n_tok, seq_idx, pos, w_dkv, w_kr, rope_cos, rope_sin, rope_rows,
                     cache: mla_cache, workspace, workspace_bytes, stream=None):
    _check(_lib.mla_append_cache(ctypes.byref(dims), _p(h), n_tok, _p(seq_idx), _p(pos), _p(w_dkv),
                                 _p(w_kr), _p(rope_cos), _p(rope_sin), rope_rows, ctypes.byref(cache),
                                 _p(workspace), workspace_bytes, _s(stream)), "mla_append_cache")


def mla_absorb_query(dims, q_nope, q_rope, q_pos, n_tok, w_uk, rope_cos, rope_sin, rope_rows,
                     q_packed, stream=None):
    _check(_lib.mla_absorb_query(ctypes.byref(dims), _p(q_nope), _p(q_rope), _p(q_pos), n_tok,
                                 _p(w_uk), _p(rope_cos), _p(rope_sin), rope_rows, _p(q_packed),
                                 _s(stream)), "mla_absorb_query")


def mla_decode_workspace_size(dims, batch, s_q, n_split, max_pages_per_seq) -> int:
    return _lib.mla_decode_workspace_size(ctypes.byref(dims), batch, s_q, n_split, max_pages_per_seq)


def mla_decode_attention(dims, q_packed, cache: mla_cache, seq_lens, batch, s_q, causal, n_split,
                         workspace, workspace_bytes, o_lat, lse, stream=None):
    _check(_lib.mla_decode_attention(ctypes.byref(dims), _p(q_packed), ctypes.byref(cache),
                                     _p(seq_lens), batch, s_q, int(causal), n_split, _p(workspace),
                                     workspace_bytes, _p(o_lat), _p(lse), _s(stream)),
           "mla_decode_attention")


def mla_decode_attention_noalloc(dims, q_packed, cache: mla_cache, seq_lens, batch, s_q, causal,
                                 n_split, o_lat, lse, stream=None):
    _check(_lib.mla_decode_attention_noalloc(ctypes.byref(dims), _p(q_packed), ctypes.byref(cache),
                                             _p(seq_lens), batch, s_q, int(causal), n_split, _p(o_lat),
                                             _p(lse), _s(stream)), "mla_decode_attention_noalloc")


def mla_output_up(dims, o_lat, n_tok, w_uv, out, stream=None):
    _check(_lib.mla_output_up(ctypes.byref(dims), _p(o_lat), n_tok, _p(w_uv), _p(out), _s(stream)),
           "mla_output_up")


def mla_check_device_error(stream=None):
    """Returns (status, detail) without raising."""
    detail = ctypes.c_int32(0)
    st = _lib.mla_check_device_error(_s(stream), ctypes.byref(detail))
    return st, detail.value
