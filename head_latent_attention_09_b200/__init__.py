"""Python binding of libmla.so, the decode-time Multi-head Latent Attention
library for B200 (sm_100a).

Argument marshalling only: every function here has the name of the C entry
point it forwards to (include/mla.h) and converts torch tensors / ints /
streams to pointers.  All arithmetic runs in the library's CUDA kernels; if
the library is missing, loading fails with an error (there is no fallback).
"""

from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmla.so")

MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_WORKSPACE = 3
MLA_ERR_CUDA = 4
MLA_ERR_TIMEOUT = 5
MLA_ERR_DEVICE_BOUNDS = 6
MLA_BF16 = 0
MLA_FP32 = 1

EXPORTED = (
    "mla_status_string", "mla_config_validate", "mla_create", "mla_destroy",
    "mla_cache_append", "mla_absorb_q", "mla_decode_workspace_size",
    "mla_default_num_parts", "mla_decode_attn", "mla_combine_splits", "mla_out_proj",
    "mla_query_proj",
    "mla_get_device_status", "mla_plan_pieces", "mla_decode_attn_combine_noalloc",
    "mla_noalloc_scratch_bytes", "mla_set_rope_scaling",
    "mla_fp8_scale_groups", "mla_cache_append_fp8_workspace_size", "mla_cache_append_fp8",
    "mla_quantize_rows_fp8", "mla_decode_attn_fp8", "mla_selftest_wait_timeout",
    "mla_set_strict", "mla_decode_attn_range", "mla_combine_splits_f32", "mla_merge_ranges",
    "mla_combine_out_proj", "mla_plan_pieces_tiled", "mla_plan_tile",
)


class MlaError(RuntimeError):
    def __init__(self, status: int, where: str):
        super().__init__(f"{where}: {mla_status_string(status)} ({status})")
        self.status = status


class mla_config(ctypes.Structure):
    _fields_ = [("n_h", ctypes.c_int), ("d_h", ctypes.c_int), ("d_c", ctypes.c_int),
                ("d_r", ctypes.c_int), ("d_model", ctypes.c_int), ("page_size", ctypes.c_int),
                ("rope_base", ctypes.c_double), ("dtype", ctypes.c_int)]


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libmla.so (raises OSError if it has not been built)."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    p = path or LIB_PATH
    if not os.path.exists(p):
        raise OSError(f"{p} is missing: build it with head_latent_attention_09_b200.build.build()")
    lib = ctypes.CDLL(p)
    vp, i, ll, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_longlong, ctypes.c_size_t
    sig = {
        "mla_status_string": (ctypes.c_char_p, [i]),
        "mla_config_validate": (i, [ctypes.POINTER(mla_config)]),
        "mla_create": (i, [ctypes.POINTER(mla_config), ctypes.POINTER(vp)]),
        "mla_destroy": (None, [vp]),
        "mla_cache_append": (i, [vp, vp, i, i, vp, vp, vp, vp, ll, vp, i, vp]),
        "mla_absorb_q": (i, [vp, vp, vp, vp, vp, vp, i, vp]),
        "mla_decode_workspace_size": (sz, [vp, i, i]),
        "mla_default_num_parts": (i, [vp]),
        "mla_decode_attn": (i, [vp, vp, vp, ll, vp, i, vp, i, i, vp, sz, vp]),
        "mla_combine_splits": (i, [vp, vp, sz, i, i, vp, vp, vp]),
        "mla_out_proj": (i, [vp, vp, vp, vp, vp, vp, i, vp]),
        "mla_query_proj": (i, [vp, vp, i, vp, i, vp, vp, vp, vp, vp, vp]),
        "mla_get_device_status": (i, [vp, vp]),
        "mla_plan_pieces": (ll, [vp, i, i, vp]),
        "mla_decode_attn_combine_noalloc": (i, [vp, vp, vp, ll, vp, i, vp, i, i, vp, vp, vp]),
        "mla_noalloc_scratch_bytes": (sz, []),
        "mla_set_rope_scaling": (i, [vp, ctypes.c_double, i, ctypes.c_double, ctypes.c_double,
                                     ctypes.c_double]),
        "mla_fp8_scale_groups": (i, [vp]),
        "mla_cache_append_fp8_workspace_size": (sz, [vp, i, i]),
        "mla_cache_append_fp8": (i, [vp, vp, i, i, vp, vp, vp, vp, vp, ll, vp, i, vp, sz, vp]),
        "mla_quantize_rows_fp8": (i, [vp, vp, ll, vp, vp, vp]),
        "mla_decode_attn_fp8": (i, [vp, vp, vp, vp, ll, vp, i, vp, i, i, vp, sz, vp]),
        "mla_selftest_wait_timeout": (i, [vp, ll, vp]),
        "mla_set_strict": (i, [vp, i]),
        "mla_decode_attn_range": (i, [vp, vp, vp, ll, vp, i, vp, vp, i, i, vp, sz, vp]),
        "mla_combine_splits_f32": (i, [vp, vp, sz, i, i, vp, vp, vp]),
        "mla_merge_ranges": (i, [vp, vp, vp, i, i, vp, vp, vp]),
        "mla_combine_out_proj": (i, [vp, vp, sz, i, i, vp, vp, vp, vp, vp, vp, vp]),
        "mla_plan_pieces_tiled": (ll, [vp, i, i, i, vp]),
        "mla_plan_tile": (i, [vp, i]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path is None:
        _lib = lib
    return lib


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------

def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if hasattr(x, "data_ptr"):
        return x.data_ptr()
    if isinstance(x, ctypes.c_void_p):
        return x.value
    raise TypeError(f"cannot pass {type(x).__name__} as a pointer")


def _stream(s):
    if s is None:
        import torch
        return torch.cuda.current_stream().cuda_stream if torch.cuda.is_available() else None
    if isinstance(s, int):
        return s
    return s.cuda_stream


def _check(status: int, where: str):
    if status != MLA_OK:
        raise MlaError(status, where)


# ----------------------------------------------------------------------------
# entry points (same names as the C ABI)
# ----------------------------------------------------------------------------

def mla_status_string(status: int) -> str:
    return load().mla_status_string(int(status)).decode()


def mla_config_validate(cfg: mla_config) -> int:
    return load().mla_config_validate(ctypes.byref(cfg))


def mla_create(cfg: mla_config) -> int:
    """Returns the handle as an integer address."""
    h = ctypes.c_void_p()
    _check(load().mla_create(ctypes.byref(cfg), ctypes.byref(h)), "mla_create")
    return h.value


def mla_destroy(handle: int) -> None:
    load().mla_destroy(handle)


def mla_set_rope_scaling(handle, factor, original_ctx, alpha, beta, mscale_coef) -> None:
    _check(load().mla_set_rope_scaling(handle, float(factor), int(original_ctx), float(alpha),
                                       float(beta), float(mscale_coef)), "mla_set_rope_scaling")


def mla_set_strict(handle, strict) -> None:
    _check(load().mla_set_strict(handle, int(bool(strict))), "mla_set_strict")


def mla_cache_append(handle, h, B, T, start_pos, w_dkv, w_kr, cache, cache_len,
                     block_table=None, max_blocks_per_seq=0, stream=None):
    _check(load().mla_cache_append(handle, _ptr(h), B, T, _ptr(start_pos), _ptr(w_dkv),
                                   _ptr(w_kr), _ptr(cache), cache_len, _ptr(block_table),
                                   max_blocks_per_seq, _stream(stream)), "mla_cache_append")


def mla_absorb_q(handle, q_nope, q_rope, pos, w_uk, q_abs, B, stream=None):
    _check(load().mla_absorb_q(handle, _ptr(q_nope), _ptr(q_rope), _ptr(pos), _ptr(w_uk),
                               _ptr(q_abs), B, _stream(stream)), "mla_absorb_q")


def mla_decode_workspace_size(handle, B, num_parts=0) -> int:
    return load().mla_decode_workspace_size(handle, B, num_parts)


def mla_default_num_parts(handle) -> int:
    return load().mla_default_num_parts(handle)


def mla_fp8_scale_groups(handle):
    return load().mla_fp8_scale_groups(handle)


def mla_cache_append_fp8_workspace_size(handle, B, T):
    return load().mla_cache_append_fp8_workspace_size(handle, B, T)


def mla_cache_append_fp8(handle, h, B, T, start_pos, w_dkv, w_kr, cache, kv_scale, cache_len,
                         block_table, max_blocks_per_seq, workspace, ws_bytes, stream=None):
    _check(load().mla_cache_append_fp8(handle, _ptr(h), B, T, _ptr(start_pos), _ptr(w_dkv),
                                       _ptr(w_kr), _ptr(cache), _ptr(kv_scale), cache_len,
                                       _ptr(block_table), max_blocks_per_seq, _ptr(workspace),
                                       ws_bytes, _stream(stream)), "mla_cache_append_fp8")


def mla_quantize_rows_fp8(handle, rows, n_rows, codes, kv_scale, stream=None):
    _check(load().mla_quantize_rows_fp8(handle, _ptr(rows), n_rows, _ptr(codes), _ptr(kv_scale),
                                        _stream(stream)), "mla_quantize_rows_fp8")


def mla_decode_attn_fp8(handle, q_abs, cache, kv_scale, cache_len, block_table, max_blocks_per_seq,
                        ctx_len, B, num_parts, workspace, ws_bytes, stream=None):
    _check(load().mla_decode_attn_fp8(handle, _ptr(q_abs), _ptr(cache), _ptr(kv_scale), cache_len,
                                      _ptr(block_table), max_blocks_per_seq, _ptr(ctx_len), B,
                                      num_parts, _ptr(workspace), ws_bytes, _stream(stream)),
           "mla_decode_attn_fp8")


def mla_selftest_wait_timeout(handle, limit_ns, stream=None):
    _check(load().mla_selftest_wait_timeout(handle, limit_ns, _stream(stream)),
           "mla_selftest_wait_timeout")


def mla_decode_attn(handle, q_abs, cache, cache_len, block_table, max_blocks_per_seq, ctx_len, B,
                    num_parts, workspace, ws_bytes, stream=None):
    _check(load().mla_decode_attn(handle, _ptr(q_abs), _ptr(cache), cache_len, _ptr(block_table),
                                  max_blocks_per_seq, _ptr(ctx_len), B, num_parts,
                                  _ptr(workspace), ws_bytes, _stream(stream)), "mla_decode_attn")


def mla_decode_attn_range(handle, q_abs, cache, cache_len, block_table, max_blocks_per_seq, ctx_begin,
                          ctx_len, B, num_parts, workspace, ws_bytes, stream=None):
    _check(load().mla_decode_attn_range(handle, _ptr(q_abs), _ptr(cache), cache_len, _ptr(block_table),
                                        max_blocks_per_seq, _ptr(ctx_begin), _ptr(ctx_len), B, num_parts,
                                        _ptr(workspace), ws_bytes, _stream(stream)), "mla_decode_attn_range")


def mla_combine_splits_f32(handle, workspace, ws_bytes, B, num_parts, ctx_lat, lse, stream=None):
    _check(load().mla_combine_splits_f32(handle, _ptr(workspace), ws_bytes, B, num_parts, _ptr(ctx_lat),
                                         _ptr(lse), _stream(stream)), "mla_combine_splits_f32")


def mla_merge_ranges(handle, ctx_parts, lse_parts, R, B, ctx_lat, lse=None, stream=None):
    _check(load().mla_merge_ranges(handle, _ptr(ctx_parts), _ptr(lse_parts), R, B, _ptr(ctx_lat), _ptr(lse),
                                   _stream(stream)), "mla_merge_ranges")


def mla_combine_splits(handle, workspace, ws_bytes, B, num_parts, ctx_lat, lse=None, stream=None):
    _check(load().mla_combine_splits(handle, _ptr(workspace), ws_bytes, B, num_parts,
                                     _ptr(ctx_lat), _ptr(lse), _stream(stream)),
           "mla_combine_splits")


def mla_query_proj(handle, x, B, w_dq, d_cq, w_uq, w_qr, c_q, q_nope, q_rope, stream=None):
    _check(load().mla_query_proj(handle, _ptr(x), B, _ptr(w_dq), d_cq, _ptr(w_uq), _ptr(w_qr),
                                 _ptr(c_q), _ptr(q_nope), _ptr(q_rope), _stream(stream)),
           "mla_query_proj")


def mla_out_proj(handle, ctx_lat, w_uv, w_o, o, u, B, stream=None):
    _check(load().mla_out_proj(handle, _ptr(ctx_lat), _ptr(w_uv), _ptr(w_o), _ptr(o), _ptr(u), B,
                               _stream(stream)), "mla_out_proj")


def mla_combine_out_proj(handle, workspace, ws_bytes, B, num_parts, w_uv, w_o, o, u=None, ctx_lat=None, lse=None,
                         stream=None):
    _check(load().mla_combine_out_proj(handle, _ptr(workspace), ws_bytes, B, num_parts, _ptr(w_uv), _ptr(w_o),
                                       _ptr(o), _ptr(u), _ptr(ctx_lat), _ptr(lse), _stream(stream)),
           "mla_combine_out_proj")


def mla_get_device_status(handle, stream=None) -> int:
    return load().mla_get_device_status(handle, _stream(stream))


def mla_decode_attn_combine_noalloc(handle, q_abs, cache, cache_len, block_table,
                                    max_blocks_per_seq, ctx_len, B, num_parts, ctx_lat, lse=None,
                                    stream=None):
    """Attention plus combine with the library's fixed scratch array (no
    device allocation; see include/mla.h)."""
    _check(load().mla_decode_attn_combine_noalloc(
        handle, _ptr(q_abs), _ptr(cache), cache_len, _ptr(block_table), max_blocks_per_seq,
        _ptr(ctx_len), B, num_parts, _ptr(ctx_lat), _ptr(lse), _stream(stream)),
        "mla_decode_attn_combine_noalloc")


def mla_noalloc_scratch_bytes() -> int:
    return load().mla_noalloc_scratch_bytes()


def mla_plan_pieces_tiled(ctx_len, num_parts, tile_tokens):
    """Host mirror of the split plan with tiles of tile_tokens tokens."""
    B = len(ctx_len)
    arr = (ctypes.c_int * max(B, 1))(*[int(c) for c in ctx_len])
    base = (ctypes.c_longlong * (B + 1))()
    n = load().mla_plan_pieces_tiled(ctypes.cast(arr, ctypes.c_void_p), B, num_parts, tile_tokens,
                                     ctypes.cast(base, ctypes.c_void_p))
    return n, list(base)


def mla_plan_tile(handle, fp8=False):
    return load().mla_plan_tile(handle, 1 if fp8 else 0)


def mla_plan_pieces(ctx_len, num_parts):
    """Host mirror of the split plan: returns (n_pieces, piece_base list of B+1)."""
    B = len(ctx_len)
    arr = (ctypes.c_int * max(B, 1))(*[int(c) for c in ctx_len])
    base = (ctypes.c_longlong * (B + 1))()
    n = load().mla_plan_pieces(ctypes.cast(arr, ctypes.c_void_p), B, num_parts,
                               ctypes.cast(base, ctypes.c_void_p))
    return n, list(base)
