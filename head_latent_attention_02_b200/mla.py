"""Python binding of libmla (include/mla.h): argument marshalling only.

Every step runs in the library's CUDA kernels; this module turns torch
tensors into pointers and sizes, calls the C ABI and raises on a non-OK
status.  It fails loudly when libmla.so is missing -- there is no fallback.
"""
from __future__ import annotations

import ctypes
import os
import re
from typing import Optional, Sequence

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmla.so")
HEADER = os.path.join(os.path.dirname(_PKG), "include", "mla.h")

MLA_F32, MLA_BF16 = 0, 1
STATUS = {0: "MLA_OK", 1: "MLA_ERR_INVALID_ARG", 2: "MLA_ERR_UNSUPPORTED", 3: "MLA_ERR_WORKSPACE",
          4: "MLA_ERR_CUDA", 5: "MLA_ERR_TIMEOUT", 6: "MLA_ERR_BAD_INDEX"}


class MLAError(RuntimeError):
    def __init__(self, fn: str, code: int):
        super().__init__(f"{fn} returned {STATUS.get(code, code)}")
        self.code = code


class Dims(ctypes.Structure):
    _fields_ = [("H", ctypes.c_int32), ("d_c", ctypes.c_int32), ("d_r", ctypes.c_int32),
                ("d_n", ctypes.c_int32), ("d_v", ctypes.c_int32), ("d_model", ctypes.c_int32),
                ("page_size", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("scale", ctypes.c_float), ("rope_base", ctypes.c_double)]


_lib = None
_vp, _i32, _i64, _sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t
_SIGS = {
    "mla_abi_version": ([], _i32),
    "mla_status_str": ([_i32], ctypes.c_char_p),
    "mla_get_status": ([_vp], _i32),
    "mla_absorb_q": ([ctypes.POINTER(Dims), _i32, _vp, _vp, _vp, ctypes.POINTER(_i32), _i32, _vp,
                      _vp, _vp], _i32),
    "mla_decode": ([ctypes.POINTER(Dims), _i32, _i32, _vp, _i32, _vp, _i32, _vp, _i64, _vp, _i32,
                    _vp, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp], _i32),
    "mla_decode_workspace_size": ([ctypes.POINTER(Dims), _i32, _i32, _i32, _i32], _sz),
    "mla_decode_static_ws": ([ctypes.POINTER(Dims), _i32, _i32, _vp, _i32, _vp, _i32, _vp, _i64,
                              _vp, _i32, _vp, _i32, _vp, _vp, _i32, _vp, _vp, _vp, _vp], _i32),
    "mla_decode_static_ws_init": ([], _i32),
    "mla_merge_lse": ([_i32, _i32, _vp, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _vp, _vp], _i32),
    "mla_out_proj": ([ctypes.POINTER(Dims), _i32, _vp, _vp, _vp, _vp, _vp, _vp], _i32),
    "mla_append_rows": ([ctypes.POINTER(Dims), _i32, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i64,
                         _vp, _i32, _vp, ctypes.c_float, _vp, _vp], _i32),
    "mla_qknorm_query": ([ctypes.POINTER(Dims), _i32, _vp, _vp, _vp, ctypes.c_float, _vp, _vp],
                         _i32),
    "mla_qknorm_key_gram": ([ctypes.POINTER(Dims), _vp, _vp, _vp], _i32),
    "mla_debug_wait_probe": ([_i64, _vp, _vp], _i32),
    "mla_pack_rows": ([ctypes.POINTER(Dims), _i32, _i32, _i64, _vp, _vp, _vp, _vp, _vp], _i32),
    "mla_decode_lowbit": ([ctypes.POINTER(Dims), _i32, _i32, _i32, _i32, _vp, _i32, _vp, _i32,
                           _vp, _vp, _vp, _i64, _vp, _i32, _vp, _i32, _vp, _vp, _i32, _vp, _vp,
                           _vp, _vp], _i32),
    "mla_lowbit_dequant_bytes": ([ctypes.POINTER(Dims), _i64], _sz),
    "mla_dequant_rows": ([ctypes.POINTER(Dims), _i32, _i32, _i64, _vp, _vp, _vp, _vp, _vp], _i32),
    "mla_decode_lowbit_tc": ([ctypes.POINTER(Dims), _i32, _i32, _i32, _i32, _vp, _i32, _vp, _i32,
                              _vp, _vp, _vp, _i64, _vp, _i32, _vp, _i32, _vp, _vp, _i32, _vp, _vp,
                              _vp, _vp, _sz, _vp, _sz, _vp], _i32),
    "mla_decode_qknorm": ([ctypes.POINTER(Dims), _i32, _i32, _vp, _i32, _vp, _i32, _vp, _vp, _i64,
                           _vp, _i32, _vp, _i32, _vp, _vp, _vp, _vp, _sz, _vp], _i32),
}


def lib() -> ctypes.CDLL:
    """Load libmla.so (built in-tree); raises if it is missing."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libmla.so not built at {LIB_PATH}: run "
                               "`python -m head_latent_attention_02_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            f = getattr(L, name)
            f.argtypes = args
            f.restype = res
        _lib = L
    return _lib


def header_symbols() -> list:
    """Entry points declared in include/mla.h."""
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?[\w\*]+\s+\*?(mla_\w+)\s*\(", txt, re.M)))


def make_dims(wl, dtype: Optional[int] = None) -> Dims:
    return Dims(wl.H, wl.d_c, wl.d_r, wl.d_n, wl.d_v, wl.d_model, 64,
                (MLA_BF16 if wl.dtype == "bf16" else MLA_F32) if dtype is None else dtype,
                wl.scale, wl.rope_base)


def _p(t: Optional[torch.Tensor]):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return t.data_ptr()


def _s(stream) -> Optional[int]:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(fn: str, code: int):
    if code != 0:
        raise MLAError(fn, code)


def status_str(code: int) -> str:
    return lib().mla_status_str(code).decode()


def get_status(stream=None) -> int:
    """Waits for the stream and returns (and clears) the device status word."""
    return int(lib().mla_get_status(_s(stream)))


def absorb_q(dims: Dims, q_nope, q_rope, q_pos, deltas: Sequence[int], w_uk, q_abs, stream=None):
    n_q = q_nope.shape[0]
    arr = (_i32 * len(deltas))(*[int(d) for d in deltas])
    _check("mla_absorb_q", lib().mla_absorb_q(ctypes.byref(dims), n_q, _p(q_nope), _p(q_rope),
                                              _p(q_pos), arr, len(deltas), _p(w_uk), _p(q_abs),
                                              _s(stream)))


def workspace_size(dims: Dims, B: int, s_q: int, n_h: int, n_ver: int = 1) -> int:
    return int(lib().mla_decode_workspace_size(ctypes.byref(dims), B, s_q, n_ver, n_h))


def decode(dims: Dims, B: int, s_q: int, q_abs, n_ver: int, head_ids, n_h: int, cache,
           block_table, segs, q_pos, o_lat, lse, workspace, gather_rows=None, n_gather=None,
           stream=None):
    """mla_decode; ``head_ids`` is an int32 device tensor of n_h head ids, or
    None for heads 0 .. n_h-1."""
    n_pages = cache.shape[0]
    max_pages = block_table.shape[1]
    max_segs = segs.shape[1]
    max_gather = gather_rows.shape[1] if gather_rows is not None else 0
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("mla_decode", lib().mla_decode(
        ctypes.byref(dims), B, s_q, _p(q_abs), n_ver, _p(head_ids), n_h, _p(cache), n_pages,
        _p(block_table), max_pages, _p(segs), max_segs, _p(gather_rows), _p(n_gather),
        max_gather, _p(q_pos), _p(o_lat), _p(lse), _p(workspace), ws_bytes, _s(stream)))


def decode_static_ws(dims: Dims, B: int, s_q: int, q_abs, n_ver: int, head_ids, n_h: int, cache,
                     block_table, segs, q_pos, o_lat, lse, gather_rows=None, n_gather=None,
                     stream=None):
    """mla_decode with the library's fixed scratch array instead of a workspace."""
    max_gather = gather_rows.shape[1] if gather_rows is not None else 0
    _check("mla_decode_static_ws", lib().mla_decode_static_ws(
        ctypes.byref(dims), B, s_q, _p(q_abs), n_ver, _p(head_ids), n_h, _p(cache), cache.shape[0],
        _p(block_table), block_table.shape[1], _p(segs), segs.shape[1], _p(gather_rows),
        _p(n_gather), max_gather, _p(q_pos), _p(o_lat), _p(lse), _s(stream)))


def decode_static_ws_init():
    """Loads the static scratch array on the current device."""
    _check("mla_decode_static_ws_init", lib().mla_decode_static_ws_init())


def merge_lse(n_q: int, H: int, head_ids, n_h: int, d: int, o_a, lse_a, o_b, lse_b, o, lse,
              stream=None):
    _check("mla_merge_lse", lib().mla_merge_lse(n_q, H, _p(head_ids), n_h, d, _p(o_a), _p(lse_a),
                                                _p(o_b), _p(lse_b), _p(o), _p(lse), _s(stream)))


def out_proj(dims: Dims, o_lat, w_uv, w_o, v, out, stream=None):
    n_q = o_lat.shape[0]
    _check("mla_out_proj", lib().mla_out_proj(ctypes.byref(dims), n_q, _p(o_lat), _p(w_uv),
                                              _p(w_o), _p(v), _p(out), _s(stream)))


def append_rows(dims, c_new, k_rope_raw, cache_pos, seq, row, cache, block_table,
                key_gram=None, qk_eps=0.0, key_inv_rms=None, stream=None):
    """mla_append_rows: entries i -> cache row (seq[i], row[i]) = [c | R(cache_pos) k_raw]
    (QK-normed caches: with key_gram, also key_inv_rms and a rescaled k_rope)."""
    _check("mla_append_rows", lib().mla_append_rows(
        ctypes.byref(dims), c_new.shape[0], _p(c_new), _p(k_rope_raw), _p(cache_pos), _p(seq),
        _p(row), block_table.shape[0], _p(cache), cache.shape[0], _p(block_table),
        block_table.shape[1], _p(key_gram), qk_eps, _p(key_inv_rms), _s(stream)))


def qknorm_query(dims, q_nope, g_q, g_k, eps, q_out, stream=None):
    _check("mla_qknorm_query", lib().mla_qknorm_query(
        ctypes.byref(dims), q_nope.shape[0], _p(q_nope), _p(g_q), _p(g_k), eps, _p(q_out),
        _s(stream)))


def qknorm_key_gram(dims, w_uk, gram, stream=None):
    _check("mla_qknorm_key_gram", lib().mla_qknorm_key_gram(ctypes.byref(dims), _p(w_uk),
                                                            _p(gram), _s(stream)))


def decode_qknorm(dims, B, s_q, q_abs, n_ver, head_ids, n_h, cache, key_inv_rms, block_table,
                  segs, q_pos, o_lat, lse, workspace, stream=None):
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("mla_decode_qknorm", lib().mla_decode_qknorm(
        ctypes.byref(dims), B, s_q, _p(q_abs), n_ver, _p(head_ids), n_h, _p(cache),
        _p(key_inv_rms), cache.shape[0], _p(block_table), block_table.shape[1], _p(segs),
        segs.shape[1], _p(q_pos), _p(o_lat), _p(lse), _p(workspace), ws_bytes, _s(stream)))


def pack_rows(dims, bits_c, bits_r, rows, scale_c, scale_r, packed, stream=None):
    """mla_pack_rows: rows [n, d_c + d_r] -> packed codes [n, row bytes]."""
    _check("mla_pack_rows", lib().mla_pack_rows(ctypes.byref(dims), bits_c, bits_r,
                                                rows.shape[0], _p(rows), _p(scale_c),
                                                _p(scale_r), _p(packed), _s(stream)))


def decode_lowbit(dims, bits_c, bits_r, B, s_q, q_abs, n_ver, head_ids, n_h, cache, scale_c,
                  scale_r, block_table, segs, q_pos, o_lat, lse, gather_rows=None, n_gather=None,
                  stream=None):
    """mla_decode_lowbit over a packed pool cache [n_pages, 64, row bytes] (uint8)."""
    max_gather = gather_rows.shape[1] if gather_rows is not None else 0
    _check("mla_decode_lowbit", lib().mla_decode_lowbit(
        ctypes.byref(dims), bits_c, bits_r, B, s_q, _p(q_abs), n_ver, _p(head_ids), n_h,
        _p(cache), _p(scale_c), _p(scale_r), cache.shape[0], _p(block_table),
        block_table.shape[1], _p(segs), segs.shape[1], _p(gather_rows), _p(n_gather),
        max_gather, _p(q_pos), _p(o_lat), _p(lse), _s(stream)))


def lowbit_dequant_bytes(dims, n_pages):
    """mla_lowbit_dequant_bytes: bytes of a dequantised pool of n_pages pages."""
    return lib().mla_lowbit_dequant_bytes(ctypes.byref(dims), n_pages)


def dequant_rows(dims, bits_c, bits_r, packed, scale_c, scale_r, out, stream=None):
    """mla_dequant_rows: packed codes [n, row bytes] -> out [n, d_c + d_r] (dtype)."""
    _check("mla_dequant_rows", lib().mla_dequant_rows(ctypes.byref(dims), bits_c, bits_r,
                                                      packed.shape[0], _p(packed), _p(scale_c),
                                                      _p(scale_r), _p(out), _s(stream)))


def decode_lowbit_tc(dims, bits_c, bits_r, B, s_q, q_abs, n_ver, head_ids, n_h, cache, scale_c,
                     scale_r, block_table, segs, q_pos, o_lat, lse, dequant, workspace,
                     gather_rows=None, n_gather=None, stream=None):
    """mla_decode_lowbit_tc over a packed pool cache [n_pages, 64, row bytes]
    (uint8), dequantising into ``dequant`` and decoding with ``workspace``."""
    max_gather = gather_rows.shape[1] if gather_rows is not None else 0
    dq_bytes = dequant.numel() * dequant.element_size()
    ws_bytes = workspace.numel() * workspace.element_size() if workspace is not None else 0
    _check("mla_decode_lowbit_tc", lib().mla_decode_lowbit_tc(
        ctypes.byref(dims), bits_c, bits_r, B, s_q, _p(q_abs), n_ver, _p(head_ids), n_h,
        _p(cache), _p(scale_c), _p(scale_r), cache.shape[0], _p(block_table),
        block_table.shape[1], _p(segs), segs.shape[1], _p(gather_rows), _p(n_gather),
        max_gather, _p(q_pos), _p(o_lat), _p(lse), _p(dequant), dq_bytes, _p(workspace),
        ws_bytes, _s(stream)))
