"""ctypes binding of ``libmla.so`` (include/mla.h): the same names, argument
marshalling only. Every step of the decode runs in the library's CUDA
kernels; there is no fallback. Importing this module without the built
library raises ``RuntimeError``.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.environ.get("MLA_LIB", os.path.join(_HERE, "libmla.so"))

MLA_OK = 0
MLA_ERR_INVALID_ARG = 1
MLA_ERR_UNSUPPORTED = 2
MLA_ERR_WORKSPACE_TOO_SMALL = 3
MLA_ERR_CUDA = 4
MLA_ERR_DEVICE_BOUNDS = 5
MLA_ERR_DEVICE_TIMEOUT = 6

MLA_DEVERR_SEQ_LEN = 0x1
MLA_DEVERR_PAGE_ID = 0x2
MLA_DEVERR_INDEX = 0x4
MLA_DEVERR_TIMEOUT = 0x8
MLA_DEVERR_POSITION = 0x10

EXPORTED = (
    "mla_plan_bytes", "mla_workspace_bytes", "mla_num_workers", "mla_decode_plan", "mla_decode",
    "mla_combine", "mla_get_error", "mla_status_string", "mla_decode_noalloc", "mla_cache_insert",
    "mla_absorb_query", "mla_unabsorb_output", "mla_index_scores", "mla_topk", "mla_merge", "mla_decode_fp8",
    "mla_cache_insert_fp8",
)

DEFAULT_SOFTMAX_SCALE = 1.0 / math.sqrt(192.0)


class mla_decode_desc_t(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("q_len", ctypes.c_int32),
        ("num_heads", ctypes.c_int32),
        ("d_latent", ctypes.c_int32),
        ("d_rope", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32),
        ("topk", ctypes.c_int32),
        ("causal", ctypes.c_int32),
        ("softmax_scale", ctypes.c_float),
        ("num_sms", ctypes.c_int32),
    ]


def make_desc(*, batch: int, q_len: int, num_heads: int, num_pages: int, max_pages_per_seq: int, topk: int = 0,
              causal: bool = False, softmax_scale: float = DEFAULT_SOFTMAX_SCALE, num_sms: int = 0,
              d_latent: int = 512, d_rope: int = 64, page_size: int = 64) -> mla_decode_desc_t:
    return mla_decode_desc_t(batch, q_len, num_heads, d_latent, d_rope, page_size, num_pages, max_pages_per_seq,
                             topk, int(bool(causal)), softmax_scale, num_sms)


class mla_insert_desc_t(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int32),
        ("batch", ctypes.c_int32),
        ("max_pages_per_seq", ctypes.c_int32),
        ("num_pages", ctypes.c_int32),
        ("max_positions", ctypes.c_int32),
        ("d_latent", ctypes.c_int32),
        ("d_rope", ctypes.c_int32),
        ("page_size", ctypes.c_int32),
        ("eps", ctypes.c_float),
    ]


def make_insert_desc(*, num_tokens: int, batch: int, max_pages_per_seq: int, num_pages: int, max_positions: int,
                     eps: float = 1e-6, d_latent: int = 512, d_rope: int = 64,
                     page_size: int = 64) -> mla_insert_desc_t:
    return mla_insert_desc_t(num_tokens, batch, max_pages_per_seq, num_pages, max_positions, d_latent, d_rope,
                             page_size, eps)


class mla_absorb_desc_t(ctypes.Structure):
    _fields_ = [
        ("num_tokens", ctypes.c_int32),
        ("num_heads", ctypes.c_int32),
        ("d_nope", ctypes.c_int32),
        ("d_rope", ctypes.c_int32),
        ("d_latent", ctypes.c_int32),
        ("d_v", ctypes.c_int32),
    ]


def make_absorb_desc(*, num_tokens: int, num_heads: int, d_nope: int = 128, d_rope: int = 64, d_latent: int = 512,
                     d_v: int = 128) -> mla_absorb_desc_t:
    return mla_absorb_desc_t(num_tokens, num_heads, d_nope, d_rope, d_latent, d_v)


class mla_index_desc_t(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32),
        ("q_len", ctypes.c_int32),
        ("num_heads", ctypes.c_int32),
        ("head_dim", ctypes.c_int32),
        ("num_keys", ctypes.c_int32),
    ]


def make_index_desc(*, batch: int, q_len: int, num_heads: int, num_keys: int, head_dim: int = 128) -> mla_index_desc_t:
    return mla_index_desc_t(batch, q_len, num_heads, head_dim, num_keys)


class mla_topk_desc_t(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int32),
        ("num_keys", ctypes.c_int32),
        ("k", ctypes.c_int32),
    ]


def make_topk_desc(*, rows: int, num_keys: int, k: int) -> mla_topk_desc_t:
    return mla_topk_desc_t(rows, num_keys, k)


class mla_merge_desc_t(ctypes.Structure):
    _fields_ = [
        ("parts", ctypes.c_int32),
        ("d_latent", ctypes.c_int32),
        ("rows", ctypes.c_int64),
    ]


def make_merge_desc(*, parts: int, rows: int, d_latent: int = 512) -> mla_merge_desc_t:
    return mla_merge_desc_t(parts, d_latent, rows)


def load_library(path: str) -> ctypes.CDLL:
    """A handle on a build of the library at ``path`` with every C signature set."""
    if not os.path.exists(path):
        raise RuntimeError(
            f"libmla.so is not built ({path} missing): run `python -m mla_latent_kv_26_b200.build` "
            "(there is no non-CUDA fallback)")
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    D = ctypes.POINTER(mla_decode_desc_t)
    sig = {
        "mla_plan_bytes": (ctypes.c_size_t, [D]),
        "mla_workspace_bytes": (ctypes.c_size_t, [D]),
        "mla_num_workers": (ctypes.c_int32, [D]),
        "mla_decode_plan": (ctypes.c_int, [D, P, P, ctypes.c_size_t, P]),
        "mla_decode": (ctypes.c_int, [D, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]),
        "mla_combine": (ctypes.c_int, [D, P, P, ctypes.c_size_t, P, P, P]),
        "mla_get_error": (ctypes.c_int, [P, ctypes.POINTER(ctypes.c_uint32), P]),
        "mla_status_string": (ctypes.c_char_p, [ctypes.c_int]),
        "mla_decode_noalloc": (ctypes.c_int, [D, P, P, P, P, P, P, P, P]),
        "mla_cache_insert": (ctypes.c_int, [ctypes.POINTER(mla_insert_desc_t), P, P, P, P, P, P, P, P, P, P]),
        "mla_absorb_query": (ctypes.c_int, [ctypes.POINTER(mla_absorb_desc_t), P, P, P, P, P]),
        "mla_unabsorb_output": (ctypes.c_int, [ctypes.POINTER(mla_absorb_desc_t), P, P, P, P, P]),
        "mla_index_scores": (ctypes.c_int, [ctypes.POINTER(mla_index_desc_t), P, P, P, P, P, P, P]),
        "mla_topk": (ctypes.c_int, [ctypes.POINTER(mla_topk_desc_t), P, P, P, P]),
        "mla_merge": (ctypes.c_int, [ctypes.POINTER(mla_merge_desc_t), P, P, P, P, P]),
        "mla_decode_fp8": (ctypes.c_int, [D, P, P, P, P, P, P, P, P, P, ctypes.c_size_t, P]),
        "mla_cache_insert_fp8": (ctypes.c_int, [ctypes.POINTER(mla_insert_desc_t), P, P, P, P, P, P, P, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


_lib = load_library(LIB_PATH)


def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(s) -> Optional[int]:
    if s is None:
        return None
    if isinstance(s, int):
        return s
    return s.cuda_stream


class MlaError(RuntimeError):
    def __init__(self, status: int, what: str):
        super().__init__(f"{what}: {mla_status_string(status)} ({status})")
        self.status = status


def mla_status_string(status: int) -> str:
    return _lib.mla_status_string(int(status)).decode()


def mla_plan_bytes(desc: mla_decode_desc_t) -> int:
    return int(_lib.mla_plan_bytes(ctypes.byref(desc)))


def mla_workspace_bytes(desc: mla_decode_desc_t) -> int:
    return int(_lib.mla_workspace_bytes(ctypes.byref(desc)))


def mla_num_workers(desc: mla_decode_desc_t) -> int:
    return int(_lib.mla_num_workers(ctypes.byref(desc)))


def mla_decode_plan(desc, seq_lens, plan, plan_bytes: int, stream=None) -> int:
    return int(_lib.mla_decode_plan(ctypes.byref(desc), _ptr(seq_lens), _ptr(plan), int(plan_bytes),
                                    _stream(stream)))


def mla_decode(desc, plan, q, kv_cache, block_table, seq_lens, topk_indices, out, lse, workspace,
               workspace_bytes: int, stream=None) -> int:
    return int(_lib.mla_decode(ctypes.byref(desc), _ptr(plan), _ptr(q), _ptr(kv_cache), _ptr(block_table),
                               _ptr(seq_lens), _ptr(topk_indices), _ptr(out), _ptr(lse), _ptr(workspace),
                               int(workspace_bytes), _stream(stream)))


def mla_decode_fp8(desc, plan, q, kv_cache_fp8, block_table, seq_lens, topk_indices, out, lse, workspace,
                   workspace_bytes: int, stream=None) -> int:
    """mla_decode over an fp8 latent cache [pages, 64, 656] bytes."""
    return int(_lib.mla_decode_fp8(ctypes.byref(desc), _ptr(plan), _ptr(q), _ptr(kv_cache_fp8), _ptr(block_table),
                                   _ptr(seq_lens), _ptr(topk_indices), _ptr(out), _ptr(lse), _ptr(workspace),
                                   int(workspace_bytes), _stream(stream)))


def mla_cache_insert_fp8(desc, kv, weight, cos_table, sin_table, seq_ids, positions, block_table, kv_cache_fp8,
                         error_word=None, stream=None) -> int:
    """mla_cache_insert writing the fp8 cache format."""
    return int(_lib.mla_cache_insert_fp8(ctypes.byref(desc), _ptr(kv), _ptr(weight), _ptr(cos_table),
                                         _ptr(sin_table), _ptr(seq_ids), _ptr(positions), _ptr(block_table),
                                         _ptr(kv_cache_fp8), _ptr(error_word), _stream(stream)))


def mla_combine(desc, plan, workspace, workspace_bytes: int, out, lse, stream=None) -> int:
    return int(_lib.mla_combine(ctypes.byref(desc), _ptr(plan), _ptr(workspace), int(workspace_bytes), _ptr(out),
                                _ptr(lse), _stream(stream)))


def mla_decode_noalloc(desc, seq_lens, q, kv_cache, block_table, topk_indices, out, lse, stream=None) -> int:
    """Plan + decode + combine with the library's fixed device scratch (no allocation)."""
    return int(_lib.mla_decode_noalloc(ctypes.byref(desc), _ptr(seq_lens), _ptr(q), _ptr(kv_cache), _ptr(block_table),
                                       _ptr(topk_indices), _ptr(out), _ptr(lse), _stream(stream)))


def mla_cache_insert(desc, kv, weight, cos_table, sin_table, seq_ids, positions, block_table, kv_cache,
                     error_word=None, stream=None) -> int:
    """kv_norm + RoPE of new tokens, written into their rows of the paged cache."""
    return int(_lib.mla_cache_insert(ctypes.byref(desc), _ptr(kv), _ptr(weight), _ptr(cos_table), _ptr(sin_table),
                                     _ptr(seq_ids), _ptr(positions), _ptr(block_table), _ptr(kv_cache),
                                     _ptr(error_word), _stream(stream)))


def mla_absorb_query(desc, q, wkv_b, q_abs, error_word=None, stream=None) -> int:
    """q [T,H,192] -> q_abs [T,H,576] = (W_UK^T q_nope || q_pe)."""
    return int(_lib.mla_absorb_query(ctypes.byref(desc), _ptr(q), _ptr(wkv_b), _ptr(q_abs), _ptr(error_word),
                                     _stream(stream)))


def mla_unabsorb_output(desc, o_lat, wkv_b, out, error_word=None, stream=None) -> int:
    """o_lat [T,H,512] -> out [T,H,128] = W_UV o_lat."""
    return int(_lib.mla_unabsorb_output(ctypes.byref(desc), _ptr(o_lat), _ptr(wkv_b), _ptr(out), _ptr(error_word),
                                        _stream(stream)))


def mla_index_scores(desc, q, q_s, k, k_s, scores, error_word=None, stream=None) -> int:
    """fp8 index scores [b, m, n] of every key for every query token."""
    return int(_lib.mla_index_scores(ctypes.byref(desc), _ptr(q), _ptr(q_s), _ptr(k), _ptr(k_s), _ptr(scores),
                                     _ptr(error_word), _stream(stream)))


def mla_topk(desc, scores, valid_lens, indices, stream=None) -> int:
    """Top-k positions of each score row, increasing, -1 padded."""
    return int(_lib.mla_topk(ctypes.byref(desc), _ptr(scores), _ptr(valid_lens), _ptr(indices), _stream(stream)))


def mla_merge(desc, part_out, part_lse, out, lse, stream=None) -> int:
    """LSE merge of per-shard decode results [parts, rows, 512] / [parts, rows]."""
    return int(_lib.mla_merge(ctypes.byref(desc), _ptr(part_out), _ptr(part_lse), _ptr(out), _ptr(lse),
                              _stream(stream)))


def mla_get_error(plan, stream=None):
    """Synchronises ``stream``; returns ``(status, error_bits)``."""
    bits = ctypes.c_uint32(0)
    st = int(_lib.mla_get_error(_ptr(plan), ctypes.byref(bits), _stream(stream)))
    return st, int(bits.value)


def check(status: int, what: str) -> None:
    if status != MLA_OK:
        raise MlaError(status, what)
