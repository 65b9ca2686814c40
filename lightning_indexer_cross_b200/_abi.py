"""ctypes binding of ``libindexcache.so`` (declared in ``include/indexcache.h``).

Argument marshalling only: each function here forwards to the C entry point of
the same name. There is no Python or CPU implementation behind any of them;
if the library is missing the import of this module fails loudly.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libindexcache.so")

IC_OK = 0
IC_ERR_INVALID_ARG = 1
IC_ERR_UNSUPPORTED = 2
IC_ERR_CUDA = 3
IC_ERR_TIMEOUT = 4
IC_ERR_BAD_INDEX = 5

IC_BF16 = 0
IC_FP8_E4M3 = 1
IC_F32 = 2

# every symbol include/indexcache.h declares
EXPORTED = [
    "ic_status_string",
    "ic_indexer_score",
    "ic_indexer_workspace_size",
    "ic_topk",
    "ic_topk_workspace_size",
    "ic_topk_noalloc",
    "ic_indexer_topk",
    "ic_indexer_topk_workspace_size",
    "ic_sparse_mla_decode",
    "ic_sparse_mla_workspace_size",
    "ic_layer_stack",
    "ic_layer_stack_workspace_size",
    "ic_cache_append",
    "ic_cache_append_workspace_size",
    "ic_decompress_gate",
    "ic_decompress_gate_workspace_size",
    "ic_last_device_status",
    "ic_last_launch_count",
    "ic_set_wait_limit_ns",
    "ic_wait_limit_ns",
    "ic_cp_candidates",
    "ic_cp_workspace_size",
    "ic_cp_merge_topk",
    "ic_cp_combine",
    "ic_index_overlap",
]


class ICError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__(f"{where}: {ic_status_string(code)}")


if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python -m lightning_indexer_cross_b200.build` "
        "(there is no fallback implementation)")

_lib = ctypes.CDLL(LIB_PATH)

_p = ctypes.c_void_p
_i = ctypes.c_int
_i64 = ctypes.c_int64
_sz = ctypes.c_size_t
_f = ctypes.c_float


class ic_stack_shape_t(ctypes.Structure):
    _fields_ = [
        ("B", _i), ("N", _i64), ("H_I", _i), ("d_I", _i), ("k_dtype", _i), ("topk", _i), ("H", _i),
        ("sm_scale", _f), ("out_dtype", _i), ("k_batch_stride", _i64), ("scale_batch_stride", _i64),
        ("kv_batch_stride", _i64), ("n_valid", _p), ("rows_per_pass", _i),
    ]


class ic_layer_t(ctypes.Structure):
    _fields_ = [
        ("q_idx", _p), ("w", _p), ("k_idx", _p), ("k_scale", _p), ("q", _p), ("kv", _p), ("sink", _p),
        ("gate", _p), ("out", _p), ("lse", _p), ("wait_event", _p),
    ]


def _sig(name, res, args):
    fn = getattr(_lib, name)
    fn.restype = res
    fn.argtypes = args
    return fn


_status_string = _sig("ic_status_string", ctypes.c_char_p, [_i])
_indexer = _sig("ic_indexer_score", _i, [_p, _p, _p, _p, _i, _i, _i, _i, _i64, _i64, _i64, _p, _p, _p, _sz, _p])
_indexer_ws = _sig("ic_indexer_workspace_size", _sz, [])
_topk = _sig("ic_topk", _i, [_p, _i, _i64, _p, _i, _p, _p, _sz, _p])
_topk_ws = _sig("ic_topk_workspace_size", _sz, [_i, _i64, _i])
_indexer_topk = _sig("ic_indexer_topk", _i,
                     [_p, _p, _p, _p, _i, _i, _i, _i, _i64, _i64, _i64, _p, _i, _i, _p, _p, _sz, _p])
_indexer_topk_ws = _sig("ic_indexer_topk_workspace_size", _sz, [_i, _i64, _i, _i])
_topk_noalloc = _sig("ic_topk_noalloc", _i, [_p, _i, _i64, _p, _i, _p, _p])
_mla = _sig("ic_sparse_mla_decode", _i,
            [_p, _p, _i64, _i64, _p, _i, _p, _p, _f, _i, _i, _i, _p, _p, _p, _sz, _p])
_mla_ws = _sig("ic_sparse_mla_workspace_size", _sz, [_i, _i, _i])
_stack = _sig("ic_layer_stack", _i,
              [ctypes.POINTER(ic_layer_t), _i, ctypes.c_char_p, ctypes.POINTER(ic_stack_shape_t), _p, _p, _p,
               _sz, _p])
_stack_ws = _sig("ic_layer_stack_workspace_size", _sz, [ctypes.POINTER(ic_stack_shape_t)])
_append = _sig("ic_cache_append", _i,
               [_p, _p, _p, _f, _i, _p, _p, _i64, _i64, _p, _p, _i64, _p, _i, _i, _i64, _f, _p, _p, _i, _i, _p, _sz,
                _p])
_append_ws = _sig("ic_cache_append_workspace_size", _sz, [])
_gate = _sig("ic_decompress_gate", _i, [_p, _p, _p, _i, _i, _i, _i, _p, _p, _sz, _p])
_gate_ws = _sig("ic_decompress_gate_workspace_size", _sz, [])
_last_status = _sig("ic_last_device_status", _i, [_p, _p])
_last_launches = _sig("ic_last_launch_count", _i, [])
_cp_cand = _sig("ic_cp_candidates", _i, [_p, _p, _i, _i64, _i, _i64, _p, _p, _p, _sz, _p])
_cp_ws = _sig("ic_cp_workspace_size", _sz, [])
_cp_merge = _sig("ic_cp_merge_topk", _i, [_p, _p, _i64, _i, _i, _i, _i, _i64, _i64, _p, _p, _p])
_cp_combine = _sig("ic_cp_combine", _i, [_p, _i64, _p, _i64, _i, _i, _i, _p, _p, _i, _p, _p, _p])
_overlap = _sig("ic_index_overlap", _i, [_p, _p, _i, _i, _i64, _p, _p])
_set_wait = _sig("ic_set_wait_limit_ns", None, [ctypes.c_uint64])
_get_wait = _sig("ic_wait_limit_ns", ctypes.c_uint64, [])


def ic_status_string(code: int) -> str:
    return _status_string(int(code)).decode()


def _check(code: int, where: str) -> None:
    if code != IC_OK:
        raise ICError(code, where)


def ic_indexer_score(q, w, k, k_scale, k_dtype, B, H_I, d_I, N, k_batch_stride, scale_batch_stride, n_valid,
                     scores, workspace, ws_bytes, stream) -> None:
    _check(_indexer(q, w, k, k_scale, k_dtype, B, H_I, d_I, N, k_batch_stride, scale_batch_stride, n_valid,
                    scores, workspace, ws_bytes, stream), "ic_indexer_score")


def ic_indexer_workspace_size() -> int:
    return int(_indexer_ws())


def ic_topk(scores, B, N, n_valid, k, idx, workspace, ws_bytes, stream) -> None:
    _check(_topk(scores, B, N, n_valid, k, idx, workspace, ws_bytes, stream), "ic_topk")


def ic_indexer_topk(q, w, k, k_scale, k_dtype, B, H_I, d_I, N, k_batch_stride, scale_batch_stride, n_valid, topk,
                    rows_per_pass, idx, workspace, ws_bytes, stream) -> None:
    _check(_indexer_topk(q, w, k, k_scale, k_dtype, B, H_I, d_I, N, k_batch_stride, scale_batch_stride, n_valid,
                         topk, rows_per_pass, idx, workspace, ws_bytes, stream), "ic_indexer_topk")


def ic_indexer_topk_workspace_size(B, N, k, rows_per_pass) -> int:
    return int(_indexer_topk_ws(B, N, k, rows_per_pass))


def ic_topk_noalloc(scores, B, N, n_valid, k, idx, stream) -> None:
    """Top-k with the library's built-in scratch (no workspace argument)."""
    _check(_topk_noalloc(scores, B, N, n_valid, k, idx, stream), "ic_topk_noalloc")


IC_TOPK_NOALLOC_MAX_ROWS = 64


def ic_topk_workspace_size(B, N, k) -> int:
    return int(_topk_ws(B, N, k))


def ic_sparse_mla_decode(q, kv, kv_batch_stride, N, idx, k, sink, gate, sm_scale, B, H, out_dtype, out, lse,
                         workspace, ws_bytes, stream) -> None:
    _check(_mla(q, kv, kv_batch_stride, N, idx, k, sink, gate, sm_scale, B, H, out_dtype, out, lse, workspace,
                ws_bytes, stream), "ic_sparse_mla_decode")


def ic_sparse_mla_workspace_size(B, H, k) -> int:
    return int(_mla_ws(B, H, k))


def ic_layer_stack(layers, L, schedule: bytes, shape, index_buf, idx_trace, workspace, ws_bytes, stream) -> None:
    _check(_stack(layers, L, schedule, ctypes.byref(shape), index_buf, idx_trace, workspace, ws_bytes, stream),
           "ic_layer_stack")


def ic_layer_stack_workspace_size(shape) -> int:
    return int(_stack_ws(ctypes.byref(shape)))


def ic_cache_append(k_raw, ln_gamma, ln_beta, ln_eps, k_dtype, key_cache, key_scale, k_batch_stride,
                    scale_batch_stride, kv_raw, kv_cache, kv_batch_stride, pos, T, d_I, N, rope_base, q, q_pos, B,
                    H, workspace, ws_bytes, stream) -> None:
    _check(_append(k_raw, ln_gamma, ln_beta, ln_eps, k_dtype, key_cache, key_scale, k_batch_stride,
                   scale_batch_stride, kv_raw, kv_cache, kv_batch_stride, pos, T, d_I, N, rope_base, q, q_pos, B, H,
                   workspace, ws_bytes, stream), "ic_cache_append")


def ic_cache_append_workspace_size() -> int:
    return int(_append_ws())


def ic_decompress_gate(o_latent, wv_b, gate, B, H, d_v, out_dtype, out, workspace, ws_bytes, stream) -> None:
    _check(_gate(o_latent, wv_b, gate, B, H, d_v, out_dtype, out, workspace, ws_bytes, stream),
           "ic_decompress_gate")


def ic_decompress_gate_workspace_size() -> int:
    return int(_gate_ws())


def ic_last_device_status(workspace, stream) -> int:
    return int(_last_status(workspace, stream))


def ic_last_launch_count() -> int:
    return int(_last_launches())


def ic_cp_candidates(scores, idx, B, N_local, k, offset, cand_score, cand_idx, workspace, ws_bytes, stream) -> None:
    _check(_cp_cand(scores, idx, B, N_local, k, offset, cand_score, cand_idx, workspace, ws_bytes, stream),
           "ic_cp_candidates")


def ic_cp_workspace_size() -> int:
    return int(_cp_ws())


def ic_cp_merge_topk(cand_score, cand_idx, seg_stride, G, B, kin, k, lo, hi, idx_global, idx_local, stream) -> None:
    _check(_cp_merge(cand_score, cand_idx, seg_stride, G, B, kin, k, lo, hi, idx_global, idx_local, stream),
           "ic_cp_merge_topk")


def ic_cp_combine(part_out, out_stride, part_lse, lse_stride, G, B, H, sink, gate, out_dtype, out, lse,
                  stream) -> None:
    _check(_cp_combine(part_out, out_stride, part_lse, lse_stride, G, B, H, sink, gate, out_dtype, out, lse, stream),
           "ic_cp_combine")


def ic_index_overlap(a, b, B, k, N, count, stream) -> None:
    _check(_overlap(a, b, B, k, N, count, stream), "ic_index_overlap")


IC_CP_MAX_CANDIDATES = 16384


def ic_set_wait_limit_ns(ns: int) -> None:
    """Bound (ns) of every wait inside kernels enqueued from now on; 0 gives up
    any wait not already satisfied (failure-path tests)."""
    _set_wait(int(ns))


def ic_wait_limit_ns() -> int:
    return int(_get_wait())


def raw_function(name: str):
    """The raw ctypes function object of an exported symbol (for tests)."""
    return getattr(_lib, name)
