"""ctypes binding of ``libstd_b200.so`` -- the C ABI declared in include/std_b200.h.

Argument marshalling only: every function here has the name of a C entry
point, turns torch tensors into device pointers and the current torch stream
into a ``cudaStream_t``, calls the library and raises ``StdError`` on a
non-zero status.  No step of the method runs in Python, and nothing falls
back to another implementation: if the library is missing, the first call
raises.
"""
from __future__ import annotations

import ctypes
import os
import threading
from typing import Optional

PKG = os.path.dirname(os.path.abspath(__file__))
# STD_B200_DEBUG=1 loads the debug build: the same kernels compiled with device-side
# bounds checks of every index and cache row (STD_DEVERR_DEBUG), for tests and bug hunts.
LIB_PATH = os.path.join(PKG, "libstd_b200_debug.so" if os.environ.get("STD_B200_DEBUG") == "1" else "libstd_b200.so")

STD_OK = 0
STD_ERR_INVALID_ARG = -1
STD_ERR_UNSUPPORTED = -2
STD_ERR_CAPACITY = -3
STD_ERR_CUDA = -4
STD_ERR_DEVICE = -5
STD_ERR_TIMEOUT = -6
STD_ERR_WORKSPACE = -7

STD_F32 = 0
STD_BF16 = 1

STD_DEVERR_CAPACITY = 1
STD_DEVERR_LENGTH = 2
STD_DEVERR_K_RANGE = 4
STD_DEVERR_NVIS_MAX = 8
STD_DEVERR_TIMEOUT = 16
STD_DEVERR_DEBUG = 32

# every function the header declares, with (restype, argtypes)
_P = ctypes.c_void_p
_I = ctypes.c_int
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t


class StdDims(ctypes.Structure):
    _fields_ = [("L", ctypes.c_int32), ("B", ctypes.c_int32), ("Hq", ctypes.c_int32),
                ("Hkv", ctypes.c_int32), ("d", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("cap_full", ctypes.c_int64), ("cap_sparse", ctypes.c_int64)]


class StdCache(ctypes.Structure):
    _fields_ = [("k_full", _P), ("v_full", _P), ("k_sparse", _P), ("v_sparse", _P),
                ("len_full", _P), ("len_sparse", _P)]


class StdRoundIO(ctypes.Structure):
    _fields_ = [("q_draft", _P), ("k_draft", _P), ("v_draft", _P), ("q_verify", _P),
                ("k_verify", _P), ("v_verify", _P), ("draft_tokens", _P), ("dense_tokens", _P),
                ("o_draft", _P), ("o_verify", _P), ("n_plus_1", _P), ("accepted", _P)]


_DP = ctypes.POINTER(StdDims)
SIGNATURES = {
    "std_version": (_I, []),
    "std_launch_count": (ctypes.c_ulonglong, []),
    "std_last_error": (ctypes.c_char_p, []),
    "std_get_device_error": (_I, [ctypes.POINTER(ctypes.c_int32), _I, _P]),
    "std_select_workspace_size": (_SZ, [_DP, _I, _I]),
    "std_select_topk": (_I, [_DP, _P, _I, _P, _P, _P, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "std_select_topk_ex": (_I, [_DP, _P, _I, _P, _P, _P, _I, _I, _I, _I, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "std_topk_from_scores": (_I, [_P, _I, _I, _I, _P, _P]),
    "std_streaming_indices": (_I, [_DP, _P, _I, _I, _P, _P]),
    "std_gather_sparse": (_I, [_DP, _P, _P, _P, _P, _I, _I, _I, _P, _P, _P, _P]),
    "std_select_rowstats": (_I, [_DP, _P, _I, _P, _P, _I, _I, _P, _P, _P]),
    "std_merge_rowstats": (_I, [_I64, _I, _P, _P, _P, _P, _P]),
    "std_select_candidates_workspace_size": (_SZ, [_DP, _I]),
    "std_select_candidates": (_I, [_DP, _P, _I, _P, _P, _I, _I, _P, _P, _I, _P, _P, _P, _P, _SZ, _P]),
    "std_merge_candidates_workspace_size": (_SZ, [_DP, _I, _I]),
    "std_merge_candidates": (_I, [_DP, _I, _I, _P, _P, _P, _P, _P, _SZ, _P]),
    "std_gather_sparse_part": (_I, [_DP, _P, _P, _P, _P, _I, _I, _I, _I64, _I64, _P, _P, _P, _P]),
    "std_attn_workspace_size": (_SZ, [_DP, _I, _I64, _I]),
    "std_attn_splits": (_I, [_DP, _I, _I64, _I]),
    "std_attn_splits_ex": (_I, [_DP, _I, _I64, _I, _I]),
    "std_sparse_decode_attn": (_I, [_DP, _P, _P, _P, _P, _I, _P, _I, _P, _SZ, _P]),
    "std_dense_verify_attn": (_I, [_DP, _P, _I, _P, _P, _P, _P, _I, _P, _SZ, _P]),
    "std_dense_verify_attn_noalloc": (_I, [_DP, _P, _I, _P, _P, _P, _P, _I, _P]),
    "std_dense_verify_attn_partial": (_I, [_DP, _P, _I, _P, _P, _P, _I64, _I64, _I64, _P, _P, _I, _P, _SZ, _P]),
    "std_sparse_decode_attn_partial": (_I, [_DP, _P, _P, _P, _P, _I, _I64, _I64, _I64, _P, _P, _I, _P, _SZ, _P]),
    "std_merge_partials": (_I, [_I64, _I, _I, _P, _P, _P, _P]),
    "std_sparse_decode_attn_append": (_I, [_DP, _P, _P, _P, _P, _I, _P, _P, _P, _I, _P, _SZ, _P]),
    "std_sparse_decode_attn_append_ex": (_I, [_DP, _P, _P, _P, _P, _I, _P, _P, _P, _I, _I, _P, _SZ, _P]),
    "std_dense_verify_attn_append": (_I, [_DP, _P, _I, _P, _P, _P, _P, _P, _P, _I, _P, _SZ, _P]),
    "std_accept_prefix": (_I, [_I, _I, _P, _P, _P, _P, _P]),
    "std_kv_append": (_I, [_DP, _P, _P, _I64, _P, _I, _P, _P, _I, _P]),
    "std_kv_commit": (_I, [_DP, _P, _P, _P, _P, _P, _P, _P, _I, _P]),
    "std_round_workspace_size": (_SZ, [_DP, _I, _I, _I]),
    "std_probe_exp2": (_I, [_P, _P, _P, _I, _P]),
    "std_probe_wait_timeout": (_I, [_P, _P]),
    "std_decode_round": (_I, [_DP, _I, ctypes.POINTER(StdCache), ctypes.POINTER(StdRoundIO), _I, _I,
                              _P, _SZ, _P]),
}


class StdError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"std_b200 error {code}: {msg}")
        self.code = code


_lib = None
_lock = threading.Lock()


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                       "`python -m sparse_top_kv_std_b200.build`")
                h = ctypes.CDLL(LIB_PATH)
                for name, (res, args) in SIGNATURES.items():
                    f = getattr(h, name)
                    f.restype = res
                    f.argtypes = args
                _lib = h
    return _lib


# ----------------------------------------------------------------------------- marshalling

def _ptr(x) -> Optional[int]:
    if x is None:
        return None
    if isinstance(x, int):
        return x
    if not x.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not x.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return x.data_ptr()


def _nbytes(x) -> int:
    return 0 if x is None else x.numel() * x.element_size()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(rc: int) -> None:
    if rc != STD_OK:
        raise StdError(rc, lib().std_last_error().decode())


def dims(L, B, Hq, Hkv, d, dtype, cap_full, cap_sparse) -> StdDims:
    return StdDims(int(L), int(B), int(Hq), int(Hkv), int(d), int(dtype), int(cap_full), int(cap_sparse))


# ----------------------------------------------------------------------------- entry points

def std_version() -> int:
    return lib().std_version()


def std_launch_count() -> int:
    return int(lib().std_launch_count())


def std_last_error() -> str:
    return lib().std_last_error().decode()


def std_get_device_error(clear: bool = True, stream=None) -> int:
    flags = ctypes.c_int32(0)
    rc = lib().std_get_device_error(ctypes.byref(flags), int(clear), _stream(stream))
    if rc not in (STD_OK, STD_ERR_DEVICE):
        _check(rc)
    return flags.value


def std_select_workspace_size(d: StdDims, T: int, nvis_max: int) -> int:
    return lib().std_select_workspace_size(ctypes.byref(d), T, nvis_max)


def std_select_topk(d: StdDims, q_text, T, k_full, v_full, nvis, nvis_max, K, idx_out, k_sparse,
                    v_sparse, len_sparse, scores_out, ws, stream=None) -> None:
    _check(lib().std_select_topk(ctypes.byref(d), _ptr(q_text), T, _ptr(k_full), _ptr(v_full), _ptr(nvis),
                                 nvis_max, K, _ptr(idx_out), _ptr(k_sparse), _ptr(v_sparse), _ptr(len_sparse),
                                 _ptr(scores_out), _ptr(ws), _nbytes(ws), _stream(stream)))


STD_SELECT_CAUSAL_TEXT = 1


def std_select_topk_ex(d: StdDims, q_text, T, k_full, v_full, nvis, nvis_max, K, n_prefix, flags, idx_out,
                       k_sparse, v_sparse, len_sparse, scores_out, ws, stream=None) -> None:
    _check(lib().std_select_topk_ex(ctypes.byref(d), _ptr(q_text), T, _ptr(k_full), _ptr(v_full), _ptr(nvis),
                                    nvis_max, K, n_prefix, flags, _ptr(idx_out), _ptr(k_sparse), _ptr(v_sparse),
                                    _ptr(len_sparse), _ptr(scores_out), _ptr(ws), _nbytes(ws), _stream(stream)))


def std_topk_from_scores(scores, rows, n, K, idx_out, stream=None) -> None:
    _check(lib().std_topk_from_scores(_ptr(scores), rows, n, K, _ptr(idx_out), _stream(stream)))


def std_streaming_indices(d: StdDims, nvis, K, n_sink, idx_out, stream=None) -> None:
    _check(lib().std_streaming_indices(ctypes.byref(d), _ptr(nvis), K, n_sink, _ptr(idx_out), _stream(stream)))


def std_gather_sparse(d: StdDims, k_full, v_full, nvis, idx, K, T, k_sparse, v_sparse, len_sparse,
                      n_prefix=0, stream=None) -> None:
    _check(lib().std_gather_sparse(ctypes.byref(d), _ptr(k_full), _ptr(v_full), _ptr(nvis), _ptr(idx), K, T,
                                   n_prefix, _ptr(k_sparse), _ptr(v_sparse), _ptr(len_sparse), _stream(stream)))


# selection over a cache split by position (one part per GPU)

def std_select_rowstats(d: StdDims, q_text, T, k_full, nvis, nvis_max, n_prefix, row_m, row_l, stream=None) -> None:
    _check(lib().std_select_rowstats(ctypes.byref(d), _ptr(q_text), T, _ptr(k_full), _ptr(nvis), nvis_max, n_prefix,
                                     _ptr(row_m), _ptr(row_l), _stream(stream)))


def std_merge_rowstats(n, n_parts, m_parts, l_parts, row_m, row_l, stream=None) -> None:
    _check(lib().std_merge_rowstats(n, n_parts, _ptr(m_parts), _ptr(l_parts), _ptr(row_m), _ptr(row_l),
                                    _stream(stream)))


def std_select_candidates_workspace_size(d: StdDims, nvis_max: int) -> int:
    return lib().std_select_candidates_workspace_size(ctypes.byref(d), nvis_max)


def std_select_candidates(d: StdDims, q_text, T, k_full, nvis, nvis_max, n_prefix, row_m, row_l, K, cand_idx,
                          cand_score, scores_out, ws, stream=None) -> None:
    _check(lib().std_select_candidates(ctypes.byref(d), _ptr(q_text), T, _ptr(k_full), _ptr(nvis), nvis_max, n_prefix,
                                       _ptr(row_m), _ptr(row_l), K, _ptr(cand_idx), _ptr(cand_score),
                                       _ptr(scores_out), _ptr(ws), _nbytes(ws), _stream(stream)))


def std_merge_candidates_workspace_size(d: StdDims, n_parts: int, K: int) -> int:
    return lib().std_merge_candidates_workspace_size(ctypes.byref(d), n_parts, K)


def std_merge_candidates(d: StdDims, n_parts, K, cand_idx, cand_score, part_offset, idx_out, ws, stream=None) -> None:
    _check(lib().std_merge_candidates(ctypes.byref(d), n_parts, K, _ptr(cand_idx), _ptr(cand_score), _ptr(part_offset),
                                      _ptr(idx_out), _ptr(ws), _nbytes(ws), _stream(stream)))


def std_gather_sparse_part(d: StdDims, k_full, v_full, nvis, idx, K, T, n_prefix, part_pos0, part_rows, k_sparse,
                           v_sparse, len_sparse, stream=None) -> None:
    _check(lib().std_gather_sparse_part(ctypes.byref(d), _ptr(k_full), _ptr(v_full), _ptr(nvis), _ptr(idx), K, T,
                                        n_prefix, part_pos0, part_rows, _ptr(k_sparse), _ptr(v_sparse),
                                        _ptr(len_sparse), _stream(stream)))


def std_attn_workspace_size(d: StdDims, q_rows: int, cap: int, splits: int) -> int:
    return lib().std_attn_workspace_size(ctypes.byref(d), q_rows, cap, splits)


def std_attn_splits(d: StdDims, q_rows: int, cap: int, splits: int = 0) -> int:
    rc = lib().std_attn_splits(ctypes.byref(d), q_rows, cap, splits)
    if rc < 0:
        _check(rc)
    return rc


def std_attn_splits_ex(d: StdDims, q_rows: int, cap: int, splits: int = 0, flags: int = 0) -> int:
    rc = lib().std_attn_splits_ex(ctypes.byref(d), q_rows, cap, splits, flags)
    if rc < 0:
        _check(rc)
    return rc


def std_sparse_decode_attn(d: StdDims, q, k_sparse, v_sparse, len_sparse, len_offset, o, splits=0,
                           ws=None, stream=None) -> None:
    _check(lib().std_sparse_decode_attn(ctypes.byref(d), _ptr(q), _ptr(k_sparse), _ptr(v_sparse),
                                        _ptr(len_sparse), len_offset, _ptr(o), splits, _ptr(ws), _nbytes(ws),
                                        _stream(stream)))


def std_dense_verify_attn(d: StdDims, q, gamma, k_full, v_full, len_full, o, splits=0, ws=None,
                          stream=None) -> None:
    _check(lib().std_dense_verify_attn(ctypes.byref(d), _ptr(q), gamma, _ptr(k_full), _ptr(v_full),
                                       _ptr(len_full), _ptr(o), splits, _ptr(ws), _nbytes(ws), _stream(stream)))


def std_sparse_decode_attn_append(d: StdDims, q, k_sparse, v_sparse, len_sparse, len_offset, k_new, v_new, o,
                                  splits=0, ws=None, stream=None) -> None:
    _check(lib().std_sparse_decode_attn_append(ctypes.byref(d), _ptr(q), _ptr(k_sparse), _ptr(v_sparse),
                                               _ptr(len_sparse), len_offset, _ptr(k_new), _ptr(v_new), _ptr(o),
                                               splits, _ptr(ws), _nbytes(ws), _stream(stream)))


STD_ATTN_EARLY_KV = 1
STD_ATTN_EARLY_Q = 2


def std_sparse_decode_attn_append_ex(d: StdDims, q, k_sparse, v_sparse, len_sparse, len_offset, k_new, v_new, o,
                                     splits=0, flags=0, ws=None, stream=None) -> None:
    _check(lib().std_sparse_decode_attn_append_ex(ctypes.byref(d), _ptr(q), _ptr(k_sparse), _ptr(v_sparse),
                                                  _ptr(len_sparse), len_offset, _ptr(k_new), _ptr(v_new), _ptr(o),
                                                  splits, flags, _ptr(ws), _nbytes(ws), _stream(stream)))


def std_dense_verify_attn_append(d: StdDims, q, gamma, k_full, v_full, len_full, k_new, v_new, o, splits=0,
                                 ws=None, stream=None) -> None:
    _check(lib().std_dense_verify_attn_append(ctypes.byref(d), _ptr(q), gamma, _ptr(k_full), _ptr(v_full),
                                              _ptr(len_full), _ptr(k_new), _ptr(v_new), _ptr(o), splits, _ptr(ws),
                                              _nbytes(ws), _stream(stream)))


def std_dense_verify_attn_partial(d: StdDims, q, gamma, k_full, v_full, len_full, pos0, row_begin, row_end, o_part,
                                  ml_part, splits=0, ws=None, stream=None) -> None:
    _check(lib().std_dense_verify_attn_partial(ctypes.byref(d), _ptr(q), gamma, _ptr(k_full), _ptr(v_full),
                                               _ptr(len_full), pos0, row_begin, row_end, _ptr(o_part), _ptr(ml_part),
                                               splits, _ptr(ws), _nbytes(ws), _stream(stream)))


def std_sparse_decode_attn_partial(d: StdDims, q, k_sparse, v_sparse, len_sparse, len_offset, pos0, row_begin,
                                   row_end, o_part, ml_part, splits=0, ws=None, stream=None) -> None:
    _check(lib().std_sparse_decode_attn_partial(ctypes.byref(d), _ptr(q), _ptr(k_sparse), _ptr(v_sparse),
                                                _ptr(len_sparse), len_offset, pos0, row_begin, row_end, _ptr(o_part),
                                                _ptr(ml_part), splits, _ptr(ws), _nbytes(ws), _stream(stream)))


def std_merge_partials(rows, d, n_parts, o_parts, ml_parts, o, stream=None) -> None:
    _check(lib().std_merge_partials(rows, d, n_parts, _ptr(o_parts), _ptr(ml_parts), _ptr(o), _stream(stream)))


STD_NOALLOC_SCRATCH_BYTES = 16 << 20


def std_dense_verify_attn_noalloc(d: StdDims, q, gamma, k_full, v_full, len_full, o, splits=0,
                                  stream=None) -> None:
    _check(lib().std_dense_verify_attn_noalloc(ctypes.byref(d), _ptr(q), gamma, _ptr(k_full), _ptr(v_full),
                                               _ptr(len_full), _ptr(o), splits, _stream(stream)))


def std_accept_prefix(B, gamma, draft, dense_argmax, n_plus_1, accepted, stream=None) -> None:
    _check(lib().std_accept_prefix(B, gamma, _ptr(draft), _ptr(dense_argmax), _ptr(n_plus_1), _ptr(accepted),
                                   _stream(stream)))


def std_kv_append(d: StdDims, k_cache, v_cache, cap, length, pos_offset, k_new, v_new, n_new,
                  stream=None) -> None:
    _check(lib().std_kv_append(ctypes.byref(d), _ptr(k_cache), _ptr(v_cache), cap, _ptr(length), pos_offset,
                               _ptr(k_new), _ptr(v_new), n_new, _stream(stream)))


def std_kv_commit(d: StdDims, k_full, v_full, k_sparse, v_sparse, len_full, len_sparse, n_plus_1, max_n,
                  stream=None) -> None:
    _check(lib().std_kv_commit(ctypes.byref(d), _ptr(k_full), _ptr(v_full), _ptr(k_sparse), _ptr(v_sparse),
                               _ptr(len_full), _ptr(len_sparse), _ptr(n_plus_1), max_n, _stream(stream)))


def std_round_workspace_size(d: StdDims, gamma: int, splits_draft: int = 0, splits_verify: int = 0) -> int:
    return lib().std_round_workspace_size(ctypes.byref(d), gamma, splits_draft, splits_verify)


def std_decode_round(d: StdDims, gamma, cache: dict, io: dict, splits_draft=0, splits_verify=0, ws=None,
                     stream=None) -> None:
    """cache / io: dicts of tensors keyed by the std_cache / std_round_io field names."""
    c = StdCache(*[_ptr(cache[f]) for f, _ in StdCache._fields_])
    r = StdRoundIO(*[_ptr(io[f]) for f, _ in StdRoundIO._fields_])
    _check(lib().std_decode_round(ctypes.byref(d), gamma, ctypes.byref(c), ctypes.byref(r), splits_draft,
                                  splits_verify, _ptr(ws), _nbytes(ws), _stream(stream)))


def std_probe_exp2(x, y_fma, y_sfu, stream=None) -> None:
    _check(lib().std_probe_exp2(_ptr(x), _ptr(y_fma), _ptr(y_sfu), x.numel(), _stream(stream)))


def std_probe_wait_timeout(completed, stream=None) -> None:
    _check(lib().std_probe_wait_timeout(_ptr(completed), _stream(stream)))
