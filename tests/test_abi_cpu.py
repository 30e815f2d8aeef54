"""The C-ABI library loads, exports every entry point the header declares, and
rejects bad arguments on the host before touching the GPU (no GPU needed)."""
import ctypes
import os
import re

import pytest

from sparse_top_kv_std_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "std_b200.h")


def header_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(std_[a-z0-9_]+)\s*\(", src)))


@pytest.fixture(scope="module")
def lib():
    if not os.path.exists(B.LIB_PATH):
        from sparse_top_kv_std_b200 import build
        build.build()
    return B.lib()


def test_every_declared_symbol_is_exported(lib):
    names = header_functions()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(B.SIGNATURES), "binding and header disagree"


def test_version_and_error_string(lib):
    assert B.std_version() == 10000
    assert isinstance(B.std_last_error(), str)


def _dims(**kw):
    base = dict(L=2, B=1, Hq=28, Hkv=4, d=128, dtype=B.STD_BF16, cap_full=1000, cap_sparse=300)
    base.update(kw)
    return B.dims(**base)


def test_workspace_queries_host_only(lib):
    d = _dims()
    ws = B.std_select_workspace_size(d, 64, 512)
    assert ws >= (2 * 4 * 7 * 64 * 2 + 2 * 4 * 512) * 4
    # explicit splits: no device query.  bf16: tensor-core kernel with splits x problems CTAs
    # (problems + CTAs) partial slots of 63 rows x (d + 2) floats and a merge counter per problem
    probs = 2 * 1 * 4
    a = B.std_attn_workspace_size(d, 9, 1000, 4)
    assert a == (probs + 4 * probs) * 63 * (128 + 2) * 4 + probs * 8   # + one merge counter per problem
    # fp32: split-K, no workspace with one split
    f = _dims(dtype=B.STD_F32, d=64)
    assert B.std_attn_workspace_size(f, 9, 1000, 1) == 0
    assert B.std_attn_workspace_size(f, 9, 1000, 4) == probs * 4 * 63 * (64 + 2) * 4
    assert B.std_select_workspace_size(_dims(dtype=7), 64, 512) == 0
    assert B.std_attn_workspace_size(_dims(Hq=5), 1, 1000, 4) == 0
    # explicit splits: the CTA count needs no device, with or without early-start flags
    assert B.std_attn_splits(d, 1, 300, 4) == 4 * probs
    assert B.std_attn_splits_ex(d, 1, 300, 4, B.STD_ATTN_EARLY_KV | B.STD_ATTN_EARLY_Q) == 4 * probs
    assert lib.std_attn_splits_ex(ctypes.byref(d), 1, 300, 4, 4) == B.STD_ERR_INVALID_ARG
    assert lib.std_attn_splits_ex(ctypes.byref(d), 1, 300, 4, B.STD_ATTN_EARLY_Q) == B.STD_ERR_INVALID_ARG


FAKE = 1 << 40  # a 16-byte aligned non-null "pointer": never dereferenced, checks fail first


def _gpu_visible():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


# The calls below hand made-up device addresses to the library and rely on its host checks
# rejecting them first.  They belong to the CPU suite: where a GPU is visible they are
# skipped, so that a check that stopped firing can never become a launch on invalid memory.
no_gpu_only = pytest.mark.skipif(_gpu_visible(), reason="made-up device addresses: host-only test")


@pytest.mark.parametrize("call,code", [
    (lambda: lib_().std_select_topk(None, FAKE, 64, FAKE, FAKE, FAKE, 512, 16, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_topk(ctypes.byref(_dims(dtype=5)), FAKE, 64, FAKE, FAKE, FAKE, 512, 16, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_UNSUPPORTED),
    (lambda: lib_().std_select_topk(ctypes.byref(_dims(d=80)), FAKE, 64, FAKE, FAKE, FAKE, 512, 16, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_UNSUPPORTED),
    (lambda: lib_().std_select_topk(ctypes.byref(_dims()), None, 64, FAKE, FAKE, FAKE, 512, 16, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_topk(ctypes.byref(_dims()), FAKE + 2, 64, FAKE, FAKE, FAKE, 512, 16, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_topk(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, FAKE, 512, 513, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_topk(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, FAKE, 512, 0, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_topk(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, FAKE, 512, 256, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_CAPACITY),
    (lambda: lib_().std_select_topk(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, FAKE, 990, 16, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_CAPACITY),
    (lambda: lib_().std_select_topk(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, FAKE, 512, 16, FAKE, FAKE, FAKE, FAKE, None, FAKE, 16, None), B.STD_ERR_WORKSPACE),
    (lambda: lib_().std_select_topk_ex(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, FAKE, 512, 16, 0, 2, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_topk_ex(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, FAKE, 512, 256, 0, 1, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_CAPACITY),
    (lambda: lib_().std_select_topk_ex(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, FAKE, 512, 16, -1, 0, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_topk_ex(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, FAKE, 512, 16, 425, 0, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_CAPACITY),
    (lambda: lib_().std_select_topk_ex(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, FAKE, 800, 16, 200, 0, FAKE, FAKE, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_CAPACITY),
    (lambda: lib_().std_topk_from_scores(FAKE, 4, 100, 101, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_streaming_indices(ctypes.byref(_dims()), FAKE, 16, 17, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_streaming_indices(ctypes.byref(_dims()), FAKE, 0, 0, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_streaming_indices(ctypes.byref(_dims()), None, 16, 4, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_gather_sparse(ctypes.byref(_dims()), FAKE, FAKE, FAKE, FAKE, 256, 64, 0, FAKE, FAKE, FAKE, None), B.STD_ERR_CAPACITY),
    (lambda: lib_().std_gather_sparse(ctypes.byref(_dims()), FAKE, FAKE, FAKE, FAKE, 200, 64, 37, FAKE, FAKE, FAKE, None), B.STD_ERR_CAPACITY),
    (lambda: lib_().std_gather_sparse(ctypes.byref(_dims()), FAKE, FAKE, FAKE, FAKE, 16, 64, -1, FAKE, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_gather_sparse(ctypes.byref(_dims()), FAKE, FAKE, FAKE, None, 16, 64, 0, FAKE, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_topk_from_scores(None, 4, 100, 10, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_dense_verify_attn(ctypes.byref(_dims()), FAKE, 32, FAKE, FAKE, FAKE, FAKE, 1, None, 0, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_dense_verify_attn(ctypes.byref(_dims()), FAKE, -1, FAKE, FAKE, FAKE, FAKE, 1, None, 0, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_dense_verify_attn(ctypes.byref(_dims()), FAKE, 18, FAKE, FAKE, FAKE, FAKE, 1, None, 0, None), B.STD_ERR_UNSUPPORTED),
    (lambda: lib_().std_dense_verify_attn(ctypes.byref(_dims()), FAKE, 4, FAKE, FAKE, FAKE, FAKE, 8, None, 0, None), B.STD_ERR_WORKSPACE),
    (lambda: lib_().std_dense_verify_attn(ctypes.byref(_dims()), FAKE, 4, FAKE, FAKE, FAKE, FAKE, 2000, None, 0, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_sparse_decode_attn(ctypes.byref(_dims()), FAKE, FAKE, FAKE, FAKE, -1, FAKE, 1, None, 0, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_sparse_decode_attn(ctypes.byref(_dims()), FAKE, FAKE, FAKE, None, 0, FAKE, 1, None, 0, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_accept_prefix(0, 4, FAKE, FAKE, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_accept_prefix(2, 32, FAKE, FAKE, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_accept_prefix(2, 4, FAKE, FAKE, None, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_kv_append(ctypes.byref(_dims()), FAKE, FAKE, 100, FAKE, 90, FAKE, FAKE, 20, None), B.STD_ERR_CAPACITY),
    (lambda: lib_().std_kv_append(ctypes.byref(_dims()), FAKE, FAKE, 100, FAKE, -1, FAKE, FAKE, 2, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_kv_commit(ctypes.byref(_dims()), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 33, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_decode_round(ctypes.byref(_dims()), 4, None, None, 0, 0, None, 0, None), B.STD_ERR_INVALID_ARG),
    # the selection over a cache split by position
    (lambda: lib_().std_select_rowstats(None, FAKE, 64, FAKE, FAKE, 512, 0, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_rowstats(ctypes.byref(_dims()), FAKE, 0, FAKE, FAKE, 512, 0, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_rowstats(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, 0, 0, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_rowstats(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, 512, -1, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_rowstats(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, 900, 101, FAKE, FAKE, None), B.STD_ERR_CAPACITY),
    (lambda: lib_().std_select_rowstats(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, 512, 0, None, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_merge_rowstats(0, 2, FAKE, FAKE, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_merge_rowstats(100, 0, FAKE, FAKE, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_merge_rowstats(100, 2, None, FAKE, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_candidates(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, 512, 0, FAKE, FAKE, 0, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_candidates(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, 512, 0, FAKE, FAKE, 513, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_select_candidates(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, 512, 0, FAKE, FAKE, 16, FAKE, FAKE, None, FAKE, 16, None), B.STD_ERR_WORKSPACE),
    (lambda: lib_().std_select_candidates(ctypes.byref(_dims()), FAKE, 64, FAKE, FAKE, 512, 0, None, FAKE, 16, FAKE, FAKE, None, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_merge_candidates(ctypes.byref(_dims()), 0, 16, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_merge_candidates(ctypes.byref(_dims()), 2, 0, FAKE, FAKE, FAKE, FAKE, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_merge_candidates(ctypes.byref(_dims()), 2, 16, FAKE, FAKE, FAKE, FAKE, FAKE, 16, None), B.STD_ERR_WORKSPACE),
    (lambda: lib_().std_merge_candidates(ctypes.byref(_dims()), 2, 16, FAKE, FAKE, None, FAKE, FAKE, 1 << 30, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_gather_sparse_part(ctypes.byref(_dims()), FAKE, FAKE, FAKE, FAKE, 16, 64, 0, 0, 0, FAKE, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_gather_sparse_part(ctypes.byref(_dims()), FAKE, FAKE, FAKE, FAKE, 16, 64, 0, 0, 1001, FAKE, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_gather_sparse_part(ctypes.byref(_dims()), FAKE, FAKE, FAKE, FAKE, 16, 64, 0, -5, 100, FAKE, FAKE, FAKE, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_gather_sparse_part(ctypes.byref(_dims()), FAKE, FAKE, FAKE, FAKE, 240, 64, 0, 0, 100, FAKE, FAKE, FAKE, None), B.STD_ERR_CAPACITY),
    (lambda: lib_().std_probe_wait_timeout(None, None), B.STD_ERR_INVALID_ARG),
    (lambda: lib_().std_probe_wait_timeout(FAKE + 2, None), B.STD_ERR_INVALID_ARG),
])
@no_gpu_only
def test_host_side_rejections(lib, call, code):
    assert call() == code
    assert B.std_last_error() != ""


def lib_():
    return B.lib()


@no_gpu_only
def test_launch_count_ignores_rejected_calls(lib):
    n0 = B.std_launch_count()
    assert n0 >= 0
    rc = lib_().std_accept_prefix(0, 4, FAKE, FAKE, FAKE, FAKE, None)  # rejected before any launch
    assert rc == B.STD_ERR_INVALID_ARG
    assert B.std_launch_count() == n0


def test_binding_constants_match_the_header():
    """The Python copies of the header's constants (status codes, dtypes, device error bits,
    the built-in scratch size of the no-alloc verify) have the header's values."""
    src = re.sub(r"/\*.*?\*/", "", open(HEADER).read(), flags=re.S)
    values = {n: int(v) for n, v in re.findall(r"\b(STD_[A-Z0-9_]+)\s*=\s*(-?\d+)", src)}
    values.update({n: int(v) for n, v in re.findall(r"#define\s+(STD_[A-Z0-9_]+)\s+(-?\d+)\s*$", src, re.M)})
    assert "STD_ATTN_EARLY_KV" in values and "STD_DEVERR_DEBUG" in values
    shift = re.search(r"#define\s+STD_NOALLOC_SCRATCH_BYTES\s+\((\d+)u\s*<<\s*(\d+)\)", src)
    assert shift, "STD_NOALLOC_SCRATCH_BYTES must stay of the form (a << b)"
    values["STD_NOALLOC_SCRATCH_BYTES"] = int(shift.group(1)) << int(shift.group(2))
    assert len(values) >= 15
    for name, v in values.items():
        assert getattr(B, name) == v, (name, getattr(B, name), v)
