"""C-ABI checks that need no GPU: the library loads, exports every entry
point include/sparse_mla.h declares, and rejects bad arguments on the host
before making any CUDA call."""
import ctypes
import math
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sparse_mla.h")


def _ensure_built():
    from sparse_mla_decode_05_b200 import build
    if not os.path.exists(build.LIB):
        build.build_library()


_ensure_built()
from sparse_mla_decode_05_b200 import api  # noqa: E402


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(sparse_mla_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for must in ("sparse_mla_decode", "sparse_mla_decode_split", "sparse_mla_combine",
                 "sparse_mla_workspace_size", "sparse_mla_plan_nsplit", "sparse_mla_status_string",
                 "sparse_mla_abi_version", "sparse_mla_get_device_error", "sparse_mla_plan_merge",
                 "sparse_mla_decode_static_scratch", "sparse_mla_decode_host", "sparse_mla_host_staging_size",
                 "sparse_mla_indexer", "sparse_mla_indexer_scores", "sparse_mla_indexer_topk",
                 "sparse_mla_decode_stalled"):
        assert must in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(api.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_abi_version_and_status_strings():
    assert api.lib.sparse_mla_abi_version() == 2
    for code, name in api.STATUS.items():
        assert api.lib.sparse_mla_status_string(code).decode() == name
    assert api.lib.sparse_mla_status_string(99).decode() == "SMLA_ERR_UNKNOWN"


def test_struct_layout_matches_header():
    assert ctypes.sizeof(api.SmlaShape) == 48
    assert api.SmlaShape.num_kv_rows.offset == 24
    # smla_indexer_shape: eight int32 fields, then the int64 row count
    assert ctypes.sizeof(api.IndexerShape) == 40
    assert api.IndexerShape.num_key_rows.offset == 32


def _decode(shape, q=16, kv=16, rs=None, pt=None, idx=16, scale=0.04, out=16, lse=16, ws=None, nbytes=0):
    return api.lib.sparse_mla_decode(ctypes.byref(shape) if shape is not None else None, q, kv, rs, pt, idx,
                                     scale, out, lse, ws, nbytes, None)


GOOD = dict(batch=2, topk=100, num_kv_rows=1000)


def shape(**kw):
    d = dict(GOOD)
    d.update(kw)
    s = api.make_shape(d.pop("batch"), d.pop("topk"), d.pop("num_kv_rows"), fp8=d.pop("fp8", False),
                       page_size=d.pop("page_size", 0), pages_per_seq=d.pop("pages_per_seq", 0),
                       nsplit=d.pop("nsplit", 0))
    for k, v in d.items():
        setattr(s, k, v)
    return s


INVALID, UNSUPPORTED = 1, 2


@pytest.mark.parametrize("kw,code", [
    (dict(batch=0), INVALID), (dict(batch=70000), INVALID), (dict(topk=0), INVALID),
    (dict(num_kv_rows=0), INVALID), (dict(nsplit=-2), INVALID),
    # multi-token decode: 0..16 tokens per sequence, at most 65535 decode rows
    (dict(tokens_per_seq=-1), INVALID), (dict(tokens_per_seq=17), INVALID),
    (dict(batch=5000, tokens_per_seq=16), INVALID),
    (dict(num_heads=32), UNSUPPORTED), (dict(d_qk=512), UNSUPPORTED), (dict(d_v=576), UNSUPPORTED),
    (dict(kv_dtype=7), UNSUPPORTED), (dict(page_size=32, pages_per_seq=4), UNSUPPORTED),
    (dict(page_size=64, pages_per_seq=0), INVALID),
    # DeepSeek-V4 pages: d_qk 512, paged with 64-token pages, whole pages
    (dict(kv_dtype=2), UNSUPPORTED), (dict(kv_dtype=2, d_qk=512), UNSUPPORTED),
    (dict(kv_dtype=2, d_qk=512, page_size=64, pages_per_seq=4, num_kv_rows=1000), UNSUPPORTED),
])
def test_bad_shapes_rejected_without_cuda(kw, code):
    assert _decode(shape(**kw)) == code
    assert api.lib.sparse_mla_workspace_size(ctypes.byref(shape(**kw))) == 0
    assert api.lib.sparse_mla_plan_nsplit(ctypes.byref(shape(**kw))) == 0
    assert api.lib.sparse_mla_plan_merge(ctypes.byref(shape(**kw))) == -1
    assert api.lib.sparse_mla_decode_static_scratch(ctypes.byref(shape(**kw)), 16, 16, None, None, 16, 0.04,
                                                    16, 16, None) == code


def test_partials_size_formula():
    # B * nsplit * 64 * (512 + 1) fp32, rounded up to 256 bytes
    assert api.partials_size(1, 1) == 131328
    assert api.partials_size(3, 5) == (3 * 5 * 64 * 513 * 4 + 255) // 256 * 256


def test_null_and_misaligned_pointers_rejected():
    s = shape()
    assert _decode(None) == INVALID
    assert _decode(s, q=None) == INVALID
    assert _decode(s, kv=None) == INVALID
    assert _decode(s, idx=None) == INVALID
    assert _decode(s, out=None) == INVALID
    assert _decode(s, lse=None) == INVALID
    assert _decode(s, q=24) == INVALID            # not 16-byte aligned
    assert _decode(s, kv=8) == INVALID
    assert _decode(s, out=40) == INVALID
    assert _decode(s, idx=18) == INVALID           # not 4-byte aligned
    assert _decode(s, scale=math.nan) == INVALID
    assert _decode(s, scale=math.inf) == INVALID
    assert _decode(shape(fp8=True)) == INVALID      # fp8 without row scales
    assert _decode(shape(page_size=64, pages_per_seq=3)) == INVALID   # paged without a table


def test_combine_argument_checks():
    c = api.lib.sparse_mla_combine
    assert c(0, 64, 512, 2, 16, 16, 16, 16, None) == INVALID
    assert c(1, 64, 512, 0, 16, 16, 16, 16, None) == INVALID
    assert c(1, 64, 512, 5000, 16, 16, 16, 16, None) == INVALID
    assert c(1, 32, 512, 2, 16, 16, 16, 16, None) == UNSUPPORTED
    assert c(1, 64, 256, 2, 16, 16, 16, 16, None) == UNSUPPORTED
    assert c(1, 64, 512, 2, None, 16, 16, 16, None) == INVALID
    assert c(1, 64, 512, 2, 8, 16, 16, 16, None) == INVALID


def test_python_binding_rejects_cpu_tensors():
    import torch
    q = torch.zeros(1, 64, 576, dtype=torch.bfloat16)
    kv = torch.zeros(10, 576, dtype=torch.bfloat16)
    idx = torch.zeros(1, 4, dtype=torch.int32)
    with pytest.raises(ValueError):
        api.decode(q, kv, idx, 0.04)
    with pytest.raises(ValueError):
        api.decode(q[:, :32], kv, idx, 0.04)


def test_dsv4_shape_accepted_and_row_scale_rejected():
    s = api.make_shape(2, 100, 64 * 16, dsv4=True, page_size=64, pages_per_seq=8)
    assert s.d_qk == 512 and s.kv_dtype == api.KV_DSV4_PAGED
    assert api.lib.sparse_mla_plan_merge(ctypes.byref(s)) >= 0
    # the pages carry their own scales: a row-scale pointer is an error,
    # found before any CUDA call
    assert _decode(s, rs=16, pt=16) == INVALID


# ------------------------------------------------ sparse_mla_decode_host
def _r256(x):
    return (x + 255) // 256 * 256


def test_host_staging_size_is_the_sum_of_its_regions():
    # q, indices, page table, out, lse (workspace 0: one split without a device)
    s = api.make_shape(16, 512, 67000)
    assert api.host_staging_size(s) == (_r256(16 * 64 * 576 * 2) + _r256(16 * 512 * 4) + _r256(16 * 64 * 512 * 2)
                                        + _r256(16 * 64 * 4))
    s = api.make_shape(3, 100, 64 * 40, fp8=True, page_size=64, pages_per_seq=7)
    assert api.host_staging_size(s) == (_r256(3 * 64 * 576 * 2) + _r256(3 * 100 * 4) + _r256(3 * 7 * 4)
                                        + _r256(3 * 64 * 512 * 2) + _r256(3 * 64 * 4))
    s = api.make_shape(2, 100, 64 * 16, dsv4=True, page_size=64, pages_per_seq=8)
    assert api.host_staging_size(s) == (_r256(2 * 64 * 512 * 2) + _r256(2 * 100 * 4) + _r256(2 * 8 * 4)
                                        + _r256(2 * 64 * 512 * 2) + _r256(2 * 64 * 4))
    assert api.host_staging_size(shape(batch=0)) == 0


def _host(s, q=16, kv=16, rs=None, pt=None, idx=16, scale=0.04, out=16, lse=16, st=256, nbytes=1 << 30):
    return api.lib.sparse_mla_decode_host(ctypes.byref(s) if s is not None else None, q, kv, rs, pt, idx, scale,
                                          out, lse, st, nbytes, None)


WORKSPACE = 3


def test_decode_host_rejects_bad_arguments_before_any_copy():
    s = shape()
    assert _host(None) == INVALID
    assert _host(shape(batch=0)) == INVALID
    for kw in (dict(q=None), dict(kv=None), dict(idx=None), dict(out=None), dict(lse=None)):
        assert _host(s, **kw) == INVALID
    assert _host(s, kv=8) == INVALID                     # cache not 16-byte aligned
    assert _host(s, pt=16) == INVALID                    # page table without paging
    assert _host(shape(page_size=64, pages_per_seq=4)) == INVALID   # paging without a page table
    assert _host(s, rs=16) == INVALID                    # row scale with a bf16 cache
    assert _host(shape(fp8=True)) == INVALID             # fp8 cache without row scales
    assert _host(s, scale=float("nan")) == INVALID
    assert _host(s, st=None) == WORKSPACE
    assert _host(s, st=128) == WORKSPACE                 # staging not 256-byte aligned
    assert _host(s, nbytes=api.host_staging_size(s) - 1) == WORKSPACE


# ------------------------------------------------------------ indexer
def _ix_shape(**kw):
    d = dict(batch=2, topk=16, max_ctx=256, pages_per_seq=4, num_key_rows=64 * 8)
    d.update(kw)
    s = api.indexer_shape(d.pop("batch"), d.pop("topk"), d.pop("max_ctx"), d.pop("pages_per_seq"),
                          d.pop("num_key_rows"))
    for k, v in d.items():
        setattr(s, k, v)
    return s


@pytest.mark.parametrize("kw,code", [
    (dict(batch=0), INVALID), (dict(topk=0), INVALID), (dict(topk=65537), INVALID), (dict(max_ctx=0), INVALID),
    (dict(max_ctx=(1 << 20) + 1), INVALID), (dict(reserved=1), INVALID), (dict(heads=32), UNSUPPORTED),
    (dict(dim=64), UNSUPPORTED), (dict(page_size=32), UNSUPPORTED), (dict(pages_per_seq=3), INVALID),
    (dict(num_key_rows=100), INVALID), (dict(num_key_rows=0), INVALID),
])
def test_indexer_bad_shapes_rejected_without_cuda(kw, code):
    s = _ix_shape(**kw)
    assert api.lib.sparse_mla_indexer_scores(ctypes.byref(s), 16, 16, 16, 16, 16, 16, None) == code
    assert api.lib.sparse_mla_indexer_topk(ctypes.byref(s), 16, 16, 16, None) == code
    assert api.lib.sparse_mla_indexer(ctypes.byref(s), 16, 16, 16, 16, 16, 16, 16, None) == code


def test_indexer_null_and_misaligned_pointers_rejected():
    s = _ix_shape()
    f = api.lib.sparse_mla_indexer_scores
    assert f(None, 16, 16, 16, 16, 16, 16, None) == INVALID
    for i in range(6):
        args = [16] * 6
        args[i] = None
        assert f(ctypes.byref(s), *args, None) == INVALID
    assert f(ctypes.byref(s), 8, 16, 16, 16, 16, 16, None) == INVALID     # q not 16-byte aligned
    assert f(ctypes.byref(s), 16, 16, 8, 16, 16, 16, None) == INVALID     # keys not 16-byte aligned
    assert f(ctypes.byref(s), 16, 2, 16, 16, 16, 16, None) == INVALID     # w not 4-byte aligned
    g = api.lib.sparse_mla_indexer_topk
    assert g(ctypes.byref(s), None, 16, 16, None) == INVALID
    assert g(ctypes.byref(s), 16, 16, 2, None) == INVALID
    assert api.lib.sparse_mla_indexer(ctypes.byref(s), 16, 16, 16, 16, 16, 16, None, None) == INVALID


# ------------------------------------------------ bounded-wait test hook
def test_stalled_hook_checks_before_any_cuda_call():
    f = api.lib.sparse_mla_decode_stalled
    s = shape()
    assert f(None, 16, 16, 16, 0.04, 16, 16, 100000, None) == INVALID
    assert f(ctypes.byref(shape(fp8=True)), 16, 16, 16, 0.04, 16, 16, 100000, None) == UNSUPPORTED
    assert f(ctypes.byref(shape(page_size=64, pages_per_seq=4)), 16, 16, 16, 0.04, 16, 16, 100000,
             None) == UNSUPPORTED
    for lim in (-1, 0, 999, 4_000_000_001):
        assert f(ctypes.byref(s), 16, 16, 16, 0.04, 16, 16, lim, None) == INVALID
