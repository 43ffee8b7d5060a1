"""Thin Python binding over the C ABI in include/sparse_mla.h.

Argument marshalling only: every step of the decode runs in the CUDA
library.  Torch tensors supply device pointers and the current stream.
There is no fallback: if the shared library is missing this module raises
on import.
"""
from __future__ import annotations

import ctypes
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsparse_mla.so")

H, D_QK, D_V, TILE = 64, 576, 512, 64
NSPLIT_STREAMK = -1          # smla_shape.nsplit asking for the stream-K plan
KV_BF16, KV_FP8_E4M3_ROWSCALE, KV_DSV4_PAGED = 0, 1, 2
DSV4_PAGE_BYTES, DSV4_D_QK = 37376, 512   # DeepSeek-V4 page: 64 x 576 slot bytes + 64 x 8 scale bytes

STATUS = {0: "SMLA_OK", 1: "SMLA_ERR_INVALID_ARG", 2: "SMLA_ERR_UNSUPPORTED", 3: "SMLA_ERR_WORKSPACE",
          4: "SMLA_ERR_CUDA", 5: "SMLA_ERR_DEVICE_TIMEOUT", 6: "SMLA_ERR_DEVICE_INDEX",
          7: "SMLA_ERR_DEVICE_LAYOUT"}


class SmlaError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {STATUS.get(code, code)}")
        self.code = code


class SmlaShape(ctypes.Structure):
    _fields_ = [
        ("batch", ctypes.c_int32), ("num_heads", ctypes.c_int32), ("d_qk", ctypes.c_int32),
        ("d_v", ctypes.c_int32), ("topk", ctypes.c_int32), ("kv_dtype", ctypes.c_int32),
        ("num_kv_rows", ctypes.c_int64), ("page_size", ctypes.c_int32),
        ("pages_per_seq", ctypes.c_int32), ("nsplit", ctypes.c_int32), ("tokens_per_seq", ctypes.c_int32),
    ]


class IndexerShape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("heads", ctypes.c_int32), ("dim", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("max_ctx", ctypes.c_int32), ("page_size", ctypes.c_int32),
                ("pages_per_seq", ctypes.c_int32), ("reserved", ctypes.c_int32), ("num_key_rows", ctypes.c_int64)]


IX_HEADS, IX_DIM = 64, 128


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with "
                          "`python -m sparse_mla_decode_05_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, I32, SZ, F32 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t, ctypes.c_float
    SP = ctypes.POINTER(SmlaShape)
    lib.sparse_mla_abi_version.restype = I32
    lib.sparse_mla_status_string.restype = ctypes.c_char_p
    lib.sparse_mla_status_string.argtypes = [I32]
    lib.sparse_mla_plan_nsplit.restype = I32
    lib.sparse_mla_plan_nsplit.argtypes = [SP]
    lib.sparse_mla_plan_merge.restype = I32
    lib.sparse_mla_plan_merge.argtypes = [SP]
    lib.sparse_mla_workspace_size.restype = SZ
    lib.sparse_mla_workspace_size.argtypes = [SP]
    lib.sparse_mla_decode.restype = I32
    lib.sparse_mla_decode.argtypes = [SP, P, P, P, P, P, F32, P, P, P, SZ, P]
    lib.sparse_mla_decode_split.restype = I32
    lib.sparse_mla_decode_split.argtypes = [SP, P, P, P, P, P, F32, P, P, P, SZ,
                                            ctypes.POINTER(I32), P]
    lib.sparse_mla_combine.restype = I32
    lib.sparse_mla_combine.argtypes = [I32, I32, I32, I32, P, P, P, P, P]
    lib.sparse_mla_get_device_error.restype = I32
    lib.sparse_mla_get_device_error.argtypes = [ctypes.POINTER(ctypes.c_uint32)]
    lib.sparse_mla_decode_static_scratch.restype = I32
    lib.sparse_mla_decode_static_scratch.argtypes = [SP, P, P, P, P, P, F32, P, P, P]
    lib.sparse_mla_decode_stalled.restype = I32
    lib.sparse_mla_decode_stalled.argtypes = [SP, P, P, P, F32, P, P, ctypes.c_int64, P]
    IP = ctypes.POINTER(IndexerShape)
    lib.sparse_mla_indexer_scores.restype = I32
    lib.sparse_mla_indexer_scores.argtypes = [IP, P, P, P, P, P, P, P]
    lib.sparse_mla_indexer_topk.restype = I32
    lib.sparse_mla_indexer_topk.argtypes = [IP, P, P, P, P]
    lib.sparse_mla_indexer.restype = I32
    lib.sparse_mla_indexer.argtypes = [IP, P, P, P, P, P, P, P, P]
    lib.sparse_mla_host_staging_size.restype = SZ
    lib.sparse_mla_host_staging_size.argtypes = [SP]
    lib.sparse_mla_decode_host.restype = I32
    lib.sparse_mla_decode_host.argtypes = [SP, P, P, P, P, P, F32, P, P, P, SZ, P]
    return lib


lib = _load()


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(device) -> int:
    return torch.cuda.current_stream(device).cuda_stream


def make_shape(batch: int, topk: int, num_kv_rows: int, *, fp8: bool = False, dsv4: bool = False,
               page_size: int = 0, pages_per_seq: int = 0, nsplit: int = 0, tokens_per_seq: int = 0) -> SmlaShape:
    kind = KV_DSV4_PAGED if dsv4 else (KV_FP8_E4M3_ROWSCALE if fp8 else KV_BF16)
    return SmlaShape(batch, H, DSV4_D_QK if dsv4 else D_QK, D_V, topk, kind,
                     num_kv_rows, page_size, pages_per_seq, nsplit, tokens_per_seq)


def _tokens(q) -> int:
    """Query tokens per sequence: q is [B, 64, d] (one) or [B, T, 64, d]."""
    return q.shape[1] if q.dim() == 4 else 1


def _result_shapes(q):
    """(out, lse) shapes for q [B, (T,) 64, d]."""
    lead = tuple(q.shape[:-2])
    return lead + (H, D_V), lead + (H,)


def is_dsv4(kv) -> bool:
    """A DeepSeek-V4 paged cache: uint8 [pages, 37376]."""
    return kv.dtype == torch.uint8 and kv.dim() == 2 and kv.shape[1] == DSV4_PAGE_BYTES


def shape_for(q, kv, indices, *, page_table=None, page_size: int = 0, nsplit: int = 0) -> SmlaShape:
    """The shape of one call: q [B, 64, d] with indices [B, topk], or q
    [B, T, 64, d] with indices [B, T, topk] (T query tokens per sequence)."""
    dsv4 = is_dsv4(kv)
    T = _tokens(q)
    return make_shape(q.shape[0], indices.shape[-1], kv.shape[0] * (64 if dsv4 else 1),
                      fp8=(kv.dtype == torch.uint8 and not dsv4), dsv4=dsv4, page_size=page_size,
                      pages_per_seq=0 if page_table is None else page_table.shape[1], nsplit=nsplit,
                      tokens_per_seq=T if T > 1 else 0)


def plan_nsplit(shape: SmlaShape) -> int:
    return lib.sparse_mla_plan_nsplit(ctypes.byref(shape))


def plan_merge(shape: SmlaShape) -> int:
    """0: one split; 1: splits merged inside the split kernel (cluster);
    2: partials merged by the combine kernel; 3: stream-K (one CTA per SM
    over the rows' tiles, a shared row merged by its last CTA)."""
    return lib.sparse_mla_plan_merge(ctypes.byref(shape))


def workspace_size(shape: SmlaShape) -> int:
    return lib.sparse_mla_workspace_size(ctypes.byref(shape))


def _check_inputs(q, kv, indices, kv_row_scale, page_table, page_size):
    dsv4 = is_dsv4(kv)
    d_qk = DSV4_D_QK if dsv4 else D_QK
    if q.dtype != torch.bfloat16 or q.dim() not in (3, 4) or q.shape[-2:] != (H, d_qk):
        raise ValueError(f"q must be bf16 [B, 64, {d_qk}] or [B, T, 64, {d_qk}]")
    if not dsv4 and (kv.dim() != 2 or kv.shape[1] != D_QK or kv.dtype not in (torch.bfloat16, torch.uint8)):
        raise ValueError("kv must be [N, 576] bf16 or uint8 (fp8 e4m3fn codes), or uint8 [pages, 37376] "
                         "DeepSeek-V4 pages")
    if indices.dtype != torch.int32 or indices.dim() != q.dim() - 1 or indices.shape[:-1] != q.shape[:-2]:
        raise ValueError("indices must be int32 [B, topk] ([B, T, topk] for q [B, T, 64, d])")
    if dsv4:
        if kv_row_scale is not None:
            raise ValueError("DeepSeek-V4 pages carry their own scales: kv_row_scale must be None")
        if page_size != 64:
            raise ValueError("DeepSeek-V4 pages are paged: page_size must be 64")
    elif kv.dtype == torch.uint8 and (kv_row_scale is None or kv_row_scale.dtype != torch.float32):
        raise ValueError("fp8 cache needs float32 kv_row_scale [N]")
    if page_size and (page_table is None or page_table.dtype != torch.int32):
        raise ValueError("paged cache needs int32 page_table [B, pages_per_seq]")
    for t in (q, kv, indices, kv_row_scale, page_table):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError("all tensors must be contiguous CUDA tensors")


def decode(q, kv, indices, scale: float, *, kv_row_scale=None, page_table=None, page_size: int = 0,
           nsplit: int = 0, out=None, lse=None, workspace=None):
    """out [B,64,512] bf16, lse [B,64] fp32 = sparse-MLA decode (one call to
    sparse_mla_decode).  Allocates out / lse / workspace with torch when not
    given."""
    _check_inputs(q, kv, indices, kv_row_scale, page_table, page_size)
    shape = shape_for(q, kv, indices, page_table=page_table, page_size=page_size, nsplit=nsplit)
    dev = q.device
    o_shape, l_shape = _result_shapes(q)
    if out is None:
        out = torch.empty(o_shape, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(l_shape, dtype=torch.float32, device=dev)
    ws_bytes = workspace_size(shape)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    st = lib.sparse_mla_decode(ctypes.byref(shape), _ptr(q), _ptr(kv), _ptr(kv_row_scale),
                               _ptr(page_table), _ptr(indices), float(scale), _ptr(out), _ptr(lse),
                               _ptr(workspace), 0 if workspace is None else workspace.numel(),
                               _stream(dev))
    if st != 0:
        raise SmlaError(st, "sparse_mla_decode")
    return out, lse


# Scratch size of decode_static_scratch (SMLA_STATIC_SCRATCH_BYTES).
STATIC_SCRATCH_BYTES = 24 << 20


def decode_static_scratch(q, kv, indices, scale: float, out, lse, *, kv_row_scale=None, page_table=None,
                          page_size: int = 0, nsplit: int = 0):
    """sparse_mla_decode_static_scratch: the decode step into caller-given
    ``out`` [B,64,512] bf16 and ``lse`` [B,64] fp32, with the split partials
    in the library's own static device scratch (STATIC_SCRATCH_BYTES), for
    callers that cannot allocate.  Calls that overlap in time on one device
    share that scratch and race; issue them on one stream."""
    _check_inputs(q, kv, indices, kv_row_scale, page_table, page_size)
    shape = shape_for(q, kv, indices, page_table=page_table, page_size=page_size, nsplit=nsplit)
    st = lib.sparse_mla_decode_static_scratch(ctypes.byref(shape), _ptr(q), _ptr(kv), _ptr(kv_row_scale),
                                              _ptr(page_table), _ptr(indices), float(scale), _ptr(out),
                                              _ptr(lse), _stream(q.device))
    if st != 0:
        raise SmlaError(st, "sparse_mla_decode_static_scratch")
    return out, lse


def decode_split(q, kv, indices, scale: float, *, kv_row_scale=None, page_table=None,
                 page_size: int = 0, nsplit: int = 0, out=None, lse=None, workspace=None):
    """The split kernel alone.  Returns (nsplit, out, lse, workspace); with
    nsplit > 1 the partial results are in the workspace (see the header)."""
    _check_inputs(q, kv, indices, kv_row_scale, page_table, page_size)
    shape = shape_for(q, kv, indices, page_table=page_table, page_size=page_size, nsplit=nsplit)
    dev = q.device
    o_shape, l_shape = _result_shapes(q)
    if out is None:
        out = torch.empty(o_shape, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(l_shape, dtype=torch.float32, device=dev)
    nplan = plan_nsplit(shape)
    ws_bytes = partials_size(q.shape[0] * _tokens(q), nplan) if nplan > 1 else 0
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    n = ctypes.c_int32(0)
    st = lib.sparse_mla_decode_split(ctypes.byref(shape), _ptr(q), _ptr(kv), _ptr(kv_row_scale),
                                     _ptr(page_table), _ptr(indices), float(scale), _ptr(out),
                                     _ptr(lse), _ptr(workspace),
                                     0 if workspace is None else workspace.numel(), ctypes.byref(n),
                                     _stream(dev))
    if st != 0:
        raise SmlaError(st, "sparse_mla_decode_split")
    return n.value, out, lse, workspace


def partials_size(batch: int, nsplit: int) -> int:
    """Workspace bytes sparse_mla_decode_split needs to hold the partials of
    `nsplit` splits (fp32 O and lse), rounded up to 256."""
    b = batch * nsplit * H * (D_V + 1) * 4
    return (b + 255) // 256 * 256


def partial_views(workspace, batch: int, nsplit: int):
    """(partial_o [B, nsplit, 64, 512] fp32, partial_lse [B, nsplit, 64] fp32)
    views of a split workspace."""
    n_o = batch * nsplit * H * D_V
    f = workspace.view(torch.float32)
    return f[:n_o].view(batch, nsplit, H, D_V), f[n_o:n_o + batch * nsplit * H].view(batch, nsplit, H)


def combine(partial_o, partial_lse, out=None, lse=None):
    """out, lse = log-sum-exp combine of per-split partials (sparse_mla_combine)."""
    B, n, h, dv = partial_o.shape
    dev = partial_o.device
    if out is None:
        out = torch.empty((B, h, dv), dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty((B, h), dtype=torch.float32, device=dev)
    st = lib.sparse_mla_combine(B, h, dv, n, _ptr(partial_o), _ptr(partial_lse), _ptr(out), _ptr(lse),
                                _stream(dev))
    if st != 0:
        raise SmlaError(st, "sparse_mla_combine")
    return out, lse


def decode_stalled(q, kv, indices, scale: float, wait_limit_cycles: int, out=None, lse=None):
    """sparse_mla_decode_stalled (a test hook): launches the decode kernel
    on a flat bf16 cache with the score-MMA warp waiting on a barrier that
    nothing arrives on and every pipeline wait limited to
    ``wait_limit_cycles``.  Every wait runs out and the kernel sets the
    device error word's timeout bit; ``out`` and ``lse`` are left
    unwritten.  Returns (out, lse)."""
    _check_inputs(q, kv, indices, None, None, 0)
    shape = shape_for(q, kv, indices)
    dev = q.device
    o_shape, l_shape = _result_shapes(q)
    if out is None:
        out = torch.empty(o_shape, dtype=torch.bfloat16, device=dev)
    if lse is None:
        lse = torch.empty(l_shape, dtype=torch.float32, device=dev)
    st = lib.sparse_mla_decode_stalled(ctypes.byref(shape), _ptr(q), _ptr(kv), _ptr(indices), float(scale),
                                       _ptr(out), _ptr(lse), int(wait_limit_cycles), _stream(dev))
    if st != 0:
        raise SmlaError(st, "sparse_mla_decode_stalled")
    return out, lse


def device_error() -> int:
    """Reads and clears the device error word (synchronous)."""
    code = ctypes.c_uint32(0)
    st = lib.sparse_mla_get_device_error(ctypes.byref(code))
    if st not in (0, 5, 6, 7):
        raise SmlaError(st, "sparse_mla_get_device_error")
    return code.value


class DecodePlan:
    """A decode call with its arguments marshalled once.

    For repeated calls on fixed buffers (serving loops, CUDA-graph capture,
    benchmarking): run() is a single call into the library with no
    per-call Python-side checks.  The tensors must stay alive and keep their
    addresses while the plan is in use.
    """

    def __init__(self, q, kv, indices, scale: float, *, kv_row_scale=None, page_table=None,
                 page_size: int = 0, nsplit: int = 0, out=None, lse=None, workspace=None):
        _check_inputs(q, kv, indices, kv_row_scale, page_table, page_size)
        self.shape = shape_for(q, kv, indices, page_table=page_table, page_size=page_size, nsplit=nsplit)
        dev = q.device
        self.nsplit = plan_nsplit(self.shape)
        self.merge = plan_merge(self.shape)
        # the splits merge inside the split kernel (one launch, no combine):
        # in a thread-block cluster, or (stream-K) by the last CTA of a row
        self.clustered = self.merge == 1
        self.streamk = self.merge == 3
        o_shape, l_shape = _result_shapes(q)
        self.out = out if out is not None else torch.empty(o_shape, dtype=torch.bfloat16, device=dev)
        self.lse = lse if lse is not None else torch.empty(l_shape, dtype=torch.float32, device=dev)
        ws = workspace_size(self.shape)
        self.workspace = workspace if workspace is not None or ws == 0 else \
            torch.empty(ws, dtype=torch.uint8, device=dev)
        self._keep = (q, kv, indices, kv_row_scale, page_table)
        wsp = _ptr(self.workspace)
        wsn = 0 if self.workspace is None else self.workspace.numel()
        self._stream = _stream(dev)
        self._args = (ctypes.byref(self.shape), _ptr(q), _ptr(kv), _ptr(kv_row_scale), _ptr(page_table),
                      _ptr(indices), float(scale), _ptr(self.out), _ptr(self.lse), wsp, wsn)
        self._split_args = self._args + (None,)
        if self.nsplit > 1 and not self.clustered:
            rows = q.shape[0] * _tokens(q)
            po, pl = partial_views(self.workspace, rows, self.nsplit)
            self._combine_args = (rows, H, D_V, self.nsplit, _ptr(po), _ptr(pl), _ptr(self.out),
                                  _ptr(self.lse))
        else:
            self._combine_args = None

    def run(self, stream=None):
        st = lib.sparse_mla_decode(*self._args, self._stream if stream is None else stream)
        if st != 0:
            raise SmlaError(st, "sparse_mla_decode")

    def run_split(self, stream=None):
        """The split kernel of run(): all of run() when the splits reduce on chip."""
        if self.clustered or self.streamk:
            return self.run(stream)
        st = lib.sparse_mla_decode_split(*self._split_args, self._stream if stream is None else stream)
        if st != 0:
            raise SmlaError(st, "sparse_mla_decode_split")

    def run_combine(self, stream=None):
        if self._combine_args is None:
            return
        st = lib.sparse_mla_combine(*self._combine_args, self._stream if stream is None else stream)
        if st != 0:
            raise SmlaError(st, "sparse_mla_combine")


# ------------------------------------------------- per-step tensors on the host
def host_staging_size(shape: SmlaShape) -> int:
    """Device staging bytes of sparse_mla_decode_host for ``shape``."""
    return lib.sparse_mla_host_staging_size(ctypes.byref(shape))


def _check_host_inputs(q_host, kv, indices_host, kv_row_scale, page_table_host, page_size, out_host, lse_host):
    dsv4 = is_dsv4(kv)
    d_qk = DSV4_D_QK if dsv4 else D_QK
    for name, t in (("q_host", q_host), ("indices_host", indices_host), ("page_table_host", page_table_host),
                    ("out_host", out_host), ("lse_host", lse_host)):
        if t is not None and (t.is_cuda or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous host tensor")
    for name, t in (("kv", kv), ("kv_row_scale", kv_row_scale)):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if q_host.dtype != torch.bfloat16 or q_host.dim() not in (3, 4) or q_host.shape[-2:] != (H, d_qk):
        raise ValueError(f"q_host must be bf16 [B, 64, {d_qk}] or [B, T, 64, {d_qk}]")
    if (indices_host.dtype != torch.int32 or indices_host.dim() != q_host.dim() - 1
            or indices_host.shape[:-1] != q_host.shape[:-2]):
        raise ValueError("indices_host must be int32 [B, topk] ([B, T, topk] for q [B, T, 64, d])")
    if page_size and (page_table_host is None or page_table_host.dtype != torch.int32):
        raise ValueError("paged cache needs int32 page_table_host [B, pages_per_seq]")
    o_shape, l_shape = _result_shapes(q_host)
    if out_host.dtype != torch.bfloat16 or tuple(out_host.shape) != o_shape:
        raise ValueError("out_host must be bf16 [B, (T,) 64, 512]")
    if lse_host.dtype != torch.float32 or tuple(lse_host.shape) != l_shape:
        raise ValueError("lse_host must be float32 [B, (T,) 64]")


class HostDecodePlan:
    """sparse_mla_decode_host with its arguments marshalled once.

    q_host, indices_host (and page_table_host) are host tensors the caller
    refills between steps; out_host and lse_host receive each step's
    results.  Pinned host tensors make the copies asynchronous.  kv and
    kv_row_scale are device tensors.  run(stream) enqueues one step (copies
    in, decode, copies out) on ``stream`` (default: the current stream) and
    returns; the results are ready once that stream has reached it.  Plans
    used on different streams at the same time need their own staging,
    which each plan allocates unless one is given."""

    def __init__(self, q_host, kv, indices_host, scale: float, *, kv_row_scale=None, page_table_host=None,
                 page_size: int = 0, nsplit: int = 0, out_host=None, lse_host=None, staging=None):
        pin = q_host.is_pinned()
        o_shape, l_shape = _result_shapes(q_host)
        if out_host is None:
            out_host = torch.empty(o_shape, dtype=torch.bfloat16, pin_memory=pin)
        if lse_host is None:
            lse_host = torch.empty(l_shape, dtype=torch.float32, pin_memory=pin)
        _check_host_inputs(q_host, kv, indices_host, kv_row_scale, page_table_host, page_size, out_host,
                           lse_host)
        if is_dsv4(kv):
            if kv_row_scale is not None or page_size != 64:
                raise ValueError("DeepSeek-V4 pages: no kv_row_scale, page_size 64")
        elif (kv.dtype == torch.uint8) != (kv_row_scale is not None):
            raise ValueError("an fp8 cache needs kv_row_scale, a bf16 cache none")
        self.shape = shape_for(q_host, kv, indices_host, page_table=page_table_host, page_size=page_size,
                               nsplit=nsplit)
        need = host_staging_size(self.shape)
        if staging is None:
            staging = torch.empty(need, dtype=torch.uint8, device=kv.device)
        self.out_host, self.lse_host, self.staging = out_host, lse_host, staging
        self._keep = (q_host, kv, indices_host, kv_row_scale, page_table_host)
        self._device = kv.device
        self._args = (ctypes.byref(self.shape), _ptr(q_host), _ptr(kv), _ptr(kv_row_scale), _ptr(page_table_host),
                      _ptr(indices_host), float(scale), _ptr(out_host), _ptr(lse_host), _ptr(staging),
                      staging.numel())

    def run(self, stream=None):
        s = _stream(self._device) if stream is None else (stream.cuda_stream if hasattr(stream, "cuda_stream")
                                                          else stream)
        st = lib.sparse_mla_decode_host(*self._args, s)
        if st != 0:
            raise SmlaError(st, "sparse_mla_decode_host")


def decode_host(q_host, kv, indices_host, scale: float, *, kv_row_scale=None, page_table_host=None,
                page_size: int = 0, nsplit: int = 0, out_host=None, lse_host=None):
    """One decode step with the per-step tensors on the host: returns
    (out_host, lse_host) after synchronising the current stream."""
    plan = HostDecodePlan(q_host, kv, indices_host, scale, kv_row_scale=kv_row_scale,
                          page_table_host=page_table_host, page_size=page_size, nsplit=nsplit,
                          out_host=out_host, lse_host=lse_host)
    plan.run()
    torch.cuda.current_stream(kv.device).synchronize()
    return plan.out_host, plan.lse_host


# ------------------------------------------------------------------ indexer
def indexer_shape(batch: int, topk: int, max_ctx: int, pages_per_seq: int, num_key_rows: int) -> IndexerShape:
    return IndexerShape(batch, IX_HEADS, IX_DIM, topk, max_ctx, 64, pages_per_seq, 0, num_key_rows)


def _check_indexer(q, w, k_cache, page_table, ctx_len):
    for name, t in (("q", q), ("w", w), ("k_cache", k_cache), ("page_table", page_table), ("ctx_len", ctx_len)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if q.dtype != torch.bfloat16 or q.dim() != 3 or q.shape[1:] != (IX_HEADS, IX_DIM):
        raise ValueError("q must be bf16 [B, 64, 128]")
    B = q.shape[0]
    if w.dtype != torch.float32 or tuple(w.shape) != (B, IX_HEADS):
        raise ValueError("w must be float32 [B, 64]")
    if k_cache.dtype != torch.bfloat16 or k_cache.dim() != 2 or k_cache.shape[1] != IX_DIM:
        raise ValueError("k_cache must be bf16 [rows, 128]")
    if page_table.dtype != torch.int32 or page_table.dim() != 2 or page_table.shape[0] != B:
        raise ValueError("page_table must be int32 [B, pages_per_seq]")
    if ctx_len.dtype != torch.int32 or tuple(ctx_len.shape) != (B,):
        raise ValueError("ctx_len must be int32 [B]")


class IndexerPlan:
    """The indexer step with its arguments marshalled once: scores
    ([B, max_ctx] fp32) and the top-k positions ([B, topk] int32) into
    buffers the plan owns (or the caller gives).  run() is one call into
    the library (two launches)."""

    def __init__(self, q, w, k_cache, page_table, ctx_len, topk: int, *, max_ctx: int | None = None,
                 scores=None, indices=None):
        _check_indexer(q, w, k_cache, page_table, ctx_len)
        B = q.shape[0]
        if max_ctx is None:
            max_ctx = page_table.shape[1] * 64
        self.shape = indexer_shape(B, topk, max_ctx, page_table.shape[1], k_cache.shape[0])
        dev = q.device
        self.scores = scores if scores is not None else torch.empty((B, max_ctx), dtype=torch.float32, device=dev)
        self.indices = indices if indices is not None else torch.empty((B, topk), dtype=torch.int32, device=dev)
        self._keep = (q, w, k_cache, page_table, ctx_len)
        self._stream = _stream(dev)
        self._args = (ctypes.byref(self.shape), _ptr(q), _ptr(w), _ptr(k_cache), _ptr(page_table), _ptr(ctx_len),
                      _ptr(self.scores), _ptr(self.indices))

    def run(self, stream=None):
        st = lib.sparse_mla_indexer(*self._args, self._stream if stream is None else stream)
        if st != 0:
            raise SmlaError(st, "sparse_mla_indexer")

    def run_scores(self, stream=None):
        st = lib.sparse_mla_indexer_scores(*self._args[:7], self._stream if stream is None else stream)
        if st != 0:
            raise SmlaError(st, "sparse_mla_indexer_scores")

    def run_topk(self, stream=None):
        st = lib.sparse_mla_indexer_topk(self._args[0], self._args[6], self._args[5], self._args[7],
                                         self._stream if stream is None else stream)
        if st != 0:
            raise SmlaError(st, "sparse_mla_indexer_topk")


def indexer(q, w, k_cache, page_table, ctx_len, topk: int, *, max_ctx: int | None = None):
    """One indexer step: returns (indices [B, topk] int32, scores [B, max_ctx]
    fp32), enqueued on the current stream."""
    plan = IndexerPlan(q, w, k_cache, page_table, ctx_len, topk, max_ctx=max_ctx)
    plan.run()
    return plan.indices, plan.scores
