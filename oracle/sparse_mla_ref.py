"""fp64 CPU oracle for the sparse-MLA decode step.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm use it.  It shares no code, table
or constant generator with the CUDA library; it never reads a value the CUDA
path produced.

Pages cited (titles of the source web pages):
  [Design]    "The MMA Sparse-MLA Decode Kernel: A Deep Dive into AI Inference
               Optimization on Blackwell GPUs"
  [Truth]     "The Moment of Truth: Analyzing a Custom MMA Kernel's Performance
               on Blackwell GPUs"
  [Pivot]     "The Pivot Point: When a 6.3x Kernel Speedup Reveals the Next
               Bottleneck"

What it computes (the plain definition, no tiling, no online softmax):
for every sequence b and head h, over the valid entries j of the top-k index
list (index -1 = padding, skipped),

    s_j       = scale * sum_{d < d_qk} q[b,h,d] * k_j[d]
    out[b,h,:] = sum_j exp(s_j - M) * k_j[:d_v] / sum_j exp(s_j - M)
    lse[b,h]  = M + ln sum_j exp(s_j - M),          M = max_j s_j

where k_j is the gathered cache row (its first d_v dims are the value).
[Design] "The Agent Reasoning" -> "Kernel Structure Analysis" (one query
attends over the gathered rows; scores then output accumulation),
"Design Decisions" item 6 (fp32 accumulation; the oracle uses fp64) and
"Edge Case Handling" (invalid tokens take no part in the softmax).  A sequence
with no valid entry yields out = 0, lse = -inf (the pages use a -1e30 score
sentinel; with every entry masked that sentinel would give equal weights, so
this library defines the all-padding case instead).

Split-K identity used by the kernels and pinned here: partial results over a
partition of the index list combine exactly by log-sum-exp weights,
[Truth] "The Split-K Solution: Reasoning About the Fix"; [Pivot] "The
Reasoning: Weighing Two Paths".

Parity status: every function here is pinned by ``tests/test_oracle_pins.py``
against closed forms, library routines (torch float64 attention, torch's
bf16 / float8_e4m3fn decoders) and brute force; none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "bf16_bits_to_f64",
    "e4m3fn_to_f64",
    "ue8m0_to_f64",
    "dsv4_rows_f64",
    "f64_to_bf16_bits_rne",
    "resolve_rows",
    "gather_rows_f64",
    "attend_rows",
    "sparse_mla_decode",
    "sparse_mla_decode_multi_token",
    "combine_partials",
]


# --------------------------------------------------------------------------
# Number decoding (exact).
# --------------------------------------------------------------------------
def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Decode bfloat16 bit patterns (uint16) to float64 exactly.

    A bfloat16 value is, by definition, the upper 16 bits of an IEEE-754
    binary32; placing the bits there and widening is exact.
    """
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def e4m3fn_to_f64(codes: np.ndarray) -> np.ndarray:
    """Decode OCP FP8 E4M3 ("fn" variant, as torch.float8_e4m3fn) to float64.

    Layout S.EEEE.MMM, exponent bias 7.  E = 0: subnormal, value m/8 * 2^-6.
    Otherwise 2^(E-7) * (1 + m/8).  There is no infinity; S.1111.111 is NaN
    (so the largest finite magnitude is 1.75 * 2^8 = 448).
    [Design] "Potential Mistakes ..." -> "The Validation Strategy Risk" warns
    that random fp8 bytes may be NaN codes; the input generators never emit
    them, and this decoder returns NaN for them.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where((c & 0x80) != 0, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    normal = np.ldexp(1.0 + m / 8.0, (e - 7).astype(np.int64))
    sub = np.ldexp(m / 8.0, -6)
    val = sign * np.where(e == 0, sub, normal)
    return np.where((e == 15) & ((c & 0x7) == 7), np.nan, val)


def f64_to_bf16_bits_rne(x: np.ndarray) -> np.ndarray:
    """Round float64 to the nearest bfloat16 (ties to even), returning bits.

    Used only for diagnostics (distance of a result from bf16(oracle) in
    bf16 ulps).  Written from the format: 8 significant bits for normal
    numbers (exponent >= -126), a fixed 2^-133 step below that, overflow to
    +-inf beyond the largest finite bf16 (0x7F7F).
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.uint16)
    flat = x.reshape(-1)
    of = out.reshape(-1)
    _, ex = np.frexp(flat)                         # flat = mant * 2^ex, |mant| in [0.5,1)
    # unit in the last place of the bf16 result: 2^(ex-8) for normals,
    # 2^-133 for subnormals (ex - 1 < -126).
    ulp_exp = np.maximum(ex - 8, -133)
    q = np.rint(np.ldexp(flat, -ulp_exp))          # rint = round half to even
    r = np.copysign(np.ldexp(q, ulp_exp), flat)   # keeps the sign of zero
    with np.errstate(over="ignore", invalid="ignore"):
        r32 = r.astype(np.float32)                 # exact: r is a bf16 value (or overflows)
    big = np.abs(r) > 3.3895313892515355e38        # max finite bf16
    r32 = np.where(big, np.copysign(np.float32(np.inf), flat).astype(np.float32), r32)
    bits = (r32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    bits = np.where(np.isnan(flat), np.uint16(0x7FC0), bits)
    of[:] = bits
    return out


def ue8m0_to_f64(e: np.ndarray) -> np.ndarray:
    """UE8M0 scale bytes (OCP microscaling E8M0: an unsigned biased exponent,
    no sign, no mantissa) -> 2^(e - 127); the byte 0xFF is NaN."""
    e = np.asarray(e).astype(np.int64)
    out = np.ldexp(1.0, e - 127)
    return np.where(e == 255, np.nan, out)


# DeepSeek-V4 paged cache layout ([Design] "The Agent Reasoning" -> "Cache
# Layout Understanding"; reading: a 64-token page holds the 64 token slots of
# 576 bytes first, then the 64 scale blocks of 8 bytes, 584 bytes per token):
#   slot i, bytes [576 i, 576 i + 448): 448 fp8 e4m3fn codes, the "nope" dims
#   slot i, bytes [576 i + 448, 576 (i+1)): 64 bf16 values, the "rope" dims
#   bytes [36864 + 8 i, 36864 + 8 i + 7): UE8M0 scale of nope group g (dims
#   64 g .. 64 g + 63), g = 0..6; byte 7 unused
DSV4_PAGE_TOKENS = 64
DSV4_SLOT_BYTES = 576
DSV4_PAGE_BYTES = 64 * 584          # 37,376
DSV4_NOPE = 448
DSV4_ROPE = 64


def dsv4_rows_f64(pages: np.ndarray, rows: np.ndarray) -> np.ndarray:
    """Decode physical rows (page * 64 + slot) of a DeepSeek-V4 paged cache
    (uint8 [num_pages, 37376]) to float64 [n, 512]: the 448 nope dims, each
    e4m3fn code times its group's UE8M0 scale, then the 64 bf16 rope dims.
    The whole 512-dim row is both key and value ([Design] "Kernel Structure
    Analysis": the output accumulates nope and rope values)."""
    pages = np.asarray(pages, dtype=np.uint8)
    rows = np.asarray(rows, dtype=np.int64)
    page, slot = rows // DSV4_PAGE_TOKENS, rows % DSV4_PAGE_TOKENS
    base = slot * DSV4_SLOT_BYTES
    codes = pages[page[:, None], base[:, None] + np.arange(DSV4_NOPE)]
    rope_lo = pages[page[:, None], (base + DSV4_NOPE)[:, None] + 2 * np.arange(DSV4_ROPE)].astype(np.uint16)
    rope_hi = pages[page[:, None], (base + DSV4_NOPE + 1)[:, None] + 2 * np.arange(DSV4_ROPE)].astype(np.uint16)
    rope = bf16_bits_to_f64(rope_lo | (rope_hi << 8))
    sb = DSV4_PAGE_TOKENS * DSV4_SLOT_BYTES + 8 * slot
    scales = ue8m0_to_f64(pages[page[:, None], sb[:, None] + np.arange(DSV4_NOPE // 64)])
    nope = e4m3fn_to_f64(codes) * np.repeat(scales, 64, axis=1)
    return np.concatenate([nope, rope], axis=1)


# --------------------------------------------------------------------------
# Index resolution.
# --------------------------------------------------------------------------
def resolve_rows(idx: np.ndarray, *, page_table_row: np.ndarray | None,
                 page_size: int, num_rows: int) -> np.ndarray:
    """Map one sequence's index entries to physical cache rows.

    Flat pool (page_size == 0): an entry is the physical row itself.
    Paged pool: an entry r is a logical position in the sequence; its row is
    page_table_row[r // page_size] * page_size + r % page_size.
    Entries equal to -1 are padding and are returned as -1.  Anything else
    out of range is a caller error (ValueError).
    """
    idx = np.asarray(idx, dtype=np.int64)
    if np.any(idx < -1):
        raise ValueError("index below -1")
    valid = idx >= 0
    rows = np.full(idx.shape, -1, dtype=np.int64)
    if page_size == 0:
        if np.any(idx[valid] >= num_rows):
            raise ValueError("index beyond the pool")
        rows[valid] = idx[valid]
    else:
        pt = np.asarray(page_table_row, dtype=np.int64)
        if np.any(idx[valid] >= pt.shape[0] * page_size):
            raise ValueError("logical position beyond the page table")
        pages = pt[idx[valid] // page_size]
        rows[valid] = pages * page_size + idx[valid] % page_size
        if np.any(rows[valid] >= num_rows) or np.any(pages < 0):
            raise ValueError("page table entry outside the pool")
    return rows


def gather_rows_f64(kv: np.ndarray, rows: np.ndarray, *, kv_format: str,
                    row_scale: np.ndarray | None) -> np.ndarray:
    """Decode the cache rows ``rows`` (all >= 0) to float64.

    kv_format "bf16": kv holds bf16 bit patterns (uint16).
    kv_format "fp8_e4m3_rowscale": kv holds e4m3fn codes (uint8); each row is
    multiplied by its fp32 row scale (in fp64).
    kv_format "dsv4_paged": kv holds DeepSeek-V4 pages (uint8 [pages, 37376]).
    """
    if kv_format == "dsv4_paged":
        return dsv4_rows_f64(kv, rows)
    raw = kv[rows]
    if kv_format == "bf16":
        return bf16_bits_to_f64(raw)
    if kv_format == "fp8_e4m3_rowscale":
        sc = np.asarray(row_scale, dtype=np.float32).astype(np.float64)[rows]
        return e4m3fn_to_f64(raw) * sc[:, None]
    raise ValueError(f"unknown kv_format {kv_format!r}")


# --------------------------------------------------------------------------
# The definition.
# --------------------------------------------------------------------------
def attend_rows(qh: np.ndarray, k: np.ndarray, scale: float, d_v: int):
    """Attention of queries qh [H, d_qk] over rows k [n, d_qk] (float64).

    Returns (out [H, d_v], lse [H]).  n == 0 gives out = 0, lse = -inf.
    """
    H = qh.shape[0]
    if k.shape[0] == 0:
        return np.zeros((H, d_v)), np.full(H, -np.inf)
    s = scale * (qh @ k.T)                         # [H, n]
    M = s.max(axis=1, keepdims=True)
    e = np.exp(s - M)
    W = e.sum(axis=1, keepdims=True)
    out = (e @ k[:, :d_v]) / W
    lse = (M + np.log(W))[:, 0]
    return out, lse


def sparse_mla_decode(q_bits: np.ndarray, kv: np.ndarray, indices: np.ndarray,
                      scale: float, *, d_v: int = 512, kv_format: str = "bf16",
                      kv_row_scale: np.ndarray | None = None,
                      page_table: np.ndarray | None = None, page_size: int = 0,
                      seqs=None):
    """fp64 sparse-MLA decode.

    q_bits      [B, H, d_qk] uint16 (bf16 bits)
    kv          [N, d_qk] uint16 (bf16 bits) or uint8 (e4m3fn codes)
    indices     [B, k] int32, -1 = padding
    page_table  [B, pages_per_seq] int32 when page_size > 0
    seqs        optional iterable of sequence ids to compute (others are NaN)

    Returns out [B, H, d_v] float64 and lse [B, H] float64 (natural log,
    scale inside the exponent).
    """
    q_bits = np.asarray(q_bits)
    B, H, d_qk = q_bits.shape
    if kv_format == "dsv4_paged":
        if d_qk != DSV4_NOPE + DSV4_ROPE or kv.shape[1] != DSV4_PAGE_BYTES:
            raise ValueError("DeepSeek-V4 pages need a 512-dim query and 37376-byte pages")
        num_rows = kv.shape[0] * DSV4_PAGE_TOKENS
    else:
        if kv.shape[1] != d_qk:
            raise ValueError("row width differs from the query width")
        num_rows = kv.shape[0]
    out = np.full((B, H, d_v), np.nan)
    lse = np.full((B, H), np.nan)
    for b in (range(B) if seqs is None else seqs):
        rows = resolve_rows(indices[b],
                            page_table_row=None if page_table is None else page_table[b],
                            page_size=page_size, num_rows=num_rows)
        rows = rows[rows >= 0]
        k = gather_rows_f64(kv, rows, kv_format=kv_format, row_scale=kv_row_scale)
        qh = bf16_bits_to_f64(q_bits[b])
        out[b], lse[b] = attend_rows(qh, k, scale, d_v)
    return out, lse


def sparse_mla_decode_multi_token(q_bits: np.ndarray, kv: np.ndarray, indices: np.ndarray, scale: float, *,
                                  d_v: int = 512, kv_format: str = "bf16", kv_row_scale: np.ndarray | None = None,
                                  page_table: np.ndarray | None = None, page_size: int = 0):
    """fp64 decode of s_q query tokens per sequence (speculative / multi-token
    decode): token t of sequence b attends over its own index list
    indices[b, t] through the sequence's page table, exactly as one decode
    token does.  A list shared by all tokens is the special case.

    q_bits  [B, s_q, H, d_qk] uint16, indices [B, s_q, k] int32,
    page_table [B, pages_per_seq] int32 when page_size > 0.
    Returns out [B, s_q, H, d_v] and lse [B, s_q, H] (float64)."""
    q_bits = np.asarray(q_bits)
    B, T, H, d_qk = q_bits.shape
    out = np.empty((B, T, H, d_v))
    lse = np.empty((B, T, H))
    for t in range(T):
        out[:, t], lse[:, t] = sparse_mla_decode(q_bits[:, t], kv, np.asarray(indices)[:, t], scale, d_v=d_v,
                                                 kv_format=kv_format, kv_row_scale=kv_row_scale,
                                                 page_table=page_table, page_size=page_size)
    return out, lse


def combine_partials(outs, lses):
    """Merge per-split results over disjoint parts of the index list.

    outs: sequence of [..., d_v] arrays (each already normalised by its own
    softmax sum), lses: matching [...] log-sum-exp values.  With
    L = ln sum_s exp(lse_s), the merged output is sum_s exp(lse_s - L) o_s and
    the merged lse is L.  Splits with lse = -inf carry weight 0; if every
    split is empty the result is out = 0, lse = -inf.
    [Truth] "The Split-K Solution: Reasoning About the Fix".
    """
    lses = np.stack([np.asarray(x, dtype=np.float64) for x in lses])
    outs = np.stack([np.asarray(x, dtype=np.float64) for x in outs])
    mx = lses.max(axis=0)
    finite = np.isfinite(mx)
    mx_safe = np.where(finite, mx, 0.0)
    w = np.where(np.isfinite(lses), np.exp(lses - mx_safe), 0.0)
    tot = w.sum(axis=0)
    L = np.where(finite, mx_safe + np.log(np.where(finite, tot, 1.0)), -np.inf)
    wn = np.where(finite, w / np.where(finite, tot, 1.0), 0.0)
    out = (wn[..., None] * np.where(np.isfinite(lses)[..., None], outs, 0.0)).sum(axis=0)
    return out, L


def lse_rel_err(lse_test, lse_ref):
    """|dlse| / max(|lse_ref|, 1): the relative lse error, made well defined
    near lse = 0; -inf == -inf counts as exact."""
    a = np.asarray(lse_test, dtype=np.float64)
    r = np.asarray(lse_ref, dtype=np.float64)
    both_inf = np.isneginf(a) & np.isneginf(r)
    d = np.where(both_inf, 0.0, np.abs(a - r))
    return d / np.maximum(np.abs(np.where(np.isfinite(r), r, 1.0)), 1.0)

