"""Seeded synthetic inputs for the sparse-MLA decode step.

This module generates inputs only.  It holds none of the method's
arithmetic, and both the CUDA library's tests/bench and the fp64 oracle take
their inputs from it.  All tensors are CPU torch tensors; callers copy them
to the device.

Workload recipes (shapes, value distributions, index structure):

  c1  B=1,  H=64, q bf16 ~N(0,1); flat bf16 pool [4096, 576] ~N(0,1);
      top-k = 512 distinct uniform rows.
  c2  B=16; per-sequence cache lengths uniform in [256, 8192] in one flat
      bf16 pool (sequence b owns a contiguous run of rows); top-k = 512
      distinct uniform rows of its own run; when a run is shorter than 512
      all its rows are used in random order and the list is padded with -1.
  c3  B=64; 16384 rows per sequence; top-k = 512: 256 distinct rows from the
      last 1024 (recency-skewed) and 256 distinct uniform rows from the rest,
      sorted ascending.
  c4a/c4b  B=1 / B=2; 65536 rows per sequence; top-k = 2048 distinct
      uniform; q multiplied by 4 (peaky softmax).
  c5  B=128; paged pool of 16384 pages of 64 rows (1,048,576 rows), fp8
      e4m3fn codes with one fp32 scale per row (row amax / 448 of an N(0,1)
      row); each sequence maps 8192 logical positions through a 128-entry
      page table (a random permutation of all pages); top-k = 2048 distinct
      uniform logical positions.

scale = 1/sqrt(576) everywhere.  Seeds: workload ci uses seed 1000 + i unless
one is given.  Normals come from torch's CPU generator (fp32, rounded to
bf16); index sets from numpy's PCG64 generator.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np
import torch

H = 64
D_QK = 576
D_V = 512
SCALE = 1.0 / math.sqrt(D_QK)


@dataclasses.dataclass
class Workload:
    name: str
    q: torch.Tensor                      # [B, H, D_QK] bfloat16
    kv: torch.Tensor                     # [N, D_QK] bfloat16, or uint8 (e4m3fn codes)
    indices: torch.Tensor                # [B, topk] int32, -1 = padding
    scale: float = SCALE
    kv_row_scale: torch.Tensor | None = None   # [N] float32 (fp8 pools)
    page_table: torch.Tensor | None = None     # [B, pages_per_seq] int32
    page_size: int = 0
    d_v: int = D_V
    meta: dict = dataclasses.field(default_factory=dict)
    layout: str = ""                           # "dsv4": DeepSeek-V4 pages (uint8 [pages, 37376])

    @property
    def batch(self) -> int:
        return self.q.shape[0]

    @property
    def topk(self) -> int:
        return self.indices.shape[-1]

    @property
    def tokens(self) -> int:
        """Query tokens per sequence (q [B, T, 64, d] for T > 1)."""
        return self.q.shape[1] if self.q.dim() == 4 else 1

    @property
    def rows(self) -> int:
        """Decode rows: sequences x query tokens."""
        return self.batch * self.tokens

    @property
    def kv_format(self) -> str:
        if self.layout == "dsv4":
            return "dsv4_paged"
        return "fp8_e4m3_rowscale" if self.kv.dtype == torch.uint8 else "bf16"

    def valid_count(self) -> int:
        return int((self.indices >= 0).sum())

    # numpy views for the oracle (bit patterns, no arithmetic)
    def np_q_bits(self) -> np.ndarray:
        return self.q.view(torch.int16).numpy().view(np.uint16)

    def np_kv(self) -> np.ndarray:
        if self.kv.dtype == torch.uint8:
            return self.kv.numpy()
        return self.kv.view(torch.int16).numpy().view(np.uint16)


def _normal_bf16(gen: torch.Generator, shape, mult: float = 1.0,
                 chunk_rows: int = 65536) -> torch.Tensor:
    """N(0,1) (times ``mult``) in fp32, rounded to bf16; generated in row
    chunks to bound host memory."""
    rows = shape[0]
    out = torch.empty(shape, dtype=torch.bfloat16)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=gen, dtype=torch.float32)
        if mult != 1.0:
            x.mul_(mult)
        out[r0:r1] = x.to(torch.bfloat16)
    return out


def _fp8_rows(gen: torch.Generator, rows: int, chunk_rows: int = 65536):
    """N(0,1) rows quantised to e4m3fn with a per-row scale amax/448."""
    codes = torch.empty((rows, D_QK), dtype=torch.uint8)
    scales = torch.empty((rows,), dtype=torch.float32)
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        x = torch.randn((r1 - r0, D_QK), generator=gen, dtype=torch.float32)
        s = x.abs().amax(dim=1) / 448.0
        s = torch.where(s > 0, s, torch.ones_like(s))
        codes[r0:r1] = (x / s[:, None]).to(torch.float8_e4m3fn).view(torch.uint8)
        scales[r0:r1] = s
    return codes, scales


def _distinct(rng: np.random.Generator, n: int, k: int) -> np.ndarray:
    return rng.choice(n, size=k, replace=False).astype(np.int64)


def flat_per_seq(B: int, rows_per_seq: int, topk: int, *, seed: int,
                 q_mult: float = 1.0, index_mode: str = "uniform",
                 recent_window: int = 1024, name: str = "flat") -> Workload:
    """Flat bf16 pool of B * rows_per_seq rows; sequence b owns rows
    [b*R, (b+1)*R).  index_mode "uniform": topk distinct uniform rows;
    "recency": half from the last ``recent_window`` rows, half uniform from
    the rest, all distinct, sorted ascending."""
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    q = _normal_bf16(gen, (B, H, D_QK), mult=q_mult)
    kv = _normal_bf16(gen, (B * rows_per_seq, D_QK))
    idx = np.empty((B, topk), dtype=np.int64)
    for b in range(B):
        if index_mode == "uniform":
            sel = _distinct(rng, rows_per_seq, topk)
        elif index_mode == "recency":
            w = min(recent_window, rows_per_seq)
            n_recent = topk // 2
            recent = rows_per_seq - w + _distinct(rng, w, n_recent)
            rest_pool = np.setdiff1d(np.arange(rows_per_seq), recent, assume_unique=True)
            rest = rest_pool[_distinct(rng, rest_pool.size, topk - n_recent)]
            sel = np.sort(np.concatenate([recent, rest]))
        else:
            raise ValueError(index_mode)
        idx[b] = sel + b * rows_per_seq
    return Workload(name=name, q=q, kv=kv, indices=torch.from_numpy(idx.astype(np.int32)),
                    meta=dict(B=B, rows_per_seq=rows_per_seq, topk=topk, seed=seed,
                              q_mult=q_mult, index_mode=index_mode))


def flat_varlen(B: int, len_lo: int, len_hi: int, topk: int, *, seed: int,
                name: str = "varlen") -> Workload:
    """One flat bf16 pool holding B runs with lengths uniform in
    [len_lo, len_hi]; runs shorter than topk are used whole (shuffled) and
    padded with -1 at the tail."""
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    lens = rng.integers(len_lo, len_hi + 1, size=B)
    offs = np.concatenate([[0], np.cumsum(lens)[:-1]])
    q = _normal_bf16(gen, (B, H, D_QK))
    kv = _normal_bf16(gen, (int(lens.sum()), D_QK))
    idx = np.full((B, topk), -1, dtype=np.int64)
    for b in range(B):
        if lens[b] >= topk:
            idx[b] = _distinct(rng, int(lens[b]), topk) + offs[b]
        else:
            idx[b, :lens[b]] = rng.permutation(int(lens[b])) + offs[b]
    return Workload(name=name, q=q, kv=kv, indices=torch.from_numpy(idx.astype(np.int32)),
                    meta=dict(B=B, lens=lens.tolist(), topk=topk, seed=seed))


def paged_fp8(B: int, rows_per_seq: int, total_pages: int, topk: int, *, seed: int,
              page_size: int = 64, name: str = "paged_fp8") -> Workload:
    """Paged fp8 e4m3fn pool with per-row fp32 scales; each sequence's page
    table row is a slice of one random permutation of all pages."""
    pps = rows_per_seq // page_size
    if B * pps > total_pages:
        raise ValueError("not enough pages for distinct page tables")
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    q = _normal_bf16(gen, (B, H, D_QK))
    codes, scales = _fp8_rows(gen, total_pages * page_size)
    perm = rng.permutation(total_pages)[: B * pps].reshape(B, pps)
    idx = np.stack([_distinct(rng, rows_per_seq, topk) for _ in range(B)])
    return Workload(name=name, q=q, kv=codes, indices=torch.from_numpy(idx.astype(np.int32)),
                    kv_row_scale=scales, page_table=torch.from_numpy(perm.astype(np.int32)),
                    page_size=page_size,
                    meta=dict(B=B, rows_per_seq=rows_per_seq, total_pages=total_pages,
                              topk=topk, seed=seed))


def paged_bf16(B: int, rows_per_seq: int, total_pages: int, topk: int, *, seed: int,
               name: str = "paged_bf16") -> Workload:
    """Paged bf16 pool [total_pages * 64, 576] of N(0,1) rows; page tables
    and index lists as in paged_fp8."""
    pps = rows_per_seq // 64
    if B * pps > total_pages:
        raise ValueError("not enough pages for distinct page tables")
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    q = _normal_bf16(gen, (B, H, D_QK))
    kv = _normal_bf16(gen, (total_pages * 64, D_QK))
    perm = rng.permutation(total_pages)[: B * pps].reshape(B, pps)
    idx = np.stack([_distinct(rng, rows_per_seq, topk) for _ in range(B)])
    return Workload(name=name, q=q, kv=kv, indices=torch.from_numpy(idx.astype(np.int32)),
                    page_table=torch.from_numpy(perm.astype(np.int32)), page_size=64,
                    meta=dict(B=B, rows_per_seq=rows_per_seq, total_pages=total_pages, topk=topk, seed=seed))


def _token_lists(rng, B: int, T: int, R: int, topk: int, overlap: float, *, flat: bool) -> np.ndarray:
    """[B, T, topk] index lists: token 0 takes topk distinct uniform
    positions of [0, R); token t > 0 keeps round(overlap * topk) of them (a
    random subset) and draws the rest afresh, distinct within its list.
    flat: sequence b's positions are offset to rows [b R, (b+1) R)."""
    idx = np.empty((B, T, topk), dtype=np.int64)
    keep = int(round(overlap * topk))
    for b in range(B):
        first = _distinct(rng, R, topk)
        idx[b, 0] = first
        for t in range(1, T):
            kept = rng.choice(first, size=keep, replace=False)
            rest_pool = np.setdiff1d(np.arange(R), kept, assume_unique=True)
            fresh = rest_pool[_distinct(rng, rest_pool.size, topk - keep)]
            idx[b, t] = rng.permutation(np.concatenate([kept, fresh]))
        if flat:
            idx[b] += b * R
    return idx


def multi_token(B: int, T: int, rows_per_seq: int, total_pages: int, topk: int, *, seed: int,
                fp8: bool = False, paged: bool = True, overlap: float = 0.75,
                name: str = "multi_token") -> Workload:
    """Several query tokens per sequence (multi-token / speculative decode),
    each with its own top-k list.  q [B, T, 64, 576] ~N(0,1) bf16; the cache
    is a 64-row paged pool (bf16, or fp8 e4m3fn with an amax/448 row scale)
    with one page table row per sequence, or, with paged=False, a flat pool
    where sequence b owns rows [b R, (b+1) R).  Token 0 draws topk distinct
    uniform positions; token t > 0 keeps round(overlap * topk) of token 0's
    positions (a random subset) and draws the rest afresh, distinct within
    its list, so that consecutive tokens of a step share most of their
    rows.  indices [B, T, topk]."""
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    q = _normal_bf16(gen, (B * T, H, D_QK)).view(B, T, H, D_QK)
    n_rows = total_pages * 64 if paged else B * rows_per_seq
    if fp8:
        kv, scales = _fp8_rows(gen, n_rows)
    else:
        kv, scales = _normal_bf16(gen, (n_rows, D_QK)), None
    pt = None
    if paged:
        pps = rows_per_seq // 64
        if B * pps > total_pages:
            raise ValueError("not enough pages for distinct page tables")
        pt = torch.from_numpy(rng.permutation(total_pages)[: B * pps].reshape(B, pps).astype(np.int32))
    idx = _token_lists(rng, B, T, rows_per_seq, topk, overlap, flat=not paged)
    return Workload(name=name, q=q, kv=kv, indices=torch.from_numpy(idx.astype(np.int32)),
                    kv_row_scale=scales, page_table=pt, page_size=64 if paged else 0,
                    meta=dict(B=B, T=T, rows_per_seq=rows_per_seq, total_pages=total_pages, topk=topk,
                              seed=seed, overlap=overlap))


DSV4_PAGE_BYTES = 64 * 584          # 64 slots of 576 bytes, then 64 scale blocks of 8 bytes


def paged_dsv4(B: int, rows_per_seq: int, total_pages: int, topk: int, *, seed: int,
               name: str = "paged_dsv4") -> Workload:
    """DeepSeek-V4 paged cache: 64-token pages of 37,376 bytes.  Slot i holds
    448 fp8 e4m3fn "nope" codes then 64 bf16 "rope" values (576 bytes);
    after the 64 slots come 64 scale blocks of 8 bytes, 7 UE8M0 exponents
    (one per 64 nope dims) and a zero byte.  Values are N(0,1); a group's
    scale is the power of two 2^ceil(log2(amax / 448)), so every code is in
    range.  q is [B, 64, 512] (448 nope + 64 rope dims); indices are logical
    positions through a page table (a slice of one random permutation of
    all pages per sequence)."""
    pps = rows_per_seq // 64
    if B * pps > total_pages:
        raise ValueError("not enough pages for distinct page tables")
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    q = _normal_bf16(gen, (B, H, 512))
    pages = torch.zeros((total_pages, DSV4_PAGE_BYTES), dtype=torch.uint8)
    for p0 in range(0, total_pages, 256):
        p1 = min(total_pages, p0 + 256)
        n = (p1 - p0) * 64
        nope = torch.randn((n, 448), generator=gen, dtype=torch.float32).view(n, 7, 64)
        amax = nope.abs().amax(dim=2).clamp_min(1e-30)
        e = torch.ceil(torch.log2(amax / 448.0))
        codes = (nope / torch.exp2(e)[:, :, None]).view(n, 448).to(torch.float8_e4m3fn).view(torch.uint8)
        rope = torch.randn((n, 64), generator=gen, dtype=torch.float32).to(torch.bfloat16).view(torch.uint8)
        slots = torch.cat([codes, rope.view(n, 128)], dim=1).view(p1 - p0, 64 * 576)
        sc = torch.zeros((n, 8), dtype=torch.uint8)
        sc[:, :7] = (e + 127).to(torch.uint8)
        pages[p0:p1, :64 * 576] = slots
        pages[p0:p1, 64 * 576:] = sc.view(p1 - p0, 64 * 8)
    perm = rng.permutation(total_pages)[: B * pps].reshape(B, pps)
    idx = np.stack([_distinct(rng, rows_per_seq, topk) for _ in range(B)])
    return Workload(name=name, q=q, kv=pages, indices=torch.from_numpy(idx.astype(np.int32)),
                    scale=1.0 / math.sqrt(512), page_table=torch.from_numpy(perm.astype(np.int32)),
                    page_size=64, layout="dsv4",
                    meta=dict(B=B, rows_per_seq=rows_per_seq, total_pages=total_pages, topk=topk, seed=seed))


@dataclasses.dataclass
class IndexerWorkload:
    """Inputs of the indexer step: the decode token's indexer query and head
    weights per sequence, a paged bf16 key cache, page tables and context
    lengths."""
    name: str
    q: torch.Tensor            # [B, H, D] bfloat16
    w: torch.Tensor            # [B, H] float32
    k: torch.Tensor            # [pages * 64, D] bfloat16
    page_table: torch.Tensor   # [B, pages_per_seq] int32
    ctx_len: torch.Tensor      # [B] int32
    max_ctx: int
    topk: int
    meta: dict = dataclasses.field(default_factory=dict)

    @property
    def batch(self) -> int:
        return self.q.shape[0]


def indexer_workload(B: int, max_ctx: int, total_pages: int, *, seed: int, topk: int = 512, H: int = 64,
                     D: int = 128, ctx_lo: int | None = None, name: str = "indexer") -> IndexerWorkload:
    """Seeded indexer inputs: q and k N(0,1) in bf16, w N(0,1)/sqrt(H) in
    fp32 (signed), context lengths uniform in [ctx_lo, max_ctx] (all equal to
    max_ctx when ctx_lo is None), page tables slices of one random
    permutation of all pages."""
    pps = (max_ctx + 63) // 64
    if B * pps > total_pages:
        raise ValueError("not enough pages for distinct page tables")
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    q = _normal_bf16(gen, (B, H, D))
    w = (torch.randn((B, H), generator=gen, dtype=torch.float32) / math.sqrt(H)).contiguous()
    k = _normal_bf16(gen, (total_pages * 64, D))
    perm = rng.permutation(total_pages)[: B * pps].reshape(B, pps)
    if ctx_lo is None:
        ctx = np.full(B, max_ctx)
    else:
        ctx = rng.integers(ctx_lo, max_ctx + 1, size=B)
    return IndexerWorkload(name=name, q=q, w=w, k=k, page_table=torch.from_numpy(perm.astype(np.int32)),
                           ctx_len=torch.from_numpy(ctx.astype(np.int32)), max_ctx=max_ctx, topk=topk,
                           meta=dict(B=B, max_ctx=max_ctx, total_pages=total_pages, seed=seed, H=H, D=D))


INDEXER_DESCRIPTION = ("B=32, 8192-token contexts, top-512 of 64 heads x 128 bf16 dims, "
                       "paged keys (4096 pages, 67 MB)")


def make_indexer_config(seed: int | None = None) -> IndexerWorkload:
    """The full-size indexer workload: batch 32 (the pages' steady batch),
    contexts of 8,192 tokens (the pages' context cap), top-512."""
    return indexer_workload(32, 8192, 4096, seed=1007 if seed is None else seed, topk=512, name="indexer")


def indexer_algorithmic_bytes(w: IndexerWorkload) -> int:
    """Bytes the indexer step must move at minimum: the keys of every
    context position (D bf16 each), q, w, the page tables, the context
    lengths and the selected index lists."""
    D = w.q.shape[2]
    n = int(w.ctx_len.sum())
    return int(n * D * 2 + w.q.numel() * 2 + w.w.numel() * 4 + w.page_table.numel() * 4 + w.batch * 4
               + w.batch * w.topk * 4)


CONFIG_NAMES = ("c1", "c2", "c3", "c4a", "c4b", "c5")

CONFIG_DESCRIPTIONS = {
    "c1": "B=1 k=512 flat bf16 pool 4096 rows, uniform distinct",
    "c2": "B=16 k=512 flat bf16 varlen [256,8192], -1 padded",
    "c3": "B=64 k=512 flat bf16 16384 rows/seq, recency-skewed sorted",
    "c4a": "B=1 k=2048 flat bf16 65536 rows/seq, q x4 (split-K stress)",
    "c4b": "B=2 k=2048 flat bf16 65536 rows/seq, q x4 (split-K stress)",
    "c5": "B=128 k=2048 paged(64) fp8 e4m3 + row scale, 8192 rows/seq",
}

# Workloads beyond the headline set, measured and parity-tested the same way
EXTRA_NAMES = ("dsv4", "mt2")
EXTRA_DESCRIPTIONS = {
    "dsv4": "B=32 k=512 DeepSeek-V4 pages (448 fp8 + UE8M0 group scales, 64 bf16 rope), 8192 rows/seq",
    "mt2": "B=64 x 2 query tokens, k=2048 per token (75% shared), paged(64) fp8 e4m3 + row scale, 8192 rows/seq",
}
_BASE_SEEDS = {"c1": 1001, "c2": 1002, "c3": 1003, "c4a": 1004, "c4b": 1004, "c5": 1005, "dsv4": 1006,
               "mt2": 1008}


def make_config(name: str, seed: int | None = None) -> Workload:
    """The full-size workload ``name`` (one of CONFIG_NAMES or EXTRA_NAMES)."""
    base = _BASE_SEEDS[name]
    s = base if seed is None else seed
    if name == "c1":
        return flat_per_seq(1, 4096, 512, seed=s, name="c1")
    if name == "c2":
        return flat_varlen(16, 256, 8192, 512, seed=s, name="c2")
    if name == "c3":
        return flat_per_seq(64, 16384, 512, seed=s, index_mode="recency", name="c3")
    if name == "c4a":
        return flat_per_seq(1, 65536, 2048, seed=s, q_mult=4.0, name="c4a")
    if name == "c4b":
        return flat_per_seq(2, 65536, 2048, seed=s, q_mult=4.0, name="c4b")
    if name == "c5":
        return paged_fp8(128, 8192, 16384, 2048, seed=s, name="c5")
    if name == "dsv4":
        return paged_dsv4(32, 8192, 4096, 512, seed=s, name="dsv4")
    if name == "mt2":
        return multi_token(64, 2, 8192, 16384, 2048, seed=s, fp8=True, overlap=0.75, name="mt2")
    raise KeyError(name)


def reindexed(w: Workload, seed: int) -> Workload:
    """Another batch of the same workload over the same cache: fresh queries
    and fresh index lists drawn by ``w``'s own recipe (the pool, row scales
    and page tables are shared, not copied).  Used to rotate distinct
    batches through a timed loop so that successive steps gather different
    rows of a pool larger than L2."""
    gen = torch.Generator().manual_seed(seed)
    rng = np.random.default_rng(seed)
    m = w.meta
    B, topk = w.batch, w.topk
    q_mult = m.get("q_mult", 1.0)
    q = _normal_bf16(gen, tuple(w.q.shape), mult=q_mult)
    idx = np.full((B, topk), -1, dtype=np.int64)
    if w.tokens > 1:                                  # multi_token: same recipe, new draws
        idx = _token_lists(rng, B, w.tokens, m["rows_per_seq"], topk, m["overlap"], flat=not w.page_size)
        return dataclasses.replace(w, q=q, indices=torch.from_numpy(idx.astype(np.int32)),
                                   meta=dict(m, reindexed_seed=seed))
    if "lens" in m:                                   # flat_varlen
        lens = np.asarray(m["lens"])
        offs = np.concatenate([[0], np.cumsum(lens)[:-1]])
        for b in range(B):
            if lens[b] >= topk:
                idx[b] = _distinct(rng, int(lens[b]), topk) + offs[b]
            else:
                idx[b, :lens[b]] = rng.permutation(int(lens[b])) + offs[b]
    elif w.page_size:                                 # paged pools: logical positions
        for b in range(B):
            idx[b] = _distinct(rng, m["rows_per_seq"], topk)
    else:                                             # flat_per_seq
        R = m["rows_per_seq"]
        for b in range(B):
            if m.get("index_mode", "uniform") == "recency":
                win = min(1024, R)
                n_recent = topk // 2
                recent = R - win + _distinct(rng, win, n_recent)
                rest_pool = np.setdiff1d(np.arange(R), recent, assume_unique=True)
                rest = rest_pool[_distinct(rng, rest_pool.size, topk - n_recent)]
                sel = np.sort(np.concatenate([recent, rest]))
            else:
                sel = _distinct(rng, R, topk)
            idx[b] = sel + b * R
    return dataclasses.replace(w, q=q, indices=torch.from_numpy(idx.astype(np.int32)),
                               meta=dict(m, reindexed_seed=seed))


def shard_seed(name: str, rank: int) -> int | None:
    """Seed of rank ``rank``'s batch of workload ``name`` when the step runs
    as independent per-GPU batches (the op shards over sequences): rank 0
    keeps the workload's own seed (None), rank r > 0 draws a distinct one."""
    if rank < 0:
        raise ValueError("rank must be >= 0")
    if rank == 0:
        return None
    return _BASE_SEEDS[name] + 100_000 * rank


def gathered_row_count(w: Workload) -> int:
    """Cache rows the step must read at least once: the valid entries of
    each index list; with several query tokens per sequence, the union of
    the tokens' lists of a sequence (a row two tokens share is needed from
    memory once)."""
    if w.tokens == 1:
        return w.valid_count()
    idx = w.indices.numpy()
    return int(sum(np.unique(idx[b][idx[b] >= 0]).size for b in range(w.batch)))


def algorithmic_bytes(w: Workload) -> int:
    """Bytes the step must move at minimum: the gathered rows
    (gathered_row_count; row bytes, plus the 4-byte row scale for fp8 pools;
    a DeepSeek-V4 slot's 576 bytes plus its 7 scale bytes), q, out, lse,
    the index lists and the page table.  Padding entries gather nothing."""
    n_valid = gathered_row_count(w)
    if w.layout == "dsv4":
        row, d_qk = 576 + 7, 512
    else:
        row = D_QK * (1 if w.kv.dtype == torch.uint8 else 2) + (4 if w.kv_row_scale is not None else 0)
        d_qk = D_QK
    R = w.rows
    b = n_valid * row
    b += R * H * d_qk * 2          # q
    b += R * H * w.d_v * 2         # out
    b += R * H * 4                 # lse
    b += w.indices.numel() * 4     # indices
    if w.page_table is not None:
        b += w.page_table.numel() * 4
    return int(b)


def algorithmic_flops(w: Workload) -> int:
    """2*H*(d_qk + d_v) flops per valid (decode row, index entry): the
    score and the value contractions."""
    return int(w.valid_count() * 2 * H * (w.q.shape[-1] + w.d_v))
