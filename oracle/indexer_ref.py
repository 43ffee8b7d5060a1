"""fp64 CPU oracle for the indexer step that produces the decode's index list.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
execute this module: only ``tests/``, ``__graft_entry__.smoke()`` and
``bench.py``'s CPU-baseline / reference arm use it.  It shares no code, table
or constant generator with the CUDA library; it never reads a value the CUDA
path produced, except where a test hands it the kernel's own scores to take
the top-k decision in the kernel's precision.

Pages cited (titles of the source web pages):
  [Pivot]     "The Pivot Point: When a 6.3x Kernel Speedup Reveals the Next
               Bottleneck": "The Context: A Campaign in Full Swing" (the
               indexer's batched matrix product, moved from fp32 CUDA cores
               to bf16 tensor cores), "Input Knowledge Required" (the indexer
               selects the top ~512 cache positions per decode step; the
               decode attends to those only) and "Assumptions and Potential
               Mistakes" (the top-512 selection is sensitive to precision).
  [Bench]     "The Moment of Truth: Benchmarking a Custom MMA Kernel for
               DeepSeek-V4-Flash on Blackwell", "Broader Context": the indexer
               must score only the real context (capped at 8192 tokens), not
               the maximum context.

What it computes.  The pages name the step (a batched matrix product of the
decode token's indexer query with the indexer keys of every context position,
then the top-k positions) but not its head combination.  The reading taken
here is the published form of the DeepSeek sparse-attention indexer: per
head h a dot product, a ReLU, and a weighted sum over heads,

    I[b, s] = sum_h w[b, h] * max(0, sum_d q[b, h, d] * k_s[d]),   s < ctx[b]

where k_s is the indexer key of logical position s of sequence b, found
through the sequence's page table (page size 64):
row = page_table[b, s // 64] * 64 + s % 64.  Positions at or past ctx[b]
take no part.  The selection returns the min(topk, ctx[b]) positions with
the largest scores, a tie at the boundary going to the lower position, in
ascending order, padded with -1 to topk.

Parity status: pinned by ``tests/test_oracle_indexer.py`` against a
hand-worked fixture (tests/golden/indexer_handworked.json), torch float64
einsum, a brute-force flat pool, closed forms (w = 0, negative dots) and a
brute-force selection by Python's sorted(); none is "parity unpinned".
"""
from __future__ import annotations

import numpy as np

__all__ = ["bf16_bits_to_f64", "key_rows", "indexer_scores", "topk_positions"]

PAGE = 64


def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) -> float64, exactly: a bf16 is the upper
    half of an IEEE binary32."""
    b = np.asarray(bits).astype(np.uint32) << 16
    return b.view(np.float32).astype(np.float64)


def key_rows(page_table_row: np.ndarray, n: int) -> np.ndarray:
    """Physical key-cache rows of logical positions 0 .. n-1 of one sequence
    (the same 64-token page mapping as the decode's cache)."""
    s = np.arange(n, dtype=np.int64)
    return np.asarray(page_table_row, np.int64)[s // PAGE] * PAGE + s % PAGE


def indexer_scores(q_bits: np.ndarray, w: np.ndarray, k_bits: np.ndarray, page_table: np.ndarray,
                   ctx_len: np.ndarray, max_ctx: int) -> np.ndarray:
    """Scores [B, max_ctx] float64: I[b, s] for s < ctx_len[b], -inf after.

    q_bits [B, H, D] uint16 (bf16), w [B, H] float32, k_bits [rows, D] uint16
    (bf16 key cache), page_table [B, pages_per_seq] int32, ctx_len [B]."""
    B, H, D = q_bits.shape
    out = np.full((B, max_ctx), -np.inf)
    for b in range(B):
        n = int(ctx_len[b])
        if n <= 0:
            continue
        if n > max_ctx or n > page_table.shape[1] * PAGE:
            raise ValueError("context longer than the score row or the page table")
        rows = key_rows(page_table[b], n)
        if rows.min() < 0 or rows.max() >= k_bits.shape[0]:
            raise ValueError("page table points outside the key cache")
        k = bf16_bits_to_f64(k_bits[rows])                   # [n, D]
        q = bf16_bits_to_f64(q_bits[b])                      # [H, D]
        wb = np.asarray(w[b], np.float64)
        acc = np.zeros(n)
        for h in range(H):                                   # head by head, as the definition reads
            dots = k @ q[h]
            acc += wb[h] * np.maximum(dots, 0.0)
        out[b, :n] = acc
    return out


def topk_positions(scores: np.ndarray, ctx_len: np.ndarray, topk: int) -> np.ndarray:
    """[B, topk] int32: the min(topk, ctx_len[b]) positions with the largest
    scores[b, :ctx_len[b]] (ties to the lower position), ascending, -1 after.
    ``scores`` may be any real dtype; the comparison is in that dtype."""
    B = scores.shape[0]
    out = np.full((B, topk), -1, dtype=np.int32)
    for b in range(B):
        n = int(ctx_len[b])
        if n <= 0:
            continue
        sc = scores[b, :n]
        # descending score, then ascending position
        order = np.lexsort((np.arange(n), -sc.astype(np.float64)))
        pick = np.sort(order[:min(topk, n)])
        out[b, :pick.size] = pick
    return out
