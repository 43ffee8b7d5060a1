"""Pins for the indexer oracle (oracle/indexer_ref.py), on the CPU.

Each pin checks the oracle against something other than itself: values
worked out by hand (tests/golden/indexer_handworked.json), torch float64
einsum over a flat copy of the cache, closed forms, and a brute-force
selection by Python's sorted().  Planted mistakes in copies of the oracle
(no ReLU, a swapped page mapping, the context cap ignored, ties to the
higher position) each fail at least one pin.
"""
import json
import os

import numpy as np
import pytest
import torch

from oracle import indexer_ref as ix

GOLD = os.path.join(os.path.dirname(__file__), "golden", "indexer_handworked.json")


def bf16(x) -> np.ndarray:
    """float array -> bf16 bit patterns (uint16), round to nearest even (torch)."""
    t = torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _case_inputs(c):
    q = bf16(np.asarray(c["q"])[None])                       # [1, H, D]
    k = np.asarray(c["keys"], np.float64)
    n_rows = max(64, len(k))
    kc = np.zeros((n_rows, k.shape[1]))
    kc[:len(k)] = k
    pt = np.zeros((1, 1), np.int32)                          # one page, page 0
    return q, np.asarray(c["w"], np.float32)[None], bf16(kc), pt, np.array([c["ctx"]], np.int32)


def _random_problem(seed, B=3, H=8, D=32, pps=4, pages=16, ctx=None):
    rng = np.random.default_rng(seed)
    q = bf16(rng.standard_normal((B, H, D)))
    w = (rng.standard_normal((B, H)) / np.sqrt(H)).astype(np.float32)
    k = bf16(rng.standard_normal((pages * 64, D)))
    pt = np.stack([rng.permutation(pages)[:pps] for _ in range(B)]).astype(np.int32)
    ctx = np.array(ctx if ctx is not None else rng.integers(1, pps * 64 + 1, size=B), np.int32)
    return q, w, k, pt, ctx


# ------------------------------------------------------------ hand-worked
def _golden_cases():
    return json.load(open(GOLD))["cases"]


@pytest.mark.parametrize("c", _golden_cases(), ids=lambda c: c["name"])
def test_handworked(c):
    q, w, k, pt, ctx = _case_inputs(c)
    width = len(c["keys"])
    s = ix.indexer_scores(q, w, k, pt, ctx, width)
    want = np.full(width, -np.inf)
    want[:c["ctx"]] = c["scores"]
    assert np.array_equal(s[0], want)
    assert ix.topk_positions(s, ctx, c["topk"])[0].tolist() == c["indices"]


# ------------------------------------------------------- library routine
def test_scores_equal_torch_einsum_on_a_flat_copy():
    q, w, k, pt, ctx = _random_problem(1)
    s = ix.indexer_scores(q, w, k, pt, ctx, 256)
    kt = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16).double()
    qt = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double()
    for b in range(q.shape[0]):
        n = int(ctx[b])
        # the sequence's keys rebuilt as a flat, contiguous block, page by page
        flat = torch.cat([kt[int(p) * 64:(int(p) + 1) * 64] for p in pt[b]])[:n]
        dots = torch.einsum("hd,sd->hs", qt[b], flat)
        want = torch.einsum("h,hs->s", torch.from_numpy(w[b]).double(), torch.relu(dots))
        np.testing.assert_allclose(s[b, :n], want.numpy(), rtol=1e-12, atol=1e-12)
        assert np.all(np.isneginf(s[b, n:]))


# ------------------------------------------------------------ closed forms
def test_zero_weight_removes_a_head_and_weights_scale_linearly():
    q, w, k, pt, ctx = _random_problem(2)
    s = ix.indexer_scores(q, w, k, pt, ctx, 256)
    w0 = w.copy()
    w0[:, 3] = 0.0
    q_drop = q.copy()
    q_drop[:, 3] = bf16(-np.abs(np.ones(q.shape[2])))[None]  # any values: its weight is zero
    assert np.array_equal(ix.indexer_scores(q_drop, w0, k, pt, ctx, 256), ix.indexer_scores(q, w0, k, pt, ctx, 256))
    s2 = ix.indexer_scores(q, (2.0 * w).astype(np.float32), k, pt, ctx, 256)
    finite = np.isfinite(s)
    assert np.array_equal(s2[finite], 2.0 * s[finite])


def test_negative_dots_contribute_nothing():
    # every key has positive entries; a head whose query is all negative has
    # only negative dots, so flipping its weight changes nothing
    rng = np.random.default_rng(3)
    q = bf16(np.abs(rng.standard_normal((1, 2, 16))))
    q[0, 1] = bf16(-np.abs(rng.standard_normal(16)))
    k = bf16(np.abs(rng.standard_normal((64, 16))) + 0.1)
    pt = np.zeros((1, 1), np.int32)
    ctx = np.array([64], np.int32)
    a = ix.indexer_scores(q, np.array([[1.0, 5.0]], np.float32), k, pt, ctx, 64)
    b = ix.indexer_scores(q, np.array([[1.0, -7.0]], np.float32), k, pt, ctx, 64)
    assert np.array_equal(a, b)


# ------------------------------------------------------------ selection
def test_selection_equals_brute_force_sorted():
    rng = np.random.default_rng(4)
    for trial in range(20):
        n = int(rng.integers(1, 200))
        topk = int(rng.integers(1, 80))
        sc = rng.integers(-5, 6, size=n).astype(np.float64)   # many ties
        got = ix.topk_positions(sc[None], np.array([n]), topk)[0]
        ranked = sorted(range(n), key=lambda i: (-sc[i], i))[:min(topk, n)]
        want = sorted(ranked) + [-1] * (topk - min(topk, n))
        assert got.tolist() == want, trial


def test_context_cap_and_empty_sequences():
    q, w, k, pt, _ = _random_problem(5, B=2)
    ctx = np.array([0, 10], np.int32)
    s = ix.indexer_scores(q, w, k, pt, ctx, 256)
    assert np.all(np.isneginf(s[0])) and np.all(np.isneginf(s[1, 10:]))
    sel = ix.topk_positions(s, ctx, 16)
    assert sel[0].tolist() == [-1] * 16
    assert sel[1].tolist() == list(range(10)) + [-1] * 6


def test_out_of_range_inputs_are_rejected():
    q, w, k, pt, _ = _random_problem(6, B=1)
    with pytest.raises(ValueError):
        ix.indexer_scores(q, w, k, pt, np.array([300], np.int32), 256)     # past the score row
    bad = pt.copy()
    bad[0, 0] = 10_000
    with pytest.raises(ValueError):
        ix.indexer_scores(q, w, k, bad, np.array([5], np.int32), 256)      # page outside the cache


# ------------------------------------------------------- planted mistakes
def _mutant(kind):
    def scores(q_bits, w, k_bits, page_table, ctx_len, max_ctx):
        B, H, D = q_bits.shape
        out = np.full((B, max_ctx), -np.inf)
        for b in range(B):
            n = int(ctx_len[b]) if kind != "no_cap" else max_ctx
            s = np.arange(n)
            if kind == "pages_swapped":
                rows = page_table[b][s % 64 % page_table.shape[1]] * 64 + s // 64
            else:
                rows = page_table[b][s // 64] * 64 + s % 64
            rows = np.clip(rows, 0, k_bits.shape[0] - 1)
            k = ix.bf16_bits_to_f64(k_bits[rows])
            q = ix.bf16_bits_to_f64(q_bits[b])
            dots = k @ q.T
            act = dots if kind == "no_relu" else np.maximum(dots, 0)
            out[b, :n] = act @ np.asarray(w[b], np.float64)
        return out

    def topk(sc, ctx_len, k):
        if kind != "ties_high":
            return ix.topk_positions(sc, ctx_len, k)
        out = np.full((sc.shape[0], k), -1, np.int32)
        for b in range(sc.shape[0]):
            n = int(ctx_len[b])
            order = sorted(range(n), key=lambda i: (-sc[b, i], -i))[:min(k, n)]
            out[b, :len(order)] = sorted(order)
        return out
    return scores, topk


def _pins_pass(scores, topk) -> bool:
    for c in _golden_cases():
        q, w, k, pt, ctx = _case_inputs(c)
        width = len(c["keys"])
        s = scores(q, w, k, pt, ctx, width)
        want = np.full(width, -np.inf)
        want[:c["ctx"]] = c["scores"]
        if not np.array_equal(s[0], want) or topk(s, ctx, c["topk"])[0].tolist() != c["indices"]:
            return False
    q, w, k, pt, ctx = _random_problem(1)
    s = scores(q, w, k, pt, ctx, 256)
    kt = torch.from_numpy(k.view(np.int16)).view(torch.bfloat16).double()
    qt = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double()
    for b in range(q.shape[0]):
        n = int(ctx[b])
        flat = torch.cat([kt[int(p) * 64:(int(p) + 1) * 64] for p in pt[b]])[:n]
        want = torch.einsum("h,hs->s", torch.from_numpy(w[b]).double(),
                            torch.relu(torch.einsum("hd,sd->hs", qt[b], flat)))
        if not np.allclose(s[b, :n], want.numpy(), rtol=1e-12, atol=1e-12):
            return False
    return True


def test_the_pins_accept_the_oracle():
    assert _pins_pass(ix.indexer_scores, ix.topk_positions)


@pytest.mark.parametrize("kind", ["no_relu", "pages_swapped", "no_cap", "ties_high"])
def test_planted_mistakes_are_caught(kind):
    assert not _pins_pass(*_mutant(kind))
