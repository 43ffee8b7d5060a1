"""GPU parity for the indexer step (sparse_mla_indexer*): scores against the
fp64 oracle, the top-k selection exactly.

Scores: |GPU - oracle| <= 2^-15 * sum_h |w_h| sum_d |q_hd k_d| per position
(each head's 128-term dot product accumulates in fp32, <= 128 * 2^-23 of
its absolute sum, then 64 weighted fp32 additions).  Selection: a decision
taken on floating-point scores, so both sides take it in the kernel's
precision: the oracle's selection rule applied to the kernel's own scores
must give exactly the kernel's index lists.  It must also be a valid top-k
of the fp64 scores up to the score tolerance.
"""
import numpy as np
import pytest
import torch

from oracle import indexer_ref as ix
from oracle import sparse_mla_ref as ref
from sparse_mla_decode_05_b200 import inputs

from _helpers import assert_parity

pytestmark = pytest.mark.gpu


def api():
    from sparse_mla_decode_05_b200 import api as a
    return a


@pytest.fixture(autouse=True)
def _no_device_errors():
    yield
    if torch.cuda.is_available():
        torch.cuda.synchronize()
        assert api().device_error() == 0


def _bits(t):
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def _plan(w, max_ctx=None):
    d = "cuda"
    return api().IndexerPlan(w.q.to(d), w.w.to(d), w.k.to(d), w.page_table.to(d), w.ctx_len.to(d), w.topk,
                             max_ctx=max_ctx if max_ctx is not None else w.max_ctx)


def _oracle(w):
    return ix.indexer_scores(_bits(w.q), w.w.numpy(), _bits(w.k), w.page_table.numpy(), w.ctx_len.numpy(),
                             w.max_ctx)


def _tolerance(w):
    """2^-15 * sum_h |w_h| sum_d |q_hd k_sd| for every (b, s < ctx)."""
    q = np.abs(ix.bf16_bits_to_f64(_bits(w.q)))
    k = np.abs(ix.bf16_bits_to_f64(_bits(w.k)))
    tol = np.zeros((w.batch, w.max_ctx))
    for b in range(w.batch):
        n = int(w.ctx_len[b])
        if n == 0:
            continue
        rows = ix.key_rows(w.page_table[b].numpy(), n)
        tol[b, :n] = (k[rows] @ q[b].T) @ np.abs(w.w[b].numpy().astype(np.float64))
    return 2.0 ** -15 * tol


def _check(w, plan):
    torch.cuda.synchronize()
    got = plan.scores.cpu().numpy()
    sel = plan.indices.cpu().numpy()
    want = _oracle(w)
    tol = _tolerance(w)
    ctx = w.ctx_len.numpy()
    for b in range(w.batch):
        n = int(ctx[b])
        assert np.all(np.abs(got[b, :n] - want[b, :n]) <= tol[b, :n]), f"seq {b}: scores"
        assert np.all(np.isneginf(got[b, n:])), f"seq {b}: past the context"
    # the selection, in the kernel's precision
    assert np.array_equal(sel, ix.topk_positions(got, ctx, w.topk))
    # a valid top-k of the fp64 scores, up to the score tolerance
    for b in range(w.batch):
        n = int(ctx[b])
        if n <= w.topk:
            continue
        chosen = sel[b][sel[b] >= 0]
        rest = np.setdiff1d(np.arange(n), chosen)
        assert want[b, chosen].min() >= want[b, rest].max() - 2 * tol[b, :n].max(), f"seq {b}: selection"
    return got, sel


@pytest.mark.parametrize("B,max_ctx,topk,ctx_lo,pages", [
    (3, 1000, 64, 1, 64),        # ragged tails: contexts not multiples of 64 or 128
    (2, 256, 512, None, 16),     # top-k wider than the context: all positions, then -1
    (4, 700, 100, 100, 48),
    (1, 128, 1, None, 4),        # one tile, top-1
    (2, 8192, 512, 4000, 300),   # long contexts, several thousand candidates
    (5, 2048, 2048, 1500, 200),  # top-k equal to the score row
    (2, 12000, 512, 9000, 400),  # contexts past 8192: the top-k path that re-reads the scores
])
def test_indexer_parity(B, max_ctx, topk, ctx_lo, pages):
    w = inputs.indexer_workload(B, max_ctx, pages, seed=B * 1000 + topk, topk=topk, ctx_lo=ctx_lo)
    plan = _plan(w)
    plan.run()
    _check(w, plan)


def test_indexer_bs32_workload():
    """Batch 32, 8192-token contexts, top-512: the bench's indexer line."""
    w = inputs.make_indexer_config()
    plan = _plan(w)
    plan.run()
    _check(w, plan)


def test_context_edges():
    lens = [0, 1, 63, 64, 65, 127, 128, 129, 255, 256, 257, 1024]
    w = inputs.indexer_workload(len(lens), 1024, 16 * len(lens) + 4, seed=77, topk=256)
    w.ctx_len = torch.tensor(lens, dtype=torch.int32)
    plan = _plan(w)
    plan.run()
    _, sel = _check(w, plan)
    assert sel[0].tolist() == [-1] * 256
    assert sel[1].tolist() == [0] + [-1] * 255


def test_ties_go_to_the_lower_position():
    """Sequence 0's keys take only five distinct values, so thousands of
    positions tie and the boundary falls inside a tie; sequence 1 has q = 0,
    so every score is 0 and the first topk positions are taken."""
    w = inputs.indexer_workload(2, 4096, 140, seed=91, topk=500)
    rng = np.random.default_rng(91)
    rows0 = ix.key_rows(w.page_table[0].numpy(), 4096)
    pick = rng.integers(0, 5, size=4096)
    k = w.k.clone()
    k[torch.from_numpy(rows0)] = k[torch.from_numpy(rows0[:5][pick])]
    w.k = k
    q = w.q.clone()
    q[1] = 0
    w.q = q
    plan = _plan(w)
    plan.run()
    got, sel = _check(w, plan)
    assert sel[1].tolist() == list(range(500))
    assert len(np.unique(got[0, :4096])) <= 5


def test_ties_past_8192_positions():
    """The long-context top-k path with the boundary inside a tie."""
    w = inputs.indexer_workload(1, 10000, 160, seed=93, topk=700)
    rows0 = ix.key_rows(w.page_table[0].numpy(), 10000)
    pick = np.random.default_rng(93).integers(0, 7, size=10000)
    k = w.k.clone()
    k[torch.from_numpy(rows0)] = k[torch.from_numpy(rows0[:7][pick])]
    w.k = k
    plan = _plan(w)
    plan.run()
    got, _ = _check(w, plan)
    assert len(np.unique(got[0, :10000])) <= 7


def test_context_longer_than_the_row_is_clamped():
    w = inputs.indexer_workload(2, 512, 20, seed=5, topk=64)
    w_long = inputs.IndexerWorkload(name=w.name, q=w.q, w=w.w, k=w.k, page_table=w.page_table,
                                    ctx_len=torch.tensor([512, 9999], dtype=torch.int32), max_ctx=512, topk=64)
    plan = _plan(w_long)
    plan.run()
    torch.cuda.synchronize()
    assert api().device_error() == 4
    w_long.ctx_len = torch.tensor([512, 512], dtype=torch.int32)
    _check(w_long, plan)


def test_graph_replay_is_identical():
    w = inputs.indexer_workload(4, 2048, 140, seed=13, topk=512, ctx_lo=600)
    plan = _plan(w)
    plan.run()
    torch.cuda.synchronize()
    s0, i0 = plan.scores.clone(), plan.indices.clone()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        plan.run(torch.cuda.current_stream().cuda_stream)
    plan.scores.zero_()
    plan.indices.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(plan.scores, s0) and torch.equal(plan.indices, i0)


@pytest.mark.parametrize("kv_kind", ["bf16", "dsv4"])
def test_indexer_feeds_the_decode(kv_kind):
    """The indexer's index lists drive the decode through one page table:
    the decode's result equals the oracle's on those same lists."""
    B, max_ctx, pages = 4, 2048, 140
    wi = inputs.indexer_workload(B, max_ctx, pages, seed=21, topk=256, ctx_lo=200)
    plan = _plan(wi)
    plan.run()
    torch.cuda.synchronize()
    idx = plan.indices.cpu()
    if kv_kind == "dsv4":
        wd = inputs.paged_dsv4(B, max_ctx, pages, 256, seed=22)
    else:
        wd = inputs.paged_bf16(B, max_ctx, pages, 256, seed=22)
    wd = inputs.Workload(name="indexed", q=wd.q, kv=wd.kv, indices=idx, scale=wd.scale,
                         page_table=wi.page_table, page_size=64, layout=wd.layout)
    d = "cuda"
    out, lse = api().decode(wd.q.to(d), wd.kv.to(d), idx.to(d), wd.scale, page_table=wi.page_table.to(d),
                            page_size=64)
    torch.cuda.synchronize()
    want_o, want_l = ref.sparse_mla_decode(wd.np_q_bits(), wd.np_kv(), idx.numpy(), wd.scale,
                                           kv_format=wd.kv_format, page_table=wi.page_table.numpy(),
                                           page_size=64)
    assert_parity(out, lse, want_o, want_l, tag=f"indexer -> decode ({kv_kind})")
