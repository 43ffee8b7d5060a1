"""GPU parity of the stream-K plan (asked for with nsplit = -1; fp8 rows,
more than half as many decode rows as SMs, lists of 16 tiles or more): one
CTA per SM over the rows' tiles laid end to end, a row shared by two or
three CTAs merged inside the kernel by the CTA that finishes its part last.

Every row is checked against the fp64 oracle (the rows that one CTA holds
whole, and the shared ones), with padding that empties whole pieces of a
row, multi-token rows, the index-counting workload (bit-exact), and the
result is the same bit for bit whichever CTA merges (repeated calls, graph
replays) and needs no zeroed workspace."""
import numpy as np
import pytest
import torch

from sparse_mla_decode_05_b200 import inputs

from _helpers import Dev, assert_parity, counting_workload, oracle

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


def sms():
    return torch.cuda.get_device_properties(0).multi_processor_count


def owner_ranges(rows, nt, g):
    """For each row, the CTAs (first, last) that hold its tiles."""
    W = rows * nt
    own = lambda t: ((t + 1) * g - 1) // W
    return [(own(r * nt), own((r + 1) * nt - 1)) for r in range(rows)]


SK = -1    # nsplit asking for stream-K


def shape_of(w, d, nsplit=SK):
    return api().shape_for(d.q, d.kv, d.indices, page_table=d.page_table, page_size=w.page_size, nsplit=nsplit)


def test_plan_is_streamk_only_where_it_applies():
    g = sms()
    a = api()
    cases = [
        (g // 2 + 1, 1024, True),     # just over half the SMs
        (g - 20, 2048, True),         # c5-like
        (g + 1, 1024, True),          # one row more than the SMs
        (g, 1024, False),             # a multiple of the SMs: one wave already
        (g - 20, 960, False),         # 15 tiles: too short
        (g // 2, 1024, False),        # cluster split plan
    ]
    for rows, topk, want in cases:
        w = inputs.paged_fp8(rows, 2048, rows * 32, min(topk, 2048), seed=rows)
        d = Dev(w)
        s = shape_of(w, d)
        assert (a.plan_merge(s) == 3) == want, (rows, topk)
        if want:
            assert a.plan_nsplit(s) == 1 and a.workspace_size(s) >= 2 * g * 64 * 512 * 4
            # an explicit split count or the automatic plan never takes it
            assert a.plan_merge(shape_of(w, d, nsplit=1)) == 0
            assert a.plan_merge(shape_of(w, d, nsplit=0)) != 3
        else:
            # not applicable: the automatic plan
            assert a.plan_nsplit(s) == a.plan_nsplit(shape_of(w, d, nsplit=0))
    # bf16 rows keep the split plan
    wb = inputs.paged_bf16(g - 20, 1024, (g - 20) * 16, 1024, seed=3)
    db = Dev(wb)
    assert a.plan_merge(shape_of(wb, db)) != 3


def rows_for(kind, g):
    return {"half+1": g // 2 + 1, "half+27": g // 2 + 27, "sms-20": g - 20, "sms+2": g + 2}[kind]


@pytest.mark.parametrize("kind,topk", [("half+1", 1024), ("half+27", 1500), ("sms-20", 1088), ("sms+2", 1024)])
def test_streamk_every_row_matches_oracle(kind, topk):
    g = sms()
    rows = rows_for(kind, g)
    w = inputs.paged_fp8(rows, 2048, rows * 32, topk, seed=7 * rows + topk)
    d = Dev(w)
    assert api().plan_merge(shape_of(w, d)) == 3
    nt = (topk + 63) // 64
    spans = owner_ranges(rows, nt, g)
    shared = [r for r, (j0, j1) in enumerate(spans) if j1 > j0]
    whole = [r for r, (j0, j1) in enumerate(spans) if j1 == j0]
    assert shared and max(j1 - j0 for j0, j1 in spans) <= 2
    out, lse = d.run(nsplit=SK)
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle(w)
    assert_parity(out, lse, out_ref, lse_ref, seqs=shared, tag=f"streamk rows={rows} k={topk} shared")
    if whole:
        assert_parity(out, lse, out_ref, lse_ref, seqs=whole, tag=f"streamk rows={rows} k={topk} whole")


def test_streamk_padding_empties_pieces():
    """Rows whose list is all padding, whose second half is padding (the
    later pieces are empty: lse -inf, weight 0), or whose first half is."""
    g = sms()
    rows, topk = g - 20, 2048
    w = inputs.paged_fp8(rows, 2048, rows * 32, topk, seed=11)
    w.indices[3] = -1
    w.indices[10, 1024:] = -1
    w.indices[40, :1024] = -1
    w.indices[77, ::2] = -1
    w.indices[rows - 1, 64:] = -1
    d = Dev(w)
    assert api().plan_merge(shape_of(w, d)) == 3
    out, lse = d.run(nsplit=SK)
    torch.cuda.synchronize()
    assert torch.all(out[3].float() == 0) and torch.all(torch.isneginf(lse[3]))
    out_ref, lse_ref = oracle(w)
    keep = [r for r in range(rows) if r != 3]
    assert_parity(out, lse, out_ref, lse_ref, seqs=keep, tag="streamk padding")


def test_streamk_counting_exact():
    """q = 0: every valid entry weighs the same, so out * n is an exact count
    of the rows read per value dim; a row read twice, dropped or misplaced
    between the pieces of a shared row changes an integer."""
    g = sms()
    B = g - 20
    w, weights, nval = counting_workload(B, 1024, 1024, fp8=True, paged=True, pad_frac=0.3, seed=5)
    d = Dev(w)
    assert api().plan_merge(shape_of(w, d)) == 3
    out, lse = d.run(nsplit=SK)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy().astype(np.float64)       # [B, 64, 512]
    for b in range(B):
        got = np.rint(o[b] * nval[b] * 2) / 2                # weights are multiples of 0.5
        assert np.array_equal(got, np.broadcast_to(weights[b], got.shape)), f"row {b}"
        np.testing.assert_allclose(lse[b].cpu().numpy(), np.log(nval[b]), rtol=1e-6)


def test_streamk_multi_token_rows():
    """Two query tokens per sequence: rows = 2 B decode rows share out the
    tiles; a row's page-table row is its sequence's."""
    g = sms()
    B = g // 3 + 5                                   # 2 B > g / 2
    w = inputs.multi_token(B, 2, 2048, B * 32 + 64, 1024, seed=17, fp8=True, paged=True)
    d = Dev(w)
    s = api().shape_for(d.q, d.kv, d.indices, page_table=d.page_table, page_size=w.page_size, nsplit=SK)
    assert api().plan_merge(s) == 3
    out, lse = d.run(nsplit=SK)
    torch.cuda.synchronize()
    from test_gpu_multitoken import oracle_mt
    o_ref, l_ref = oracle_mt(w)
    assert_parity(out, lse, o_ref, l_ref, tag="streamk T=2")


def test_streamk_bits_do_not_depend_on_arrival():
    """Repeated calls, a call on a garbage-filled workspace and graph replays
    give the same bits (the merge sums the pieces in CTA order whichever CTA
    merges, and the row counters need no initialisation)."""
    g = sms()
    rows = g - 20
    w = inputs.paged_fp8(rows, 2048, rows * 32, 2048, seed=23)
    d = Dev(w)
    a = api()
    s = shape_of(w, d)
    assert a.plan_merge(s) == 3
    ref_out, ref_lse = d.run(nsplit=SK)
    for _ in range(3):
        o, l = d.run(nsplit=SK)
        torch.cuda.synchronize()
        assert torch.equal(o.view(torch.int16), ref_out.view(torch.int16))
        assert torch.equal(l.view(torch.int32), ref_lse.view(torch.int32))
    ws = torch.randint(0, 256, (a.workspace_size(s),), dtype=torch.uint8, device="cuda:0")
    out = torch.empty_like(ref_out)
    lse = torch.empty_like(ref_lse)
    pl = a.DecodePlan(d.q, d.kv, d.indices, w.scale, kv_row_scale=d.kv_row_scale, page_table=d.page_table,
                      page_size=w.page_size, nsplit=SK, out=out, lse=lse, workspace=ws)
    assert pl.streamk
    pl.run()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
    g_ = torch.cuda.CUDAGraph()
    st = torch.cuda.Stream()
    st.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(st):
        pl.run(st.cuda_stream)
    torch.cuda.current_stream().wait_stream(st)
    with torch.cuda.graph(g_):
        pl.run(torch.cuda.current_stream().cuda_stream)
    for _ in range(3):
        out.zero_()
        lse.zero_()
        g_.replay()
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), ref_lse.view(torch.int32))
    del g_


def test_streamk_workspace_too_small_is_rejected():
    g = sms()
    rows = g - 20
    w = inputs.paged_fp8(rows, 2048, rows * 32, 1024, seed=29)
    d = Dev(w)
    a = api()
    s = shape_of(w, d)
    need = a.workspace_size(s)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda:0")
    out = torch.empty((rows, 64, 512), dtype=torch.bfloat16, device="cuda:0")
    lse = torch.empty((rows, 64), dtype=torch.float32, device="cuda:0")
    st = a.lib.sparse_mla_decode(a.ctypes.byref(s), a._ptr(d.q), a._ptr(d.kv), a._ptr(d.kv_row_scale),
                                 a._ptr(d.page_table), a._ptr(d.indices), float(w.scale), a._ptr(out),
                                 a._ptr(lse), a._ptr(ws), ws.numel(), None)
    assert st == 3                                    # SMLA_ERR_WORKSPACE, nothing launched
