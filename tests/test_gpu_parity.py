"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle.

Tolerances: bf16 out max abs error <= 2e-2, lse relative error
(|d| / max(|lse|, 1)) <= 1e-3; index and padding handling bit-exact
(counting, single-index and NaN-poison tests).
"""
import numpy as np
import pytest
import torch

from oracle import sparse_mla_ref as ref
from sparse_mla_decode_05_b200 import inputs

from _helpers import Dev, assert_parity, compare, counting_workload, oracle

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


# ------------------------------------------------------------ full configs
@pytest.mark.parametrize("name", inputs.CONFIG_NAMES)
def test_full_config_parity(name):
    w = inputs.make_config(name)
    d = Dev(w)
    out, lse = d.run()
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle(w)
    err, lerr, ulps = assert_parity(out, lse, out_ref, lse_ref, tag=name)
    print(f"{name}: nsplit={api().plan_nsplit(api().shape_for(d.q, d.kv, d.indices, page_table=d.page_table, page_size=w.page_size))} "
          f"max|dout|={err:.3e} lse_rel={lerr:.3e} max_err_ulps={ulps:.2f}")


@pytest.mark.parametrize("name", ["c2", "c4b"])
def test_full_config_every_nsplit_agrees(name):
    """The same answer (within tolerance) for one split, the plan's split and
    the maximum split."""
    w = inputs.make_config(name)
    d = Dev(w)
    out_ref, lse_ref = oracle(w)
    tiles = (w.topk + 63) // 64
    for n in (1, 3, tiles):
        out, lse = d.run(nsplit=n)
        torch.cuda.synchronize()
        assert_parity(out, lse, out_ref, lse_ref, tag=f"{name} nsplit={n}")


# ------------------------------------------------------------ small shapes
@pytest.mark.parametrize("topk", [1, 2, 63, 64, 65, 127, 128, 129, 511])
@pytest.mark.parametrize("nsplit", [0, 1, 2, 1000])
def test_small_flat_bf16(topk, nsplit):
    w = inputs.flat_per_seq(3, max(700, topk), topk, seed=topk * 7 + nsplit, q_mult=2.0)
    d = Dev(w)
    out, lse = d.run(nsplit=nsplit)
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle(w)
    assert_parity(out, lse, out_ref, lse_ref, tag=f"k={topk} n={nsplit}")


@pytest.mark.parametrize("topk", [1, 64, 100, 333])
@pytest.mark.parametrize("nsplit", [0, 1, 3])
def test_small_paged_fp8(topk, nsplit):
    w = inputs.paged_fp8(4, 1024, 96, topk, seed=5 + topk + nsplit)
    d = Dev(w)
    out, lse = d.run(nsplit=nsplit)
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle(w)
    assert_parity(out, lse, out_ref, lse_ref, tag=f"fp8 k={topk} n={nsplit}")


def test_varlen_with_padding_small():
    w = inputs.flat_varlen(9, 10, 300, 256, seed=77)
    d = Dev(w)
    for n in (0, 1, 4):
        out, lse = d.run(nsplit=n)
        torch.cuda.synchronize()
        out_ref, lse_ref = oracle(w)
        assert_parity(out, lse, out_ref, lse_ref, tag=f"varlen n={n}")


def test_paged_bf16():
    """A bf16 pool addressed through a page table."""
    w = inputs.flat_per_seq(1, 64 * 40, 200, seed=3)   # pool of 40 pages
    rng = np.random.default_rng(3)
    B, pps = 3, 10
    pt = np.stack([rng.permutation(40)[:pps] for _ in range(B)]).astype(np.int32)
    idx = np.stack([rng.choice(pps * 64, 200, replace=False) for _ in range(B)]).astype(np.int32)
    idx[1, ::7] = -1
    q = inputs._normal_bf16(torch.Generator().manual_seed(9), (B, 64, 576))
    w2 = inputs.Workload(name="paged_bf16", q=q, kv=w.kv, indices=torch.from_numpy(idx),
                         page_table=torch.from_numpy(pt), page_size=64)
    d = Dev(w2)
    out, lse = d.run()
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle(w2)
    assert_parity(out, lse, out_ref, lse_ref, tag="paged bf16")


# ------------------------------------------------------ index exactness
@pytest.mark.parametrize("fp8,paged", [(False, False), (False, True), (True, True), (True, False)])
@pytest.mark.parametrize("topk,nsplit", [(1, 0), (64, 0), (200, 0), (200, 1), (777, 0), (2048, 5)])
def test_counting_exact(fp8, paged, topk, nsplit):
    w, weights, nval = counting_workload(3, topk, 4096, fp8=fp8, paged=paged, seed=topk + nsplit)
    d = Dev(w)
    out, lse = d.run(nsplit=nsplit)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy().astype(np.float64)       # [B, 64, 512]
    for b in range(3):
        if nval[b] == 0:
            assert np.all(o[b] == 0)
            continue
        got = np.rint(o[b] * nval[b] * 2) / 2                # weights are multiples of 0.5
        assert np.array_equal(got, np.broadcast_to(weights[b], got.shape)), f"seq {b}"
        np.testing.assert_allclose(lse[b].cpu().numpy(), np.log(nval[b]), rtol=1e-6)


def test_single_index_is_bit_exact_value_row():
    w = inputs.flat_per_seq(4, 1000, 1, seed=12, q_mult=3.0)
    d = Dev(w)
    out, lse = d.run()
    torch.cuda.synchronize()
    rows = w.indices[:, 0].long()
    want = w.kv[rows, :512].view(torch.int16)                  # [B, 512]
    got = out.cpu().view(torch.int16)                           # [B, 64, 512]
    assert torch.equal(got, want[:, None, :].expand_as(got))
    _, lse_ref = oracle(w)
    np.testing.assert_allclose(lse.cpu().numpy(), lse_ref, rtol=1e-5, atol=1e-5)


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("n", [2, 4, 8, 16])
def test_cluster_merge_every_size(n, fp8):
    """nsplit a power of two no larger than the cluster limit: the CTAs of a
    sequence merge their splits inside the split kernel.  Oracle parity,
    including a sequence whose later splits hold only padding (weight 0) and
    an all-padding sequence (out 0, lse -inf)."""
    if fp8:
        w = inputs.paged_fp8(3, 4096, 256, 2048, seed=60 + n)
    else:
        w = inputs.flat_per_seq(3, 8192, 2048, seed=40 + n)
    w.indices[1, 700:] = -1
    w.indices[2] = -1
    d = Dev(w)
    a = api()
    shape = a.shape_for(d.q, d.kv, d.indices, page_table=d.page_table, page_size=w.page_size, nsplit=n)
    assert a.plan_nsplit(shape) == n
    if n <= 8:                      # portable cluster sizes always launch
        assert a.plan_merge(shape) == 1
    out, lse = d.run(nsplit=n)
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle(w, seqs=[0, 1])
    assert_parity(out, lse, out_ref, lse_ref, seqs=[0, 1], tag=f"cluster n={n}")
    assert torch.all(out[2].float() == 0) and torch.all(torch.isneginf(lse[2]))


@pytest.mark.parametrize("fp8", [False, True])
@pytest.mark.parametrize("n", [2, 16])
@pytest.mark.parametrize("c", [1e3, 1e6, 1e-3])
def test_cluster_merge_large_and_small_values(c, n, fp8):
    """Value rows scaled by c with q scaled by 1/c, so the scores keep their
    size and out scales by c (|out| ~ 0.25 c with top-2048 lists: ~2.5e5 at
    c = 1e6, legal bf16 and far beyond the fp16 range).  The in-cluster
    merge exchanges each split's result as scaled fp16, so out must stay
    finite and within the usual bar scaled by c (the step is
    scale-equivariant up to rounding: 2e-2 c on out, 1e-3 on lse)."""
    if fp8:
        w = inputs.paged_fp8(2, 4096, 128, 2048, seed=90 + n)
        w = inputs.Workload(name="fp8_scaled", q=(w.q.float() / c).to(torch.bfloat16), kv=w.kv,
                            indices=w.indices, kv_row_scale=w.kv_row_scale * c, page_table=w.page_table,
                            page_size=w.page_size)
    else:
        w = inputs.flat_per_seq(2, 8192, 2048, seed=95 + n)
        w = inputs.Workload(name="bf16_scaled", q=(w.q.float() / c).to(torch.bfloat16),
                            kv=(w.kv.float() * c).to(torch.bfloat16), indices=w.indices)
    d = Dev(w)
    a = api()
    shape = a.shape_for(d.q, d.kv, d.indices, page_table=d.page_table, page_size=w.page_size, nsplit=n)
    if n <= 8:
        assert a.plan_merge(shape) == 1
    out, lse = d.run(nsplit=n)
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle(w)
    o = out.float().cpu().numpy().astype(np.float64)
    assert np.all(np.isfinite(o))
    assert np.abs(out_ref).max() > 0.1 * c                    # the values really are that large
    err = np.abs(o - out_ref).max()
    assert err <= 2e-2 * c, f"c={c} n={n}: out err {err:.3e} > {2e-2 * c:.3e}"
    assert ref.lse_rel_err(lse.cpu().numpy().astype(np.float64), lse_ref).max() <= 1e-3


def test_cluster_merge_counting_exact():
    """On-chip merge over 8 splits recovers the exact set of gathered rows."""
    w, weights, nval = counting_workload(3, 2048, 8192, fp8=False, paged=False, seed=77)
    d = Dev(w)
    out, lse = d.run(nsplit=8)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy().astype(np.float64)
    for b in range(3):
        got = np.rint(o[b] * nval[b] * 2) / 2
        assert np.array_equal(got, np.broadcast_to(weights[b], got.shape)), f"seq {b}"
        np.testing.assert_allclose(lse[b].cpu().numpy(), np.log(nval[b]), rtol=1e-6)


def test_fp8_every_code_decodes_exactly():
    """One index per sequence gives out = the gathered value row, so every
    non-NaN e4m3fn code, times a power-of-two row scale, must come back as
    its exact bf16 value (subnormal codes included).  Values are compared,
    so -0 equals +0: the weighted sum over a tile adds +0 from the padding
    rows, which turns the code -0 into +0."""
    codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    N = 16
    kv = np.stack([codes[(np.arange(576) + 37 * r) % codes.size] for r in range(N)])
    scales = np.array([2.0 ** ((r % 7) - 3) for r in range(N)], dtype=np.float32)
    idx = np.array([[2], [7], [11], [13]], dtype=np.int32)
    q = inputs._normal_bf16(torch.Generator().manual_seed(21), (4, 64, 576))
    w = inputs.Workload(name="fp8_codes", q=q, kv=torch.from_numpy(kv), indices=torch.from_numpy(idx),
                        kv_row_scale=torch.from_numpy(scales))
    d = Dev(w)
    out, lse = d.run()
    torch.cuda.synchronize()
    for b in range(4):
        r = int(idx[b, 0])
        vals = ref.e4m3fn_to_f64(kv[r, :512]) * float(scales[r])    # exact in bf16
        got = out[b].float().cpu().numpy().astype(np.float64)
        assert np.array_equal(got, np.broadcast_to(vals, got.shape)), f"row {r}"
    # lse = the one score, an fp32 sum of 576 products of magnitude up to
    # 448 |q| (rounding ~1e-3 absolute): the parity gate
    _, lse_ref = oracle(w)
    assert np.max(ref.lse_rel_err(lse.cpu().numpy(), lse_ref)) <= 1e-3


def test_all_padding_sequence_and_mixed():
    w = inputs.flat_per_seq(3, 800, 130, seed=4)
    w.indices[1] = -1
    w.indices[2, 64:] = -1            # second tile fully padded
    d = Dev(w)
    for n in (0, 1, 2, 3):
        out, lse = d.run(nsplit=n)
        torch.cuda.synchronize()
        assert torch.all(out[1].float() == 0) and torch.all(torch.isneginf(lse[1]))
        out_ref, lse_ref = oracle(w)
        assert_parity(out, lse, out_ref, lse_ref, seqs=[0, 2], tag=f"pad n={n}")


@pytest.mark.parametrize("fp8", [False, True])
def test_nan_poisoned_unreferenced_rows_and_guards(fp8):
    """Every row no index names, and guard rows before and after the pool, are
    NaN: a stray read (or a padding entry clamped to a real row) turns the
    output into NaN through 0 * NaN.  The result must equal the clean run."""
    if fp8:
        w = inputs.paged_fp8(3, 512, 30, 300, seed=8)
    else:
        w = inputs.flat_varlen(5, 100, 700, 256, seed=8)
    d = Dev(w)
    clean_out, clean_lse = d.run()
    G = 64
    nan_code = 0x7F if fp8 else 0x7FC0
    dtype = torch.uint8 if fp8 else torch.int16
    big = torch.full((w.kv.shape[0] + 2 * G, 576), nan_code, dtype=dtype)
    ref_rows = torch.zeros(w.kv.shape[0], dtype=torch.bool)
    if w.page_table is not None:
        pt = w.page_table.long()
        for b in range(w.batch):
            logical = w.indices[b][w.indices[b] >= 0].long()
            ref_rows[pt[b, logical // 64] * 64 + logical % 64] = True
    else:
        ref_rows[w.indices[w.indices >= 0].long()] = True
    body = big[G:G + w.kv.shape[0]]
    src = w.kv if fp8 else w.kv.view(torch.int16)
    body[ref_rows] = src[ref_rows]
    big_dev = big.to("cuda:0")
    kv_view = big_dev[G:G + w.kv.shape[0]]
    if not fp8:
        kv_view = kv_view.view(torch.bfloat16)
    d2 = Dev(w, kv_override=kv_view)
    for n in (0, 1, 3):
        out, lse = d2.run(nsplit=n)
        ref_out, ref_lse = d.run(nsplit=n)
        torch.cuda.synchronize()
        assert torch.isfinite(out.float()).all()
        assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))
        assert torch.equal(lse, ref_lse)
    assert torch.equal(clean_out.view(torch.int16), d.run()[0].view(torch.int16))


# ------------------------------------------------------------ combine
def test_combine_kernel_on_oracle_partials():
    w = inputs.flat_per_seq(3, 3000, 700, seed=21, q_mult=4.0)
    cuts = [0, 100, 101, 450, 700]
    parts = []
    for a, b in zip(cuts[:-1], cuts[1:]):
        sub = inputs.Workload(name="part", q=w.q, kv=w.kv, indices=w.indices[:, a:b].contiguous())
        parts.append(oracle(sub))
    empty = inputs.Workload(name="empty", q=w.q, kv=w.kv, indices=torch.full((3, 5), -1, dtype=torch.int32))
    parts.append(oracle(empty))
    po = torch.from_numpy(np.stack([p[0] for p in parts], axis=1).astype(np.float32)).cuda()
    pl = torch.from_numpy(np.stack([p[1] for p in parts], axis=1).astype(np.float32)).cuda()
    out, lse = api().combine(po.contiguous(), pl.contiguous())
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle(w)
    err, lerr, _ = assert_parity(out, lse, out_ref, lse_ref, tag="combine")
    assert lerr < 1e-6
    # all splits empty -> out 0, lse -inf
    out2, lse2 = api().combine(po[:, -1:].contiguous(), pl[:, -1:].contiguous())
    torch.cuda.synchronize()
    assert torch.all(out2.float() == 0) and torch.all(torch.isneginf(lse2))


def test_split_partials_match_oracle_per_split():
    """sparse_mla_decode_split alone: each split's partial (normalised output
    and lse) equals the oracle on that split's slice of the index list."""
    w = inputs.flat_per_seq(2, 4000, 300, seed=33)
    d = Dev(w)
    n, _, _, ws = api().decode_split(d.q, d.kv, d.indices, w.scale, nsplit=3)
    torch.cuda.synchronize()
    assert n == 3
    po, pl = api().partial_views(ws, 2, 3)
    tiles = (300 + 63) // 64
    for s in range(3):
        t0, t1 = s * tiles // 3, (s + 1) * tiles // 3
        sub = inputs.Workload(name="s", q=w.q, kv=w.kv,
                              indices=w.indices[:, t0 * 64:min(300, t1 * 64)].contiguous())
        o_ref, l_ref = oracle(sub)
        o = po[:, s].cpu().numpy().astype(np.float64)
        assert np.max(np.abs(o - o_ref)) < 5e-3
        assert np.max(ref.lse_rel_err(pl[:, s].cpu().numpy(), l_ref)) < 1e-4


# ------------------------------------------------ determinism and graphs
def test_deterministic_bits():
    w = inputs.make_config("c1")
    d = Dev(w)
    a = d.run()
    b = d.run()
    torch.cuda.synchronize()
    assert torch.equal(a[0].view(torch.int16), b[0].view(torch.int16)) and torch.equal(a[1], b[1])


@pytest.mark.parametrize("name", ["c1", "c3", "c4a"])     # c4a: the in-cluster merge
def test_cuda_graph_replay_bit_identical(name):
    w = inputs.make_config(name)
    d = Dev(w)
    a = api()
    shape = a.shape_for(d.q, d.kv, d.indices)
    ws_bytes = a.workspace_size(shape)
    ws = torch.empty(max(ws_bytes, 256), dtype=torch.uint8, device="cuda:0")
    out = torch.empty((w.batch, 64, 512), dtype=torch.bfloat16, device="cuda:0")
    lse = torch.empty((w.batch, 64), dtype=torch.float32, device="cuda:0")
    eager_out, eager_lse = d.run()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        d.run(out=out, lse=lse, workspace=ws)
    torch.cuda.current_stream().wait_stream(s)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        d.run(out=out, lse=lse, workspace=ws)
    out.zero_()
    lse.zero_()
    g.replay()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), eager_out.view(torch.int16))
    assert torch.equal(lse, eager_lse)
    del g


def test_cuda_graph_back_to_back_calls():
    """Several decode calls in one CUDA graph (each launch may start before
    the previous one ends: programmatic dependent launch), on different
    inputs and plans: partials + combine, in-cluster merge, one split, fp8.
    Replays equal the eager results bit for bit."""
    a = api()
    ws = [inputs.flat_per_seq(2, 2048, 700, seed=91),          # explicit 3 splits: combine kernel
          inputs.flat_per_seq(2, 2048, 700, seed=92),          # 4 splits: in-cluster merge
          inputs.paged_fp8(3, 1024, 64, 300, seed=93),         # fp8, planned
          inputs.flat_per_seq(4, 1000, 64, seed=94)]           # one tile: one split
    nsplits = [3, 4, 0, 0]
    plans, eager = [], []
    for w, n in zip(ws, nsplits):
        d = Dev(w)
        pl = a.DecodePlan(d.q, d.kv, d.indices, w.scale, kv_row_scale=d.kv_row_scale, page_table=d.page_table,
                          page_size=w.page_size, nsplit=n)
        pl.run()
        torch.cuda.synchronize()
        eager.append((pl.out.clone(), pl.lse.clone()))
        plans.append((d, pl))
    assert plans[0][1].nsplit == 3 and not plans[0][1].clustered     # combine kernel path
    assert plans[1][1].nsplit == 4 and plans[1][1].clustered         # in-cluster merge
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for _, pl in plans:
            pl.run(torch.cuda.current_stream().cuda_stream)
    for _, pl in plans:
        pl.out.zero_()
        pl.lse.zero_()
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    for (_, pl), (o, l) in zip(plans, eager):
        assert torch.equal(pl.out.view(torch.int16), o.view(torch.int16))
        assert torch.equal(pl.lse.view(torch.int32), l.view(torch.int32))
    del g


def test_workspace_checks():
    w = inputs.flat_per_seq(2, 1000, 300, seed=1)
    d = Dev(w)
    a = api()
    shape = a.shape_for(d.q, d.kv, d.indices, nsplit=3)
    need = a.workspace_size(shape)
    assert need > 0 and need % 256 == 0 and a.plan_nsplit(shape) == 3
    small = torch.empty(need - 256, dtype=torch.uint8, device="cuda:0")
    with pytest.raises(a.SmlaError) as e:
        d.run(nsplit=3, workspace=small)
    assert e.value.code == 3
    big = torch.empty(need + 512, dtype=torch.uint8, device="cuda:0")
    with pytest.raises(a.SmlaError) as e:
        d.run(nsplit=3, workspace=big[16:])          # not 256-byte aligned
    assert e.value.code == 3
    one = a.shape_for(d.q, d.kv, d.indices, nsplit=1)
    assert a.workspace_size(one) == 0
    d.run(nsplit=1, workspace=None)                  # no workspace needed


# ------------------------------------------------ entries naming no row
@pytest.mark.parametrize("kind", ["flat_bf16", "paged_fp8", "dsv4"])
def test_out_of_range_entries_read_as_padding(kind):
    """An index past the pool (flat), past the page table's width (paged),
    or resolving through a page-table entry outside the pool, is read as
    padding and sets bit 2 of the device error word: the result equals the
    oracle's with those entries replaced by -1."""
    if kind == "flat_bf16":
        w = inputs.flat_per_seq(3, 700, 300, seed=91)
        n_rows = w.kv.shape[0]
        bad = [n_rows, n_rows + 12345, 2 ** 31 - 1]
    elif kind == "paged_fp8":
        w = inputs.paged_fp8(3, 1024, 96, 300, seed=92)
        bad = [1024, 1024 + 63, 2 ** 31 - 1]
    else:
        w = inputs.paged_dsv4(3, 1024, 96, 300, seed=93)
        bad = [1024, 5000, 2 ** 31 - 1]
    idx = w.indices.clone()
    idx[0, 5] = bad[0]
    idx[1, 100] = bad[1]
    idx[2, 299] = bad[2]
    clean = idx.clone()
    clean[0, 5] = clean[1, 100] = clean[2, 299] = -1
    if w.page_table is not None:
        # a page-table entry that points past the pool
        pt = w.page_table.clone()
        pt[1, 0] = 96 + 5
        pt[2, 1] = -3
        hit = (idx >= 0) & (idx < 1024) & (((idx // 64 == 0) & (torch.arange(3)[:, None] == 1)) |
                                            ((idx // 64 == 1) & (torch.arange(3)[:, None] == 2)))
        clean[hit] = -1
        w = inputs.Workload(name=w.name, q=w.q, kv=w.kv, indices=idx, scale=w.scale,
                            kv_row_scale=w.kv_row_scale, page_table=pt, page_size=w.page_size,
                            layout=w.layout)
    else:
        w = inputs.Workload(name=w.name, q=w.q, kv=w.kv, indices=idx, scale=w.scale)
    w_clean = inputs.Workload(name=w.name, q=w.q, kv=w.kv, indices=clean, scale=w.scale,
                              kv_row_scale=w.kv_row_scale, page_table=w.page_table,
                              page_size=w.page_size, layout=w.layout)
    d = Dev(w)
    for n in (0, 1):
        out, lse = d.run(nsplit=n)
        torch.cuda.synchronize()
        assert api().device_error() == 4
        out_ref, lse_ref = oracle(w_clean)
        assert_parity(out, lse, out_ref, lse_ref, tag=f"{kind} out-of-range n={n}")
