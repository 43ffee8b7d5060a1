"""GPU parity for the DeepSeek-V4 paged cache layout (kv_dtype
SMLA_KV_DSV4_PAGED): 64-token pages of 37,376 bytes, each slot 448 e4m3fn
codes with one UE8M0 scale per 64 dims plus 64 bf16 rope dims; the whole
512-dim row is both key and value.

Same bar as the other layouts: out max abs error <= 2e-2 and lse relative
error <= 1e-3 against the fp64 oracle; index, page and scale handling exact
(counting and single-index tests, whose expected values come from brute
force and from the UE8M0 / e4m3 definitions, not from the oracle).
"""
import numpy as np
import pytest
import torch

from oracle import sparse_mla_ref as ref
from sparse_mla_decode_05_b200 import inputs

from _helpers import Dev, assert_parity, oracle

pytestmark = pytest.mark.gpu

PAGE = 37376
SLOT = 576
SCALE_OFF = 64 * SLOT


def api():
    from sparse_mla_decode_05_b200 import api as a
    return a


@pytest.fixture(autouse=True)
def _no_device_errors():
    yield
    if torch.cuda.is_available():
        torch.cuda.synchronize()
        assert api().device_error() == 0


@pytest.mark.parametrize("topk", [1, 64, 100, 333])
@pytest.mark.parametrize("nsplit", [0, 1, 3])
def test_small_dsv4(topk, nsplit):
    w = inputs.paged_dsv4(4, 1024, 96, topk, seed=31 + topk + nsplit)
    d = Dev(w)
    out, lse = d.run(nsplit=nsplit)
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle(w)
    assert_parity(out, lse, out_ref, lse_ref, tag=f"dsv4 k={topk} n={nsplit}")


@pytest.mark.parametrize("nsplit", [2, 4, 8, 16])
def test_dsv4_in_cluster_merge(nsplit):
    """Power-of-two split counts merge inside the split kernel."""
    w = inputs.paged_dsv4(2, 2048, 64, 1100, seed=40 + nsplit)
    d = Dev(w)
    shape = api().shape_for(d.q, d.kv, d.indices, page_table=d.page_table, page_size=64, nsplit=nsplit)
    assert api().plan_nsplit(shape) == nsplit
    out, lse = d.run(nsplit=nsplit)
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle(w)
    assert_parity(out, lse, out_ref, lse_ref, tag=f"dsv4 cluster n={nsplit}")


def test_dsv4_bs32_workload():
    """The batch-32, top-512, 8192-token DeepSeek-V4 workload (the bench's
    dsv4 line), in the launch configuration the planner picks."""
    w = inputs.make_config("dsv4")
    d = Dev(w)
    out, lse = d.run()
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle(w)
    err, lerr, _ = assert_parity(out, lse, out_ref, lse_ref, tag="dsv4 bs32")
    print(f"dsv4 bs32: max|dout|={err:.3e} lse_rel={lerr:.3e}")


def _write_row(pages, r, dims_codes, rope_vals, scale_bytes):
    pg, sl = r // 64, r % 64
    base = sl * SLOT
    pages[pg, base:base + 448] = dims_codes
    rv = torch.from_numpy(np.asarray(rope_vals, dtype=np.float32)).to(torch.bfloat16).view(torch.uint8).numpy()
    pages[pg, base + 448:base + 576] = rv
    pages[pg, SCALE_OFF + 8 * sl:SCALE_OFF + 8 * sl + 7] = scale_bytes


@pytest.mark.parametrize("topk,nsplit", [(1, 0), (64, 0), (200, 0), (200, 1), (777, 0), (2048, 5), (2048, 4)])
def test_dsv4_counting_exact(topk, nsplit):
    """q = 0, so every valid entry weighs the same; row r carries a single
    1.0 at dim r % 512.  Below dim 448 that 1.0 is an e4m3 code 2^(127-e)
    times its group's UE8M0 scale 2^(e-127), with e drawn per row and group
    from {126, 127, 128}; at 448 and above it is a bf16 rope value.  Then
    out[b, h, d] * n_b is the number of valid entries whose row is d mod 512
    (brute-force bincount); a misread page, slot, group scale or rope chunk
    changes an integer."""
    rng = np.random.default_rng(topk + 7 * nsplit)
    B, rows_per_seq = 3, 4096
    pps = rows_per_seq // 64
    P = B * pps
    N = P * 64
    pages = np.zeros((P, PAGE), dtype=np.uint8)
    code_of = {126: 0x40, 127: 0x38, 128: 0x30}     # e4m3fn 2.0, 1.0, 0.5
    for r in range(N):
        d = r % 512
        e = rng.choice([126, 127, 128], size=7)
        codes = np.zeros(448, dtype=np.uint8)
        rope = np.zeros(64)
        if d < 448:
            codes[d] = code_of[int(e[d // 64])]
        else:
            rope[d - 448] = 1.0
        _write_row(pages, r, codes, rope, e.astype(np.uint8))
    perm = rng.permutation(P).reshape(B, pps)
    idx = np.full((B, topk), -1, dtype=np.int64)
    phys = np.full((B, topk), -1, dtype=np.int64)
    for b in range(B):
        n_valid = min(rows_per_seq, topk - int(round(0.25 * topk)))
        pos = np.sort(rng.choice(topk, n_valid, replace=False))
        logical = rng.choice(rows_per_seq, n_valid, replace=False)
        idx[b, pos] = logical
        phys[b, pos] = perm[b, logical // 64] * 64 + logical % 64
    w = inputs.Workload(name="dsv4_counting", q=torch.zeros((B, 64, 512), dtype=torch.bfloat16),
                        kv=torch.from_numpy(pages), indices=torch.from_numpy(idx.astype(np.int32)),
                        scale=0.0625, page_table=torch.from_numpy(perm.astype(np.int32)), page_size=64,
                        layout="dsv4")
    d = Dev(w)
    out, lse = d.run(nsplit=nsplit)
    torch.cuda.synchronize()
    o = out.float().cpu().numpy().astype(np.float64)
    for b in range(B):
        r = phys[b][phys[b] >= 0]
        counts = np.bincount(r % 512, minlength=512).astype(np.float64)
        n = r.size
        got = np.rint(o[b] * n)
        assert np.array_equal(got, np.broadcast_to(counts, got.shape)), f"seq {b}"
        np.testing.assert_allclose(lse[b].cpu().numpy(), np.log(n), rtol=1e-6)


def test_dsv4_single_index_is_the_decoded_row():
    """topk = 1: every head's output is the decoded row.  Codes sweep every
    non-NaN e4m3fn code and scales e in [60, 194], so every product
    code * 2^(e-127) is a bf16 normal number (or zero) and the decode is
    exact: the output equals the row by value (signed zeros may differ)."""
    rng = np.random.default_rng(5)
    B, P = 4, 8
    pages = np.zeros((P, PAGE), dtype=np.uint8)
    all_codes = np.array([c for c in range(256) if c not in (0x7F, 0xFF)], dtype=np.uint8)
    for r in range(P * 64):
        codes = rng.choice(all_codes, size=448)
        rope = rng.standard_normal(64) * 4.0
        e = rng.integers(60, 195, size=7).astype(np.uint8)
        _write_row(pages, r, codes, rope, e)
    pt = np.stack([rng.permutation(P)[:2] for _ in range(B)]).astype(np.int32)
    idx = rng.integers(0, 128, size=(B, 1)).astype(np.int32)
    q = inputs._normal_bf16(torch.Generator().manual_seed(6), (B, 64, 512), mult=2.0)
    w = inputs.Workload(name="dsv4_single", q=q, kv=torch.from_numpy(pages), indices=torch.from_numpy(idx),
                        scale=1.0 / np.sqrt(512), page_table=torch.from_numpy(pt), page_size=64, layout="dsv4")
    d = Dev(w)
    out, lse = d.run()
    torch.cuda.synchronize()
    rows = pt[np.arange(B), idx[:, 0] // 64] * 64 + idx[:, 0] % 64
    want = ref.dsv4_rows_f64(pages, rows)                      # [B, 512] fp64, exact
    got = out.float().cpu().numpy().astype(np.float64)          # [B, 64, 512]
    assert np.array_equal(got, np.broadcast_to(want[:, None, :], got.shape))
    # scores reach ~1e20 here (scales up to 2^67): lse is held to the parity
    # bar, relative error <= 1e-3 (fp32 accumulation of the dot products)
    _, lse_ref = oracle(w)
    assert ref.lse_rel_err(lse.cpu().numpy().astype(np.float64), lse_ref).max() <= 1e-3


@pytest.mark.parametrize("nsplit", [0, 1, 4])
def test_dsv4_rope_alone_decides(nsplit):
    """Every nope code is zero, so the scores come from the 64 bf16 rope dims
    alone and the output is zero except in dims 448..511, where it is a
    softmax-weighted mean of rope values.  A rope chunk that is not copied,
    or copied to the wrong place, changes both (checked against the oracle
    at the usual bar), and the nope part of the output must be exactly 0."""
    w = inputs.paged_dsv4(3, 2048, 96, 700, seed=77 + nsplit)
    pages = w.kv.numpy().copy()
    for sl in range(64):
        pages[:, sl * SLOT:sl * SLOT + 448] = 0
    w = inputs.Workload(name="dsv4_rope_only", q=w.q, kv=torch.from_numpy(pages), indices=w.indices,
                        scale=w.scale, page_table=w.page_table, page_size=64, layout="dsv4")
    d = Dev(w)
    out, lse = d.run(nsplit=nsplit)
    torch.cuda.synchronize()
    out_ref, lse_ref = oracle(w)
    assert np.abs(out_ref[..., 448:]).max() > 0.1          # the rope part carries the result
    assert_parity(out, lse, out_ref, lse_ref, tag=f"dsv4 rope only n={nsplit}")
    assert np.array_equal(out[..., :448].float().cpu().numpy(), np.zeros((3, 64, 448), dtype=np.float32))


def test_dsv4_input_checks():
    w = inputs.paged_dsv4(2, 256, 16, 50, seed=3)
    d = Dev(w)
    a = api()
    with pytest.raises(ValueError):
        a.decode(d.q, d.kv, d.indices, w.scale, kv_row_scale=torch.ones(16 * 64, device="cuda"),
                 page_table=d.page_table, page_size=64)
    with pytest.raises(ValueError):
        a.decode(d.q, d.kv, d.indices, w.scale)                 # not paged
    with pytest.raises(ValueError):
        q576 = torch.zeros((2, 64, 576), dtype=torch.bfloat16, device="cuda")
        a.decode(q576, d.kv, d.indices, w.scale, page_table=d.page_table, page_size=64)
