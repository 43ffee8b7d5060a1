"""Pins for the fp64 oracle (CPU only).

Each pin ties the oracle to something other than itself: a library routine
(torch's float64 attention, bf16 and float8_e4m3fn decoders), a closed form,
hand-worked fixtures under tests/golden/, or brute force.  The mutation tests
at the end plant plausible mistakes in a copy of the oracle and check that
some pin catches each one.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import sparse_mla_ref as ref
from sparse_mla_decode_05_b200 import inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def bf16_bits(x) -> np.ndarray:
    t = torch.as_tensor(np.asarray(x, dtype=np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def rand_problem(seed, B=2, H=4, d_qk=24, d_v=16, N=40, k=12, q_mult=1.0):
    rng = np.random.default_rng(seed)
    q = bf16_bits(rng.standard_normal((B, H, d_qk)) * q_mult)
    kv = bf16_bits(rng.standard_normal((N, d_qk)))
    idx = np.stack([rng.choice(N, k, replace=False) for _ in range(B)]).astype(np.int32)
    return q, kv, idx


# ---------------------------------------------------------------- decoders
def test_bf16_decode_matches_torch_all_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    mine = ref.bf16_bits_to_f64(bits)
    lib = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], lib[~nan])
    assert np.array_equal(np.signbit(mine[~nan]), np.signbit(lib[~nan]))


def test_e4m3fn_decode_matches_torch_all_codes():
    codes = np.arange(256, dtype=np.uint8)
    mine = ref.e4m3fn_to_f64(codes)
    lib = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    nan = np.isnan(lib)
    assert nan.sum() == 2                       # 0x7F, 0xFF
    assert np.array_equal(np.isnan(mine), nan)
    assert np.array_equal(mine[~nan], lib[~nan])
    assert np.array_equal(np.signbit(mine[~nan]), np.signbit(lib[~nan]))


def test_e4m3fn_spec_points():
    pts = json.load(open(os.path.join(GOLDEN, "e4m3fn_spec_points.json")))["points"]
    for p in pts:
        v = ref.e4m3fn_to_f64(np.array([int(p["code"], 16)], dtype=np.uint8))[0]
        want = float(p["value"])
        if math.isnan(want):
            assert math.isnan(v), p
        else:
            assert v == want and math.copysign(1, v) == math.copysign(1, want), p


def test_bf16_rounding_matches_torch_on_fp32_values():
    rng = np.random.default_rng(7)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-39).astype(np.float32),      # subnormals
        (rng.standard_normal(2000) * 3e38).astype(np.float32),       # near overflow
        np.array([0.0, -0.0, np.inf, -np.inf, 1.0 + 2**-8, 1.0 + 3 * 2**-8,
                  1.0 + 2**-8 + 2**-20, 3.3961e38], dtype=np.float32),
    ])
    mine = ref.f64_to_bf16_bits_rne(x.astype(np.float64))
    lib = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(mine, lib)


# ------------------------------------------------------------ hand-worked
def _golden_cases():
    return json.load(open(os.path.join(GOLDEN, "tiny_handworked.json")))["cases"]


@pytest.mark.parametrize("case", _golden_cases(), ids=lambda c: c["name"])
def test_handworked_golden(case):
    q = bf16_bits(case["q"])[None]                 # [1, H, d_qk]
    kv = bf16_bits(case["rows"])
    idx = np.array([case["indices"]], dtype=np.int32)
    scale = math.log(case["scale_is_ln_of"])
    out, lse = ref.sparse_mla_decode(q, kv, idx, scale, d_v=case["d_v"])
    np.testing.assert_allclose(out[0], np.array(case["out"]), rtol=0, atol=1e-15)
    want_lse = np.array([float(v) for v in case["lse"]])
    if np.isneginf(want_lse).all():
        assert np.isneginf(lse[0]).all()
    else:
        np.testing.assert_allclose(lse[0], want_lse, rtol=1e-15, atol=1e-15)


# ------------------------------------------------------- the four checks
def test_dense_case_equals_torch_attention_real_sizes():
    """top-k covering the whole cache == dense softmax(scale q K^T) V."""
    rng = np.random.default_rng(11)
    N = 300
    q = bf16_bits(rng.standard_normal((2, 64, 576)))
    kv = bf16_bits(rng.standard_normal((N, 576)))
    idx = np.stack([rng.permutation(N), np.arange(N)]).astype(np.int32)
    scale = 1 / math.sqrt(576)
    out, lse = ref.sparse_mla_decode(q, kv, idx, scale)
    qt = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    kt = torch.from_numpy(kv.view(np.int16)).view(torch.bfloat16).to(torch.float64)
    for b in range(2):
        want = torch.nn.functional.scaled_dot_product_attention(
            qt[b][None], kt[None], kt[None, :, :512], scale=scale)[0]
        np.testing.assert_allclose(out[b], want.numpy(), rtol=0, atol=1e-12)
        want_lse = torch.logsumexp(scale * qt[b] @ kt.T, dim=1)
        np.testing.assert_allclose(lse[b], want_lse.numpy(), rtol=1e-13, atol=0)


def test_single_index_returns_the_value_row_exactly():
    q, kv, _ = rand_problem(3, B=1, H=64, d_qk=576, d_v=512, N=50, k=2)
    for r in (0, 17, 49):
        out, lse = ref.sparse_mla_decode(q, kv, np.array([[r]], np.int32), 0.1)
        v = ref.bf16_bits_to_f64(kv[r])
        assert np.array_equal(out[0], np.broadcast_to(v[:512], (64, 512)))
        qf = ref.bf16_bits_to_f64(q[0])
        s = np.array([0.1 * math.fsum(qf[h] * v) for h in range(64)])
        np.testing.assert_allclose(lse[0], s, rtol=1e-13, atol=1e-13)


def test_zero_query_gives_mean_of_values_and_log_count():
    _, kv, idx = rand_problem(5, B=2, H=3, d_qk=20, d_v=12, N=30, k=10)
    idx[1, [2, 5, 7]] = -1
    q = np.zeros((2, 3, 20), dtype=np.uint16)
    out, lse = ref.sparse_mla_decode(q, kv, idx, 0.3, d_v=12)
    for b in range(2):
        rows = idx[b][idx[b] >= 0]
        mean = ref.bf16_bits_to_f64(kv[rows])[:, :12].mean(axis=0)
        np.testing.assert_allclose(out[b], np.broadcast_to(mean, (3, 12)), rtol=0, atol=1e-14)
        np.testing.assert_allclose(lse[b], math.log(rows.size), rtol=1e-15)


def test_permutation_invariance_and_padding_insertion():
    q, kv, idx = rand_problem(9, B=2, H=5, d_qk=32, d_v=16, N=64, k=20)
    out, lse = ref.sparse_mla_decode(q, kv, idx, 0.2, d_v=16)
    rng = np.random.default_rng(1)
    perm = np.stack([rng.permutation(idx[b]) for b in range(2)])
    out_p, lse_p = ref.sparse_mla_decode(q, kv, perm, 0.2, d_v=16)
    np.testing.assert_allclose(out_p, out, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse_p, lse, rtol=1e-13)
    padded = np.full((2, 31), -1, np.int32)
    for b in range(2):
        pos = np.sort(rng.choice(31, 20, replace=False))
        padded[b, pos] = idx[b]
    out_q, lse_q = ref.sparse_mla_decode(q, kv, padded, 0.2, d_v=16)
    assert np.array_equal(out_q, out) and np.array_equal(lse_q, lse)


def test_two_row_closed_form():
    q, kv, _ = rand_problem(12, B=1, H=6, d_qk=40, d_v=24, N=10, k=2, q_mult=3.0)
    scale = 0.37
    out, lse = ref.sparse_mla_decode(q, kv, np.array([[4, 7]], np.int32), scale, d_v=24)
    qf = ref.bf16_bits_to_f64(q[0])
    v1, v2 = ref.bf16_bits_to_f64(kv[4]), ref.bf16_bits_to_f64(kv[7])
    for h in range(6):
        s1 = scale * math.fsum(qf[h] * v1)
        s2 = scale * math.fsum(qf[h] * v2)
        sig = 1 / (1 + math.exp(s2 - s1))
        want = sig * v1[:24] + (1 - sig) * v2[:24]
        np.testing.assert_allclose(out[0, h], want, rtol=0, atol=1e-13)
        np.testing.assert_allclose(lse[0, h], np.logaddexp(s1, s2), rtol=1e-13)


def test_all_padding_sequence():
    q, kv, idx = rand_problem(4, B=2, H=3, d_qk=8, d_v=4, N=16, k=5)
    idx[1] = -1
    out, lse = ref.sparse_mla_decode(q, kv, idx, 1.0, d_v=4)
    assert np.all(out[1] == 0) and np.all(np.isneginf(lse[1]))
    assert np.all(np.isfinite(out[0])) and np.all(np.isfinite(lse[0]))


def test_split_combine_identity():
    q, kv, idx = rand_problem(21, B=2, H=4, d_qk=32, d_v=16, N=80, k=30, q_mult=4.0)
    full_o, full_l = ref.sparse_mla_decode(q, kv, idx, 0.25, d_v=16)
    parts = [idx[:, :7], idx[:, 7:19], idx[:, 19:]]
    res = [ref.sparse_mla_decode(q, kv, p, 0.25, d_v=16) for p in parts]
    o, l = ref.combine_partials([r[0] for r in res], [r[1] for r in res])
    np.testing.assert_allclose(o, full_o, rtol=0, atol=1e-12)
    np.testing.assert_allclose(l, full_l, rtol=1e-13)
    # an empty part (all padding) carries zero weight
    empty = np.full((2, 4), -1, np.int32)
    res.append(ref.sparse_mla_decode(q, kv, empty, 0.25, d_v=16))
    o2, l2 = ref.combine_partials([r[0] for r in res], [r[1] for r in res])
    np.testing.assert_allclose(o2, full_o, rtol=0, atol=1e-12)
    # every part empty
    o3, l3 = ref.combine_partials([res[-1][0]] * 2, [res[-1][1]] * 2)
    assert np.all(o3 == 0) and np.all(np.isneginf(l3))


def test_paged_equals_flat_with_brute_force_mapping():
    rng = np.random.default_rng(31)
    page, pps, pages_total = 4, 6, 20
    kv = bf16_bits(rng.standard_normal((pages_total * page, 16)))
    q = bf16_bits(rng.standard_normal((2, 3, 16)))
    pt = np.stack([rng.permutation(pages_total)[:pps] for _ in range(2)]).astype(np.int32)
    logical = np.stack([rng.choice(pps * page, 9, replace=False) for _ in range(2)]).astype(np.int32)
    logical[0, 3] = -1
    out_p, lse_p = ref.sparse_mla_decode(q, kv, logical, 0.5, d_v=8, page_table=pt, page_size=page)
    phys = np.full_like(logical, -1)
    for b in range(2):
        for j in range(logical.shape[1]):
            r = int(logical[b, j])
            if r >= 0:
                phys[b, j] = int(pt[b, r // page]) * page + (r % page)
    out_f, lse_f = ref.sparse_mla_decode(q, kv, phys, 0.5, d_v=8)
    assert np.array_equal(out_p, out_f) and np.array_equal(lse_p, lse_f)


def test_fp8_rowscale_rows_match_torch_decode():
    rng = np.random.default_rng(41)
    x = torch.from_numpy(rng.standard_normal((12, 576)).astype(np.float32))
    s = x.abs().amax(dim=1) / 448
    codes = (x / s[:, None]).to(torch.float8_e4m3fn)
    rows = np.array([3, 0, 11])
    mine = ref.gather_rows_f64(codes.view(torch.uint8).numpy(), rows,
                               kv_format="fp8_e4m3_rowscale", row_scale=s.numpy())
    lib = codes.to(torch.float64)[rows] * s.to(torch.float64)[rows, None]
    assert np.array_equal(mine, lib.numpy())


def test_out_of_range_indices_are_rejected():
    q, kv, idx = rand_problem(2, B=1, H=2, d_qk=8, d_v=4, N=10, k=3)
    with pytest.raises(ValueError):
        ref.sparse_mla_decode(q, kv, np.array([[1, -2]], np.int32), 1.0, d_v=4)
    with pytest.raises(ValueError):
        ref.sparse_mla_decode(q, kv, np.array([[10]], np.int32), 1.0, d_v=4)


def test_lse_rel_err_conventions():
    assert ref.lse_rel_err(np.array([-np.inf]), np.array([-np.inf]))[0] == 0
    assert ref.lse_rel_err(np.array([0.001]), np.array([0.0]))[0] == pytest.approx(0.001)
    assert ref.lse_rel_err(np.array([10.01]), np.array([10.0]))[0] == pytest.approx(0.001)


def test_generators_are_deterministic_and_shaped():
    w1 = inputs.flat_varlen(4, 20, 90, 64, seed=5)
    w2 = inputs.flat_varlen(4, 20, 90, 64, seed=5)
    assert torch.equal(w1.indices, w2.indices) and torch.equal(w1.q.view(torch.int16), w2.q.view(torch.int16))
    for b, L in enumerate(w1.meta["lens"]):
        row = w1.indices[b].numpy()
        valid = row[row >= 0]
        assert len(set(valid.tolist())) == valid.size == min(L, 64)
        if L < 64:
            assert np.all(row[L:] == -1)
    w = inputs.flat_per_seq(2, 4096, 512, seed=3, index_mode="recency")
    for b in range(2):
        r = w.indices[b].numpy() - b * 4096
        assert np.all(np.diff(r) > 0) and (r >= 4096 - 1024).sum() >= 256
    p = inputs.paged_fp8(3, 256, 20, 64, seed=9)
    assert p.kv.dtype == torch.uint8 and p.page_table.shape == (3, 4)
    assert len(set(p.page_table.flatten().tolist())) == 12
    codes = p.kv.numpy()
    assert not np.any((codes & 0x7F) == 0x7F)          # no NaN codes


# ------------------------------------------------------- planted mistakes
def _mutant(kind):
    """A copy of the oracle's definition with one plausible mistake."""
    def decode(q_bits, kv, indices, scale, *, d_v=512, kv_format="bf16", kv_row_scale=None,
               page_table=None, page_size=0):
        B, H, d_qk = q_bits.shape
        out = np.zeros((B, H, d_v))
        lse = np.zeros((B, H))
        for b in range(B):
            idx = np.asarray(indices[b], np.int64)
            if kind == "padding_as_row0":
                idx = np.where(idx < 0, 0, idx)
            if page_size:
                v = idx >= 0
                rows = np.full(idx.shape, -1)
                if kind == "paged_swapped":
                    rows[v] = page_table[b][idx[v] % page_size] * page_size + idx[v] // page_size
                else:
                    rows[v] = page_table[b][idx[v] // page_size] * page_size + idx[v] % page_size
            else:
                rows = idx
            rows = rows[rows >= 0]
            k = ref.gather_rows_f64(kv, rows, kv_format=kv_format,
                                    row_scale=None if kind == "fp8_no_scale" else kv_row_scale)
            if kind == "fp8_no_scale" and kv_format != "bf16":
                k = ref.e4m3fn_to_f64(kv[rows])
            qh = ref.bf16_bits_to_f64(q_bits[b])
            if kind == "no_rope":
                s = scale * (qh[:, :d_v] @ k[:, :d_v].T)
            elif kind == "no_scale":
                s = qh @ k.T
            else:
                s = scale * (qh @ k.T)
            if rows.size == 0:
                out[b], lse[b] = 0, -np.inf
                continue
            M = s.max(1, keepdims=True)
            e = np.exp(M - s) if kind == "sign" else np.exp(s - M)
            W = e.sum(1, keepdims=True)
            val = k[:, -d_v:] if kind == "value_tail" else k[:, :d_v]
            out[b] = (e @ val) / W
            lse[b] = (np.log(W) if kind == "lse_no_max" else M + np.log(W))[:, 0]
        return out, lse
    return decode


def _pins_pass(decode) -> bool:
    """Run a subset of the pins against ``decode``; True if all hold."""
    try:
        # dense vs torch attention
        rng = np.random.default_rng(11)
        q = bf16_bits(rng.standard_normal((1, 8, 40)) * 2)
        kv = bf16_bits(rng.standard_normal((30, 40)))
        idx = rng.permutation(30)[None].astype(np.int32)
        out, lse = decode(q, kv, idx, 0.3, d_v=32)
        qt = torch.from_numpy(q.view(np.int16)).view(torch.bfloat16).double()[0]
        kt = torch.from_numpy(kv.view(np.int16)).view(torch.bfloat16).double()
        want = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], kt[None, :, :32], scale=0.3)[0]
        if not np.allclose(out[0], want.numpy(), atol=1e-12, rtol=0):
            return False
        if not np.allclose(lse[0], torch.logsumexp(0.3 * qt @ kt.T, 1).numpy(), rtol=1e-12):
            return False
        # padding insertion
        pad = np.full((1, 60), -1, np.int32)
        pad[0, ::2] = idx[0]
        o2, l2 = decode(q, kv, pad, 0.3, d_v=32)
        if not (np.allclose(o2, out, atol=1e-12) and np.allclose(l2, lse, rtol=1e-12)):
            return False
        # paged == flat
        pt = np.array([[2, 0, 1]], np.int32)
        logical = np.array([[0, 5, 7, 11]], np.int32)
        phys = np.array([[2 * 4 + 0, 0 * 4 + 1, 0 * 4 + 3, 1 * 4 + 3]], np.int32)
        kv12 = kv[:12]
        op, lp = decode(q, kv12, logical, 0.3, d_v=32, page_table=pt, page_size=4)
        of, lf = decode(q, kv12, phys, 0.3, d_v=32)
        if not (np.allclose(op, of, atol=1e-12) and np.allclose(lp, lf, rtol=1e-12)):
            return False
        # fp8 rows vs torch decode
        x = torch.from_numpy(rng.standard_normal((6, 40)).astype(np.float32))
        s = x.abs().amax(1) / 448
        codes = (x / s[:, None]).to(torch.float8_e4m3fn)
        o8, _ = decode(q, codes.view(torch.uint8).numpy(), np.array([[0, 1, 2, 3, 4, 5]], np.int32), 0.3,
                       d_v=32, kv_format="fp8_e4m3_rowscale", kv_row_scale=s.numpy())
        k8 = (codes.double() * s.double()[:, None])
        w8 = torch.nn.functional.scaled_dot_product_attention(qt[None], k8[None], k8[None, :, :32], scale=0.3)[0]
        if not np.allclose(o8[0], w8.numpy(), atol=1e-12, rtol=0):
            return False
    except Exception:
        return False
    return True


def test_pins_accept_the_oracle():
    assert _pins_pass(ref.sparse_mla_decode)


@pytest.mark.parametrize("kind", ["padding_as_row0", "paged_swapped", "fp8_no_scale", "no_rope",
                                  "no_scale", "sign", "value_tail", "lse_no_max"])
def test_pins_reject_planted_mistakes(kind):
    assert not _pins_pass(_mutant(kind))


# ------------------------------------------------ DeepSeek-V4 paged layout
def test_ue8m0_decode_all_codes():
    e = np.arange(256)
    got = ref.ue8m0_to_f64(e)
    for v in range(255):
        assert got[v] == math.ldexp(1.0, v - 127)
    assert np.isnan(got[255])


def _hand_page(mistake=None):
    """Page 2 of 3, slot 5, written byte by byte; returns (pages, row, want)."""
    pages = np.zeros((3, 64 * 584), np.uint8)
    slot, page = 5, 2
    base = 576 * slot
    codes = np.full(448, 0x38, np.uint8)            # e4m3fn 0x38 = 1.0
    codes[0] = 0xC0                                 # -2.0
    codes[64] = 0x30                                # 0.5
    codes[447] = 0x01                               # 2^-9 (smallest subnormal)
    pages[page, base:base + 448] = codes
    rope = np.zeros(64, np.uint16)
    rope[0], rope[63] = 0x3FC0, 0xBE80              # bf16 1.5, -0.25
    pages[page, base + 448:base + 576] = rope.view(np.uint8)     # little-endian bytes
    sc = np.full(7, 127, np.uint8)
    sc[0], sc[1], sc[6] = 128, 126, 130             # x2, x0.5, x8
    pages[page, 64 * 576 + 8 * slot:64 * 576 + 8 * slot + 7] = sc
    want = np.ones(512)
    want[0:64] = 2.0
    want[0] = -4.0
    want[64:128] = 0.5
    want[64] = 0.25
    want[384:448] = 8.0
    want[447] = 8.0 * 2.0 ** -9
    want[448:512] = 0.0
    want[448], want[511] = 1.5, -0.25
    rows_fn = ref.dsv4_rows_f64
    if mistake == "scale_group_shift":
        def rows_fn(p, r):
            v = ref.dsv4_rows_f64(p, r)
            nope = ref.e4m3fn_to_f64(p[r // 64][:, (r % 64)[0] * 576:(r % 64)[0] * 576 + 448])
            sc_ = ref.ue8m0_to_f64(p[r // 64][:, 64 * 576 + 8 * (r % 64)[0]:64 * 576 + 8 * (r % 64)[0] + 7])
            v[:, :448] = nope * np.repeat(np.roll(sc_, 1, axis=1), 64, axis=1)
            return v
    if mistake == "rope_big_endian":
        def rows_fn(p, r):
            v = ref.dsv4_rows_f64(p, r)
            b = p[r // 64][:, (r % 64)[0] * 576 + 448:(r % 64)[0] * 576 + 576].astype(np.uint16)
            v[:, 448:] = ref.bf16_bits_to_f64((b[:, 0::2] << 8) | b[:, 1::2])
            return v
    if mistake == "scale_on_rope":
        def rows_fn(p, r):
            v = ref.dsv4_rows_f64(p, r)
            v[:, 448:] *= 2.0
            return v
    return pages, np.array([page * 64 + slot]), want, rows_fn


@pytest.mark.parametrize("mistake", [None, "scale_group_shift", "rope_big_endian", "scale_on_rope"])
def test_dsv4_hand_built_page(mistake):
    pages, row, want, rows_fn = _hand_page(mistake)
    got = rows_fn(pages, row)[0]
    assert np.array_equal(got, want) == (mistake is None)


def test_dsv4_decode_equals_the_plain_path_on_decoded_rows():
    """The paged DeepSeek-V4 decode equals the (torch-pinned) bf16 path run on
    a flat pool holding the decoded rows: e4m3fn value x power of two and
    bf16 rope are exact in bf16, and V is the whole 512-dim row."""
    w = inputs.paged_dsv4(3, 512, 32, 200, seed=12)
    pages = w.kv.numpy()
    idx = w.indices.numpy()
    pt = w.page_table.numpy()
    o, l = ref.sparse_mla_decode(w.np_q_bits(), pages, idx, w.scale, kv_format="dsv4_paged",
                                 page_table=pt, page_size=64)
    n_rows = pages.shape[0] * 64
    flat = ref.dsv4_rows_f64(pages, np.arange(n_rows))
    flat_bits = ref.f64_to_bf16_bits_rne(flat)
    assert np.array_equal(ref.bf16_bits_to_f64(flat_bits), flat)          # exact in bf16
    of, lf = ref.sparse_mla_decode(w.np_q_bits(), flat_bits, idx, w.scale, d_v=512, page_table=pt, page_size=64)
    assert np.allclose(o, of, atol=1e-12, rtol=0) and np.allclose(l, lf, atol=1e-12, rtol=0)
