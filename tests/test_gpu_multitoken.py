"""GPU parity for multi-token decode (tokens_per_seq = T > 1): every query
token of a sequence attends over its own index list through the sequence's
page table.  Checked against the fp64 oracle's multi-token definition at the
usual bar (out max abs error <= 2e-2, lse relative error <= 1e-3), and
structurally: a multi-token call equals the single-token call on the B * T
flattened rows with each sequence's page-table row repeated T times, bit for
bit, and a token whose list is all padding gets out = 0, lse = -inf while
the other tokens of its sequence are unchanged."""
import numpy as np
import pytest
import torch

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


def oracle_mt(w, seqs=None):
    rsc = None if w.kv_row_scale is None else w.kv_row_scale.numpy()
    pt = None if w.page_table is None else w.page_table.numpy()
    q, idx = w.np_q_bits(), w.indices.numpy()
    if seqs is not None:
        q, idx = q[seqs], idx[seqs]
        pt = None if pt is None else pt[seqs]
    return ref.sparse_mla_decode_multi_token(q, w.np_kv(), idx, w.scale, d_v=512, kv_format=w.kv_format,
                                             kv_row_scale=rsc, page_table=pt, page_size=w.page_size)


def run(w, nsplit=0):
    dev = "cuda:0"
    rsc = None if w.kv_row_scale is None else w.kv_row_scale.to(dev)
    pt = None if w.page_table is None else w.page_table.to(dev)
    return api().decode(w.q.to(dev), w.kv.to(dev), w.indices.to(dev), w.scale, kv_row_scale=rsc, page_table=pt,
                        page_size=w.page_size, nsplit=nsplit)


@pytest.mark.parametrize("fp8,paged,T,topk,nsplit", [
    (False, True, 2, 333, 0), (False, True, 2, 333, 1), (True, True, 4, 700, 0), (False, False, 3, 257, 3),
    (True, True, 2, 64, 2), (False, True, 16, 65, 0), (True, False, 2, 2048, 4)])
def test_multi_token_parity(fp8, paged, T, topk, nsplit):
    w = inputs.multi_token(3, T, 4096, 256, topk, seed=200 + T + topk + nsplit, fp8=fp8, paged=paged)
    out, lse = run(w, nsplit)
    torch.cuda.synchronize()
    assert out.shape == (3, T, 64, 512) and lse.shape == (3, T, 64)
    o_ref, l_ref = oracle_mt(w)
    assert_parity(out, lse, o_ref, l_ref, tag=f"mt fp8={fp8} paged={paged} T={T} k={topk} n={nsplit}")


@pytest.mark.parametrize("fp8", [False, True])
def test_multi_token_equals_flattened_rows(fp8):
    """Row b*T + t of a multi-token call is the single-token decode of q[b, t]
    over indices[b, t] through page-table row b: bit-identical results."""
    w = inputs.multi_token(4, 3, 2048, 256, 300, seed=17, fp8=fp8)
    out, lse = run(w)
    B, T = 4, 3
    flat = inputs.Workload(name="flat_rows", q=w.q.reshape(B * T, 64, 576).contiguous(), kv=w.kv,
                           indices=w.indices.reshape(B * T, -1).contiguous(), scale=w.scale,
                           kv_row_scale=w.kv_row_scale,
                           page_table=w.page_table.repeat_interleave(T, dim=0).contiguous(), page_size=64)
    o1, l1 = run(flat)
    torch.cuda.synchronize()
    assert torch.equal(out.reshape(B * T, 64, 512), o1) and torch.equal(lse.reshape(B * T, 64), l1)


def test_padding_only_token():
    w = inputs.multi_token(2, 3, 2048, 128, 200, seed=23)
    idx = w.indices.clone()
    idx[1, 1] = -1                                          # sequence 1, token 1: nothing valid
    w2 = inputs.Workload(name="mt_pad", q=w.q, kv=w.kv, indices=idx, scale=w.scale, page_table=w.page_table,
                         page_size=64)
    out, lse = run(w)
    out2, lse2 = run(w2)
    torch.cuda.synchronize()
    assert torch.all(out2[1, 1] == 0) and torch.all(torch.isneginf(lse2[1, 1]))
    keep = [(0, 0), (0, 1), (0, 2), (1, 0), (1, 2)]
    for b, t in keep:
        assert torch.equal(out2[b, t], out[b, t]) and torch.equal(lse2[b, t], lse[b, t])
    o_ref, l_ref = oracle_mt(w2)
    assert_parity(out2, lse2, o_ref, l_ref, tag="mt padding-only token")


def test_mt2_workload_sampled():
    """The full-size multi-token workload (the bench's mt2 line: 64
    sequences x 2 tokens, top-2048 per token, paged fp8), in the launch
    configuration the planner picks, checked on sampled sequences."""
    w = inputs.make_config("mt2")
    out, lse = run(w)
    torch.cuda.synchronize()
    seqs = [0, 13, 31, 47, 63]
    o_ref, l_ref = oracle_mt(w, seqs)
    err, lerr, _ = assert_parity(out[seqs], lse[seqs], o_ref, l_ref, tag="mt2 sampled")
    print(f"mt2: max|dout|={err:.3e} lse_rel={lerr:.3e}")


def test_multi_token_host_buffers():
    """sparse_mla_decode_host with T = 2: q, indices and the page table
    copied in, out and lse copied back; bit-identical to the device call."""
    w = inputs.multi_token(3, 2, 2048, 128, 500, seed=29, fp8=True)
    out, lse = run(w)
    a = api()
    dev = torch.device("cuda:0")
    hp = a.HostDecodePlan(w.q.pin_memory(), w.kv.to(dev), w.indices.pin_memory(), w.scale,
                          kv_row_scale=w.kv_row_scale.to(dev), page_table_host=w.page_table.pin_memory(),
                          page_size=64)
    hp.run()
    torch.cuda.synchronize()
    assert torch.equal(hp.out_host, out.cpu()) and torch.equal(hp.lse_host, lse.cpu())
