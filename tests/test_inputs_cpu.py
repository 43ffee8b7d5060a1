"""The byte and flop accounting behind every GB/s and roofline figure
(inputs.algorithmic_bytes, algorithmic_flops, indexer_algorithmic_bytes),
checked against sums written out by hand for small workloads, and the
seeded generators' determinism."""
import numpy as np
import torch

from sparse_mla_decode_05_b200 import inputs


def test_bf16_flat_bytes_and_flops():
    w = inputs.flat_per_seq(2, 300, 100, seed=1)
    w.indices[0, :10] = -1                               # 10 padding entries gather nothing
    n = 2 * 100 - 10
    want = n * 1152 + 2 * 64 * 576 * 2 + 2 * 64 * 512 * 2 + 2 * 64 * 4 + 2 * 100 * 4
    assert inputs.algorithmic_bytes(w) == want
    assert inputs.algorithmic_flops(w) == n * 2 * 64 * (576 + 512)


def test_fp8_paged_bytes():
    w = inputs.paged_fp8(3, 1024, 64, 200, seed=2)
    n = int((w.indices >= 0).sum())
    want = n * (576 + 4) + 3 * 64 * 576 * 2 + 3 * 64 * 512 * 2 + 3 * 64 * 4 + 3 * 200 * 4 + w.page_table.numel() * 4
    assert inputs.algorithmic_bytes(w) == want


def test_dsv4_bytes_and_flops():
    w = inputs.paged_dsv4(2, 512, 32, 100, seed=3)
    n = int((w.indices >= 0).sum())
    want = n * (576 + 7) + 2 * 64 * 512 * 2 + 2 * 64 * 512 * 2 + 2 * 64 * 4 + 2 * 100 * 4 + w.page_table.numel() * 4
    assert inputs.algorithmic_bytes(w) == want
    assert inputs.algorithmic_flops(w) == n * 2 * 64 * (512 + 512)


def test_indexer_bytes():
    w = inputs.indexer_workload(3, 700, 40, seed=4, topk=50, ctx_lo=10)
    ctx = int(w.ctx_len.sum())
    want = ctx * 128 * 2 + 3 * 64 * 128 * 2 + 3 * 64 * 4 + w.page_table.numel() * 4 + 3 * 4 + 3 * 50 * 4
    assert inputs.indexer_algorithmic_bytes(w) == want


def test_generators_are_deterministic_and_seed_sensitive():
    a = inputs.indexer_workload(2, 300, 16, seed=9, topk=20, ctx_lo=50)
    b = inputs.indexer_workload(2, 300, 16, seed=9, topk=20, ctx_lo=50)
    c = inputs.indexer_workload(2, 300, 16, seed=10, topk=20, ctx_lo=50)
    for x, y in ((a.q, b.q), (a.k, b.k), (a.w, b.w), (a.page_table, b.page_table), (a.ctx_len, b.ctx_len)):
        assert torch.equal(x, y)
    assert not torch.equal(a.k, c.k)
    d1, d2 = inputs.paged_dsv4(1, 128, 4, 10, seed=5), inputs.paged_dsv4(1, 128, 4, 10, seed=5)
    assert torch.equal(d1.kv, d2.kv) and torch.equal(d1.indices, d2.indices)


def test_full_indexer_config_shape():
    w = inputs.make_indexer_config()
    assert (w.batch, w.max_ctx, w.topk) == (32, 8192, 512)
    assert int(w.ctx_len.min()) == int(w.ctx_len.max()) == 8192
    # every sequence's page table is a distinct slice of one permutation
    pt = w.page_table.numpy()
    assert len(np.unique(pt)) == pt.size and pt.max() < w.k.shape[0] // 64
