"""Bounded waits running out, on the GPU, without a fault or a hang.

sparse_mla_decode_stalled launches the decode kernel with every pipeline
wait limited to a short cycle count and the score-MMA warp waiting on a
barrier that nothing arrives on.  No MMA is issued, so every other warp's
wait runs out in turn.  The kernel must return on its own (the synchronize
below finishes), set bit 0 of the device error word and nothing else,
leave out / lse unwritten, and release its tensor memory: the decodes that
follow (one CTA per sequence, and the planned multi-split launch with its
in-cluster merge) allocate it again and reproduce the results taken before
the stall, bit for bit.  The error word reports a timeout apart from an
out-of-range input (bit 2, SMLA_ERR_DEVICE_INDEX)."""
import ctypes

import torch
import pytest

from sparse_mla_decode_05_b200 import inputs

pytestmark = pytest.mark.gpu

TIMEOUT, INDEX = 5, 6
WAIT_LIMIT = 100_000          # SM cycles, about 50 us at B200 clocks


def api():
    from sparse_mla_decode_05_b200 import api as a
    return a


def read_error():
    code = ctypes.c_uint32(0)
    st = api().lib.sparse_mla_get_device_error(ctypes.byref(code))
    return st, code.value


def _bits(t):
    return t.view(torch.int16) if t.dtype == torch.bfloat16 else t.view(torch.int32)


def test_stalled_kernel_times_out_and_the_context_stays_usable():
    a = api()
    w = inputs.flat_per_seq(3, 2048, 700, seed=91)
    dev = "cuda:0"
    q, kv, idx = w.q.to(dev), w.kv.to(dev), w.indices.to(dev)
    torch.cuda.synchronize()
    assert read_error() == (0, 0)
    want1 = a.decode(q, kv, idx, w.scale, nsplit=1)
    want_planned = a.decode(q, kv, idx, w.scale)
    torch.cuda.synchronize()
    assert read_error() == (0, 0)
    for _ in range(2):
        out = torch.full((3, 64, 512), float("nan"), dtype=torch.bfloat16, device=dev)
        lse = torch.full((3, 64), float("nan"), dtype=torch.float32, device=dev)
        a.decode_stalled(q, kv, idx, w.scale, WAIT_LIMIT, out=out, lse=lse)
        torch.cuda.synchronize()                       # the kernel returned by itself
        assert read_error() == (TIMEOUT, 1)            # bit 0 alone
        assert read_error() == (0, 0)                  # the read cleared it
        assert torch.isnan(out.float()).all() and torch.isnan(lse).all()   # epilogue skipped
        for n, want in ((1, want1), (0, want_planned)):
            got = a.decode(q, kv, idx, w.scale, nsplit=n)
            torch.cuda.synchronize()
            assert torch.equal(_bits(got[0]), _bits(want[0])) and torch.equal(_bits(got[1]), _bits(want[1]))
        assert read_error() == (0, 0)


def test_timeout_and_index_errors_are_told_apart():
    a = api()
    w = inputs.flat_per_seq(2, 1024, 300, seed=92)
    dev = "cuda:0"
    q, kv = w.q.to(dev), w.kv.to(dev)
    bad = w.indices.clone()
    bad[0, 5] = 2 * 1024 + 7                           # past the pool: read as padding, bit 2
    idx, idx_bad = w.indices.to(dev), bad.to(dev)
    torch.cuda.synchronize()
    assert read_error() == (0, 0)
    a.decode(q, kv, idx_bad, w.scale)
    torch.cuda.synchronize()
    assert read_error() == (INDEX, 4)
    a.decode_stalled(q, kv, idx, w.scale, WAIT_LIMIT)
    torch.cuda.synchronize()
    assert read_error() == (TIMEOUT, 1)
    # both in one word: the timeout is reported, both bits are kept
    a.decode_stalled(q, kv, idx, w.scale, WAIT_LIMIT)
    a.decode(q, kv, idx_bad, w.scale)
    torch.cuda.synchronize()
    assert read_error() == (TIMEOUT, 5)
    assert read_error() == (0, 0)


def test_stalled_hook_rejects_what_it_does_not_cover():
    a = api()
    w = inputs.paged_fp8(2, 1024, 64, 100, seed=93)
    dev = "cuda:0"
    shape = a.shape_for(w.q.to(dev), w.kv.to(dev), w.indices.to(dev), page_table=w.page_table.to(dev),
                        page_size=64)
    st = a.lib.sparse_mla_decode_stalled(ctypes.byref(shape), 16, 16, 16, 0.04, 16, 16, WAIT_LIMIT, None)
    assert st == 2                                     # SMLA_ERR_UNSUPPORTED, nothing launched
    wb = inputs.flat_per_seq(2, 1024, 100, seed=94)
    shape = a.shape_for(wb.q.to(dev), wb.kv.to(dev), wb.indices.to(dev))
    for lim in (0, 999, 4_000_000_001):
        assert a.lib.sparse_mla_decode_stalled(ctypes.byref(shape), 16, 16, 16, 0.04, 16, 16, lim, None) == 1
    torch.cuda.synchronize()
    assert read_error() == (0, 0)
