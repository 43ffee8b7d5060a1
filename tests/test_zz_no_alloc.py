"""sparse_mla_decode_static_scratch: the decode step with the split partials
in the library's static device scratch, for callers that cannot allocate.

Collected last (file name) so that it runs after every other test as well as
alone.  The GPU tests compare two calls in a row against sparse_mla_decode
(same kernels, same split count, caller-allocated workspace): the results
must be bit-identical.  The size-limit checks run without a GPU: a shape
whose partials exceed the scratch is rejected before any CUDA call.
"""
from __future__ import annotations

import ctypes

import pytest
import torch

from sparse_mla_decode_05_b200 import api, inputs

WORKSPACE = 3
PARTIAL_BYTES = 64 * 512 * 4 + 64 * 4   # one (sequence, split) partial


def _static(shape, q=16, kv=16, idx=16, out=16, lse=16):
    return api.lib.sparse_mla_decode_static_scratch(ctypes.byref(shape), q, kv, None, None, idx, 0.04,
                                                    out, lse, None)


@pytest.mark.parametrize("batch,topk,nsplit", [(64, 512, 6), (64, 192, 3), (1, 2048 * 64, 200)])
def test_over_the_limit_rejected_before_any_cuda_call(batch, topk, nsplit):
    assert batch * nsplit * PARTIAL_BYTES > api.STATIC_SCRATCH_BYTES
    s = api.make_shape(batch, topk, 100000, nsplit=nsplit)
    assert _static(s) == WORKSPACE


@pytest.mark.skipif(torch.cuda.is_available(), reason="the shape passes the host checks and would launch")
@pytest.mark.parametrize("batch,nsplit", [(64, 4), (20, 16)])
def test_fixed_power_of_two_split_is_not_rejected_when_the_cluster_merge_fits(batch, nsplit):
    # the separate combine's partials would not fit, the in-cluster merge's
    # workspace (64 x 512 fp16 + 64 x 8 fp32 per split) does: the host
    # checks pass it on to the device query, which fails without a GPU
    assert batch * nsplit * PARTIAL_BYTES > api.STATIC_SCRATCH_BYTES
    assert batch * nsplit * (64 * 512 * 2 + 64 * 32) <= api.STATIC_SCRATCH_BYTES
    s = api.make_shape(batch, 64 * nsplit, 100000, nsplit=nsplit)
    assert _static(s) not in (WORKSPACE, 0)


@pytest.mark.parametrize("batch,nsplit", [(8, 32), (16, 24)])
def test_fixed_split_without_cluster_merge_is_rejected_on_its_partials(batch, nsplit):
    # more than 16 splits, or not a power of two: only the separate combine
    assert batch * nsplit * PARTIAL_BYTES > api.STATIC_SCRATCH_BYTES
    s = api.make_shape(batch, 64 * nsplit, 100000, nsplit=nsplit)
    assert _static(s) == WORKSPACE


def test_limit_constant_matches_header():
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(api.__file__), "..", "include", "sparse_mla.h")).read()
    m = re.search(r"#define SMLA_STATIC_SCRATCH_BYTES \(\(size_t\)(\d+) << (\d+)\)", hdr)
    assert m and int(m.group(1)) << int(m.group(2)) == api.STATIC_SCRATCH_BYTES
    # every split count the planner picks on a 148-SM part fits, merged
    # either way (an in-cluster merge needs 64 x 512 fp16 + 64 x 8 fp32 of
    # statistics per split, less than a partial)
    assert 148 * PARTIAL_BYTES <= api.STATIC_SCRATCH_BYTES
    assert 64 * 512 * 2 + 64 * 32 < PARTIAL_BYTES


def _dev(w):
    d = "cuda"
    return dict(q=w.q.to(d), kv=w.kv.to(d), indices=w.indices.to(d),
                kv_row_scale=None if w.kv_row_scale is None else w.kv_row_scale.to(d),
                page_table=None if w.page_table is None else w.page_table.to(d), page_size=w.page_size)


CASES = {
    "varlen_planned": (lambda: inputs.flat_varlen(4, 100, 900, 512, seed=77), 0),
    "flat_nsplit5": (lambda: inputs.flat_per_seq(2, 2048, 700, seed=78), 5),
    "flat_nsplit4_on_chip": (lambda: inputs.flat_per_seq(2, 2048, 700, seed=82), 4),
    "paged_fp8_planned": (lambda: inputs.paged_fp8(3, 1024, 64, 300, seed=79), 0),
    "single_split": (lambda: inputs.flat_per_seq(2, 1024, 200, seed=80), 1),
}


@pytest.mark.gpu
@pytest.mark.parametrize("case", sorted(CASES))
def test_two_calls_in_a_row_match_sparse_mla_decode(case):
    make, nsplit = CASES[case]
    w = make()
    t = _dev(w)
    kw = dict(kv_row_scale=t["kv_row_scale"], page_table=t["page_table"], page_size=t["page_size"],
              nsplit=nsplit)
    want_o, want_l = api.decode(t["q"], t["kv"], t["indices"], w.scale, **kw)
    B = w.batch
    for _ in range(2):
        out = torch.full((B, 64, 512), float("nan"), dtype=torch.bfloat16, device="cuda")
        lse = torch.full((B, 64), float("nan"), dtype=torch.float32, device="cuda")
        api.decode_static_scratch(t["q"], t["kv"], t["indices"], w.scale, out, lse, **kw)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), want_o.view(torch.int16))
        assert torch.equal(lse.view(torch.int32), want_l.view(torch.int32))
    assert api.device_error() == 0


@pytest.mark.gpu
def test_largest_fitting_and_first_rejected_shape_on_gpu():
    # 63 x 3 partials fit in the scratch, 64 x 3 do not (3 splits merge
    # through partials: not a power of two)
    assert 63 * 3 * PARTIAL_BYTES <= api.STATIC_SCRATCH_BYTES < 64 * 3 * PARTIAL_BYTES
    w = inputs.flat_per_seq(64, 256, 192, seed=81)
    t = _dev(w)
    q63, i63 = t["q"][:63].contiguous(), t["indices"][:63].contiguous()
    want_o, want_l = api.decode(q63, t["kv"], i63, w.scale, nsplit=3)
    out = torch.empty((63, 64, 512), dtype=torch.bfloat16, device="cuda")
    lse = torch.empty((63, 64), dtype=torch.float32, device="cuda")
    api.decode_static_scratch(q63, t["kv"], i63, w.scale, out, lse, nsplit=3)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), want_o.view(torch.int16))
    assert torch.equal(lse.view(torch.int32), want_l.view(torch.int32))
    out64 = torch.empty((64, 64, 512), dtype=torch.bfloat16, device="cuda")
    lse64 = torch.empty((64, 64), dtype=torch.float32, device="cuda")
    with pytest.raises(api.SmlaError) as e:
        api.decode_static_scratch(t["q"], t["kv"], t["indices"], w.scale, out64, lse64, nsplit=3)
    assert e.value.code == WORKSPACE
    assert api.device_error() == 0
