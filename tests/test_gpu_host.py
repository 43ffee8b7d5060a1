"""sparse_mla_decode_host: the decode step with q, indices and page table
read from host memory and out / lse written back to host memory, the cache
staying on the device.

The copies are plain transfers, so the results must equal sparse_mla_decode's
bit for bit (same kernels, same plan), for every cache layout and merge
kind; two plans on two streams in flight at once must not disturb each
other.
"""
import pytest
import torch

from sparse_mla_decode_05_b200 import inputs

from _helpers import Dev

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


CASES = {
    "flat_varlen_planned": (lambda: inputs.flat_varlen(16, 256, 8192, 512, seed=301), 0),
    "flat_single_split": (lambda: inputs.flat_per_seq(2, 2048, 700, seed=302), 1),
    "flat_combine_3": (lambda: inputs.flat_per_seq(2, 2048, 700, seed=303), 3),
    "paged_fp8_planned": (lambda: inputs.paged_fp8(3, 1024, 64, 300, seed=304), 0),
    "dsv4_planned": (lambda: inputs.paged_dsv4(4, 1024, 96, 333, seed=305), 0),
}


def _host_plan(w, d, nsplit, pinned=True):
    a = api()
    pin = (lambda t: t.pin_memory()) if pinned else (lambda t: t.clone())
    return a.HostDecodePlan(pin(w.q), d.kv, pin(w.indices), w.scale, kv_row_scale=d.kv_row_scale,
                            page_table_host=None if w.page_table is None else pin(w.page_table),
                            page_size=w.page_size, nsplit=nsplit)


@pytest.mark.parametrize("case", sorted(CASES))
@pytest.mark.parametrize("pinned", [True, False])
def test_host_call_equals_device_call(case, pinned):
    make, nsplit = CASES[case]
    w = make()
    d = Dev(w)
    want_o, want_l = d.run(nsplit=nsplit)
    plan = _host_plan(w, d, nsplit, pinned)
    plan.out_host.fill_(float("nan"))
    plan.lse_host.fill_(float("nan"))
    plan.run()
    torch.cuda.synchronize()
    assert torch.equal(plan.out_host.view(torch.int16), want_o.cpu().view(torch.int16))
    assert torch.equal(plan.lse_host.view(torch.int32), want_l.cpu().view(torch.int32))


def test_two_streams_in_flight():
    """Two batches, each with its own plan and staging, alternating on two
    streams for several rounds with no synchronisation in between."""
    ws = [inputs.flat_varlen(16, 256, 8192, 512, seed=311), inputs.paged_fp8(8, 1024, 128, 900, seed=312)]
    devs = [Dev(w) for w in ws]
    wants = [d.run() for d in devs]
    torch.cuda.synchronize()
    plans = [_host_plan(w, d, 0) for w, d in zip(ws, devs)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for _ in range(6):
        for p, s in zip(plans, streams):
            p.run(s)
    torch.cuda.synchronize()
    for p, (o, l) in zip(plans, wants):
        assert torch.equal(p.out_host.view(torch.int16), o.cpu().view(torch.int16))
        assert torch.equal(p.lse_host.view(torch.int32), l.cpu().view(torch.int32))


def test_decode_host_convenience_call():
    w = inputs.flat_per_seq(3, 1000, 200, seed=321)
    d = Dev(w)
    want_o, want_l = d.run()
    o, l = api().decode_host(w.q.pin_memory(), d.kv, w.indices.pin_memory(), w.scale)
    assert torch.equal(o.view(torch.int16), want_o.cpu().view(torch.int16))
    assert torch.equal(l.view(torch.int32), want_l.cpu().view(torch.int32))


def test_short_staging_rejected():
    w = inputs.flat_per_seq(2, 1000, 200, seed=322)
    d = Dev(w)
    a = api()
    shape = a.shape_for(w.q, d.kv, w.indices)
    small = torch.empty(a.host_staging_size(shape) - 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(a.SmlaError) as e:
        a.HostDecodePlan(w.q.pin_memory(), d.kv, w.indices.pin_memory(), w.scale, staging=small).run()
    assert e.value.code == 3
