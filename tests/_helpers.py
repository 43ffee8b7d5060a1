"""Shared helpers for the GPU parity tests: move a workload to the device,
run the CUDA path through the binding, run the oracle, compare."""
from __future__ import annotations

import numpy as np
import torch

from oracle import sparse_mla_ref as ref
from sparse_mla_decode_05_b200 import inputs

OUT_ATOL = 2e-2      # bf16 out: max abs error vs the fp64 oracle
LSE_RTOL = 1e-3      # lse: |d| / max(|lse|, 1)


class Dev:
    """A workload's tensors on the GPU."""

    def __init__(self, w: inputs.Workload, device="cuda:0", kv_override=None):
        self.w = w
        self.q = w.q.to(device)
        self.kv = w.kv.to(device) if kv_override is None else kv_override
        self.indices = w.indices.to(device)
        self.kv_row_scale = None if w.kv_row_scale is None else w.kv_row_scale.to(device)
        self.page_table = None if w.page_table is None else w.page_table.to(device)

    def run(self, nsplit=0, **kw):
        from sparse_mla_decode_05_b200 import api
        return api.decode(self.q, self.kv, self.indices, self.w.scale, kv_row_scale=self.kv_row_scale,
                          page_table=self.page_table, page_size=self.w.page_size, nsplit=nsplit, **kw)


def oracle(w: inputs.Workload, seqs=None):
    return ref.sparse_mla_decode(
        w.np_q_bits(), w.np_kv(), w.indices.numpy(), w.scale, d_v=w.d_v, kv_format=w.kv_format,
        kv_row_scale=None if w.kv_row_scale is None else w.kv_row_scale.numpy(),
        page_table=None if w.page_table is None else w.page_table.numpy(), page_size=w.page_size,
        seqs=seqs)


def compare(out_gpu, lse_gpu, out_ref, lse_ref, seqs=None):
    """Returns (max abs out error, max lse rel error, max error in bf16 ulps)
    over the selected sequences."""
    o = out_gpu.float().cpu().numpy().astype(np.float64)
    l = lse_gpu.cpu().numpy().astype(np.float64)
    if seqs is not None:
        o, l, out_ref, lse_ref = o[seqs], l[seqs], out_ref[seqs], lse_ref[seqs]
    err = float(np.max(np.abs(o - out_ref))) if o.size else 0.0
    lerr = float(np.max(ref.lse_rel_err(l, lse_ref))) if l.size else 0.0
    # error in units of the bf16 ulp at |ref| (|ref| floored at 2^-6 so that
    # values near zero do not blow the unit up)
    mag = np.maximum(np.abs(out_ref), 2.0 ** -6)
    ulp = 2.0 ** (np.floor(np.log2(mag)) - 7)
    ulps = float(np.max(np.abs(o - out_ref) / ulp)) if o.size else 0.0
    return err, lerr, ulps


def assert_parity(out_gpu, lse_gpu, out_ref, lse_ref, seqs=None, tag=""):
    err, lerr, ulps = compare(out_gpu, lse_gpu, out_ref, lse_ref, seqs)
    assert np.all(np.isfinite(out_gpu.float().cpu().numpy())), f"{tag}: non-finite out"
    assert err <= OUT_ATOL, f"{tag}: out max abs err {err:.3e} > {OUT_ATOL}"
    assert lerr <= LSE_RTOL, f"{tag}: lse rel err {lerr:.3e} > {LSE_RTOL}"
    return err, lerr, ulps


def counting_workload(B, topk, rows_per_seq, *, fp8=False, paged=False, pad_frac=0.25, seed=0,
                      page_size=64):
    """Index-exactness workload: q = 0 (every valid entry weighs the same) and
    row r carries a single 1.0 at value dim r % 512.  Then out[b,h,d] * n_b is
    exactly the number of valid entries whose row is = d mod 512, which a
    brute-force bincount reproduces; any dropped, duplicated or misread row
    changes an integer.  Padding (-1) is placed at random positions."""
    rng = np.random.default_rng(seed)
    N = B * rows_per_seq
    pages_per_seq = rows_per_seq // page_size if paged else 0
    vals = np.zeros((N, 576), dtype=np.float32)
    vals[np.arange(N), np.arange(N) % 512] = 1.0
    q = torch.zeros((B, 64, 576), dtype=torch.bfloat16)
    if fp8:
        kv = torch.from_numpy(vals).to(torch.float8_e4m3fn).view(torch.uint8)
        scales = torch.from_numpy(rng.choice([0.5, 1.0, 2.0], size=N).astype(np.float32))
    else:
        kv = torch.from_numpy(vals).to(torch.bfloat16)
        scales = None
    idx = np.full((B, topk), -1, dtype=np.int64)
    page_table = None
    phys = np.full((B, topk), -1, dtype=np.int64)
    if paged:
        perm = rng.permutation(N // page_size).reshape(B, pages_per_seq)
        page_table = torch.from_numpy(perm.astype(np.int32))
    for b in range(B):
        n_valid = max(0, topk - int(round(pad_frac * topk)))
        n_valid = min(n_valid, rows_per_seq)
        pos = np.sort(rng.choice(topk, n_valid, replace=False))
        logical = rng.choice(rows_per_seq, n_valid, replace=False)
        if paged:
            idx[b, pos] = logical
            phys[b, pos] = perm[b, logical // page_size] * page_size + logical % page_size
        else:
            idx[b, pos] = logical + b * rows_per_seq
            phys[b, pos] = idx[b, pos]
    w = inputs.Workload(name="counting", q=q, kv=kv, indices=torch.from_numpy(idx.astype(np.int32)),
                        scale=0.0625, kv_row_scale=scales, page_table=page_table,
                        page_size=page_size if paged else 0)
    counts = np.zeros((B, 512), dtype=np.float64)
    weights = np.zeros((B, 512), dtype=np.float64)
    nval = np.zeros(B)
    for b in range(B):
        r = phys[b][phys[b] >= 0]
        nval[b] = r.size
        np.add.at(counts[b], r % 512, 1.0)
        sc = np.ones(r.size) if scales is None else scales.numpy()[r].astype(np.float64)
        np.add.at(weights[b], r % 512, sc)
    return w, weights, nval
