"""Staggered rectification inside one decode batch, through the row map of the
cache struct: at a step, the sequences in the decode phase of their ReSA
cycle run one resa_decode_step over their rows while the sequences whose
cycle ends rectify in one resa_rectify_attention over theirs, on the same
cache (ReSA summary §3.4.2-§3.4.3; per-request rectification in continuous
batching).  Compared with the oracle stepping the same rows through views of
one cache.

Bars as in test_gpu_parity: K/V and descriptors bit-exact, block sets exact
up to fp32 near-ties of the k-th score, outputs within 2e-3 absolute,
log-sum-exp within 1e-3.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_resa_b200 import inputs
from block_sparse_long_resa_b200 import resa as R

from test_gpu_parity import (LSE_ATOL, OUT_ATOL, assert_no_device_error, bits_of,
                             check_block_sets, make, oracle_of, setup_layer)

pytestmark = pytest.mark.gpu

HQ, HKV, D = 28, 4, 128


def i32(x, dev):
    return torch.as_tensor(np.asarray(x, dtype=np.int32)).to(dev)


def gpu_mixed_step(cfg, lc, ws, dev, dec, rect, f, q, kn, vn, topk, max_topk, qc, kc, vc):
    """One step: decode the rows in ``dec``, rectify the rows in ``rect``."""
    res = {}
    if dec:
        n = len(dec)
        out = torch.empty(n, HQ, D, device=dev)
        lse = torch.empty(n, HQ, device=dev)
        idx = torch.full((n, HKV, max_topk + 1), -1, dtype=torch.int32, device=dev)
        cnt = torch.zeros(n, HKV, dtype=torch.int32, device=dev)
        rows = i32(dec, dev)
        R.resa_decode_step(cfg, lc.struct(rows=rows), q.to(dev), kn.to(dev), vn.to(dev),
                           topk.to(dev), max_topk, out, lse, idx, cnt, ws)
        res["dec"] = (out, lse, idx, cnt)
    if rect:
        n = len(rect)
        rout = torch.empty(n, f, HQ, D, device=dev)
        rlse = torch.empty(n, f, HQ, device=dev)
        rows = i32(rect, dev)
        R.resa_rectify_attention(cfg, lc.struct(rows=rows), f, qc.to(dev), kc.to(dev),
                                 vc.to(dev), rout, rlse, ws)
        res["rect"] = (rout, rlse)
    torch.cuda.synchronize()
    return res


def check_decode(o, res, dec, q, kn, vn, topk, L, max_topk, bs=16):
    out, lse, idx, cnt = res["dec"]
    view = o.rows_view(dec)
    r = view.decode_step(q, kn, vn, topk, L, max_topk)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    same = check_block_sets(gidx, gcnt, r["block_idx"], r["block_cnt"], r["scores"], topk, L, bs)
    ref, ref_lse = (r["out"], r["lse"]) if same else view.sparse_attention(q, gidx, gcnt, L)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


def check_rect(o, res, rect, qc, kc, vc, L, f):
    rout, rlse = res["rect"]
    ref, ref_lse = o.rows_view(rect).rectify(qc, kc, vc, L, f)
    np.testing.assert_allclose(rout.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(rlse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


MIXED = dict(seed=21, batch=6, num_q_heads=HQ, num_kv_heads=HKV, head_dim=D, block_size=16,
             ctx_lens=[300, 5003, 64, 2049, 777, 40], topk=[7, 60, 4, 30, 16, 16], paged=True)
# 24 sequences: the decoding rows exceed the fused step's one-wave limit
WIDE = dict(seed=22, batch=24, num_q_heads=HQ, num_kv_heads=HKV, head_dim=D, block_size=16,
            ctx_lens=[97 + 131 * i for i in range(24)], topk=[5 + i for i in range(24)],
            paged=True)


MIXED64 = dict(MIXED, seed=26, block_size=64)


@pytest.mark.parametrize("case,dec,rect", [
    (MIXED, [0, 2, 4, 5], [1, 3]),
    (MIXED, [5, 1, 3], [4, 0, 2]),
    (WIDE, [i for i in range(24) if i % 6 != 2], [2, 8, 14, 20]),
    (MIXED64, [3, 0, 5], [2, 1, 4]),
], ids=["fused", "permuted", "three-launch", "block64"])
def test_mixed_phase_step(cuda_device, case, dec, rect):
    p = make(case)
    f = 32
    cfg, lc, ws = setup_layer(p, cuda_device, max_chunk=f)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L.to(cuda_device))
    max_topk = int(p.topk[dec].max())
    qc, kc, vc = inputs.make_rectify_chunk(23, len(rect), f, HQ, HKV, D)
    if len(dec) * HKV <= 74 and p.block_size == 16:
        assert R.resa_decode_step_launches(cfg, len(dec), lc.max_pages, lc.k.shape[0]) == 1
    else:
        assert R.resa_decode_step_launches(cfg, len(dec), lc.max_pages, lc.k.shape[0]) == 3
    res = gpu_mixed_step(cfg, lc, ws, cuda_device, dec, rect, f, p.q[dec], p.k_new[dec],
                         p.v_new[dec], p.topk[dec], max_topk, qc, kc, vc)
    assert_no_device_error(ws)

    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    check_decode(o, res, dec, p.q[dec], p.k_new[dec], p.v_new[dec], p.topk[dec], L[dec],
                 max_topk, p.block_size)
    check_rect(o, res, rect, qc, kc, vc, L[rect], f)
    np.testing.assert_array_equal(bits_of(lc.k), o.K)
    np.testing.assert_array_equal(bits_of(lc.v), o.V)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)


def test_staggered_cycles(cuda_device):
    """Four sequences whose cycles of f = 8 are offset by 2 steps: at every
    step one of them rectifies while the others decode, for two periods."""
    p = make(dict(seed=24, batch=4, num_q_heads=HQ, num_kv_heads=HKV, head_dim=D,
                  block_size=16, ctx_lens=[700, 1500, 333, 2600], topk=[8, 12, 16, 20],
                  paged=True))
    f, B, max_topk = 8, 4, 20
    phase = [0, 2, 4, 6]
    cfg, lc, ws = setup_layer(p, cuda_device, max_chunk=f)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    for t in range(2 * f):
        L = p.ctx_len + t + 1
        lc.seq_len.copy_(L.to(cuda_device))
        rect = [b for b in range(B) if (t + phase[b]) % f == f - 1]
        dec = [b for b in range(B) if b not in rect]
        q, kn, vn = inputs.make_step_tokens(45, t, len(dec), HQ, HKV, D, p.k_scale)
        qc, kc, vc = inputs.make_rectify_chunk(200 + t, len(rect), f, HQ, HKV, D)
        res = gpu_mixed_step(cfg, lc, ws, cuda_device, dec, rect, f, q, kn, vn, p.topk[dec],
                             max_topk, qc, kc, vc)
        check_decode(o, res, dec, q, kn, vn, p.topk[dec], L[dec], max_topk)
        if rect:
            check_rect(o, res, rect, qc, kc, vc, L[rect], f)
        np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    np.testing.assert_array_equal(bits_of(lc.k), o.K)
    np.testing.assert_array_equal(bits_of(lc.v), o.V)
    assert_no_device_error(ws)


def test_row_outside_table_is_reported(cuda_device):
    """A mapped row outside the table: the sequence is skipped and the error
    word says so; the other rows of the call are decoded."""
    p = make(MIXED)
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L.to(cuda_device))
    dec = [0, 2]
    rows = i32([0, 6], cuda_device)   # 6 is past the 6-row table
    out = torch.empty(2, HQ, D, device=cuda_device)
    idx = torch.full((2, HKV, 8), -1, dtype=torch.int32, device=cuda_device)
    cnt = torch.zeros(2, HKV, dtype=torch.int32, device=cuda_device)
    topk = p.topk[dec].to(cuda_device)
    R.resa_decode_step(cfg, lc.struct(rows=rows), p.q[dec].to(cuda_device),
                       p.k_new[dec].to(cuda_device), p.v_new[dec].to(cuda_device), topk, 7, out,
                       None, idx, cnt, ws)
    torch.cuda.synchronize()
    code = R.resa_check_device_status(ws, raise_on_error=False)
    assert code & R.DEVERR_ROW
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    r = o.rows_view([0]).decode_step(p.q[:1], p.k_new[:1], p.v_new[:1], p.topk[:1], L[:1], 7)
    gidx, gcnt = idx.cpu().numpy()[:1], cnt.cpu().numpy()[:1]
    same = check_block_sets(gidx, gcnt, r["block_idx"], r["block_cnt"], r["scores"],
                            p.topk[:1], L[:1], 16)
    ref = r["out"] if same else o.rows_view([0]).sparse_attention(p.q[:1], gidx, gcnt, L[:1])[0]
    np.testing.assert_allclose(out[:1].cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    # nothing was appended anywhere but row 0
    o2 = oracle_of(p)
    o2.build_descriptors(p.ctx_len)
    o2.rows_view([0]).append(p.k_new[:1], p.v_new[:1], L[:1])
    np.testing.assert_array_equal(bits_of(lc.k), o2.K)


def test_dense_decode_on_mapped_rows(cuda_device):
    """Dense decoding of a subset of the table's rows, in a permuted order."""
    p = make(MIXED)
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L.to(cuda_device))
    dec = [4, 1, 5]
    out = torch.empty(3, HQ, D, device=cuda_device)
    lse = torch.empty(3, HQ, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    rows = i32(dec, cuda_device)  # kept alive until the call has run
    R.resa_dense_decode(cfg, lc.struct(rows=rows), dev(p.q[dec]), dev(p.k_new[dec]),
                        dev(p.v_new[dec]), out, lse, ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    view = o.rows_view(dec)
    view.append(p.k_new[dec], p.v_new[dec], L[dec])
    ref, ref_lse = view.dense_attention(p.q[dec], L[dec])
    np.testing.assert_array_equal(bits_of(lc.k), o.K)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)
