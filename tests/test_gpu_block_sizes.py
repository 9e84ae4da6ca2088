"""Blocks of 32 and 64 tokens (ReSA summary §3.4.3, Eq. 6: the block size b is
one of the three knobs of the memory model).  Every entry point runs with
b = 32 and b = 64 against the oracle at the same block size: descriptors
bit-exact, block sets exact up to fp32 near-ties, outputs within 2e-3, as in
test_gpu_parity.  The decode step takes the three-launch path there (the
fused step is built for 16-token blocks).
"""
import numpy as np
import pytest
import torch

from block_sparse_long_resa_b200 import inputs
from block_sparse_long_resa_b200 import resa as R

from test_gpu_parity import (LSE_ATOL, OUT_ATOL, assert_no_device_error, bits_of,
                             check_block_sets, make, oracle_of, setup_layer)

pytestmark = pytest.mark.gpu

BS = [32, 64]


def case(bs, paged=True):
    # lengths around block edges: 1 token, one block exactly, one more, long
    return dict(seed=30 + bs, batch=5, num_q_heads=28, num_kv_heads=4, head_dim=128,
                block_size=bs, ctx_lens=[1, bs - 1, bs, 777, 9001],
                topk=[4, 16, 16, 5, 40], paged=paged)


def case64d(bs):
    return dict(seed=40 + bs, batch=3, num_q_heads=8, num_kv_heads=1, head_dim=64,
                block_size=bs, ctx_lens=[2 * bs + 1, 700, 3000], topk=[100, 3, 20], paged=True)


@pytest.mark.parametrize("bs", BS)
def test_build_descriptors(cuda_device, bs):
    p = make(case(bs))
    cfg, lc, ws = setup_layer(p, cuda_device)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)


@pytest.mark.parametrize("bs", BS)
@pytest.mark.parametrize("d64", [False, True], ids=["d128", "d64"])
def test_decode_step(cuda_device, bs, d64):
    p = make(case64d(bs) if d64 else case(bs))
    cfg, lc, ws = setup_layer(p, cuda_device)
    assert R.resa_decode_step_launches(cfg, p.batch, lc.max_pages, lc.k.shape[0]) == 3
    L = p.ctx_len + 1
    lc.seq_len.copy_(L.to(cuda_device))
    max_topk = int(p.topk.max())
    B, Hq, Hkv, d = p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim
    out = torch.empty(B, Hq, d, device=cuda_device)
    lse = torch.empty(B, Hq, device=cuda_device)
    idx = torch.full((B, Hkv, max_topk + 1), -1, dtype=torch.int32, device=cuda_device)
    cnt = torch.zeros(B, Hkv, dtype=torch.int32, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    R.resa_decode_step(cfg, lc.struct(), dev(p.q), dev(p.k_new), dev(p.v_new), dev(p.topk),
                       max_topk, out, lse, idx, cnt, ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    r = o.decode_step(p.q, p.k_new, p.v_new, p.topk, L, max_topk)
    np.testing.assert_array_equal(bits_of(lc.k), o.K)
    np.testing.assert_array_equal(bits_of(lc.v), o.V)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    same = check_block_sets(gidx, gcnt, r["block_idx"], r["block_cnt"], r["scores"], p.topk, L,
                            bs)
    ref, ref_lse = (r["out"], r["lse"]) if same else o.sparse_attention(p.q, gidx, gcnt, L)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


@pytest.mark.parametrize("bs", BS)
def test_dense_decode(cuda_device, bs):
    p = make(case(bs))
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L.to(cuda_device))
    out = torch.empty(p.batch, 28, 128, device=cuda_device)
    lse = torch.empty(p.batch, 28, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    R.resa_dense_decode(cfg, lc.struct(), dev(p.q), dev(p.k_new), dev(p.v_new), out, lse, ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    o.append(p.k_new, p.v_new, L)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    ref, ref_lse = o.dense_attention(p.q, L)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


@pytest.mark.parametrize("bs", BS)
@pytest.mark.parametrize("shape,ctx,f,paged", [
    ((28, 4, 128), [4096, 1000], 32, True),
    ((28, 4, 128), [777], 13, False),
    ((8, 1, 64), [70, 300], 40, True),
])
def test_rectify(cuda_device, bs, shape, ctx, f, paged):
    hq, hkv, d = shape
    p = inputs.make_decode_problem(50 + bs, len(ctx), hq, hkv, d, bs, ctx, paged=paged)
    cfg, lc, ws = setup_layer(p, cuda_device, max_chunk=f)
    L = p.ctx_len
    qc, kc, vc = inputs.make_rectify_chunk(51, len(ctx), f, hq, hkv, d)
    out = torch.empty(len(ctx), f, hq, d, device=cuda_device)
    lse = torch.empty(len(ctx), f, hq, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    R.resa_rectify_attention(cfg, lc.struct(), f, dev(qc), dev(kc), dev(vc), out, lse, ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    ref, ref_lse = o.rectify(qc, kc, vc, L, f)
    np.testing.assert_array_equal(bits_of(lc.k), o.K)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


@pytest.mark.parametrize("bs", BS)
def test_decode_loop_with_rectification(cuda_device, bs):
    """Decode steps that fill blocks and start new ones, then a rectification
    whose chunk straddles a block edge, twice."""
    p = make(dict(seed=60 + bs, batch=2, num_q_heads=28, num_kv_heads=4, head_dim=128,
                  block_size=bs, ctx_lens=[1000, 2 * bs - 3], topk=[6, 2], paged=True))
    f, B = 8, 2
    cfg, lc, ws = setup_layer(p, cuda_device, max_chunk=f)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    L = p.ctx_len.clone()
    dev = lambda t: t.to(cuda_device)
    out = torch.empty(B, 28, 128, device=cuda_device)
    idx = torch.empty(B, 4, 9, dtype=torch.int32, device=cuda_device)
    cnt = torch.empty(B, 4, dtype=torch.int32, device=cuda_device)
    for cycle in range(2):
        for s in range(f - 1):
            q, kn, vn = inputs.make_step_tokens(61, cycle * f + s, B, 28, 4, 128, p.k_scale)
            L = L + 1
            lc.seq_len.copy_(dev(L))
            R.resa_decode_step(cfg, lc.struct(), dev(q), dev(kn), dev(vn), dev(p.topk), 8, out,
                               None, idx, cnt, ws)
            r = o.decode_step(q, kn, vn, p.topk, L, 8)
            gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
            same = check_block_sets(gidx, gcnt, r["block_idx"], r["block_cnt"], r["scores"],
                                    p.topk, L, bs)
            ref = r["out"] if same else o.sparse_attention(q, gidx, gcnt, L)[0]
            np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
        L = L + 1
        lc.seq_len.copy_(dev(L))
        qc, kc, vc = inputs.make_rectify_chunk(62 + cycle, B, f, 28, 4, 128)
        rout = torch.empty(B, f, 28, 128, device=cuda_device)
        R.resa_rectify_attention(cfg, lc.struct(), f, dev(qc), dev(kc), dev(vc), rout, None, ws)
        ref, _ = o.rectify(qc, kc, vc, L, f)
        np.testing.assert_allclose(rout.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
        np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    np.testing.assert_array_equal(bits_of(lc.k), o.K)
    assert_no_device_error(ws)
