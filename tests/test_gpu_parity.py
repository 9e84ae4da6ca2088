"""CUDA path (through the C ABI) against the CPU oracle on the same seeded inputs.

Bars: descriptors, written K/V and block sets bit-exact (block sets may differ
only on blocks whose oracle fp32 score is within 1e-6 relative of the k-th
score); attention outputs within 2e-3 absolute (bf16 K/V, fp32 accumulation);
log-sum-exp within 1e-3.
"""
import math

import numpy as np
import pytest
import torch

from block_sparse_long_resa_b200 import inputs
from block_sparse_long_resa_b200 import resa as R
from block_sparse_long_resa_b200.cache import LayerCache, workspace
from oracle import oracle as O

pytestmark = pytest.mark.gpu

OUT_ATOL = 2e-3
LSE_ATOL = 1e-3
TIE_REL = 1e-6


def oracle_of(p, desc=None):
    return O.OracleCache(p.k_cache, p.v_cache, p.page_table, p.num_q_heads, p.num_kv_heads,
                         p.head_dim, p.block_size, desc=desc)


def cfg_of(p):
    return R.make_config(p.num_q_heads, p.num_kv_heads, p.head_dim, p.block_size)


def setup_layer(p, dev, max_chunk=64):
    cfg = cfg_of(p)
    lc = LayerCache.from_problem(p, dev)
    ws = workspace(cfg, lc.batch, lc.max_pages, max_chunk, dev)
    R.resa_build_descriptors(cfg, lc.struct(), None, ws)
    return cfg, lc, ws


def assert_no_device_error(ws):
    torch.cuda.synchronize()
    assert R.resa_check_device_status(ws, raise_on_error=False) == 0


def bits_of(t):
    return O.bits(t)


def check_block_sets(gidx, gcnt, oidx, ocnt, oscores, topk, L, bs):
    """Returns True when the sets are identical; asserts differences are near-ties."""
    same = True
    B, H = ocnt.shape
    for b in range(B):
        M = (int(L[b]) - 1) // bs
        k = min(int(topk[b]), M)
        for h in range(H):
            assert int(gcnt[b, h]) == int(ocnt[b, h]) == k + 1
            g = gidx[b, h, :k + 1].tolist()
            o = oidx[b, h, :k + 1].tolist()
            assert g[-1] == o[-1] == M
            assert g[:-1] == sorted(set(g[:-1])), "GPU list must be ascending and unique"
            diff = set(g[:-1]) ^ set(o[:-1])
            if diff:
                same = False
                s = oscores[b, h, :M].astype(np.float64)
                sk = np.sort(s)[::-1][k - 1]
                for i in diff:
                    assert abs(s[i] - sk) <= TIE_REL * abs(sk), (b, h, i, s[i], sk)
    return same


# --------------------------------------------------------------------------- cases

TINY = dict(seed=1, batch=1, num_q_heads=4, num_kv_heads=2, head_dim=64, block_size=16,
            ctx_lens=[2048], topk=[16])
QWEN32K = dict(seed=2, batch=1, num_q_heads=28, num_kv_heads=4, head_dim=128, block_size=16,
               ctx_lens=[32768])  # top-k = 10% = 205
RAGGED = dict(seed=3, batch=5, num_q_heads=28, num_kv_heads=4, head_dim=128, block_size=16,
              ctx_lens=[1, 15, 16, 300, 5003], topk=[4, 16, 16, 7, 500], paged=True)
RAGGED64 = dict(seed=4, batch=3, num_q_heads=8, num_kv_heads=1, head_dim=64, block_size=16,
                ctx_lens=[33, 257, 1111], topk=[100, 3, 60], paged=True)
GQA8 = dict(seed=5, batch=2, num_q_heads=32, num_kv_heads=8, head_dim=128, block_size=16,
            ctx_lens=[20000, 7777], topk=[125, 48], paged=True)  # 8 kv heads: 16 KB stages


def make(case, device="cpu", **over):
    kw = dict(case)
    kw.update(over)
    seed = kw.pop("seed")
    B = kw.pop("batch")
    return inputs.make_decode_problem(seed, B, kw.pop("num_q_heads"), kw.pop("num_kv_heads"),
                                      kw.pop("head_dim"), kw.pop("block_size"),
                                      kw.pop("ctx_lens"), device=device, **kw)


@pytest.mark.parametrize("case", [TINY, QWEN32K, RAGGED, RAGGED64], ids=["tiny", "qwen32k",
                                                                         "ragged", "ragged64"])
def test_build_descriptors_bit_exact(cuda_device, case):
    p = make(case)
    cfg, lc, ws = setup_layer(p, cuda_device)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)


def test_build_descriptors_from_first_block(cuda_device):
    p = make(RAGGED)
    cfg, lc, ws = setup_layer(p, cuda_device)
    lc.desc.zero_()
    first = torch.tensor([0, 0, 1, 7, 300], dtype=torch.int32)
    R.resa_build_descriptors(cfg, lc.struct(), first.to(cuda_device), ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len, first)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)


@pytest.mark.parametrize("case", [TINY, QWEN32K, RAGGED, RAGGED64, GQA8],
                         ids=["tiny", "qwen32k", "ragged", "ragged64", "gqa8"])
def test_decode_step_matches_oracle(cuda_device, case):
    p = make(case)
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L.to(cuda_device))
    max_topk = int(p.topk.max())
    B, Hq, Hkv, d = p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim
    out = torch.empty(B, Hq, d, dtype=torch.float32, device=cuda_device)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=cuda_device)
    idx = torch.full((B, Hkv, max_topk + 1), -1, dtype=torch.int32, device=cuda_device)
    cnt = torch.zeros(B, Hkv, dtype=torch.int32, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    R.resa_decode_step(cfg, lc.struct(), dev(p.q), dev(p.k_new), dev(p.v_new), dev(p.topk),
                       max_topk, out, lse, idx, cnt, ws)
    assert_no_device_error(ws)

    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    r = o.decode_step(p.q, p.k_new, p.v_new, p.topk, L, max_topk)
    # append: K, V and descriptors bit-exact
    np.testing.assert_array_equal(bits_of(lc.k), o.K)
    np.testing.assert_array_equal(bits_of(lc.v), o.V)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    same = check_block_sets(gidx, gcnt, r["block_idx"], r["block_cnt"], r["scores"], p.topk, L,
                            p.block_size)
    ref_out, ref_lse = (r["out"], r["lse"]) if same else o.sparse_attention(p.q, gidx, gcnt, L)
    np.testing.assert_allclose(out.cpu().numpy(), ref_out, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)
    # the needles are found
    for b in range(B):
        M = (int(L[b]) - 1) // p.block_size
        if M - 1 >= 4 and int(p.topk[b]) >= 16:
            for h in range(Hkv):
                sel = set(gidx[b, h, :gcnt[b, h]].tolist())
                assert set(p.needle_blocks[b, h].tolist()) <= sel


@pytest.mark.parametrize("case", [TINY, QWEN32K, RAGGED, GQA8],
                         ids=["tiny", "qwen32k", "ragged", "gqa8"])
def test_select_blocks_scores(cuda_device, case):
    p = make(case)
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L.to(cuda_device))
    R.resa_append_token(cfg, lc.struct(), p.k_new.to(cuda_device), p.v_new.to(cuda_device), ws)
    max_topk = int(p.topk.max())
    B, Hkv = p.batch, p.num_kv_heads
    idx = torch.full((B, Hkv, max_topk + 1), -1, dtype=torch.int32, device=cuda_device)
    cnt = torch.zeros(B, Hkv, dtype=torch.int32, device=cuda_device)
    scores = torch.full((B, Hkv, lc.max_pages), float("nan"), device=cuda_device)
    R.resa_select_blocks(cfg, lc.struct(), p.q.to(cuda_device), p.topk.to(cuda_device), max_topk,
                         idx, cnt, scores, ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    o.append(p.k_new, p.v_new, L)
    sc = o.block_scores(o.pooled_query(p.q), L)
    oidx, ocnt = o.select(sc, p.topk, L, max_topk)
    gs = scores.cpu().numpy()
    for b in range(B):
        M = (int(L[b]) - 1) // p.block_size
        np.testing.assert_allclose(gs[b, :, :M], sc[b, :, :M], rtol=2e-6, atol=2e-6)
    check_block_sets(idx.cpu().numpy(), cnt.cpu().numpy(), oidx, ocnt, sc, p.topk, L,
                     p.block_size)


def test_select_exact_ties_and_edges(cuda_device):
    """All keys equal: every score ties, the lowest indices win."""
    p = make(RAGGED64, seed=9, ctx_lens=[333, 257, 1999])
    p.k_cache[:] = 0.5
    cfg, lc, ws = setup_layer(p, cuda_device)
    lc.seq_len.copy_((p.ctx_len + 1).to(cuda_device))
    topk = torch.tensor([5, 0, 10**6], dtype=torch.int32)
    max_topk = 80
    idx = torch.full((3, 1, max_topk + 1), -1, dtype=torch.int32, device=cuda_device)
    cnt = torch.zeros(3, 1, dtype=torch.int32, device=cuda_device)
    R.resa_select_blocks(cfg, lc.struct(), p.q.to(cuda_device), topk.to(cuda_device), max_topk,
                         idx, cnt, None, ws)
    code = R.resa_check_device_status(ws, raise_on_error=False)
    assert code == R.DEVERR_TOPK       # sequence 2 asks for more than max_topk
    idx, cnt = idx.cpu(), cnt.cpu()
    L = (p.ctx_len + 1).tolist()
    M = [(x - 1) // 16 for x in L]
    assert idx[0, 0, :cnt[0, 0]].tolist() == [0, 1, 2, 3, 4, M[0]]
    assert idx[1, 0, :cnt[1, 0]].tolist() == [M[1]]
    assert idx[2, 0, :cnt[2, 0]].tolist() == list(range(max_topk)) + [M[2]]


def test_sparse_decode_given_blocks(cuda_device):
    """Attention over caller-chosen blocks, including a partial current block
    and a block id outside the sequence (skipped, error bit set)."""
    p = make(QWEN32K, ctx_lens=[32768 + 5])
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len.clone()
    M = (int(L[0]) - 1) // 16
    rng = np.random.default_rng(5)
    blocks = np.sort(rng.choice(M, size=300, replace=False)).astype(np.int32)
    idx = np.full((1, 4, 302), -1, dtype=np.int32)
    cnt = np.full((1, 4), 301, dtype=np.int32)
    for h in range(4):
        idx[0, h, :300] = np.sort(rng.choice(M, size=300, replace=False))
        idx[0, h, 300] = M
    out = torch.empty(1, 28, 128, device=cuda_device)
    lse = torch.empty(1, 28, device=cuda_device)
    R.resa_sparse_decode(cfg, lc.struct(), p.q.to(cuda_device), torch.from_numpy(idx).to(cuda_device),
                         torch.from_numpy(cnt).to(cuda_device), 301, out, lse, ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    ref, ref_lse = o.sparse_attention(p.q, idx, cnt, L)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)
    # an out-of-range block id is skipped and reported
    idx[0, 0, 0] = M + 50
    R.resa_sparse_decode(cfg, lc.struct(), p.q.to(cuda_device), torch.from_numpy(idx).to(cuda_device),
                         torch.from_numpy(cnt).to(cuda_device), 301, out, lse, ws)
    code = R.resa_check_device_status(ws, raise_on_error=False)
    assert code & R.DEVERR_BLOCK


def test_sparse_decode_split_merge_beyond_one_wave(cuda_device):
    """38 sequences x 4 kv heads = 152 (sequence, head) units with 520+1 blocks
    each: two splits per unit (512-block cap) give 304 CTAs, more than one
    wave, so the splits are merged by the last CTA of each unit instead of
    across the grid."""
    p = make(dict(seed=9, batch=38, num_q_heads=8, num_kv_heads=4, head_dim=128,
                  block_size=16, ctx_lens=[8400] * 38, topk=[16] * 38))
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len.clone()
    B, Hkv = p.batch, p.num_kv_heads
    M = (int(L[0]) - 1) // 16
    rng = np.random.default_rng(11)
    n = 520
    idx = np.full((B, Hkv, n + 1), -1, dtype=np.int32)
    cnt = np.full((B, Hkv), n + 1, dtype=np.int32)
    for b in range(B):
        for h in range(Hkv):
            idx[b, h, :n] = np.sort(rng.choice(M, size=n, replace=False))
            idx[b, h, n] = M
    out = torch.empty(B, 8, 128, device=cuda_device)
    lse = torch.empty(B, 8, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    R.resa_sparse_decode(cfg, lc.struct(), dev(p.q), dev(torch.from_numpy(idx)),
                         dev(torch.from_numpy(cnt)), n, out, lse, ws)
    assert_no_device_error(ws)
    ref, ref_lse = oracle_of(p).sparse_attention(p.q, idx, cnt, L)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


def test_all_blocks_equals_dense(cuda_device):
    p = make(RAGGED)
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L.to(cuda_device))
    B = p.batch
    max_topk = int((L.max() - 1) // 16)
    topk = torch.full((B,), 10**6, dtype=torch.int32)
    out = torch.empty(B, 28, 128, device=cuda_device)
    idx = torch.empty(B, 4, max_topk + 1, dtype=torch.int32, device=cuda_device)
    cnt = torch.empty(B, 4, dtype=torch.int32, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    R.resa_decode_step(cfg, lc.struct(), dev(p.q), dev(p.k_new), dev(p.v_new), dev(topk),
                       max_topk, out, None, idx, cnt, ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.append(p.k_new, p.v_new, L)
    dense, _ = o.dense_attention(p.q, L)
    np.testing.assert_allclose(out.cpu().numpy(), dense, rtol=0, atol=OUT_ATOL)


@pytest.mark.parametrize("case", [TINY, QWEN32K, RAGGED, RAGGED64, GQA8],
                         ids=["tiny", "qwen32k", "ragged", "ragged64", "gqa8"])
def test_dense_decode_matches_oracle(cuda_device, case):
    """The dense baseline: append, then attention over every position."""
    p = make(case)
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L.to(cuda_device))
    B, Hq, d = p.batch, p.num_q_heads, p.head_dim
    out = torch.empty(B, Hq, d, dtype=torch.float32, device=cuda_device)
    lse = torch.empty(B, Hq, dtype=torch.float32, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    R.resa_dense_decode(cfg, lc.struct(), dev(p.q), dev(p.k_new), dev(p.v_new), out, lse, ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    o.append(p.k_new, p.v_new, L)
    np.testing.assert_array_equal(bits_of(lc.k), o.K)
    np.testing.assert_array_equal(bits_of(lc.v), o.V)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    ref, ref_lse = o.dense_attention(p.q, L)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


def test_dense_decode_long_single_sequence(cuda_device):
    """One unit over 100K positions: splits far beyond one wave of CTAs."""
    p = make(dict(seed=11, batch=1, num_q_heads=8, num_kv_heads=1, head_dim=128,
                  block_size=16, ctx_lens=[100003], paged=True))
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L.to(cuda_device))
    out = torch.empty(1, 8, 128, dtype=torch.float32, device=cuda_device)
    lse = torch.empty(1, 8, dtype=torch.float32, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    R.resa_dense_decode(cfg, lc.struct(), dev(p.q), dev(p.k_new), dev(p.v_new), out, lse, ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.append(p.k_new, p.v_new, L)
    ref, ref_lse = o.dense_attention(p.q, L)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


@pytest.mark.parametrize("shape,ctx,f,paged", [
    ((4, 2, 64), [2049], 32, True),
    ((28, 4, 128), [4096, 1000], 32, True),
    ((28, 4, 128), [777], 13, True),
    ((8, 1, 64), [40, 64, 300], 40, True),
    ((28, 4, 128), [4096, 1000], 32, False),
    ((4, 2, 64), [2049, 77], 32, False),
    ((28, 4, 128), [3000, 700], 64, True),
    ((4, 2, 64), [500, 37], 1, True),
], ids=["tiny", "qwen-aligned", "qwen-unaligned", "whole-seq", "qwen-contiguous",
        "tiny-contiguous", "qwen-two-row-groups", "one-row-chunk"])
def test_rectify_matches_oracle(cuda_device, shape, ctx, f, paged):
    """Random page order takes the per-block tensor loads; the contiguous
    layout takes the four-page loads wherever a tile's pages are consecutive
    (and the per-block ones on the ragged last tile)."""
    hq, hkv, d = shape
    p = inputs.make_decode_problem(20 + f, len(ctx), hq, hkv, d, 16, ctx, paged=paged,
                                   needles=0, topk=[1] * len(ctx))
    cfg, lc, ws = setup_layer(p, cuda_device, max_chunk=f)
    L = p.ctx_len.clone()
    qc, kc, vc = inputs.make_rectify_chunk(f, len(ctx), f, hq, hkv, d)
    B = len(ctx)
    out = torch.empty(B, f, hq, d, device=cuda_device)
    lse = torch.empty(B, f, hq, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    R.resa_rectify_attention(cfg, lc.struct(), f, dev(qc), dev(kc), dev(vc), out, lse, ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(L)
    ref, ref_lse = o.rectify(qc, kc, vc, L, f)
    np.testing.assert_array_equal(bits_of(lc.k), o.K)
    np.testing.assert_array_equal(bits_of(lc.v), o.V)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


def test_rectify_chunk_longer_than_sequence_is_reported(cuda_device):
    p = inputs.make_decode_problem(31, 2, 4, 2, 64, 16, [10, 100], needles=0, topk=[1, 1])
    cfg, lc, ws = setup_layer(p, cuda_device, max_chunk=32)
    qc, kc, vc = inputs.make_rectify_chunk(31, 2, 32, 4, 2, 64)
    out = torch.zeros(2, 32, 4, 64, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    R.resa_rectify_attention(cfg, lc.struct(), 32, dev(qc), dev(kc), dev(vc), out, None, ws)
    code = R.resa_check_device_status(ws, raise_on_error=False)
    assert code & R.DEVERR_CHUNK
    # the valid sequence was still rectified
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    res = o.rectify_rows(qc, kc, vc, p.ctx_len, 32, [0, 31])
    for r, (ref, _) in res.items():
        np.testing.assert_allclose(out[1, r].cpu().numpy(), ref[1], rtol=0, atol=OUT_ATOL)


def test_decode_loop_with_rectification(cuda_device):
    """A few ReSA cycles (f = 8): sparse decode steps appending tokens, then a
    rectification of the last f tokens; every step checked against the oracle."""
    p = make(QWEN32K, batch=2, ctx_lens=[3000, 1234], topk=[20, 16], paged=True, seed=44)
    cfg, lc, ws = setup_layer(p, cuda_device, max_chunk=8)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    f, B = 8, 2
    L = p.ctx_len.clone()
    dev = lambda t: t.to(cuda_device)
    out = torch.empty(B, 28, 128, device=cuda_device)
    idx = torch.empty(B, 4, 21, dtype=torch.int32, device=cuda_device)
    cnt = torch.empty(B, 4, dtype=torch.int32, device=cuda_device)
    for cycle in range(2):
        for s in range(f - 1):
            q, kn, vn = inputs.make_step_tokens(44, cycle * f + s, B, 28, 4, 128, p.k_scale)
            L = L + 1
            lc.seq_len.copy_(dev(L))
            R.resa_decode_step(cfg, lc.struct(), dev(q), dev(kn), dev(vn), dev(p.topk), 20, out,
                               None, idx, cnt, ws)
            r = o.decode_step(q, kn, vn, p.topk, L, 20)
            gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
            same = check_block_sets(gidx, gcnt, r["block_idx"], r["block_cnt"], r["scores"],
                                    p.topk, L, 16)
            ref = r["out"] if same else o.sparse_attention(q, gidx, gcnt, L)[0]
            np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
        L = L + 1
        lc.seq_len.copy_(dev(L))
        qc, kc, vc = inputs.make_rectify_chunk(100 + cycle, B, f, 28, 4, 128)
        rout = torch.empty(B, f, 28, 128, device=cuda_device)
        R.resa_rectify_attention(cfg, lc.struct(), f, dev(qc), dev(kc), dev(vc), rout, None, ws)
        ref, _ = o.rectify(qc, kc, vc, L, f)
        np.testing.assert_allclose(rout.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
        np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    assert_no_device_error(ws)


# --------------------------------------------------------------------------- full sizes

def test_full_size_256k_layer(cuda_device):
    """One layer of the 256K long-context decode workload (28 q / 4 kv heads,
    d 128, 262144-token cache, top-k 1638 + current block), in the launch
    configuration the benchmark times; the oracle computes every output."""
    p = inputs.make_decode_problem(7, 1, 28, 4, 128, 16, [262144], device=cuda_device)
    cfg = cfg_of(p)
    lc = LayerCache(k=p.k_cache, v=p.v_cache,
                    desc=torch.zeros(p.num_pages, 4, 2, 128, dtype=torch.bfloat16,
                                     device=cuda_device),
                    page_table=p.page_table, seq_len=p.ctx_len.clone())
    ws = workspace(cfg, 1, lc.max_pages, 32, cuda_device)
    R.resa_build_descriptors(cfg, lc.struct(), None, ws)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L)
    k = int(p.topk[0])
    assert k == 1638
    out = torch.empty(1, 28, 128, device=cuda_device)
    idx = torch.empty(1, 4, k + 1, dtype=torch.int32, device=cuda_device)
    cnt = torch.empty(1, 4, dtype=torch.int32, device=cuda_device)
    R.resa_decode_step(cfg, lc.struct(), p.q, p.k_new, p.v_new, p.topk, k, out, None, idx, cnt,
                       ws)
    assert_no_device_error(ws)
    cpu = lambda t: t.cpu()
    o = O.OracleCache(cpu(p.k_cache), cpu(p.v_cache), cpu(p.page_table), 28, 4, 128, 16)
    o.build_descriptors(cpu(p.ctx_len))
    r = o.decode_step(cpu(p.q), cpu(p.k_new), cpu(p.v_new), cpu(p.topk), cpu(L), k)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    same = check_block_sets(gidx, gcnt, r["block_idx"], r["block_cnt"], r["scores"],
                            cpu(p.topk), cpu(L), 16)
    ref = r["out"] if same else o.sparse_attention(cpu(p.q), gidx, gcnt, cpu(L))[0]
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)


def test_full_size_dense_decode_256k(cuda_device):
    """Dense decoding of one 256K layer (28 q / 4 kv heads, d 128) in the
    launch configuration of the bench's dense baseline; the oracle computes
    every output."""
    p = inputs.make_decode_problem(9, 1, 28, 4, 128, 16, [262144], device=cuda_device)
    cfg = cfg_of(p)
    lc = LayerCache(k=p.k_cache, v=p.v_cache,
                    desc=torch.zeros(p.num_pages, 4, 2, 128, dtype=torch.bfloat16,
                                     device=cuda_device),
                    page_table=p.page_table, seq_len=p.ctx_len.clone())
    ws = workspace(cfg, 1, lc.max_pages, 16, cuda_device)
    R.resa_build_descriptors(cfg, lc.struct(), None, ws)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L)
    out = torch.empty(1, 28, 128, device=cuda_device)
    lse = torch.empty(1, 28, device=cuda_device)
    R.resa_dense_decode(cfg, lc.struct(), p.q, p.k_new, p.v_new, out, lse, ws)
    assert_no_device_error(ws)
    cpu = lambda t: t.cpu()
    o = O.OracleCache(cpu(p.k_cache), cpu(p.v_cache), cpu(p.page_table), 28, 4, 128, 16)
    o.append(cpu(p.k_new), cpu(p.v_new), cpu(L))
    ref, ref_lse = o.dense_attention(cpu(p.q), cpu(L))
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


def test_rectification_beyond_one_wave(cuda_device):
    """A batch whose (sequence, kv head) units and key splits exceed one wave
    of CTAs (160 units, two splits for the longest sequences): each group's
    last split merges it.  Sampled rows against the oracle; every touched
    block's descriptor bit-exact; a second call reuses the reset tickets."""
    B, f = 40, 32
    ctx = [2000 + (i * 467) % 18000 for i in range(B)]
    p = inputs.make_decode_problem(12, B, 4, 4, 128, 16, ctx, paged=True)
    cfg, lc, ws = setup_layer(p, cuda_device, max_chunk=f)
    L = p.ctx_len
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    rows = [0, 13, 31]
    dev = lambda t: t.to(cuda_device)
    for call in range(2):
        qc, kc, vc = inputs.make_rectify_chunk(13 + call, B, f, 4, 4, 128)
        out = torch.empty(B, f, 4, 128, device=cuda_device)
        lse = torch.empty(B, f, 4, device=cuda_device)
        R.resa_rectify_attention(cfg, lc.struct(), f, dev(qc), dev(kc), dev(vc), out, lse, ws)
        assert_no_device_error(ws)
        res = o.rectify_rows(qc, kc, vc, L, f, rows)
        np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
        for r in rows:
            ref, ref_lse = res[r]
            np.testing.assert_allclose(out[:, r].cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
            np.testing.assert_allclose(lse[:, r].cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


def test_rectification_row_groups_beyond_one_wave(cuda_device):
    """Two 256-row groups a (sequence, kv head) (f = 64 chunk rows x 7 heads =
    448 rows) and two key splits (the longest sequence has more than 16384
    keys) over 48 units: 192 CTAs, more than one wave, so each group's last
    split merges it, group 1 included.  Sampled rows of both groups against
    the oracle; a second call reuses the reset tickets."""
    B, f, hq, hkv, d = 12, 64, 28, 4, 128
    ctx = [17000] + [500 + (i * 733) % 2500 for i in range(1, B)]
    p = inputs.make_decode_problem(14, B, hq, hkv, d, 16, ctx, paged=True, needles=0,
                                   topk=[1] * B)
    cfg, lc, ws = setup_layer(p, cuda_device, max_chunk=f)
    L = p.ctx_len
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    rows = [0, 36, 37, 63]  # rows 252-258 straddle the groups; 441-447 end group 1
    dev = lambda t: t.to(cuda_device)
    for call in range(2):
        qc, kc, vc = inputs.make_rectify_chunk(15 + call, B, f, hq, hkv, d)
        out = torch.empty(B, f, hq, d, device=cuda_device)
        lse = torch.empty(B, f, hq, device=cuda_device)
        R.resa_rectify_attention(cfg, lc.struct(), f, dev(qc), dev(kc), dev(vc), out, lse, ws)
        assert_no_device_error(ws)
        res = o.rectify_rows(qc, kc, vc, L, f, rows)
        np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
        for r in rows:
            ref, ref_lse = res[r]
            np.testing.assert_allclose(out[:, r].cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
            np.testing.assert_allclose(lse[:, r].cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


def test_full_size_rectification_sampled_rows(cuda_device):
    """Rectification at the decode-loop workload's size (batch 4, 65536-token
    cache, f = 32, 28 q / 4 kv heads): every output row computed, sampled rows
    compared with the oracle."""
    B, f = 4, 32
    p = inputs.make_decode_problem(8, B, 28, 4, 128, 16, [65536] * B, device=cuda_device)
    cfg = cfg_of(p)
    lc = LayerCache(k=p.k_cache, v=p.v_cache,
                    desc=torch.zeros(p.num_pages, 4, 2, 128, dtype=torch.bfloat16,
                                     device=cuda_device),
                    page_table=p.page_table, seq_len=p.ctx_len.clone())
    ws = workspace(cfg, B, lc.max_pages, f, cuda_device)
    R.resa_build_descriptors(cfg, lc.struct(), None, ws)
    kc0, vc0 = p.k_cache.cpu(), p.v_cache.cpu()
    qc, kc, vc = inputs.make_rectify_chunk(8, B, f, 28, 4, 128, device=cuda_device)
    out = torch.empty(B, f, 28, 128, device=cuda_device)
    R.resa_rectify_attention(cfg, lc.struct(), f, qc, kc, vc, out, None, ws)
    assert_no_device_error(ws)
    o = O.OracleCache(kc0, vc0, p.page_table.cpu(), 28, 4, 128, 16)
    o.build_descriptors(p.ctx_len.cpu())
    rows = [0, 13, 31]
    res = o.rectify_rows(qc.cpu(), kc.cpu(), vc.cpu(), p.ctx_len.cpu(), f, rows)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    for r in rows:
        np.testing.assert_allclose(out[:, r].cpu().numpy(), res[r][0], rtol=0, atol=OUT_ATOL)
    assert torch.isfinite(out).all()


def test_full_size_continuous_batching(cuda_device):
    """Continuous-batching workload: 32 sequences with lengths uniform in
    [8192, 131072], random physical page order, top-k 10% per sequence."""
    lens = inputs.continuous_batch_lengths(9, 32, 8192, 131072)
    p = inputs.make_decode_problem(9, 32, 28, 4, 128, 16, lens, paged=True, device=cuda_device,
                                   reserve_tokens=16)
    cfg = cfg_of(p)
    lc = LayerCache(k=p.k_cache, v=p.v_cache,
                    desc=torch.zeros(p.num_pages, 4, 2, 128, dtype=torch.bfloat16,
                                     device=cuda_device),
                    page_table=p.page_table, seq_len=p.ctx_len.clone())
    ws = workspace(cfg, 32, lc.max_pages, 0, cuda_device)
    R.resa_build_descriptors(cfg, lc.struct(), None, ws)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L)
    max_topk = int(p.topk.max())
    out = torch.empty(32, 28, 128, device=cuda_device)
    idx = torch.empty(32, 4, max_topk + 1, dtype=torch.int32, device=cuda_device)
    cnt = torch.empty(32, 4, dtype=torch.int32, device=cuda_device)
    R.resa_decode_step(cfg, lc.struct(), p.q, p.k_new, p.v_new, p.topk, max_topk, out, None, idx,
                       cnt, ws)
    assert_no_device_error(ws)
    cpu = lambda t: t.cpu()
    o = O.OracleCache(cpu(p.k_cache), cpu(p.v_cache), cpu(p.page_table), 28, 4, 128, 16)
    o.build_descriptors(cpu(p.ctx_len))
    r = o.decode_step(cpu(p.q), cpu(p.k_new), cpu(p.v_new), cpu(p.topk), cpu(L), max_topk)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    same = check_block_sets(gidx, gcnt, r["block_idx"], r["block_cnt"], r["scores"],
                            cpu(p.topk), cpu(L), 16)
    ref = r["out"] if same else o.sparse_attention(cpu(p.q), gidx, gcnt, cpu(L))[0]
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)


# --------------------------------------------------------------------------- value range
#
# Tolerance for values far from N(0, 1): the attention output is a convex
# combination of the values, and its rounding error scales with their size,
# so the 2e-3 bar (stated for N(0, 1) values) is applied relative to the
# largest |v| a head's rows attend to: |out - ref| <= 2e-3 * max|v|.

def _wide_values(p, kind, seed):
    """Replace the cache's values with wide-range ones, drawn along sequence
    positions of the contiguous layout; slots beyond the context stay zero."""
    v = p.v_cache
    P, H, T, D = v.shape
    tok = v.permute(1, 0, 2, 3).reshape(H, P * T, D)
    w = inputs.wide_range_values(seed, tok, kind, tokens_axis=1)
    w = w.reshape(H, P, T, D).permute(1, 0, 2, 3).contiguous()
    p.v_cache = torch.where(v != 0, w, torch.zeros_like(w))


def _row_tol(o, B, hkv, g, L_per_b):
    """[B][Hq] tolerance: 2e-3 * max|v| over the positions of the row's kv head."""
    tol = np.zeros((B, hkv * g))
    for b in range(B):
        for h in range(hkv):
            vmax = float(np.abs(o.values(b, h, int(L_per_b[b]))).max())
            tol[b, h * g:(h + 1) * g] = OUT_ATOL * vmax
    return tol


@pytest.mark.parametrize("kind", inputs.WIDE_KINDS)
def test_rectify_value_range(cuda_device, kind):
    """Values from 1e-6 to +-3.3e38, mixed within and across 64-key tiles:
    the fp16 staging of V is scaled per tile, so no finite bf16 value overflows
    and tiny ones keep their precision."""
    hq, hkv, d, f = 28, 4, 128, 32
    ctx = [1000, 4096]
    B = len(ctx)
    p = inputs.make_decode_problem(60, B, hq, hkv, d, 16, ctx, needles=0, topk=[1] * B)
    _wide_values(p, kind, 61)
    cfg, lc, ws = setup_layer(p, cuda_device, max_chunk=f)
    L = p.ctx_len.clone()
    qc, kc, vc = inputs.make_rectify_chunk(62, B, f, hq, hkv, d)
    vc = inputs.wide_range_values(63, vc, kind, tokens_axis=1)
    out = torch.empty(B, f, hq, d, device=cuda_device)
    lse = torch.empty(B, f, hq, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    R.resa_rectify_attention(cfg, lc.struct(), f, dev(qc), dev(kc), dev(vc), out, lse, ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(L)
    ref, ref_lse = o.rectify(qc, kc, vc, L, f)
    np.testing.assert_array_equal(bits_of(lc.v), o.V)
    got = out.cpu().numpy()
    assert np.isfinite(got).all()
    tol = _row_tol(o, B, hkv, hq // hkv, L)
    err = np.abs(got - ref).max(axis=-1)             # [B][f][Hq]
    assert (err <= tol[:, None, :]).all(), float((err / tol[:, None, :]).max())
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


@pytest.mark.parametrize("kind", ["large", "tiny", "tiles"])
def test_decode_step_value_range(cuda_device, kind):
    """The decode step's bf16 V and hi + lo P keep their precision from 1e-6 to
    1e5 (the decode paths' range is stated in include/resa.h)."""
    p = make(QWEN32K)
    _wide_values(p, kind, 71)
    if kind == "tiny":
        p.v_new = (p.v_new.float() * 1e-6).to(torch.bfloat16)
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    lc.seq_len.copy_(L.to(cuda_device))
    max_topk = int(p.topk.max())
    B, Hq, Hkv, d = p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim
    out = torch.empty(B, Hq, d, dtype=torch.float32, device=cuda_device)
    idx = torch.full((B, Hkv, max_topk + 1), -1, dtype=torch.int32, device=cuda_device)
    cnt = torch.zeros(B, Hkv, dtype=torch.int32, device=cuda_device)
    dev = lambda t: t.to(cuda_device)
    R.resa_decode_step(cfg, lc.struct(), dev(p.q), dev(p.k_new), dev(p.v_new), dev(p.topk),
                       max_topk, out, None, idx, cnt, ws)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    o.append(p.k_new, p.v_new, L)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    ref, _ = o.sparse_attention(p.q, gidx, gcnt, L)
    tol = _row_tol(o, B, Hkv, Hq // Hkv, L)
    err = np.abs(out.cpu().numpy() - ref).max(axis=-1)
    assert (err <= tol).all(), float((err / tol).max())
