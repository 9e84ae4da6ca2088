"""Pins of the CPU oracle against things other than itself.

Each oracle step is checked against a library routine (numpy min/max, sorts,
torch's scaled_dot_product_attention / logsumexp in fp64), a brute force on
tiny inputs, a closed form or an invariant the method guarantees, chosen so
that a dropped term, a wrong sign or index, or a transposed operand fails at
least one of them.
"""
import itertools
import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from block_sparse_long_resa_b200 import inputs
from oracle import oracle as O


def small_problem(seed=0, B=2, hq=4, hkv=2, d=16, bs=4, ctx=(37, 22), paged=True, needles=2,
                  topk=None):
    return inputs.make_decode_problem(seed, B, hq, hkv, d, bs, list(ctx), reserve_tokens=8,
                                      paged=paged, needles=needles,
                                      topk=topk if topk is not None else [3] * B, n_min=1)


def oracle_of(p):
    return O.OracleCache(p.k_cache, p.v_cache, p.page_table, p.num_q_heads, p.num_kv_heads,
                         p.head_dim, p.block_size)


# --------------------------------------------------------------------------- descriptors

@pytest.mark.parametrize("paged,bs,ctx", [(False, 4, (37, 22)), (True, 4, (37, 22)),
                                           (True, 32, (201, 64)), (False, 64, (150, 63))])
def test_descriptors_match_numpy_minmax(paged, bs, ctx):
    p = small_problem(paged=paged, bs=bs, ctx=ctx)
    c = oracle_of(p)
    c.build_descriptors(p.ctx_len)
    for b in range(p.batch):
        L = int(p.ctx_len[b])
        for h in range(p.num_kv_heads):
            k = c.keys(b, h, L)
            for blk in range((L + p.block_size - 1) // p.block_size):
                seg = k[blk * p.block_size: min(L, (blk + 1) * p.block_size)]
                page = c.page_table[b, blk]
                mn = O.bf16_bits_to_float(c.desc[page, h, 0])
                mx = O.bf16_bits_to_float(c.desc[page, h, 1])
                np.testing.assert_array_equal(mn, seg.min(axis=0))
                np.testing.assert_array_equal(mx, seg.max(axis=0))


def test_incremental_append_equals_rebuild():
    p = small_problem(ctx=(30, 13), paged=True)
    c = oracle_of(p)
    L0 = p.ctx_len.numpy().copy()
    c.build_descriptors(L0)
    for step in range(7):
        q, kn, vn = inputs.make_step_tokens(5, step, p.batch, p.num_q_heads, p.num_kv_heads,
                                            p.head_dim)
        L = L0 + step + 1
        c.append(kn, vn, L)
        # the new token sits at position L-1
        for b in range(p.batch):
            pos = int(L[b]) - 1
            page = c.page_table[b, pos // p.block_size]
            np.testing.assert_array_equal(c.K[page, :, pos % p.block_size], O.bits(kn)[b])
            np.testing.assert_array_equal(c.V[page, :, pos % p.block_size], O.bits(vn)[b])
    fresh = O.OracleCache(c.K, c.V, c.page_table, p.num_q_heads, p.num_kv_heads, p.head_dim,
                          p.block_size)
    fresh.build_descriptors(L0 + 7)
    for b in range(p.batch):
        for blk in range((int(L0[b]) + 7 + p.block_size - 1) // p.block_size):
            page = c.page_table[b, blk]
            np.testing.assert_array_equal(c.desc[page], fresh.desc[page])


def test_partial_block_descriptor_ignores_stale_slots():
    p = small_problem(ctx=(9, 9), paged=False)
    c = oracle_of(p)
    page = c.page_table[0, 2]
    c.K[page, :, 1:] = 0x7f00  # huge stale values beyond L=9 (slot 0 of block 2 is position 8)
    c.build_descriptors(p.ctx_len)
    k = c.keys(0, 0, 9)
    np.testing.assert_array_equal(O.bf16_bits_to_float(c.desc[page, 0, 1]), k[8])


# --------------------------------------------------------------------------- pooling / scores

def test_pooled_query_is_group_mean():
    p = small_problem()
    c = oracle_of(p)
    qbar = c.pooled_query(p.q)
    ref = p.q.double().view(p.batch, p.num_kv_heads, p.group, p.head_dim).mean(dim=2).numpy()
    np.testing.assert_allclose(qbar, ref, rtol=2e-7, atol=1e-7)
    # g = 1: the pooled query is the query itself, exactly
    c1 = O.OracleCache(p.k_cache, p.v_cache, p.page_table, 2, 2, p.head_dim, p.block_size)
    q1 = p.q[:, :2]
    np.testing.assert_array_equal(c1.pooled_query(q1), q1.float().numpy())


def test_score_equals_max_over_box_corners():
    """Eq. 4 is the maximum of q.k over the axis-aligned box [min, max]: brute
    force over all 2^d corners for d = 8."""
    p = small_problem(seed=3, d=8, bs=4, ctx=(41, 29), hq=6, hkv=2)
    c = oracle_of(p)
    L = p.ctx_len + 1
    c.append(p.k_new, p.v_new, L)
    qbar = c.pooled_query(p.q)
    sc = c.block_scores(qbar, L)
    corners = np.array(list(itertools.product((0, 1), repeat=8)), dtype=np.float64)
    for b in range(p.batch):
        M = (int(L[b]) - 1) // p.block_size
        assert np.all(np.isnan(sc[b, :, M:]))
        for h in range(p.num_kv_heads):
            for i in range(M):
                page = c.page_table[b, i]
                mn = O.bf16_bits_to_float(c.desc[page, h, 0]).astype(np.float64)
                mx = O.bf16_bits_to_float(c.desc[page, h, 1]).astype(np.float64)
                pts = mn[None] + corners * (mx - mn)[None]
                brute = (pts @ qbar[b, h].astype(np.float64)).max()
                assert sc[b, h, i] == pytest.approx(brute, rel=1e-6, abs=1e-6)


def test_score_bounds_every_key_and_is_tight_for_constant_blocks():
    p = small_problem(seed=4, d=32, bs=8, ctx=(120, 77))
    c = oracle_of(p)
    L = p.ctx_len + 1
    c.append(p.k_new, p.v_new, L)
    # make block 1 of sequence 0 constant: its box is a point, the bound is exact
    page = c.page_table[0, 1]
    c.K[page, :, :] = c.K[page, :, :1]
    c.build_descriptors(L)
    qbar = c.pooled_query(p.q)
    sc = c.block_scores(qbar, L)
    for b in range(p.batch):
        M = (int(L[b]) - 1) // p.block_size
        for h in range(p.num_kv_heads):
            k = c.keys(b, h, int(L[b])).astype(np.float64)
            dots = k @ qbar[b, h].astype(np.float64)
            slack = 1e-5 * (np.abs(k) @ np.abs(qbar[b, h].astype(np.float64)))
            for i in range(M):
                seg = slice(i * p.block_size, (i + 1) * p.block_size)
                assert np.all(sc[b, h, i] >= dots[seg] - slack[seg])
    for h in range(p.num_kv_heads):
        k = c.keys(0, h, 16)[8].astype(np.float64)
        assert sc[0, h, 1] == pytest.approx(k @ qbar[0, h].astype(np.float64), rel=1e-6, abs=1e-6)


def test_score_ranking_scale_invariant_sign_sensitive():
    """Scaling q by a positive constant scales every score; flipping q swaps the
    roles of min and max (score(-q) = -(q . min-or-max chosen the other way))."""
    p = small_problem(seed=6, d=16, bs=4, ctx=(64, 64))
    c = oracle_of(p)
    L = p.ctx_len + 1
    c.append(p.k_new, p.v_new, L)
    qbar = c.pooled_query(p.q)
    s1 = c.block_scores(qbar, L)
    s2 = c.block_scores(qbar * 2.0, L)   # power of two: exact in fp32
    np.testing.assert_array_equal(s2, 2.0 * s1)
    s3 = c.block_scores(-qbar, L)
    for b in range(p.batch):
        M = (int(L[b]) - 1) // p.block_size
        for h in range(p.num_kv_heads):
            for i in range(M):
                page = c.page_table[b, i]
                mn = O.bf16_bits_to_float(c.desc[page, h, 0]).astype(np.float64)
                mx = O.bf16_bits_to_float(c.desc[page, h, 1]).astype(np.float64)
                qn = -qbar[b, h].astype(np.float64)
                assert s3[b, h, i] == pytest.approx(np.maximum(qn * mn, qn * mx).sum(), rel=1e-5, abs=1e-5)


# --------------------------------------------------------------------------- selection

@pytest.mark.parametrize("bs,ctx,topk", [(4, (200, 150), [9, 40]), (32, (2000, 700), [7, 30])])
def test_select_matches_lexsort(bs, ctx, topk):
    p = small_problem(seed=7, d=16, bs=bs, ctx=ctx, topk=topk)
    c = oracle_of(p)
    L = p.ctx_len + 1
    c.append(p.k_new, p.v_new, L)
    sc = c.block_scores(c.pooled_query(p.q), L)
    max_topk = 64
    idx, cnt = c.select(sc, p.topk, L, max_topk)
    for b in range(p.batch):
        M = (int(L[b]) - 1) // p.block_size
        k = min(int(p.topk[b]), M)
        for h in range(p.num_kv_heads):
            s = sc[b, h, :M]
            order = np.lexsort((np.arange(M), -s.astype(np.float64)))
            want = sorted(order[:k].tolist()) + [M]
            assert cnt[b, h] == k + 1
            assert idx[b, h, :k + 1].tolist() == want


def test_select_tie_breaks_to_lower_index_and_edges():
    B, hkv, max_pages, bs = 1, 1, 12, 16
    c = O.OracleCache(np.zeros((max_pages, hkv, bs, 4), np.uint16),
                      np.zeros((max_pages, hkv, bs, 4), np.uint16),
                      np.arange(max_pages, dtype=np.int32)[None], 1, 1, 4, bs)
    sc = np.full((B, hkv, max_pages), np.nan, np.float32)
    # 10 complete blocks (L = 10*16 + 1); scores with exact ties
    vals = [1.0, 3.0, 2.0, 3.0, 3.0, 0.5, 2.0, 3.0, -1.0, 2.0]
    sc[0, 0, :10] = vals
    L = [10 * bs + 1]
    idx, cnt = c.select(sc, [3], L, 8)
    assert idx[0, 0, :cnt[0, 0]].tolist() == [1, 3, 4, 10]    # 3.0 ties: blocks 1,3,4 beat 7
    idx, cnt = c.select(sc, [5], L, 8)
    assert idx[0, 0, :cnt[0, 0]].tolist() == [1, 2, 3, 4, 7, 10]  # 2.0 ties: 2 beats 6, 9
    idx, cnt = c.select(sc, [0], L, 8)
    assert idx[0, 0, :cnt[0, 0]].tolist() == [10]
    idx, cnt = c.select(sc, [100], L, 100)                      # k >= M: every block
    assert idx[0, 0, :cnt[0, 0]].tolist() == list(range(11))
    # L = 1: no complete block; the current block 0 only
    idx, cnt = c.select(sc, [4], [1], 8)
    assert idx[0, 0, :cnt[0, 0]].tolist() == [0]
    # L = 16: position 15 completes block 0, which is the current block
    idx, cnt = c.select(sc, [4], [16], 8)
    assert idx[0, 0, :cnt[0, 0]].tolist() == [0]
    # L = 17: block 0 complete, block 1 current
    idx, cnt = c.select(sc, [4], [17], 8)
    assert idx[0, 0, :cnt[0, 0]].tolist() == [0, 1]


# --------------------------------------------------------------------------- attention

def sdpa_ref(q, k, v, scale, mask=None, causal=False):
    """torch scaled_dot_product_attention in fp64; q [H][n][d], k/v [H][L][d]."""
    return F.scaled_dot_product_attention(q.double(), k.double(), v.double(), attn_mask=mask,
                                          is_causal=causal, scale=scale)


def test_all_blocks_selected_equals_dense_sdpa():
    p = small_problem(seed=8, d=32, bs=8, ctx=(90, 47), hq=6, hkv=2)
    c = oracle_of(p)
    L = p.ctx_len + 1
    r = c.decode_step(p.q, p.k_new, p.v_new, [10**6] * p.batch, L, 64)
    dense, dlse = c.dense_attention(p.q, L)
    np.testing.assert_allclose(r["out"], dense, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["lse"], dlse, rtol=0, atol=1e-12)
    scale = float(np.float32(1.0 / math.sqrt(p.head_dim)))
    for b in range(p.batch):
        Lb = int(L[b])
        for qh in range(p.num_q_heads):
            h = qh // p.group
            k = torch.from_numpy(c.keys(b, h, Lb))[None]
            v = torch.from_numpy(c.values(b, h, Lb))[None]
            q = p.q[b, qh].float()[None, None]
            ref = sdpa_ref(q, k, v, scale)[0, 0].numpy()
            np.testing.assert_allclose(r["out"][b, qh], ref, rtol=0, atol=1e-10)
            lse = torch.logsumexp(scale * (k[0].double() @ q[0, 0].double()), dim=0).item()
            assert r["lse"][b, qh] == pytest.approx(lse, abs=1e-10)


@pytest.mark.parametrize("bs,ctx,topk", [(8, (130, 61), [4, 2]), (64, (700, 200), [3, 1])])
def test_sparse_equals_masked_sdpa_and_weights_sum_to_one(bs, ctx, topk):
    p = small_problem(seed=9, d=32, bs=bs, ctx=ctx, hq=4, hkv=2, topk=topk)
    c = oracle_of(p)
    L = p.ctx_len + 1
    r = c.decode_step(p.q, p.k_new, p.v_new, p.topk, L, 8)
    scale = float(np.float32(1.0 / math.sqrt(p.head_dim)))
    for b in range(p.batch):
        Lb = int(L[b])
        for h in range(p.num_kv_heads):
            blocks = r["block_idx"][b, h, :r["block_cnt"][b, h]]
            allowed = np.zeros(Lb, dtype=bool)
            for blk in blocks:
                allowed[blk * p.block_size: min(Lb, (blk + 1) * p.block_size)] = True
            k = torch.from_numpy(c.keys(b, h, Lb))[None]
            v = torch.from_numpy(c.values(b, h, Lb))[None]
            for j in range(p.group):
                qh = h * p.group + j
                q = p.q[b, qh].float()[None, None]
                ref = sdpa_ref(q, k, v, scale, mask=torch.from_numpy(allowed)[None, None])[0, 0]
                np.testing.assert_allclose(r["out"][b, qh], ref.numpy(), rtol=0, atol=1e-10)
    # V = 1 everywhere: the output is the sum of the softmax weights
    c.V[:] = 0x3f80  # bf16 1.0
    out, _ = c.sparse_attention(p.q, r["block_idx"], r["block_cnt"], L)
    np.testing.assert_allclose(out, 1.0, rtol=0, atol=1e-12)


def test_single_token_attention_returns_its_value():
    p = small_problem(seed=10, d=16, bs=4, ctx=(8, 8))
    c = oracle_of(p)
    L = np.array([9, 9], dtype=np.int32)   # position 8 is the only token of block 2
    c.append(p.k_new, p.v_new, L)
    idx = np.array([[[2], [2]], [[2], [2]]], dtype=np.int32)
    cnt = np.ones((2, 2), np.int32)
    out, lse = c.sparse_attention(p.q, idx, cnt, L)
    vn = O.bf16_bits_to_float(O.bits(p.v_new)).astype(np.float64)
    for b in range(2):
        for qh in range(p.num_q_heads):
            np.testing.assert_array_equal(out[b, qh], vn[b, qh // p.group])


def test_needle_blocks_are_selected():
    p = inputs.make_decode_problem(11, 1, 4, 2, 64, 16, [2048], needles=4, topk=[16])
    c = oracle_of(p)
    L = p.ctx_len + 1
    c.build_descriptors(p.ctx_len)
    r = c.decode_step(p.q, p.k_new, p.v_new, p.topk, L, 16)
    for h in range(2):
        sel = set(r["block_idx"][0, h, :r["block_cnt"][0, h]].tolist())
        assert set(p.needle_blocks[0, h].tolist()) <= sel


# --------------------------------------------------------------------------- rectification

def test_rectify_whole_sequence_is_causal_sdpa():
    """f = L: the chunk is the whole sequence, so rectification is causal
    self-attention over it."""
    B, hq, hkv, d, bs, L = 1, 4, 2, 16, 4, 23
    p = inputs.make_decode_problem(12, B, hq, hkv, d, bs, [L], reserve_tokens=0, needles=0,
                                   topk=[1])
    c = oracle_of(p)
    qc, kc, vc = inputs.make_rectify_chunk(12, B, L, hq, hkv, d)
    out, lse = c.rectify(qc, kc, vc, [L], L)
    scale = float(np.float32(1.0 / math.sqrt(d)))
    for qh in range(hq):
        h = qh // (hq // hkv)
        q = qc[0, :, qh].float()[None]
        k = kc[0, :, h].float()[None]
        v = vc[0, :, h].float()[None]
        ref = sdpa_ref(q, k, v, scale, causal=True)[0].numpy()
        np.testing.assert_allclose(out[0, :, qh], ref, rtol=0, atol=1e-10)
    fresh = oracle_of(p)
    fresh.K, fresh.V = c.K.copy(), c.V.copy()
    fresh.build_descriptors([L])
    np.testing.assert_array_equal(c.desc, fresh.desc)


@pytest.mark.parametrize("bs", [8, 32])
def test_rectify_chunk_rows_against_dense_and_refresh(bs):
    p = small_problem(seed=13, d=32, bs=bs, ctx=(100, 71), hq=6, hkv=2)
    c = oracle_of(p)
    c.build_descriptors(p.ctx_len)
    f = 12
    L = p.ctx_len.numpy() + 3           # three decode tokens appended since the last one
    for s in range(3):
        _, kn, vn = inputs.make_step_tokens(13, s, p.batch, 6, 2, 32)
        c.append(kn, vn, p.ctx_len.numpy() + s + 1)
    qc, kc, vc = inputs.make_rectify_chunk(13, p.batch, f, 6, 2, 32)
    out, lse = c.rectify(qc, kc, vc, L, f)
    # every row r equals dense decode attention over positions 0..L-f+r of the updated cache
    for r in range(f):
        Lr = L - f + r + 1
        d_out, d_lse = c.dense_attention(qc[:, r], Lr)
        np.testing.assert_allclose(out[:, r], d_out, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse[:, r], d_lse, rtol=0, atol=1e-12)
    # the chunk's K/V were written
    for b in range(p.batch):
        k = c.keys(b, 1, int(L[b]))
        np.testing.assert_array_equal(k[-f:], kc[b, :, 1].float().numpy())
    # descriptors equal a rebuild from scratch
    fresh = O.OracleCache(c.K, c.V, c.page_table, 6, 2, 32, bs)
    fresh.build_descriptors(L)
    for b in range(p.batch):
        for blk in range((int(L[b]) + bs - 1) // bs):
            page = c.page_table[b, blk]
            np.testing.assert_array_equal(c.desc[page], fresh.desc[page])


def test_decode_step_with_all_blocks_equals_last_rectify_row():
    p = small_problem(seed=14, d=32, bs=8, ctx=(95, 95), hq=4, hkv=2)
    f = 5
    L = p.ctx_len.numpy() + 1
    qc, kc, vc = inputs.make_rectify_chunk(14, p.batch, f, 4, 2, 32)
    a = oracle_of(p)
    a.build_descriptors(p.ctx_len)
    out_r, _ = a.rectify(qc, kc, vc, L, f)
    b_ = oracle_of(p)
    b_.build_descriptors(p.ctx_len)
    # same cache contents for positions < L-1, then the decode token = last chunk token
    for b in range(p.batch):
        for r in range(f - 1):
            pos = int(L[b]) - f + r
            page = b_.page_table[b, pos // 8]
            b_.K[page, :, pos % 8] = O.bits(kc[b, r])
            b_.V[page, :, pos % 8] = O.bits(vc[b, r])
    b_.build_descriptors(L - 1)
    r = b_.decode_step(qc[:, f - 1], kc[:, f - 1], vc[:, f - 1], [10**6] * p.batch, L, 64)
    np.testing.assert_allclose(r["out"], out_r[:, f - 1], rtol=0, atol=1e-12)


def test_rectify_rows_equals_rectify_and_skips_short_sequences():
    p = small_problem(seed=15, d=32, bs=8, ctx=(90, 20), hq=4, hkv=2)
    f = 24
    qc, kc, vc = inputs.make_rectify_chunk(15, p.batch, f, 4, 2, 32)
    a = oracle_of(p)
    a.build_descriptors(p.ctx_len)
    out, lse = a.rectify(qc, kc, vc, p.ctx_len, f)
    b_ = oracle_of(p)
    b_.build_descriptors(p.ctx_len)
    res = b_.rectify_rows(qc, kc, vc, p.ctx_len, f, [0, 7, 23])
    np.testing.assert_array_equal(a.K, b_.K)
    np.testing.assert_array_equal(a.desc, b_.desc)
    for r, (o_r, l_r) in res.items():
        np.testing.assert_allclose(o_r[0], out[0, r], rtol=0, atol=1e-12)
        np.testing.assert_allclose(l_r[0], lse[0, r], rtol=0, atol=1e-12)
    # sequence 1 (L = 20 < f) is left untouched by both
    fresh = oracle_of(p)
    for blk in range(3):
        page = fresh.page_table[1, blk]
        np.testing.assert_array_equal(a.K[page], fresh.K[page])


def test_rows_view_mixed_step_equals_batch_wide_steps():
    """A call over mapped rows (some sequences decode while others rectify)
    gives each sequence what a batch-wide call gives it: sequences are
    independent, so the view only changes which cache row a call reads."""
    p = small_problem(seed=16, B=4, d=16, bs=4, ctx=(37, 22, 50, 41), topk=[3, 2, 4, 3])
    f, max_topk = 8, 4
    L = p.ctx_len + 1
    q, kn, vn = p.q, p.k_new, p.v_new
    qc, kc, vc = inputs.make_rectify_chunk(16, 4, f, 4, 2, 16)
    dec, rect = [2, 0], [3, 1]

    a = oracle_of(p)
    a.build_descriptors(p.ctx_len)
    r = a.rows_view(dec).decode_step(q[dec], kn[dec], vn[dec], p.topk[dec], L[dec], max_topk)
    ro, rl = a.rows_view(rect).rectify(qc[rect], kc[rect], vc[rect], L[rect], f)

    b_ = oracle_of(p)
    b_.build_descriptors(p.ctx_len)
    rb = b_.decode_step(q, kn, vn, p.topk, L, max_topk)
    c_ = oracle_of(p)
    c_.build_descriptors(p.ctx_len)
    co, cl = c_.rectify(qc, kc, vc, L, f)

    np.testing.assert_array_equal(r["block_idx"], rb["block_idx"][dec])
    np.testing.assert_array_equal(r["out"], rb["out"][dec])
    np.testing.assert_array_equal(r["lse"], rb["lse"][dec])
    np.testing.assert_array_equal(ro, co[rect])
    np.testing.assert_array_equal(rl, cl[rect])
    for rows, ref in ((dec, b_), (rect, c_)):
        for row in rows:
            pages = a.page_table[row][a.page_table[row] >= 0]
            pages = pages[: (int(L[row]) + 3) // 4]
            np.testing.assert_array_equal(a.K[pages], ref.K[pages])
            np.testing.assert_array_equal(a.V[pages], ref.V[pages])
            np.testing.assert_array_equal(a.desc[pages], ref.desc[pages])
