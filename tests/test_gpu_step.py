"""The fused decode step (one cooperative launch per step) against the CPU
oracle, on the cases that reach its own code paths: a selection concentrated
in a few CTAs' ranges that the balanced slices of the ordered selection
spread over all CTAs, exact score ties resolved by block index (candidate
lists in shared memory and, past their room, the fallback scan of the keys),
top-k 0 and top-k >= M in one launch, and back-to-back calls that must leave
the workspace clean (histogram and barriers) and give identical results.

Bars as in test_gpu_parity: block sets exact (up to fp32 near-ties of the
k-th score), outputs within 2e-3 absolute, log-sum-exp within 1e-3.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_resa_b200 import inputs
from block_sparse_long_resa_b200 import resa as R
from block_sparse_long_resa_b200.cache import LayerCache, workspace
from oracle import oracle as O

from test_gpu_parity import (LSE_ATOL, OUT_ATOL, assert_no_device_error, bits_of,
                             check_block_sets, oracle_of, setup_layer)

pytestmark = pytest.mark.gpu


def run_step(p, lc, cfg, ws, dev, topk, max_topk, L):
    B, Hq, Hkv, d = p.batch, p.num_q_heads, p.num_kv_heads, p.head_dim
    lc.seq_len.copy_(L.to(dev))
    out = torch.empty(B, Hq, d, device=dev)
    lse = torch.empty(B, Hq, device=dev)
    idx = torch.full((B, Hkv, max_topk + 1), -1, dtype=torch.int32, device=dev)
    cnt = torch.zeros(B, Hkv, dtype=torch.int32, device=dev)
    R.resa_decode_step(cfg, lc.struct(), p.q.to(dev), p.k_new.to(dev), p.v_new.to(dev),
                       topk.to(dev), max_topk, out, lse, idx, cnt, ws)
    return out, lse, idx, cnt


def test_fused_path_is_taken(cuda_device):
    cfg = R.make_config(28, 4, 128, 16)
    assert R.resa_decode_step_launches(cfg, 1, 16400, 16400) == 1     # 256K layer
    assert R.resa_decode_step_launches(cfg, 4, 4100, 16400) == 1      # batch 4 x 64K
    assert R.resa_decode_step_launches(cfg, 32, 8200, 140000) == 3    # 128 units: three launches
    assert R.resa_decode_step_launches(R.make_config(64, 4, 128, 16), 1, 2048, 2048) == 3  # g 16
    assert R.resa_decode_step_launches(R.make_config(4, 2, 64, 16), 1, 132, 132) == 1


def test_concentrated_selection_moves_blocks_between_ctas(cuda_device):
    """Blocks 0..299 of the sequence get keys pushed along the pooled query,
    so the top 205 all lie in the first CTAs' ranges: the contiguous slices of
    the ordered selection hand them to every CTA of the unit."""
    p = inputs.make_decode_problem(61, 1, 28, 4, 128, 16, [32768], needles=0)
    hq, hkv, g = 28, 4, 7
    qbar = p.q.float().view(1, hkv, g, 128).mean(2)[0]          # [Hkv][d]
    u = qbar / qbar.norm(dim=-1, keepdim=True)
    for blk in range(300):
        page = int(p.page_table[0, blk])
        p.k_cache[page] = (p.k_cache[page].float() + 3.0 * u[:, None, :]).to(torch.bfloat16)
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    k = int(p.topk[0])
    assert k == 205
    out, lse, idx, cnt = run_step(p, lc, cfg, ws, cuda_device, p.topk, k, L)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    r = o.decode_step(p.q, p.k_new, p.v_new, p.topk, L, k)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    assert (gidx[0, :, :k] < 300).all()
    same = check_block_sets(gidx, gcnt, r["block_idx"], r["block_cnt"], r["scores"], p.topk, L, 16)
    ref, ref_lse = (r["out"], r["lse"]) if same else o.sparse_attention(p.q, gidx, gcnt, L)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


@pytest.mark.parametrize("outlier", [0.0, 60.0, 300.0],
                         ids=["zero-blocks", "top-outlier-2-octaves", "top-outlier-4-octaves"])
def test_wide_score_range(cuda_device, outlier):
    """Blocks of all-zero keys score 0, thousands of histogram bins below the
    rest (the first window still holds the boundary).  A block pushed along
    the pooled query puts the unit's top digit about two octaves (the window
    below it holds the boundary) or four octaves (more than a window: the
    chunked read of the whole touched range) above the bulk."""
    p = inputs.make_decode_problem(71, 1, 28, 4, 128, 16, [65536], needles=0)
    for blk in (3, 500, 2047, 3000):
        p.k_cache[int(p.page_table[0, blk])] = 0
    if outlier:
        qbar = p.q.float().view(1, 4, 7, 128).mean(2)[0]
        u = qbar / qbar.norm(dim=-1, keepdim=True)
        page = int(p.page_table[0, 1234])
        p.k_cache[page] = (p.k_cache[page].float() + outlier * u[:, None, :]).to(torch.bfloat16)
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    k = int(p.topk[0])
    out, lse, idx, cnt = run_step(p, lc, cfg, ws, cuda_device, p.topk, k, L)
    assert_no_device_error(ws)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    r = o.decode_step(p.q, p.k_new, p.v_new, p.topk, L, k)
    gidx, gcnt = idx.cpu().numpy(), cnt.cpu().numpy()
    same = check_block_sets(gidx, gcnt, r["block_idx"], r["block_cnt"], r["scores"], p.topk, L, 16)
    ref, ref_lse = (r["out"], r["lse"]) if same else o.sparse_attention(p.q, gidx, gcnt, L)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)
    if outlier:
        assert (gidx[0, :, :k] == 1234).any(axis=1).all()


@pytest.mark.parametrize("ctx,topk,max_topk,d", [
    ([333, 257, 1999], [5, 0, 10**6], 80, 64),  # candidate lists in shared memory
    ([65536], [300], 300, 64),                   # 4096 tied candidates
    ([131072], [500], 500, 128),                 # 8192 tied candidates: past the lists' room
], ids=["small", "4096-tied", "8192-tied"])
def test_exact_ties_go_to_lower_block_ids(cuda_device, ctx, topk, max_topk, d):
    """All keys equal: every score ties, so the lowest block ids win; top-k 0
    keeps the current block only; top-k above max_topk is clamped and
    reported."""
    B = len(ctx)
    p = inputs.make_decode_problem(9, B, 8, 1, d, 16, ctx, paged=True, needles=0,
                                   topk=[1] * B)
    p.k_cache[:] = 0.5
    p.k_new[:] = 0.5
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    tk = torch.tensor(topk, dtype=torch.int32)
    out, lse, idx, cnt = run_step(p, lc, cfg, ws, cuda_device, tk, max_topk, L)
    code = R.resa_check_device_status(ws, raise_on_error=False)
    M = [(int(x) - 1) // 16 for x in L]
    expect_err = any(t > max_topk and m > max_topk for t, m in zip(topk, M))
    assert code == (R.DEVERR_TOPK if expect_err else 0)
    idx, cnt = idx.cpu(), cnt.cpu()
    want = []
    for b in range(B):
        kk = min(min(topk[b], max_topk), M[b])
        want.append(list(range(kk)) + [M[b]])
        assert idx[b, 0, :cnt[b, 0]].tolist() == want[b], b
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    o.append(p.k_new, p.v_new, L)
    ref, ref_lse = o.sparse_attention(p.q, idx.numpy(), cnt.numpy(), L)
    np.testing.assert_allclose(out.cpu().numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.cpu().numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


def test_mixed_modes_and_repeat_calls_are_identical(cuda_device):
    """One launch with top-k 0, top-k = M and ordinary top-k, called three
    times on the same state: the append is idempotent, the histogram and the
    unit counters must be left clean (and the generation advanced), and the
    results repeat bit for bit."""
    p = inputs.make_decode_problem(12, 4, 28, 4, 128, 16, [4000, 700, 16, 12000], paged=True,
                                   topk=[0, 10**5, 3, 300])
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    max_topk = 1000
    outs = []
    for _ in range(3):
        out, lse, idx, cnt = run_step(p, lc, cfg, ws, cuda_device, p.topk, max_topk, L)
        assert_no_device_error(ws)
        outs.append((out.cpu(), lse.cpu(), idx.cpu(), cnt.cpu()))
    for o2 in outs[1:]:
        for a, b in zip(outs[0], o2):
            assert torch.equal(a, b)
    o = oracle_of(p)
    o.build_descriptors(p.ctx_len)
    r = o.decode_step(p.q, p.k_new, p.v_new, p.topk, L, max_topk)
    np.testing.assert_array_equal(bits_of(lc.desc), o.desc)
    out, lse, idx, cnt = outs[0]
    gidx, gcnt = idx.numpy(), cnt.numpy()
    same = check_block_sets(gidx, gcnt, r["block_idx"], r["block_cnt"], r["scores"], p.topk, L, 16)
    ref, ref_lse = (r["out"], r["lse"]) if same else o.sparse_attention(p.q, gidx, gcnt, L)
    np.testing.assert_allclose(out.numpy(), ref, rtol=0, atol=OUT_ATOL)
    np.testing.assert_allclose(lse.numpy(), ref_lse, rtol=0, atol=LSE_ATOL)


def test_fused_and_three_launch_paths_agree(cuda_device):
    """The same step through resa_decode_step (fused) and through
    resa_append_token + resa_select_blocks + resa_sparse_decode."""
    p = inputs.make_decode_problem(13, 2, 28, 4, 128, 16, [20000, 9000], paged=True)
    cfg, lc, ws = setup_layer(p, cuda_device)
    L = p.ctx_len + 1
    max_topk = int(p.topk.max())
    out, lse, idx, cnt = run_step(p, lc, cfg, ws, cuda_device, p.topk, max_topk, L)
    assert_no_device_error(ws)
    p2 = inputs.make_decode_problem(13, 2, 28, 4, 128, 16, [20000, 9000], paged=True)
    cfg2, lc2, ws2 = setup_layer(p2, cuda_device)
    lc2.seq_len.copy_(L.to(cuda_device))
    dev = lambda t: t.to(cuda_device)
    R.resa_append_token(cfg2, lc2.struct(), dev(p2.k_new), dev(p2.v_new), ws2)
    idx2 = torch.full_like(idx, -1)
    cnt2 = torch.zeros_like(cnt)
    R.resa_select_blocks(cfg2, lc2.struct(), dev(p2.q), dev(p2.topk), max_topk, idx2, cnt2, None,
                         ws2)
    out2 = torch.empty_like(out)
    lse2 = torch.empty_like(lse)
    R.resa_sparse_decode(cfg2, lc2.struct(), dev(p2.q), idx2, cnt2, max_topk, out2, lse2, ws2)
    assert_no_device_error(ws2)
    assert torch.equal(lc.k, lc2.k) and torch.equal(lc.v, lc2.v) and torch.equal(lc.desc, lc2.desc)
    assert torch.equal(cnt, cnt2)
    for b in range(2):
        for h in range(4):
            n = int(cnt[b, h])
            assert idx[b, h, :n].tolist() == idx2[b, h, :n].tolist()
    torch.testing.assert_close(out, out2, rtol=0, atol=1e-5)
    torch.testing.assert_close(lse, lse2, rtol=0, atol=1e-5)
