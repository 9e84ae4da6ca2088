"""resa_sparse_decode_noalloc against resa_sparse_decode and the CPU oracle.

The no-allocation variant serves callers that may not allocate device memory
(hosts that hand the library only input and output pointers, with all HBM
already owned by their own pools), so it keeps its scratch in a fixed device
array inside the library instead of a caller workspace.  This file is named to
be collected last: it must pass on its own in a fresh process and after every
other test.
"""
import numpy as np
import pytest
import torch

from block_sparse_long_resa_b200 import inputs
from block_sparse_long_resa_b200 import resa as R
from block_sparse_long_resa_b200.cache import LayerCache, workspace
from oracle import oracle as O

pytestmark = pytest.mark.gpu

OUT_ATOL = 2e-3   # the parity tolerance used for attention outputs
LSE_ATOL = 1e-3


def _select(p, dev):
    cfg = R.make_config(p.num_q_heads, p.num_kv_heads, p.head_dim, p.block_size)
    lc = LayerCache.from_problem(p, dev)
    ws = workspace(cfg, lc.batch, lc.max_pages, 0, dev)
    R.resa_build_descriptors(cfg, lc.struct(), None, ws)
    lc.seq_len.copy_((p.ctx_len + 1).to(dev))
    R.resa_append_token(cfg, lc.struct(), p.k_new.to(dev), p.v_new.to(dev), ws)
    max_topk = int(p.topk.max())
    idx = torch.empty(p.batch, p.num_kv_heads, max_topk + 1, dtype=torch.int32, device=dev)
    cnt = torch.empty(p.batch, p.num_kv_heads, dtype=torch.int32, device=dev)
    R.resa_select_blocks(cfg, lc.struct(), p.q.to(dev), p.topk.to(dev), max_topk, idx, cnt, None,
                         ws)
    return cfg, lc, ws, idx, cnt, max_topk


def _oracle_out(p, lc, idx, cnt):
    """The oracle's group block-sparse attention over the same cache and block lists."""
    o = O.OracleCache(lc.k, lc.v, lc.page_table, p.num_q_heads, p.num_kv_heads, p.head_dim,
                      p.block_size)
    return o.sparse_attention(p.q, idx, cnt, lc.seq_len)


@pytest.mark.parametrize("case", [
    dict(seed=2, B=1, hq=28, hkv=4, d=128, ctx=[32768], topk=None, paged=False),
    dict(seed=3, B=5, hq=28, hkv=4, d=128, ctx=[1, 15, 16, 300, 5003], topk=[4, 16, 16, 7, 500],
         paged=True),
    dict(seed=4, B=3, hq=8, hkv=1, d=64, ctx=[33, 257, 1111], topk=[100, 3, 60], paged=True),
    dict(seed=6, B=3, hq=28, hkv=4, d=128, ctx=[100, 2000, 7000], topk=[2, 20, 50], paged=True,
         bs=32),
], ids=["qwen32k", "ragged", "d64", "block32"])
def test_noalloc_matches_workspace_path_and_oracle_twice(case):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    p = inputs.make_decode_problem(case["seed"], case["B"], case["hq"], case["hkv"], case["d"],
                                   case.get("bs", 16), case["ctx"], paged=case["paged"],
                                   topk=case["topk"])
    cfg, lc, ws, idx, cnt, max_topk = _select(p, dev)
    q = p.q.to(dev)
    shape = (p.batch, p.num_q_heads, p.head_dim)
    ref = torch.empty(shape, device=dev)
    ref_lse = torch.empty(shape[:2], device=dev)
    R.resa_sparse_decode(cfg, lc.struct(), q, idx, cnt, max_topk, ref, ref_lse, ws)
    torch.cuda.synchronize()
    assert R.resa_check_device_status(ws, raise_on_error=False) == 0
    o_out, o_lse = _oracle_out(p, lc, idx, cnt)
    err = torch.zeros(4, dtype=torch.int32, device=dev)
    for _ in range(2):   # two calls in a row share (and must reset) the scratch array
        out = torch.full(shape, float("nan"), device=dev)
        lse = torch.full(shape[:2], float("nan"), device=dev)
        R.resa_sparse_decode_noalloc(cfg, lc.struct(), q, idx, cnt, max_topk, out, lse, err)
        torch.cuda.synchronize()
        assert int(err[0]) == 0
        np.testing.assert_allclose(out.cpu().numpy(), ref.cpu().numpy(), rtol=0, atol=OUT_ATOL)
        np.testing.assert_allclose(lse.cpu().numpy(), ref_lse.cpu().numpy(), rtol=0,
                                   atol=LSE_ATOL)
        np.testing.assert_allclose(out.cpu().numpy(), o_out, rtol=0, atol=OUT_ATOL)
        np.testing.assert_allclose(lse.cpu().numpy(), o_lse, rtol=0, atol=LSE_ATOL)


def test_noalloc_reports_device_errors_in_the_callers_word():
    """A block id outside the sequence is skipped and flagged; the flag lands in
    the caller's error word and stays there through a later clean call."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    p = inputs.make_decode_problem(5, 1, 8, 2, 64, 16, [300], topk=[4])
    cfg, lc, ws, idx, cnt, max_topk = _select(p, dev)
    bad = idx.clone()
    bad[0, 0, 0] = 10_000   # far beyond the sequence's 19 blocks
    out = torch.empty(1, 8, 64, device=dev)
    err = torch.zeros(4, dtype=torch.int32, device=dev)
    R.resa_sparse_decode_noalloc(cfg, lc.struct(), p.q.to(dev), bad, cnt, max_topk, out, None, err)
    R.resa_sparse_decode_noalloc(cfg, lc.struct(), p.q.to(dev), idx, cnt, max_topk, out, None, err)
    torch.cuda.synchronize()
    assert int(err[0]) & R.DEVERR_BLOCK


def _tiny_args(dev, batch, max_topk):
    cfg = R.make_config(28, 4, 128, 16)
    k = torch.zeros(8, 4, 16, 128, dtype=torch.bfloat16, device=dev)
    pt = torch.zeros(batch, 1, dtype=torch.int32, device=dev)
    sl = torch.ones(batch, dtype=torch.int32, device=dev)
    cache = R.make_cache(k, k, k, pt, sl)
    idx = torch.zeros(batch, 4, 2, dtype=torch.int32, device=dev)
    cnt = torch.ones(batch, 4, dtype=torch.int32, device=dev)
    q = torch.zeros(batch, 28, 128, dtype=torch.bfloat16, device=dev)
    out = torch.full((batch, 28, 128), 7.0, device=dev)
    return cfg, cache, q, idx, cnt, out


def test_noalloc_rejects_calls_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    err = torch.zeros(4, dtype=torch.int32, device=dev)
    cfg, cache, q, idx, cnt, out = _tiny_args(dev, 2048, 1)   # batch 2048 x Hkv 4 > 4096
    with pytest.raises(R.ResaError) as e:
        R.resa_sparse_decode_noalloc(cfg, cache, q, idx, cnt, 1, out, None, err)
    assert e.value.status == 2


def test_noalloc_rejects_topk_beyond_the_split_merge_and_launches_nothing():
    """max_topk + 1 > 1024 * 512 blocks needs more splits than the merge holds."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    err = torch.zeros(4, dtype=torch.int32, device=dev)
    cfg, cache, q, idx, cnt, out = _tiny_args(dev, 1, 1)
    for max_topk in (1024 * 512, 2**31 - 1):
        with pytest.raises(R.ResaError) as e:
            R.resa_sparse_decode_noalloc(cfg, cache, q, idx, cnt, max_topk, out, None, err)
        assert e.value.status == 3
    torch.cuda.synchronize()
    assert bool((out == 7.0).all()), "a rejected call must not launch"
    assert int(err[0]) == 0


def test_noalloc_requires_the_error_word():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    cfg, cache, q, idx, cnt, out = _tiny_args(dev, 1, 1)
    with pytest.raises(R.ResaError) as e:
        R.resa_sparse_decode_noalloc(cfg, cache, q, idx, cnt, 1, out, None, None)
    assert e.value.status == 1
