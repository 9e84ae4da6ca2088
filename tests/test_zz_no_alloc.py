"""resa_sparse_decode_noalloc against resa_sparse_decode.

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


@pytest.mark.parametrize("case", [
    dict(seed=2, B=1, hq=28, hkv=4, d=128, ctx=[32768], topk=None, paged=False),
    dict(seed=3, B=5, hq=28, hkv=4, d=128, ctx=[1, 15, 16, 300, 5003], topk=[4, 16, 16, 7, 500],
         paged=True),
    dict(seed=4, B=3, hq=8, hkv=1, d=64, ctx=[33, 257, 1111], topk=[100, 3, 60], paged=True),
], ids=["qwen32k", "ragged", "d64"])
def test_noalloc_matches_workspace_path_twice(case):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    p = inputs.make_decode_problem(case["seed"], case["B"], case["hq"], case["hkv"], case["d"], 16,
                                   case["ctx"], paged=case["paged"], topk=case["topk"])
    cfg, lc, ws, idx, cnt, max_topk = _select(p, dev)
    q = p.q.to(dev)
    shape = (p.batch, p.num_q_heads, p.head_dim)
    ref = torch.empty(shape, device=dev)
    ref_lse = torch.empty(shape[:2], device=dev)
    R.resa_sparse_decode(cfg, lc.struct(), q, idx, cnt, max_topk, ref, ref_lse, ws)
    torch.cuda.synchronize()
    assert R.resa_check_device_status(ws, raise_on_error=False) == 0
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


def test_noalloc_rejects_calls_beyond_its_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    dev = torch.device("cuda:0")
    cfg = R.make_config(28, 4, 128, 16)
    k = torch.zeros(8, 4, 16, 128, dtype=torch.bfloat16, device=dev)
    pt = torch.zeros(2048, 1, dtype=torch.int32, device=dev)    # batch 2048 x Hkv 4 > 4096
    sl = torch.ones(2048, dtype=torch.int32, device=dev)
    cache = R.make_cache(k, k, k, pt, sl)
    idx = torch.zeros(2048, 4, 2, dtype=torch.int32, device=dev)
    cnt = torch.ones(2048, 4, dtype=torch.int32, device=dev)
    q = torch.zeros(2048, 28, 128, dtype=torch.bfloat16, device=dev)
    out = torch.zeros(2048, 28, 128, device=dev)
    with pytest.raises(R.ResaError) as e:
        R.resa_sparse_decode_noalloc(cfg, cache, q, idx, cnt, 1, out, None)
    assert e.value.status == 2
