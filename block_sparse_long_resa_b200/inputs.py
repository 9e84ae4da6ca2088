"""Seeded synthetic inputs for the ReSA decode hot path.

This module only draws random tensors and lays them out in the paged cache
format; it performs none of the method's arithmetic (no descriptors, scores,
selection or attention).  The CPU oracle tests, the CUDA parity tests and the
benchmark all take their inputs from here, so both sides of every parity check
see the same bytes.

Recipe (the workloads of the Rectified Sparse Attention efficiency study:
Qwen2.5-7B attention shape, long-context decode, synthetic data):

* q, K, V ~ N(0, 1), rounded to bf16.
* K carries a per-(kv head, channel) scale s[h, j] ~ LogNormal(0, 0.5), the
  same for every sequence and position (a model property, not a token one).
* ``needles`` seeded complete blocks per (sequence, kv head), never the last
  complete block, get ``+2 * u_h`` added to every key, where ``u_h`` is the
  unit vector along the sum of the group's first decode query heads (the
  direction of the group-pooled query).  They make the block ranking
  non-trivial: a correct selection must find them.
* The paged layout draws physical pages as a seeded random permutation
  (``paged=True``) or uses the identity (contiguous cache); both go through the
  same page table, so there is one code path.
* Rectification chunks draw fresh q, K, V ~ N(0, 1).

Cache layout (one layer):
    K, V        [num_pages][Hkv][block_size][head_dim]  bf16
    page_table  [batch][max_pages]                      int32 (physical page of logical block i)
    ctx_len     [batch]                                  tokens already in the cache
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Sequence

import torch


@dataclass
class DecodeProblem:
    batch: int
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    ctx_len: torch.Tensor          # [B] int32, tokens in the cache before the decode token
    page_table: torch.Tensor       # [B][max_pages] int32
    k_cache: torch.Tensor          # [num_pages][Hkv][bs][d] bf16
    v_cache: torch.Tensor          # [num_pages][Hkv][bs][d] bf16
    q: torch.Tensor                # [B][Hq][d] bf16, first decode query
    k_new: torch.Tensor            # [B][Hkv][d] bf16, first decode key
    v_new: torch.Tensor            # [B][Hkv][d] bf16
    topk: torch.Tensor             # [B] int32, blocks to select (before the local block)
    k_scale: torch.Tensor          # [Hkv][d] fp32 channel scale of K
    needle_blocks: torch.Tensor    # [B][Hkv][needles] int64, logical block ids
    seed: int = 0
    extra: dict = field(default_factory=dict)

    @property
    def max_pages(self) -> int:
        return int(self.page_table.shape[1])

    @property
    def num_pages(self) -> int:
        return int(self.k_cache.shape[0])

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads


def topk_for(ctx_len: int, block_size: int, frac_num: int = 1, frac_den: int = 10,
             n_min: int = 16) -> int:
    """Workload top-k: ``max(n_min, round(M * num / den))`` capped at M.

    M = complete blocks seen by the first decode token (ctx_len // block_size).
    Round-half-up reproduces both printed workload values (205 of 2048 and
    1638 of 16384 blocks); the library itself takes k as an input.
    """
    m = ctx_len // block_size
    k = max(n_min, (m * frac_num + frac_den // 2) // frac_den)
    return min(k, m)


def _gen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def make_decode_problem(seed: int, batch: int, num_q_heads: int, num_kv_heads: int,
                        head_dim: int, block_size: int, ctx_lens: Sequence[int], *,
                        reserve_tokens: int = 64, paged: bool = False, needles: int = 4,
                        topk: Optional[Sequence[int]] = None, frac=(1, 10), n_min: int = 16,
                        device="cpu", k_scale_sigma: float = 0.5) -> DecodeProblem:
    """Draw one decode problem: a filled paged KV cache plus the first decode token.

    ``reserve_tokens`` extra token slots are allocated per sequence so that
    decode steps can append without reallocating.
    """
    assert num_q_heads % num_kv_heads == 0
    assert len(ctx_lens) == batch
    dev = torch.device(device)
    g = _gen(seed, dev)
    hkv, d, bs = num_kv_heads, head_dim, block_size
    grp = num_q_heads // num_kv_heads
    pages_per = [-(-(int(L) + reserve_tokens) // bs) for L in ctx_lens]
    max_pages = max(pages_per)
    num_pages = sum(pages_per)

    if paged:
        perm = torch.randperm(num_pages, generator=g, device=dev).to(torch.int32)
    else:
        perm = torch.arange(num_pages, device=dev, dtype=torch.int32)
    page_table = torch.zeros(batch, max_pages, dtype=torch.int32, device=dev)
    off = 0
    for b in range(batch):
        page_table[b, :pages_per[b]] = perm[off:off + pages_per[b]]
        off += pages_per[b]

    k_scale = torch.exp(k_scale_sigma * torch.randn(hkv, d, generator=g, device=dev))
    # Draw in fp32 then round to bf16 (one draw per page keeps memory bounded for long caches).
    k_cache = torch.empty(num_pages, hkv, bs, d, dtype=torch.bfloat16, device=dev)
    v_cache = torch.empty(num_pages, hkv, bs, d, dtype=torch.bfloat16, device=dev)
    chunk = max(1, (1 << 26) // (hkv * bs * d))
    for p0 in range(0, num_pages, chunk):
        p1 = min(num_pages, p0 + chunk)
        kk = torch.randn(p1 - p0, hkv, bs, d, generator=g, device=dev)
        kk.mul_(k_scale[None, :, None, :])
        k_cache[p0:p1] = kk.to(torch.bfloat16)
        vv = torch.randn(p1 - p0, hkv, bs, d, generator=g, device=dev)
        v_cache[p0:p1] = vv.to(torch.bfloat16)
        del kk, vv

    q = torch.randn(batch, num_q_heads, d, generator=g, device=dev).to(torch.bfloat16)
    k_new = (torch.randn(batch, hkv, d, generator=g, device=dev) * k_scale[None]).to(torch.bfloat16)
    v_new = torch.randn(batch, hkv, d, generator=g, device=dev).to(torch.bfloat16)

    # Token slots beyond ctx_len are zeroed so a stale read is visible.
    for b in range(batch):
        L = int(ctx_lens[b])
        first_free = L // bs
        if L % bs:
            p = int(page_table[b, first_free])
            k_cache[p, :, L % bs:, :] = 0
            v_cache[p, :, L % bs:, :] = 0
            first_free += 1
        if first_free < pages_per[b]:
            idx = page_table[b, first_free:pages_per[b]].long()
            k_cache[idx] = 0
            v_cache[idx] = 0

    needle_blocks = torch.zeros(batch, hkv, max(needles, 0), dtype=torch.int64, device=dev)
    if needles > 0:
        qf = q.float().view(batch, hkv, grp, d).sum(dim=2)          # group sum direction
        u = qf / qf.norm(dim=-1, keepdim=True).clamp_min(1e-12)
        for b in range(batch):
            m = int(ctx_lens[b]) // bs
            if m - 1 < needles:
                continue
            for h in range(hkv):
                blocks = torch.randperm(m - 1, generator=g, device=dev)[:needles]
                needle_blocks[b, h] = blocks
                pages = page_table[b, blocks].long()
                kk = k_cache[pages, h].float() + 2.0 * u[b, h][None, None, :]
                k_cache[pages, h] = kk.to(torch.bfloat16)

    if topk is None:
        topk_t = torch.tensor([topk_for(int(L), bs, frac[0], frac[1], n_min) for L in ctx_lens],
                              dtype=torch.int32, device=dev)
    else:
        topk_t = torch.tensor(list(topk), dtype=torch.int32, device=dev)

    return DecodeProblem(batch=batch, num_q_heads=num_q_heads, num_kv_heads=hkv, head_dim=d,
                         block_size=bs,
                         ctx_len=torch.tensor([int(x) for x in ctx_lens], dtype=torch.int32,
                                              device=dev),
                         page_table=page_table, k_cache=k_cache, v_cache=v_cache, q=q,
                         k_new=k_new, v_new=v_new, topk=topk_t, k_scale=k_scale,
                         needle_blocks=needle_blocks, seed=seed)


def make_step_tokens(seed: int, step: int, batch: int, num_q_heads: int, num_kv_heads: int,
                     head_dim: int, k_scale: Optional[torch.Tensor] = None, device="cpu"):
    """Decode query and the new token's key/value for step ``step`` (seeded per step)."""
    dev = torch.device(device)
    g = _gen(seed * 1_000_003 + 7919 * (step + 1), dev)
    q = torch.randn(batch, num_q_heads, head_dim, generator=g, device=dev)
    k = torch.randn(batch, num_kv_heads, head_dim, generator=g, device=dev)
    if k_scale is not None:
        k = k * k_scale.to(dev)[None]
    v = torch.randn(batch, num_kv_heads, head_dim, generator=g, device=dev)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


def make_rectify_chunk(seed: int, batch: int, f: int, num_q_heads: int, num_kv_heads: int,
                       head_dim: int, device="cpu"):
    """Fresh queries and key/values of the last f tokens for one rectification, ~N(0, 1)."""
    dev = torch.device(device)
    g = _gen(seed * 7_368_787 + 104_729, dev)
    q = torch.randn(batch, f, num_q_heads, head_dim, generator=g, device=dev)
    k = torch.randn(batch, f, num_kv_heads, head_dim, generator=g, device=dev)
    v = torch.randn(batch, f, num_kv_heads, head_dim, generator=g, device=dev)
    return q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)


WIDE_KINDS = ("large", "huge", "tiny", "tiles")


def wide_range_values(seed: int, v: torch.Tensor, kind: str, tokens_axis: int = -2) -> torch.Tensor:
    """bf16 values of ``v``'s shape spanning bf16's range, for the value-range
    parity cases (seeded; the input's own values are only used for their signs
    and shapes):

    - ``large``: N(0, 1), with about 1 token in 16 scaled by 1e5;
    - ``huge``: as ``large``, plus about 1 token in 64 set to +-(1.0 .. 3.3)e38
      (near the largest finite bf16, 3.39e38);
    - ``tiny``: N(0, 1) * 1e-6 everywhere;
    - ``tiles``: runs of 64 consecutive tokens drawn as N(0,1) * 1e-6,
      N(0,1) * 1e5 or N(0,1), so that whole tiles differ in magnitude.
    ``tokens_axis`` is the axis along which tokens are counted.
    """
    assert kind in WIDE_KINDS, kind
    g = _gen(seed * 2_654_435 + 97, "cpu")
    x = torch.randn(v.shape, generator=g)
    ax = tokens_axis % x.dim()
    ntok = x.shape[ax]
    view = [1] * x.dim()
    view[ax] = ntok
    if kind == "tiny":
        return (x * 1e-6).to(torch.bfloat16).to(v.device)
    if kind == "tiles":
        run = torch.randint(0, 3, ((ntok + 63) // 64,), generator=g)
        scale = torch.tensor([1e-6, 1e5, 1.0])[run].repeat_interleave(64)[:ntok]
        return (x * scale.view(view)).to(torch.bfloat16).to(v.device)
    big = (torch.rand(ntok, generator=g) < 1 / 16).to(torch.float32)
    x = x * (1.0 + (1e5 - 1.0) * big).view(view)
    if kind == "huge":
        hot = (torch.rand(x.shape, generator=g) < 1 / 64)
        mag = 1.0e38 + 2.3e38 * torch.rand(x.shape, generator=g)
        x = torch.where(hot, torch.sign(x) * mag, x)
    return x.to(torch.bfloat16).to(v.device)


def continuous_batch_lengths(seed: int, batch: int, lo: int, hi: int) -> List[int]:
    """Context lengths uniform in [lo, hi] for the continuous-batching workload."""
    g = _gen(seed + 4242, "cpu")
    return [int(x) for x in torch.randint(lo, hi + 1, (batch,), generator=g)]
