"""CPU oracle for the ReSA decode hot path (ctypes front end of resa_oracle.c).

TEST INFRASTRUCTURE ONLY: the tests, the smoke check and the benchmark's
CPU-baseline leg may import this module; the product path never does.  It
shares no code with the CUDA library.

Source ("ReSA summary"): the page "Rectified Sparse Attention" of the
paper-graph-ui summary of arXiv 2506.04108; section and equation numbers
refer to that page.  Every pin of this oracle lives in
tests/test_oracle_pins.py and tests/test_golden.py.
"""
from __future__ import annotations

import ctypes
import math
import os
import subprocess
import threading
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "resa_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

# -ffp-contract=off: no fused multiply-add, so every fp32 product and sum
# rounds exactly as written in the C source.
CFLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math"]


def build(force: bool = False) -> str:
    """Compile resa_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, _SRC, "-o", tmp, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            _lib = ctypes.CDLL(build())
            P = ctypes.c_void_p
            I = ctypes.c_int
            F = ctypes.c_float
            sig = {
                "oracle_build_descriptors": [P, P, P, P, P, I, I, I, I, I],
                "oracle_append": [P, P, P, P, P, P, P, I, I, I, I, I],
                "oracle_pooled_query": [P, P, I, I, I, I],
                "oracle_block_scores": [P, P, P, P, P, I, I, I, I, I],
                "oracle_select": [P, P, P, P, P, I, I, I, I, I],
                "oracle_sparse_attention": [P, P, P, P, P, P, P, I, F, P, P, I, I, I, I, I, I],
                "oracle_rectify": [P, P, P, P, P, P, P, P, I, F, P, P, I, I, I, I, I, I],
                "oracle_dense_attention": [P, P, P, P, P, F, P, P, I, I, I, I, I, I],
            }
            for name, args in sig.items():
                fn = getattr(_lib, name)
                fn.argtypes = args
                fn.restype = None
            _lib.oracle_num_threads.restype = ctypes.c_int
            _lib.oracle_set_num_threads.argtypes = [ctypes.c_int]
            _lib.oracle_set_num_threads.restype = None
        return _lib


def num_threads() -> int:
    return int(lib().oracle_num_threads())


def set_num_threads(n: int) -> None:
    """Threads of the oracle's parallel loops (results do not depend on it)."""
    lib().oracle_set_num_threads(int(n))


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data


def bits(x) -> np.ndarray:
    """bf16 data as a contiguous uint16 array of bit patterns (torch bf16 or uint16 input)."""
    try:
        import torch
        if isinstance(x, torch.Tensor):
            t = x.detach().to("cpu").contiguous()
            if t.dtype == torch.bfloat16:
                return t.view(torch.int16).numpy().view(np.uint16).copy()
            x = t.numpy()
    except ImportError:  # pragma: no cover
        pass
    a = np.ascontiguousarray(x)
    assert a.dtype == np.uint16, a.dtype
    return a.copy()


def bf16_bits_to_float(a: np.ndarray) -> np.ndarray:
    return (a.astype(np.uint32) << 16).view(np.float32)


def _i32(x) -> np.ndarray:
    try:
        import torch
        if isinstance(x, torch.Tensor):
            x = x.detach().to("cpu").numpy()
    except ImportError:  # pragma: no cover
        pass
    return np.ascontiguousarray(np.asarray(x, dtype=np.int32))


# ---------------------------------------------------------------------------
# Closed forms printed on the pages
# ---------------------------------------------------------------------------

def selection_count(num_blocks: int, p: float, n_min: int = 16) -> int:
    """Eq. 5 (ReSA summary §3.4.1): n = max(n_min, ceil(M * p))."""
    return max(n_min, math.ceil(num_blocks * p))


def memory_access_factor(b: int, p: float, f: int) -> float:
    """Eq. 6 (ReSA summary §3.4.3): average memory access per decode step
    relative to mem(KV cache): 1/b + p + 1/f."""
    return 1.0 / b + p + 1.0 / f


def touched_blocks(seq_len: int, f: int, bs: int) -> range:
    """Blocks whose descriptors a rectification of positions L-f .. L-1
    rewrites (ReSA summary §3.4.2, descriptor recomputation)."""
    return range((seq_len - f) // bs, (seq_len - 1) // bs + 1)


# ---------------------------------------------------------------------------
# Stateful oracle over one layer's cache
# ---------------------------------------------------------------------------

class OracleCache:
    """One layer of the paged cache held as numpy arrays, plus the oracle steps.

    Arrays: K, V [num_pages][hkv][bs][d] uint16 (bf16 bits), desc
    [num_pages][hkv][2][d] uint16, page_table [B][max_pages] int32.
    """

    def __init__(self, k_cache, v_cache, page_table, num_q_heads: int, num_kv_heads: int,
                 head_dim: int, block_size: int, desc=None):
        self.K = bits(k_cache)
        self.V = bits(v_cache)
        self.page_table = _i32(page_table)
        self.B, self.max_pages = self.page_table.shape
        self.hq, self.hkv, self.d, self.bs = num_q_heads, num_kv_heads, head_dim, block_size
        self.num_pages = self.K.shape[0]
        assert self.K.shape == (self.num_pages, self.hkv, self.bs, self.d)
        self.desc = (np.zeros((self.num_pages, self.hkv, 2, self.d), dtype=np.uint16)
                     if desc is None else bits(desc))

    @property
    def sm_scale_default(self) -> float:
        return 1.0 / math.sqrt(self.d)

    def build_descriptors(self, seq_len, first_block=None) -> np.ndarray:
        sl = _i32(seq_len)
        fb = None if first_block is None else _i32(first_block)
        lib().oracle_build_descriptors(_ptr(self.K), _ptr(self.desc), _ptr(self.page_table),
                                       _ptr(sl), _ptr(fb), self.B, self.hkv, self.d, self.bs,
                                       self.max_pages)
        return self.desc

    def append(self, k_new, v_new, seq_len) -> None:
        kn, vn, sl = bits(k_new), bits(v_new), _i32(seq_len)
        lib().oracle_append(_ptr(self.K), _ptr(self.V), _ptr(self.desc), _ptr(kn), _ptr(vn),
                            _ptr(self.page_table), _ptr(sl), self.B, self.hkv, self.d, self.bs,
                            self.max_pages)

    def pooled_query(self, q) -> np.ndarray:
        qb = bits(q)
        out = np.zeros((self.B, self.hkv, self.d), dtype=np.float32)
        lib().oracle_pooled_query(_ptr(qb), _ptr(out), self.B, self.hq, self.hkv, self.d)
        return out

    def block_scores(self, qbar: np.ndarray, seq_len) -> np.ndarray:
        """fp32 scores [B][hkv][max_pages]; entries of non-complete blocks are NaN."""
        qb = np.ascontiguousarray(qbar, dtype=np.float32)
        sl = _i32(seq_len)
        out = np.full((self.B, self.hkv, self.max_pages), np.nan, dtype=np.float32)
        lib().oracle_block_scores(_ptr(qb), _ptr(self.desc), _ptr(self.page_table), _ptr(sl),
                                  _ptr(out), self.B, self.hkv, self.d, self.bs, self.max_pages)
        return out

    def select(self, scores: np.ndarray, topk, seq_len, max_topk: int):
        sc = np.ascontiguousarray(scores, dtype=np.float32)
        tk, sl = _i32(topk), _i32(seq_len)
        idx = np.full((self.B, self.hkv, max_topk + 1), -1, dtype=np.int32)
        cnt = np.zeros((self.B, self.hkv), dtype=np.int32)
        lib().oracle_select(_ptr(sc), _ptr(tk), _ptr(sl), _ptr(idx), _ptr(cnt), max_topk, self.B,
                            self.hkv, self.bs, self.max_pages)
        return idx, cnt

    def sparse_attention(self, q, block_idx, block_cnt, seq_len, sm_scale: Optional[float] = None):
        qb = bits(q)
        idx = _i32(block_idx)
        cnt = _i32(block_cnt)
        sl = _i32(seq_len)
        max_topk = idx.shape[-1] - 1
        out = np.zeros((self.B, self.hq, self.d), dtype=np.float64)
        lse = np.zeros((self.B, self.hq), dtype=np.float64)
        s = self.sm_scale_default if sm_scale is None else sm_scale
        lib().oracle_sparse_attention(_ptr(qb), _ptr(self.K), _ptr(self.V), _ptr(self.page_table),
                                      _ptr(sl), _ptr(idx), _ptr(cnt), max_topk, s, _ptr(out),
                                      _ptr(lse), self.B, self.hq, self.hkv, self.d, self.bs,
                                      self.max_pages)
        return out, lse

    def dense_attention(self, q, seq_len, sm_scale: Optional[float] = None):
        qb = bits(q)
        sl = _i32(seq_len)
        out = np.zeros((self.B, self.hq, self.d), dtype=np.float64)
        lse = np.zeros((self.B, self.hq), dtype=np.float64)
        s = self.sm_scale_default if sm_scale is None else sm_scale
        lib().oracle_dense_attention(_ptr(qb), _ptr(self.K), _ptr(self.V), _ptr(self.page_table),
                                     _ptr(sl), s, _ptr(out), _ptr(lse), self.B, self.hq, self.hkv,
                                     self.d, self.bs, self.max_pages)
        return out, lse

    def decode_step(self, q, k_new, v_new, topk, seq_len, max_topk: int,
                    sm_scale: Optional[float] = None) -> dict:
        """Append, pool, score, select, attend (one ReSA sparse decode step).

        seq_len already counts the decode token."""
        self.append(k_new, v_new, seq_len)
        qbar = self.pooled_query(q)
        scores = self.block_scores(qbar, seq_len)
        idx, cnt = self.select(scores, topk, seq_len, max_topk)
        out, lse = self.sparse_attention(q, idx, cnt, seq_len, sm_scale)
        return dict(qbar=qbar, scores=scores, block_idx=idx, block_cnt=cnt, out=out, lse=lse)

    def rectify(self, q_chunk, k_new, v_new, seq_len, f: int, sm_scale: Optional[float] = None):
        qc, kn, vn, sl = bits(q_chunk), bits(k_new), bits(v_new), _i32(seq_len)
        assert qc.shape == (self.B, f, self.hq, self.d)
        assert kn.shape == (self.B, f, self.hkv, self.d)
        out = np.zeros((self.B, f, self.hq, self.d), dtype=np.float64)
        lse = np.zeros((self.B, f, self.hq), dtype=np.float64)
        s = self.sm_scale_default if sm_scale is None else sm_scale
        lib().oracle_rectify(_ptr(qc), _ptr(kn), _ptr(vn), _ptr(self.K), _ptr(self.V),
                             _ptr(self.desc), _ptr(self.page_table), _ptr(sl), f, s, _ptr(out),
                             _ptr(lse), self.B, self.hq, self.hkv, self.d, self.bs, self.max_pages)
        return out, lse

    def rectify_rows(self, q_chunk, k_new, v_new, seq_len, f: int, rows,
                     sm_scale: Optional[float] = None):
        """Rectification evaluated on a sample of chunk rows: the same three
        steps as rectify() (write-back, descriptor refresh of the touched
        blocks, causal attention), with the attention of chunk row r taken as
        dense attention of q_chunk[:, r] over positions 0 .. L-f+r.  Returns
        {r: (out [B][hq][d], lse [B][hq])}."""
        kn, vn, sl = bits(k_new), bits(v_new), _i32(seq_len)
        for b in range(self.B):
            L = int(sl[b])
            if f > L:
                continue  # a chunk longer than the sequence leaves it untouched
            for r in range(f):
                pos = L - f + r
                page = self.page_table[b, pos // self.bs]
                self.K[page, :, pos % self.bs] = kn[b, r]
                self.V[page, :, pos % self.bs] = vn[b, r]
        ok = sl >= f
        self.build_descriptors(np.where(ok, sl, 0).astype(np.int32),
                               np.where(ok, (sl - f) // self.bs, 0).astype(np.int32))
        qc = bits(q_chunk)
        res = {}
        for r in rows:
            res[int(r)] = self.dense_attention(qc[:, r], np.maximum(sl - f + int(r) + 1, 0),
                                               sm_scale)
        return res

    def rows_view(self, rows) -> "OracleCache":
        """The same cache seen by a call that covers the sequences in rows
        ``rows`` of the page table, in that order (the row map of resa.h):
        K, V and the descriptors are shared, so the view's steps update this
        cache; per-call arrays passed to the view are indexed by position in
        ``rows``."""
        v = object.__new__(OracleCache)
        v.__dict__.update(self.__dict__)
        v.page_table = np.ascontiguousarray(self.page_table[np.asarray(rows, dtype=np.int64)])
        v.B = v.page_table.shape[0]
        return v

    # Views used by tests ----------------------------------------------------
    def keys(self, b: int, h: int, L: int) -> np.ndarray:
        """Keys of sequence b, kv head h, positions 0 .. L-1 as float32 [L][d]."""
        pages = self.page_table[b, : (L + self.bs - 1) // self.bs]
        k = self.K[pages, h].reshape(-1, self.d)[:L]
        return bf16_bits_to_float(k)

    def values(self, b: int, h: int, L: int) -> np.ndarray:
        pages = self.page_table[b, : (L + self.bs - 1) // self.bs]
        v = self.V[pages, h].reshape(-1, self.d)[:L]
        return bf16_bits_to_float(v)
