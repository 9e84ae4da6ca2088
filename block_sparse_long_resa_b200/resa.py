"""ctypes binding of libresa (include/resa.h).

Argument marshalling only: every step of the hot path runs in the CUDA
kernels of libresa.so.  Tensors are torch CUDA tensors (PyTorch provides the
device memory and the stream); the functions keep the C names and raise
ResaError on any status other than RESA_OK.  There is no fallback: if the
library is missing, importing it raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libresa.so")

RESA_OK = 0
STATUS_NAMES = {0: "RESA_OK", 1: "RESA_ERR_NULL", 2: "RESA_ERR_SHAPE", 3: "RESA_ERR_RANGE",
                4: "RESA_ERR_UNSUPPORTED", 5: "RESA_ERR_CUDA", 6: "RESA_ERR_DEVICE_CHECK"}
DEVERR_SEQ_LEN, DEVERR_PAGE, DEVERR_BLOCK, DEVERR_TOPK, DEVERR_CHUNK, DEVERR_TIMEOUT, DEVERR_ROW = (
    0x1, 0x2, 0x4, 0x8, 0x10, 0x20, 0x40)


class ResaError(RuntimeError):
    def __init__(self, status: int, where: str, code: int = 0):
        self.status = status
        self.code = code
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}"
                         + (f" (device error word 0x{code:x})" if code else ""))


class resa_config_t(ctypes.Structure):
    _fields_ = [("num_q_heads", ctypes.c_int32), ("num_kv_heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("block_size", ctypes.c_int32),
                ("sm_scale", ctypes.c_float)]


class resa_cache_t(ctypes.Structure):
    _fields_ = [("k", ctypes.c_void_p), ("v", ctypes.c_void_p), ("desc", ctypes.c_void_p),
                ("page_table", ctypes.c_void_p), ("seq_len", ctypes.c_void_p),
                ("batch", ctypes.c_int32), ("max_pages", ctypes.c_int32),
                ("num_pages", ctypes.c_int32), ("rows", ctypes.c_void_p),
                ("table_rows", ctypes.c_int32)]


_lib = None

_P = ctypes.c_void_p
_I = ctypes.c_int32
_SIGS = {
    "resa_workspace_size": ([_P, _I, _I, _I], ctypes.c_size_t),
    "resa_workspace_init": ([_P, ctypes.c_size_t, _P], ctypes.c_int),
    "resa_check_device_status": ([_P, ctypes.c_size_t, _P, _P], ctypes.c_int),
    "resa_build_descriptors": ([_P, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "resa_append_token": ([_P, _P, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "resa_select_blocks": ([_P, _P, _P, _P, _I, _P, _P, _P, _P, ctypes.c_size_t, _P],
                           ctypes.c_int),
    "resa_sparse_decode": ([_P, _P, _P, _P, _P, _I, _P, _P, _P, ctypes.c_size_t, _P],
                           ctypes.c_int),
    "resa_rectify_attention": ([_P, _P, _I, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
                               ctypes.c_int),
    "resa_decode_step": ([_P, _P, _P, _P, _P, _P, _I, _P, _P, _P, _P, _P, ctypes.c_size_t, _P],
                         ctypes.c_int),
    "resa_sparse_decode_noalloc": ([_P, _P, _P, _P, _P, _I, _P, _P, _P, _P], ctypes.c_int),
    "resa_dense_decode": ([_P, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "resa_kernels_per_call": ([ctypes.c_char_p], ctypes.c_int32),
    "resa_decode_step_launches": ([_P, _I, _I, _I], ctypes.c_int32),
    "resa_status_string": ([ctypes.c_int], ctypes.c_char_p),
}


def lib() -> ctypes.CDLL:
    """Load libresa.so (built in-tree by block_sparse_long_resa_b200.build)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libresa.so is not built ({LIB_PATH}); run "
                               "`python -m block_sparse_long_resa_b200.build`")
        dll = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in _SIGS.items():
            fn = getattr(dll, name)
            fn.argtypes = args
            fn.restype = res
        _lib = dll
    return _lib


def _ptr(t) -> Optional[int]:
    if t is None:
        return None
    if isinstance(t, int):
        return t
    return t.data_ptr()


def _stream(stream) -> Optional[int]:
    if stream is None:
        import torch
        return torch.cuda.current_stream().cuda_stream
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(st: int, where: str):
    if st != RESA_OK:
        raise ResaError(st, where)


# ---------------------------------------------------------------------------
# Plain structs
# ---------------------------------------------------------------------------

def make_config(num_q_heads: int, num_kv_heads: int, head_dim: int, block_size: int = 16,
                sm_scale: float = 0.0) -> resa_config_t:
    return resa_config_t(num_q_heads, num_kv_heads, head_dim, block_size, sm_scale)


def make_cache(k, v, desc, page_table, seq_len, rows=None) -> resa_cache_t:
    """Cache struct over torch tensors k/v [pages][Hkv][b][d] bf16, desc
    [pages][Hkv][2][d] bf16, page_table [B][max_pages] int32, seq_len [B] int32.

    With ``rows`` (int32 device tensor [n]) the call covers the n sequences in
    those rows of page_table / seq_len (the row map of resa_cache_t)."""
    nrows = int(page_table.shape[0])
    if rows is None:
        return resa_cache_t(_ptr(k), _ptr(v), _ptr(desc), _ptr(page_table), _ptr(seq_len),
                            nrows, int(page_table.shape[1]), int(k.shape[0]), None, 0)
    return resa_cache_t(_ptr(k), _ptr(v), _ptr(desc), _ptr(page_table), _ptr(seq_len),
                        int(rows.numel()), int(page_table.shape[1]), int(k.shape[0]),
                        _ptr(rows), nrows)


# ---------------------------------------------------------------------------
# Entry points (same names as the C ABI)
# ---------------------------------------------------------------------------

def resa_workspace_size(cfg: resa_config_t, batch: int, max_pages: int, max_chunk: int = 0) -> int:
    n = lib().resa_workspace_size(ctypes.byref(cfg), batch, max_pages, max_chunk)
    if n == 0:
        raise ResaError(2, "resa_workspace_size")
    return int(n)


def resa_workspace_init(ws, stream=None):
    _check(lib().resa_workspace_init(_ptr(ws), ws.numel(), _stream(stream)), "resa_workspace_init")


def resa_check_device_status(ws, stream=None, raise_on_error: bool = True) -> int:
    code = ctypes.c_uint32(0)
    st = lib().resa_check_device_status(_ptr(ws), ws.numel(), _stream(stream), ctypes.byref(code))
    if st != RESA_OK and (raise_on_error or st != 6):
        raise ResaError(st, "resa_check_device_status", code.value)
    return int(code.value)


def resa_build_descriptors(cfg, cache, first_block, ws, stream=None):
    _check(lib().resa_build_descriptors(ctypes.byref(cfg), ctypes.byref(cache), _ptr(first_block),
                                        _ptr(ws), ws.numel(), _stream(stream)),
           "resa_build_descriptors")


def resa_append_token(cfg, cache, k_new, v_new, ws, stream=None):
    _check(lib().resa_append_token(ctypes.byref(cfg), ctypes.byref(cache), _ptr(k_new),
                                   _ptr(v_new), _ptr(ws), ws.numel(), _stream(stream)),
           "resa_append_token")


def resa_select_blocks(cfg, cache, q, topk, max_topk: int, block_idx, block_cnt, scores, ws,
                       stream=None):
    _check(lib().resa_select_blocks(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(topk),
                                    max_topk, _ptr(block_idx), _ptr(block_cnt), _ptr(scores),
                                    _ptr(ws), ws.numel(), _stream(stream)),
           "resa_select_blocks")


def resa_sparse_decode(cfg, cache, q, block_idx, block_cnt, max_topk: int, out, lse, ws,
                       stream=None):
    _check(lib().resa_sparse_decode(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q),
                                    _ptr(block_idx), _ptr(block_cnt), max_topk, _ptr(out),
                                    _ptr(lse), _ptr(ws), ws.numel(), _stream(stream)),
           "resa_sparse_decode")


def resa_rectify_attention(cfg, cache, f: int, q_chunk, k_new, v_new, out, lse, ws, stream=None):
    _check(lib().resa_rectify_attention(ctypes.byref(cfg), ctypes.byref(cache), f, _ptr(q_chunk),
                                        _ptr(k_new), _ptr(v_new), _ptr(out), _ptr(lse), _ptr(ws),
                                        ws.numel(), _stream(stream)),
           "resa_rectify_attention")


def resa_decode_step(cfg, cache, q, k_new, v_new, topk, max_topk: int, out, lse, block_idx,
                     block_cnt, ws, stream=None):
    _check(lib().resa_decode_step(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(k_new),
                                  _ptr(v_new), _ptr(topk), max_topk, _ptr(out), _ptr(lse),
                                  _ptr(block_idx), _ptr(block_cnt), _ptr(ws), ws.numel(),
                                  _stream(stream)),
           "resa_decode_step")


def resa_dense_decode(cfg, cache, q, k_new, v_new, out, lse, ws, stream=None):
    """Dense decode: append the decode token and attend to every position."""
    _check(lib().resa_dense_decode(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q), _ptr(k_new),
                                   _ptr(v_new), _ptr(out), _ptr(lse), _ptr(ws), ws.numel(),
                                   _stream(stream)),
           "resa_dense_decode")


def resa_sparse_decode_noalloc(cfg, cache, q, block_idx, block_cnt, max_topk: int, out, lse,
                               dev_error, stream=None):
    """resa_sparse_decode without a workspace, for callers that cannot allocate
    device memory (scratch lives in a fixed device array inside the library).
    dev_error: a device uint32 word (e.g. an int32 tensor element) that
    receives the device error bits; required."""
    _check(lib().resa_sparse_decode_noalloc(ctypes.byref(cfg), ctypes.byref(cache), _ptr(q),
                                            _ptr(block_idx), _ptr(block_cnt), max_topk, _ptr(out),
                                            _ptr(lse), _ptr(dev_error), _stream(stream)),
           "resa_sparse_decode_noalloc")


def resa_kernels_per_call(entry_point: str) -> int:
    return int(lib().resa_kernels_per_call(entry_point.encode()))


def resa_decode_step_launches(cfg, batch: int, max_pages: int, num_pages: int) -> int:
    """1 when resa_decode_step runs as one fused launch for this cache shape, else 3."""
    return int(lib().resa_decode_step_launches(ctypes.byref(cfg), batch, max_pages, num_pages))


def resa_status_string(status: int) -> str:
    return lib().resa_status_string(status).decode()
