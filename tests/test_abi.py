"""The C-ABI library loads, exports every symbol include/resa.h declares, and
its host-side validation answers without touching a GPU."""
import ctypes
import os
import re

import pytest

from block_sparse_long_resa_b200 import build as B
from block_sparse_long_resa_b200 import resa as R

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return R.lib()


def declared_functions():
    text = open(os.path.join(ROOT, "include", "resa.h")).read()
    return sorted(set(re.findall(r"RESA_API\s+[\w\s\*]*?\b(resa_\w+)\s*\(", text)))


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert len(names) >= 11
    for name in ["resa_build_descriptors", "resa_select_blocks", "resa_sparse_decode",
                 "resa_rectify_attention", "resa_decode_step"]:
        assert name in names
    for name in names:
        assert hasattr(lib, name), name
        assert name in R._SIGS, name


def test_status_strings_and_launch_table(lib):
    assert R.resa_status_string(0) == "RESA_OK"
    assert R.resa_status_string(6) == "RESA_ERR_DEVICE_CHECK"
    assert R.resa_kernels_per_call("resa_decode_step") == 1
    assert R.resa_kernels_per_call("resa_rectify_attention") == 2
    assert R.resa_kernels_per_call("nope") == -1


def test_workspace_size(lib):
    cfg = R.make_config(28, 4, 128, 16)
    small = R.resa_workspace_size(cfg, 1, 2048, 0)
    big = R.resa_workspace_size(cfg, 1, 16400, 32)
    assert 0 < small < big
    assert R.resa_workspace_size(cfg, 4, 4100, 32) > 0
    with pytest.raises(R.ResaError):
        R.resa_workspace_size(R.make_config(28, 4, 96, 16), 1, 10, 0)   # unsupported d


class FakeTensor:
    """Stands in for a device tensor: an address and a size, never dereferenced."""

    def __init__(self, addr=0x10000, n=1 << 30, shape=(1, 1)):
        self.addr, self.n, self.shape = addr, n, shape

    def data_ptr(self):
        return self.addr

    def numel(self):
        return self.n


def _cache(**kw):
    c = R.resa_cache_t(0x100000, 0x200000, 0x300000, 0x400000, 0x500000, 1, 64, 64)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def _call_select(cfg, cache, ws_bytes=1 << 30, q=0x600000):
    return R.lib().resa_select_blocks(ctypes.byref(cfg), ctypes.byref(cache), q, 0x700000, 8,
                                      0x800000, 0x900000, None, 0xa00000, ws_bytes, None)


def test_host_validation_without_gpu(lib):
    cfg = R.make_config(4, 2, 64, 16)
    assert lib.resa_select_blocks(None, ctypes.byref(_cache()), 1, 1, 8, 1, 1, None, 1, 1, None) == 1
    assert _call_select(cfg, _cache(k=None)) == 1                          # NULL k
    assert _call_select(cfg, _cache(), q=None) == 1                        # NULL q
    assert _call_select(R.make_config(4, 3, 64, 16), _cache()) == 2        # Hq % Hkv
    assert _call_select(R.make_config(4, 2, 96, 16), _cache()) == 4        # head_dim 96
    assert _call_select(R.make_config(4, 2, 64, 8), _cache()) == 4         # block size 8
    assert _call_select(R.make_config(4, 2, 64, 48), _cache()) == 4        # block size 48
    assert _call_select(R.make_config(68, 2, 64, 16), _cache()) == 4       # group 34 > 16
    assert _call_select(R.make_config(4, 2, 64, 16, -1.0), _cache()) == 3  # negative scale
    assert _call_select(cfg, _cache(batch=0)) == 2
    assert _call_select(cfg, _cache(k=0x100008)) == 4                      # misaligned
    assert _call_select(cfg, _cache(), ws_bytes=16) == 2                   # workspace too small
    assert _call_select(cfg, _cache(rows=0xb00000, table_rows=0)) == 2     # row map, no table
    assert _call_select(cfg, _cache(rows=0xb00004, table_rows=4)) == 4     # misaligned row map
    # dense decode: NULL token, misaligned query
    assert lib.resa_dense_decode(ctypes.byref(cfg), ctypes.byref(_cache()), 0x600000, None,
                                 0x610000, 0x620000, None, 0xa00000, 1 << 30, None) == 1
    assert lib.resa_dense_decode(ctypes.byref(cfg), ctypes.byref(_cache()), 0x600008, 0x610000,
                                 0x610000, 0x620000, None, 0xa00000, 1 << 30, None) == 4
    # rectify: f < 1 and chunk too large
    c = _cache()
    assert lib.resa_rectify_attention(ctypes.byref(cfg), ctypes.byref(c), 0, 1 << 20, 1 << 20,
                                      1 << 20, 1 << 20, None, 1 << 20, 1 << 30, None) == 3
    assert lib.resa_rectify_attention(ctypes.byref(cfg), ctypes.byref(c), 100000, 1 << 20,
                                      1 << 20, 1 << 20, 1 << 20, None, 1 << 20, 1 << 30,
                                      None) == 4
    assert lib.resa_workspace_init(None, 0, None) == 1
    assert lib.resa_check_device_status(None, 0, None, None) == 1


def test_host_validation_of_the_other_entry_points(lib):
    """Argument checks that return before anything is launched (status codes
    of resa.h: 1 NULL, 3 RANGE, 4 UNSUPPORTED)."""
    cfg, c, B = R.make_config(4, 2, 64, 16), _cache(), ctypes.byref

    def step(q=0x600000, topk=0x630000, max_topk=8):
        return lib.resa_decode_step(B(cfg), B(c), q, 0x610000, 0x620000, topk, max_topk,
                                    0x640000, None, None, None, 0xa00000, 1 << 30, None)
    assert step(max_topk=-1) == 3
    assert step(max_topk=65) == 3          # above max_pages with the list in the workspace
    assert step(q=None) == 1
    assert step(topk=0x630004) == 4        # misaligned
    assert lib.resa_append_token(B(cfg), B(c), None, 0x620000, 0xa00000, 1 << 30, None) == 1
    assert lib.resa_build_descriptors(None, B(c), None, 0xa00000, 1 << 30, None) == 1
    assert lib.resa_build_descriptors(B(R.make_config(4, 2, 64, 8)), B(c), None, 0xa00000,
                                      1 << 30, None) == 4
    # max_topk + 1 above the split merge's 1024 x 512 blocks
    assert lib.resa_sparse_decode(B(cfg), B(c), 0x600000, 0x700000, 0x800000, 1024 * 512,
                                  0x640000, None, 0xa00000, 1 << 30, None) == 3
    assert lib.resa_sparse_decode_noalloc(B(cfg), B(c), 0x600000, 0x700000, 0x800000, 8,
                                          0x640000, None, None, None) == 1
    assert lib.resa_sparse_decode_noalloc(B(cfg), B(c), 0x600000, 0x700000, 0x800000,
                                          1024 * 512, 0x640000, None, 0x650000, None) == 3


def test_binding_raises_on_error(lib):
    cfg = R.make_config(4, 2, 64, 16)
    with pytest.raises(R.ResaError) as e:
        R.resa_sparse_decode(cfg, _cache(), None, FakeTensor(), FakeTensor(), 8, FakeTensor(),
                             None, FakeTensor(), stream=0)
    assert e.value.status == 1
