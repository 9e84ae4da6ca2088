"""The oracle's closed forms against the numbers the pages print (tests/golden)."""
import json
import math
import os

import numpy as np
import pytest

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def test_eq5_printed_examples():
    g = load("eq5_selection_count.json")
    for case in g["cases"]:
        M = case["context_tokens"] // case["block_size"]
        assert M == case["M"]
        assert math.ceil(M * case["p"]) == case["ceil_M_p"]
        # the floor n_min then applies
        assert O.selection_count(M, case["p"], g["n_min"]) == max(g["n_min"], case["ceil_M_p"])
    fc = g["floor_case"]
    assert O.selection_count(fc["M"], fc["p"], g["n_min"]) == fc["n"]


def test_eq6_defaults():
    g = load("eq6_memory_access.json")
    assert O.memory_access_factor(g["b"], g["p"], g["f"]) == pytest.approx(g["factor"], abs=1e-12)
    assert 1.0 / g["b"] == g["terms"]["1/b"]
    assert 1.0 / g["f"] == g["terms"]["1/f"]


def test_rectify_refreshes_two_blocks_when_aligned():
    g = load("rectify_refresh.json")
    bs, f = g["block_size"], g["f"]
    for L in (64, 1024, 65536 + 32):
        assert L % bs == 0
        assert len(O.touched_blocks(L, f, bs)) == g["blocks_refreshed"]
    # not block-aligned: one more block is touched
    assert len(O.touched_blocks(1000, f, bs)) == g["blocks_refreshed"] + 1


def test_rectify_refresh_matches_oracle_writes():
    """The blocks the oracle's rectification rewrites are exactly touched_blocks."""
    bs, d, hkv, hq, f = 16, 8, 1, 1, 32
    L = 16 * 6 + 5
    pages = (L + bs - 1) // bs
    rng = np.random.default_rng(3)
    K = rng.integers(0x3c00, 0x4000, size=(pages, hkv, bs, d)).astype(np.uint16)
    V = K.copy()
    pt = np.arange(pages, dtype=np.int32)[None]
    c = O.OracleCache(K, V, pt, hq, hkv, d, bs)
    c.build_descriptors([L])
    sentinel = np.uint16(0x7f7f)
    c.desc[:] = sentinel
    kn = rng.integers(0x3c00, 0x4000, size=(1, f, hkv, d)).astype(np.uint16)
    c.rectify(kn.reshape(1, f, hq, d), kn, kn, [L], f)
    touched = [blk for blk in range(pages) if not np.all(c.desc[blk] == sentinel)]
    assert touched == list(O.touched_blocks(L, f, bs))


def test_descriptor_size():
    g = load("descriptor_size.json")
    assert 2 * g["head_dim"] == g["descriptor_values"]
    assert g["block_size"] * g["head_dim"] == g["block_key_values"]
    # the printed 1/16 is against keys + values (Eq. 6's 1/b term); against keys alone it is 1/8
    assert 2 * g["block_key_values"] // g["descriptor_values"] == g["printed_ratio"]
    assert g["block_key_values"] // g["descriptor_values"] == g["printed_ratio"] // 2


def test_printed_cache_size_is_one_tensor():
    g = load("kv_cache_size.json")
    one = g["layers"] * g["kv_heads"] * g["tokens"] * g["head_dim"] * g["bytes_per_value"]
    assert one / 1e9 == pytest.approx(g["printed_gb"], abs=0.05)
    assert 2 * one / 1e9 == pytest.approx(2 * g["printed_gb"], abs=0.1)
