"""Host check of the arithmetic behind warp_max_f32 (block_sparse_flashattention_sbfa_b200/csrc/sbfa_ptx.cuh):
floats are mapped to unsigned integers in the same order, reduced with an
integer max (redux.sync), and mapped back.  These tests replay the map with
numpy, bit for bit."""
import numpy as np


def _ordered(v):
    u = np.asarray(v, dtype=np.float32).view(np.uint32)
    return np.where(u & 0x80000000, ~u, u | 0x80000000).astype(np.uint32)


def _unordered(u):
    u = np.asarray(u, dtype=np.uint32)
    return np.where(u & 0x80000000, u & 0x7FFFFFFF, ~u).astype(np.uint32).view(np.float32)


def test_float_order_map_of_the_warp_max():
    rng = np.random.default_rng(0)
    v = np.concatenate([rng.normal(size=1000) * 50, [-np.inf, np.inf, 0.0, 1e-38, -1e-38]])
    v = v.astype(np.float32)
    u = _ordered(v)
    order = np.argsort(v, kind="stable")
    assert np.all(np.diff(u[order].astype(np.int64)) >= 0)      # same order as the floats
    np.testing.assert_array_equal(_unordered(u), v)              # and back, bit for bit
    for _ in range(100):
        w = rng.normal(size=32).astype(np.float32) * 10
        assert _unordered(_ordered(w).max()) == w.max()
