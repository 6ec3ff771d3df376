"""CPU checks of the C-ABI library: it loads, exports every entry point that
include/sbfa.h declares, and rejects bad arguments on the host before any
launch (no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sbfa.h")


def _declared():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+[\s\*]+(sbfa_\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def sb():
    import __graft_entry__
    __graft_entry__.build()
    import block_sparse_flashattention_sbfa_b200 as m
    return m


def test_header_declares_the_boundary():
    names = _declared()
    for n in ("sbfa_fwd", "sbfa_fwd_dense", "sbfa_fwd_partials", "sbfa_combine",
              "sbfa_speculative_sparse", "sbfa_fwd_gated", "sbfa_convert_vertical_slash",
              "sbfa_fwd_vertical_slash", "sbfa_check_status", "sbfa_last_error"):
        assert n in names


def test_library_exports_every_declared_symbol(sb):
    lib = ctypes.CDLL(sb.LIB_PATH)
    missing = [n for n in _declared() if not hasattr(lib, n)]
    assert not missing, missing
    assert b"sm_100a" in sb.lib.sbfa_version()


def _shape(sb, **kw):
    d = dict(B=1, Sq=128, Sk=128, Hq=2, Hkv=2, D=128, scale=0.0, causal=0)
    d.update(kw)
    return sb.Shape(**d)


def _t4(ptr=16 * 1024, sb_=128 * 2 * 128, ss=2 * 128, sh=128):
    import block_sparse_flashattention_sbfa_b200 as m
    return m.T4(ptr, sb_, ss, sh)


def test_host_validation_rejects_before_launch(sb):
    lib = sb.lib
    good = _t4()
    tab = sb.Table(16 * 1024, 0, 0, 0, 4, 64, 64)
    lse = 16 * 1024
    # null shape
    assert lib.sbfa_fwd(None, good, good, good, ctypes.byref(tab), good, lse, None, None) == \
        sb.ERR_INVALID_ARG
    # head dim other than 128
    s = _shape(sb, D=64)
    assert lib.sbfa_fwd(ctypes.byref(s), good, good, good, ctypes.byref(tab), good, lse, None,
                        None) == sb.ERR_UNSUPPORTED
    assert b"head dim" in lib.sbfa_last_error()
    # Hq not a multiple of Hkv
    s = _shape(sb, Hq=3, Hkv=2)
    assert lib.sbfa_fwd(ctypes.byref(s), good, good, good, ctypes.byref(tab), good, lse, None,
                        None) == sb.ERR_INVALID_ARG
    # null and misaligned q
    s = _shape(sb)
    assert lib.sbfa_fwd(ctypes.byref(s), _t4(ptr=0), good, good, ctypes.byref(tab), good, lse,
                        None, None) == sb.ERR_INVALID_ARG
    assert lib.sbfa_fwd(ctypes.byref(s), _t4(ptr=16 * 1024 + 2), good, good, ctypes.byref(tab),
                        good, lse, None, None) == sb.ERR_INVALID_ARG
    # strides that TMA cannot take
    assert lib.sbfa_fwd(ctypes.byref(s), _t4(ss=2 * 128 + 4), good, good, ctypes.byref(tab), good,
                        lse, None, None) == sb.ERR_INVALID_ARG
    # unsupported kv_block on the prefill path
    bad = sb.Table(16 * 1024, 0, 0, 0, 4, 64, 48)
    assert lib.sbfa_fwd(ctypes.byref(s), good, good, good, ctypes.byref(bad), good, lse, None,
                        None) == sb.ERR_UNSUPPORTED
    # null table
    assert lib.sbfa_fwd(ctypes.byref(s), good, good, good, None, good, lse, None, None) == \
        sb.ERR_INVALID_ARG
    # gated: needs Sq == Sk and causal
    s = _shape(sb, Sk=256, causal=1)
    assert lib.sbfa_fwd_gated(ctypes.byref(s), good, good, good, lse, 64, good, lse, None, None,
                              None, None) == sb.ERR_UNSUPPORTED
    # vertical-slash conversion: only 64 x 64 blocks
    assert lib.sbfa_convert_vertical_slash(lse, lse, lse, 4, lse, 4, 1, 1, 128, 32, 64, 1, lse,
                                           lse, lse, lse, None, None) == sb.ERR_UNSUPPORTED
    # combine: D must be 128
    assert lib.sbfa_combine(2, 1, 1, 1, 64, lse, lse, good, lse, None) == sb.ERR_UNSUPPORTED
    # NSA varlen: q rows are gathered from the (token x head) flattening, so the
    # token stride must be Hq head strides; and the selection block must be 64
    ws = 1 << 20
    q_bad = _t4(ss=4 * 128 + 64, sh=128)
    assert lib.sbfa_fwd_varlen_selected(lse, 1, 8, 8, 4, 4, 128, 0.0, 1, q_bad, good, good, lse,
                                        16, 64, ws, 1 << 30, good, lse, None, None) == \
        sb.ERR_UNSUPPORTED
    assert b"token stride" in lib.sbfa_last_error()
    assert lib.sbfa_fwd_varlen_selected(lse, 1, 8, 8, 4, 4, 128, 0.0, 1, good, good, good, lse,
                                        16, 32, ws, 1 << 30, good, lse, None, None) == \
        sb.ERR_UNSUPPORTED


def test_workspace_sizes(sb):
    """The NSA workspace query is host arithmetic (no GPU): the workspace
    holds the inverted index, the unit table and one fp32 accumulator row per
    (token, head) with its sum and row-maximum key -- not one partial per
    (token, head, slot).  Bad sizes give 0.  (The decode query sizes by the
    device's SM count and needs a GPU.)"""
    lib = ctypes.CDLL(sb.LIB_PATH)
    lib.sbfa_varlen_selected_workspace_size.restype = ctypes.c_size_t
    nsa = lib.sbfa_varlen_selected_workspace_size
    total, H, topk = 98304, 4, 16
    n = nsa(2, total, 65536, H, H, topk)
    acc = total * H * 128 * 4
    assert acc + 2 * total * H * 4 <= n < 0.26e9, n    # 0.23 GB on the bench workload
    assert n < total * H * topk * 128 * 4 / 10          # far below per-slot fp32 partials
    assert nsa(2, 2 * total, 65536, H, H, topk) > n
    assert nsa(2, total, 65536, 2 * H, H, topk) > n
    for bad in [(0, total, 65536, H, H, topk), (2, 0, 65536, H, H, topk),
                (2, total, 65536, H, H, 0), (2, total, 0, H, H, topk)]:
        assert nsa(*bad) == 0


def test_package_fails_loudly_without_library(tmp_path, monkeypatch):
    import importlib.util
    import sys
    src = os.path.join(ROOT, "block_sparse_flashattention_sbfa_b200", "__init__.py")
    pkg = tmp_path / "block_sparse_flashattention_sbfa_b200"
    pkg.mkdir()
    (pkg / "__init__.py").write_text(open(src).read())
    spec = importlib.util.spec_from_file_location("sbfa_nolib", str(pkg / "__init__.py"))
    mod = importlib.util.module_from_spec(spec)
    with pytest.raises(ImportError, match="missing"):
        spec.loader.exec_module(mod)
    assert "sbfa_nolib" not in sys.modules
