"""Block-sparse FlashAttention forward for NVIDIA B200 (sm_100a).

Thin Python binding over the C ABI of ``libsbfa.so`` (declared in
``include/sbfa.h``): it only marshals torch tensors into pointers, strides
and the current CUDA stream.  Every step of the computation runs in the
library's CUDA kernels; there is no fallback.  Importing the package without
the built library raises ImportError.

Layouts follow the Incremental_FlashAttention README (Usage 1):
q (B, Sq, Hq, 128), k/v (B, Sk, Hkv, 128) bf16, o like q, lse (B, Hq, Sq) fp32.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libsbfa.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_CUDA, ERR_DEVICE, ERR_TIMEOUT = range(6)
DEV_BAD_INDEX, DEV_TIMEOUT, DEV_OVERFLOW = 0x1, 0x2, 0x4
_STATUS_NAMES = {0: "SBFA_OK", 1: "SBFA_ERR_INVALID_ARG", 2: "SBFA_ERR_UNSUPPORTED",
                 3: "SBFA_ERR_CUDA", 4: "SBFA_ERR_DEVICE", 5: "SBFA_ERR_TIMEOUT"}


class T4(ctypes.Structure):
    _fields_ = [("ptr", ctypes.c_void_p), ("sb", ctypes.c_int64), ("ss", ctypes.c_int64),
                ("sh", ctypes.c_int64)]


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Sq", ctypes.c_int32), ("Sk", ctypes.c_int32),
                ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32), ("D", ctypes.c_int32),
                ("scale", ctypes.c_float), ("causal", ctypes.c_int32)]


class Table(ctypes.Structure):
    _fields_ = [("idx", ctypes.c_void_p), ("sb", ctypes.c_int64), ("sh", ctypes.c_int64),
                ("sqb", ctypes.c_int64), ("nmax", ctypes.c_int32), ("q_block", ctypes.c_int32),
                ("kv_block", ctypes.c_int32)]


_P = ctypes.c_void_p
_I = ctypes.c_int32
_SIGS = {
    "sbfa_fwd": [ctypes.POINTER(Shape), T4, T4, T4, ctypes.POINTER(Table), T4, _P, _P, _P],
    "sbfa_fwd_dense": [ctypes.POINTER(Shape), T4, T4, T4, T4, _P, _P, _P],
    "sbfa_fwd_partials": [ctypes.POINTER(Shape), T4, T4, T4, ctypes.POINTER(Table), _P, _P, _P,
                          _P],
    "sbfa_combine": [_I, _I, _I, _I, _I, _P, _P, T4, _P, _P],
    "sbfa_calibrate_thresholds": [_P, _I, _I, _I, _I, _P, _P],
    "sbfa_speculative_sparse": [ctypes.POINTER(Shape), T4, T4, T4, _I, _I, T4, T4,
                                ctypes.POINTER(Table), _P, ctypes.c_size_t, T4, _P, _P, _P],
    "sbfa_speculative_sparse_noalloc": [ctypes.POINTER(Shape), T4, T4, T4, _I, _I, T4, T4,
                                        ctypes.POINTER(Table), T4, _P, _P, _P],
    "sbfa_decode_workspace_size": [_I, _I, _I, _I],
    "sbfa_fwd_gated": [ctypes.POINTER(Shape), T4, T4, T4, _P, _I, T4, _P, _P, _P, _P, _P],
    "sbfa_convert_vertical_slash": [_P, _P, _P, _I, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P,
                                    _P, _P, _P],
    "sbfa_fwd_vertical_slash": [ctypes.POINTER(Shape), T4, T4, T4, _P, _P, _I, _P, _P, _I, _I,
                                _I, T4, _P, _P, _P],
    "sbfa_convert_vertical_slash_mergehead": [_P, _P, _P, _I, _P, _I, _P, _P, _I, _I, _I, _I, _I,
                                              _I, _P, _P, _P, _P, _P, _P],
    "sbfa_fwd_varlen": [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, T4, T4, T4,
                        ctypes.POINTER(Table), T4, _P, _P, _P],
    "sbfa_fwd_vertical_slash_varlen": [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float,
                                       _I, T4, T4, T4, _P, _P, _I, _P, _P, _I, _I, _I, T4, _P,
                                       _P, _P],
    "sbfa_fwd_window": [ctypes.POINTER(Shape), T4, T4, T4, _I, T4, _P, _P, _P],
    "sbfa_fwd_window_varlen": [_P, _P, _I, _I, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, T4, T4,
                               T4, T4, _P, _P, _P],
    "sbfa_fwd_varlen_selected": [_P, _I, _I, _I, _I, _I, _I, ctypes.c_float, _I, T4, T4, T4, _P,
                                 _I, _I, _P, ctypes.c_size_t, T4, _P, _P, _P],
    "sbfa_varlen_selected_workspace_size": [_I, _I, _I, _I, _I, _I],
    "sbfa_check_status": [_P, _P],
    "sbfa_set_wait_limit_ns": [ctypes.c_uint64],
    "sbfa_last_error": [],
    "sbfa_version": [],
}
_RESTYPES = {"sbfa_decode_workspace_size": ctypes.c_size_t,
             "sbfa_set_wait_limit_ns": ctypes.c_uint64,
             "sbfa_varlen_selected_workspace_size": ctypes.c_size_t, "sbfa_last_error": ctypes.c_char_p,
             "sbfa_version": ctypes.c_char_p}


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(
            f"{LIB_PATH} is missing: build it with "
            "`python block_sparse_flashattention_sbfa_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    for name, args in _SIGS.items():
        fn = getattr(lib, name)
        fn.argtypes = args
        fn.restype = _RESTYPES.get(name, ctypes.c_int)
    return lib


lib = _load()


class SbfaError(RuntimeError):
    def __init__(self, fn, code):
        msg = lib.sbfa_last_error().decode()
        super().__init__(f"{fn}: {_STATUS_NAMES.get(code, code)}: {msg}")
        self.code = code


def _call(name, *args):
    code = getattr(lib, name)(*args)
    if code != OK:
        raise SbfaError(name, code)


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------

def _t4(x: torch.Tensor) -> T4:
    if x.dim() != 4 or x.stride(3) != 1:
        raise ValueError("expected a (B, S, H, D) tensor with a contiguous last dim")
    return T4(x.data_ptr(), x.stride(0), x.stride(1), x.stride(2))


def _ptr(x):
    return None if x is None else x.data_ptr()


def _stream():
    return torch.cuda.current_stream().cuda_stream


def _shape(q, k, causal, scale):
    B, Sq, Hq, D = q.shape
    return Shape(B, Sq, k.shape[1], Hq, k.shape[2], D, 0.0 if scale is None else float(scale),
                 int(bool(causal)))


def _check_bf16(*ts):
    for t in ts:
        if t.dtype != torch.bfloat16 or not t.is_cuda:
            raise TypeError("q, k, v must be bf16 CUDA tensors")


def _table(table: torch.Tensor, q_block: int, kv_block: int) -> Table:
    if table.dtype != torch.int32 or not table.is_cuda:
        raise TypeError("table must be an int32 CUDA tensor")
    if table.dim() == 1:          # the README's 1-D table, shared by every row
        return Table(table.data_ptr(), 0, 0, 0, table.shape[0], q_block, kv_block)
    if table.dim() != 4 or table.stride(3) != 1:
        raise ValueError("table must be (N,) or (B, Hkv, nQB, nmax) with a contiguous last dim")
    sb, sh, sqb = (table.stride(i) if table.shape[i] > 1 else 0 for i in range(3))
    return Table(table.data_ptr(), sb, sh, sqb, table.shape[3], q_block, kv_block)


def _outputs(q, out, lse):
    B, Sq, Hq, D = q.shape
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device=q.device)
    return out, lse


# ----------------------------------------------------------------------------
# public API
# ----------------------------------------------------------------------------

def fwd(q, k, v, table, q_block, kv_block, causal=False, scale=None, out=None, lse=None,
        status=None):
    """Block-table attention (``sbfa_fwd``). Returns (o, lse)."""
    _check_bf16(q, k, v)
    out, lse = _outputs(q, out, lse)
    tb = _table(table, q_block, kv_block)
    shp = _shape(q, k, causal, scale)
    _call("sbfa_fwd", ctypes.byref(shp), _t4(q), _t4(k), _t4(v), ctypes.byref(tb), _t4(out),
          lse.data_ptr(), _ptr(status), _stream())
    return out, lse


def fwd_dense(q, k, v, causal=False, scale=None, out=None, lse=None, status=None):
    """Dense attention over all keys (``sbfa_fwd_dense``). Returns (o, lse)."""
    _check_bf16(q, k, v)
    out, lse = _outputs(q, out, lse)
    shp = _shape(q, k, causal, scale)
    _call("sbfa_fwd_dense", ctypes.byref(shp), _t4(q), _t4(k), _t4(v), _t4(out), lse.data_ptr(),
          _ptr(status), _stream())
    return out, lse


def fwd_window(q, k, v, window, scale=None, out=None, lse=None, status=None):
    """Causal sliding-window attention of ``window`` keys (``sbfa_fwd_window``).
    Returns (o, lse)."""
    _check_bf16(q, k, v)
    out, lse = _outputs(q, out, lse)
    shp = _shape(q, k, True, scale)
    _call("sbfa_fwd_window", ctypes.byref(shp), _t4(q), _t4(k), _t4(v), int(window), _t4(out),
          lse.data_ptr(), _ptr(status), _stream())
    return out, lse


def fwd_partials(q, k, v, table, q_block, kv_block, causal=False, scale=None, status=None):
    """One (o, lse) per table entry (``sbfa_fwd_partials``): fp32
    o_parts (nmax, B, Sq, Hq, D) and lse_parts (nmax, B, Hq, Sq)."""
    _check_bf16(q, k, v)
    tb = _table(table, q_block, kv_block)
    B, Sq, Hq, D = q.shape
    o_parts = torch.empty(tb.nmax, B, Sq, Hq, D, dtype=torch.float32, device=q.device)
    lse_parts = torch.empty(tb.nmax, B, Hq, Sq, dtype=torch.float32, device=q.device)
    shp = _shape(q, k, causal, scale)
    _call("sbfa_fwd_partials", ctypes.byref(shp), _t4(q), _t4(k), _t4(v), ctypes.byref(tb),
          o_parts.data_ptr(), lse_parts.data_ptr(), _ptr(status), _stream())
    return o_parts, lse_parts


def combine(o_parts, lse_parts, out=None, lse=None):
    """LSE combine of fp32 partials (``sbfa_combine``). Returns (o bf16, lse)."""
    P, B, Sq, Hq, D = o_parts.shape
    o_parts = o_parts.contiguous()
    lse_parts = lse_parts.contiguous()
    if out is None:
        out = torch.empty(B, Sq, Hq, D, dtype=torch.bfloat16, device=o_parts.device)
    if lse is None:
        lse = torch.empty(B, Hq, Sq, dtype=torch.float32, device=o_parts.device)
    _call("sbfa_combine", P, B, Sq, Hq, D, o_parts.data_ptr(), lse_parts.data_ptr(), _t4(out),
          lse.data_ptr(), _stream())
    return out, lse


def decode_workspace(B, Hkv, Sq, Hq, device=None):
    """Zero-filled workspace for ``speculative_sparse`` (reusable across calls)."""
    n = lib.sbfa_decode_workspace_size(B, Hkv, Sq, Hq)
    if n == 0:
        raise SbfaError("sbfa_decode_workspace_size", ERR_CUDA)
    return torch.zeros(n, dtype=torch.uint8, device=device)


def speculative_sparse(q, k_spec, v_spec, causal_spec, k, v, table, kv_block, scale=None,
                       ws=None, out=None, lse=None, status=None):
    """Fused two-pass speculative + sparse decode (``sbfa_speculative_sparse``)."""
    _check_bf16(q, k_spec, v_spec, k, v)
    out, lse = _outputs(q, out, lse)
    B, Sq, Hq, D = q.shape
    if ws is None:
        ws = decode_workspace(B, k.shape[2], Sq, Hq, q.device)
    tb = _table(table, max(Sq, 1), kv_block)
    shp = _shape(q, k, False, scale)
    _call("sbfa_speculative_sparse", ctypes.byref(shp), _t4(q), _t4(k_spec), _t4(v_spec),
          k_spec.shape[1], int(bool(causal_spec)), _t4(k), _t4(v), ctypes.byref(tb),
          ws.data_ptr(), ws.numel(), _t4(out), lse.data_ptr(), _ptr(status), _stream())
    return out, lse


def speculative_sparse_noalloc(q, k_spec, v_spec, causal_spec, k, v, table, kv_block,
                               scale=None, out=None, lse=None, status=None):
    """``sbfa_speculative_sparse_noalloc``: the fused decode with the
    library's fixed scratch instead of a workspace (for callers that cannot
    allocate).  Pass preallocated ``out``/``lse`` to allocate nothing here
    either.  Calls that overlap on the GPU race on the shared scratch."""
    _check_bf16(q, k_spec, v_spec, k, v)
    out, lse = _outputs(q, out, lse)
    tb = _table(table, max(q.shape[1], 1), kv_block)
    shp = _shape(q, k, False, scale)
    _call("sbfa_speculative_sparse_noalloc", ctypes.byref(shp), _t4(q), _t4(k_spec),
          _t4(v_spec), k_spec.shape[1], int(bool(causal_spec)), _t4(k), _t4(v),
          ctypes.byref(tb), _t4(out), lse.data_ptr(), _ptr(status), _stream())
    return out, lse


def fwd_gated(q, k, v, T, block=64, scale=None, out=None, lse=None, smax_out=None,
              keep_out=None, status=None):
    """BSFA gated causal prefill (``sbfa_fwd_gated``); T fp32 (Hq, nQB)."""
    _check_bf16(q, k, v)
    out, lse = _outputs(q, out, lse)
    if T.dtype != torch.float32 or not T.is_contiguous():
        raise TypeError("T must be contiguous fp32")
    shp = _shape(q, k, True, scale)
    _call("sbfa_fwd_gated", ctypes.byref(shp), _t4(q), _t4(k), _t4(v), T.data_ptr(), block,
          _t4(out), lse.data_ptr(), _ptr(smax_out), _ptr(keep_out), _ptr(status), _stream())
    return out, lse


def convert_vertical_slash(q_seqlens, kv_seqlens, vertical, slash, context_size, block_M=64,
                           block_N=64, causal=True, status=None):
    """Vertical/slash indices -> (block_count, block_offset, column_count,
    column_index) (``sbfa_convert_vertical_slash``).  Entries past a count
    are unspecified."""
    B, H, nnz_v = vertical.shape
    nnz_s = slash.shape[2]
    nqb = -(-context_size // block_M)
    dev = vertical.device
    for t in (q_seqlens, kv_seqlens, vertical, slash):
        if t.dtype != torch.int32 or not t.is_contiguous():
            raise TypeError("index inputs must be contiguous int32")
    bc = torch.empty(B, H, nqb, dtype=torch.int32, device=dev)
    bo = torch.empty(B, H, nqb, nnz_s, dtype=torch.int32, device=dev)
    cc = torch.empty(B, H, nqb, dtype=torch.int32, device=dev)
    ci = torch.empty(B, H, nqb, nnz_v, dtype=torch.int32, device=dev)
    _call("sbfa_convert_vertical_slash", q_seqlens.data_ptr(), kv_seqlens.data_ptr(),
          vertical.data_ptr(), nnz_v, slash.data_ptr(), nnz_s, B, H, context_size, block_M,
          block_N, int(bool(causal)), bc.data_ptr(), bo.data_ptr(), cc.data_ptr(),
          ci.data_ptr(), _ptr(status), _stream())
    return bc, bo, cc, ci


def convert_vertical_slash_mergehead(q_seqlens, kv_seqlens, vertical, slash, vertical_count,
                                     slash_count, context_size, block_M=64, block_N=64,
                                     causal=True, status=None):
    """``sbfa_convert_vertical_slash_mergehead``: as convert_vertical_slash,
    with head h using only the first vertical_count[h] / slash_count[h]
    entries of its rows (int32 (H,) device tensors)."""
    B, H, nnz_v = vertical.shape
    nnz_s = slash.shape[2]
    nqb = -(-context_size // block_M)
    dev = vertical.device
    for t in (q_seqlens, kv_seqlens, vertical, slash, vertical_count, slash_count):
        if t.dtype != torch.int32 or not t.is_contiguous():
            raise TypeError("index inputs must be contiguous int32")
    bc = torch.empty(B, H, nqb, dtype=torch.int32, device=dev)
    bo = torch.empty(B, H, nqb, nnz_s, dtype=torch.int32, device=dev)
    cc = torch.empty(B, H, nqb, dtype=torch.int32, device=dev)
    ci = torch.empty(B, H, nqb, nnz_v, dtype=torch.int32, device=dev)
    _call("sbfa_convert_vertical_slash_mergehead", q_seqlens.data_ptr(), kv_seqlens.data_ptr(),
          vertical.data_ptr(), nnz_v, slash.data_ptr(), nnz_s, vertical_count.data_ptr(),
          slash_count.data_ptr(), B, H, context_size, block_M, block_N, int(bool(causal)),
          bc.data_ptr(), bo.data_ptr(), cc.data_ptr(), ci.data_ptr(), _ptr(status), _stream())
    return bc, bo, cc, ci


def _varlen_args(q, k, cu_seqlens_q, cu_seqlens_k):
    for t in (cu_seqlens_q, cu_seqlens_k):
        if t.dtype != torch.int32 or not t.is_cuda or not t.is_contiguous():
            raise TypeError("cu_seqlens must be contiguous int32 CUDA tensors")
    if q.dim() != 3 or k.dim() != 3:
        raise ValueError("varlen q, k, v are (total, heads, dim)")
    return cu_seqlens_q.numel() - 1, q.shape[0], k.shape[0]


def fwd_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, table, q_block,
               kv_block, causal=False, scale=None, out=None, lse=None, status=None):
    """Block-table attention over cu_seqlens-packed sequences
    (``sbfa_fwd_varlen``).  q (total_q, Hq, D), k/v (total_k, Hkv, D), table
    int32 (nseq, Hkv, nQB, nmax) of sequence-local blocks.  Returns
    o (total_q, Hq, D), lse (Hq, total_q)."""
    _check_bf16(q, k, v)
    nseq, tq, tk = _varlen_args(q, k, cu_seqlens_q, cu_seqlens_k)
    Hq, D = q.shape[1], q.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(Hq, tq, dtype=torch.float32, device=q.device)
    tb = _table(table, q_block, kv_block)
    _call("sbfa_fwd_varlen", cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), nseq, tq, tk,
          int(max_seqlen_q), int(max_seqlen_k), Hq, k.shape[1], D,
          0.0 if scale is None else float(scale), int(bool(causal)), _t4(q[None]), _t4(k[None]),
          _t4(v[None]), ctypes.byref(tb), _t4(out[None]), lse.data_ptr(), _ptr(status), _stream())
    return out, lse


def fwd_vertical_slash_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k,
                              block_count, block_offset, column_count, column_index, causal=True,
                              scale=None, block_M=64, block_N=64, out=None, lse=None,
                              status=None):
    """``sbfa_fwd_vertical_slash_varlen``: vertical/slash attention over
    cu_seqlens-packed sequences; index arrays (nseq, Hq, ceil(max_seqlen_q /
    64), nnz).  Returns o (total_q, Hq, D), lse (Hq, total_q)."""
    _check_bf16(q, k, v)
    nseq, tq, tk = _varlen_args(q, k, cu_seqlens_q, cu_seqlens_k)
    Hq, D = q.shape[1], q.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(Hq, tq, dtype=torch.float32, device=q.device)
    _call("sbfa_fwd_vertical_slash_varlen", cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(),
          nseq, tq, tk, int(max_seqlen_q), int(max_seqlen_k), Hq, k.shape[1], D,
          0.0 if scale is None else float(scale), int(bool(causal)), _t4(q[None]), _t4(k[None]),
          _t4(v[None]), block_count.data_ptr(), block_offset.data_ptr(), block_offset.shape[-1],
          column_count.data_ptr(), column_index.data_ptr(), column_index.shape[-1], block_M,
          block_N, _t4(out[None]), lse.data_ptr(), _ptr(status), _stream())
    return out, lse


def fwd_window_varlen(q, k, v, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, window,
                      scale=None, out=None, lse=None, status=None):
    """``sbfa_fwd_window_varlen``: causal sliding window over cu_seqlens-packed
    sequences.  Returns o (total_q, Hq, D), lse (Hq, total_q)."""
    _check_bf16(q, k, v)
    nseq, tq, tk = _varlen_args(q, k, cu_seqlens_q, cu_seqlens_k)
    Hq, D = q.shape[1], q.shape[2]
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(Hq, tq, dtype=torch.float32, device=q.device)
    _call("sbfa_fwd_window_varlen", cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), nseq, tq,
          tk, int(max_seqlen_q), int(max_seqlen_k), Hq, k.shape[1], D,
          0.0 if scale is None else float(scale), int(window), _t4(q[None]), _t4(k[None]),
          _t4(v[None]), _t4(out[None]), lse.data_ptr(), _ptr(status), _stream())
    return out, lse


def calibrate_thresholds(smax, k_top, T=None):
    """BSFA thresholds from block maxima (``sbfa_calibrate_thresholds``):
    smax fp32 (B, Hq, n, n) -> T fp32 (B, Hq, n), T[b, h, i] = k-th largest
    of smax[b, h, i, :i] (-inf when i < k)."""
    if smax.dtype != torch.float32 or not smax.is_contiguous() or smax.dim() != 4:
        raise TypeError("smax must be a contiguous fp32 (B, Hq, n, n) tensor")
    B, Hq, n, n2 = smax.shape
    if n != n2:
        raise ValueError("smax must be square in its last two dims")
    if T is None:
        T = torch.empty(B, Hq, n, dtype=torch.float32, device=smax.device)
    _call("sbfa_calibrate_thresholds", smax.data_ptr(), B, Hq, n, int(k_top), T.data_ptr(),
          _stream())
    return T


def fwd_vertical_slash(q, k, v, block_count, block_offset, column_count, column_index,
                       causal=True, scale=None, block_M=64, block_N=64, out=None, lse=None,
                       status=None):
    """Sparse attention over converted vertical/slash lists
    (``sbfa_fwd_vertical_slash``)."""
    _check_bf16(q, k, v)
    out, lse = _outputs(q, out, lse)
    shp = _shape(q, k, causal, scale)
    _call("sbfa_fwd_vertical_slash", ctypes.byref(shp), _t4(q), _t4(k), _t4(v),
          block_count.data_ptr(), block_offset.data_ptr(), block_offset.shape[-1],
          column_count.data_ptr(), column_index.data_ptr(), column_index.shape[-1], block_M,
          block_N, _t4(out), lse.data_ptr(), _ptr(status), _stream())
    return out, lse


def varlen_selected_workspace(nseq, total, max_seqlen, Hq, Hkv, topk, device=None):
    n = lib.sbfa_varlen_selected_workspace_size(nseq, total, max_seqlen, Hq, Hkv, topk)
    if n == 0:
        raise SbfaError("sbfa_varlen_selected_workspace_size", ERR_INVALID_ARG)
    return torch.empty(n, dtype=torch.uint8, device=device)


def fwd_varlen_selected(q, k, v, cu_seqlens, max_seqlen, sel, block=64, causal=True,
                        scale=None, ws=None, out=None, lse=None, status=None):
    """NSA selected attention over varlen-packed sequences
    (``sbfa_fwd_varlen_selected``).  q (total, Hq, D), k/v (total, Hkv, D),
    sel int32 (total, Hkv, topk).  Returns o (total, Hq, D), lse (Hq, total)."""
    _check_bf16(q, k, v)
    total, Hq, D = q.shape
    Hkv, topk = k.shape[1], sel.shape[2]
    nseq = cu_seqlens.numel() - 1
    if sel.dtype != torch.int32 or not sel.is_contiguous() or cu_seqlens.dtype != torch.int32:
        raise TypeError("sel and cu_seqlens must be contiguous int32")
    if out is None:
        out = torch.empty_like(q)
    if lse is None:
        lse = torch.empty(Hq, total, dtype=torch.float32, device=q.device)
    if ws is None:
        ws = varlen_selected_workspace(nseq, total, max_seqlen, Hq, Hkv, topk, q.device)
    _call("sbfa_fwd_varlen_selected", cu_seqlens.data_ptr(), nseq, total, max_seqlen, Hq, Hkv, D,
          0.0 if scale is None else float(scale), int(bool(causal)), _t4(q[None]), _t4(k[None]),
          _t4(v[None]), sel.data_ptr(), topk, block, ws.data_ptr(), ws.numel(), _t4(out[None]),
          lse.data_ptr(), _ptr(status), _stream())
    return out, lse


def check_status(status):
    """Synchronise and map the device status word to an exception."""
    _call("sbfa_check_status", _ptr(status), _stream())


def set_wait_limit_ns(ns):
    """Limit of the bounded waits inside the pipelined kernels launched from
    now on (``sbfa_set_wait_limit_ns``; 0 restores the 2 s default).  Returns
    the previous limit."""
    return lib.sbfa_set_wait_limit_ns(int(ns))


def new_status(device=None):
    return torch.zeros(1, dtype=torch.int32, device=device)


def default_scale(d=128):
    return 1.0 / math.sqrt(d)
