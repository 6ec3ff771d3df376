"""Plain fp64 CPU oracle for the block-sparse FlashAttention forward.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import this module.  The product path (the
CUDA library and its Python binding) never calls it and shares no code with
it; this file imports nothing from the package.

Every function is the plain definition of what the method computes, written
as gathers, masks and matrix products in numpy fp64 -- no tiling, no online
softmax, no fusion.  Sources (page title, section):

* "Sparse FlashAttention with Incremental Repair" (Incremental_FlashAttention
  README), Usage 1-3: block-table attention, empty table -> (0, -inf),
  speculative + sparse decode merged by the LSE combine, per-block partials;
  "What's in this fork": FA(A u B) == Combine(FA(A), FA(B)).
* "Block Sparse Flash Attention" (BSFA), Abstract and Figure 2: exact
  per-block maxima s_max(i,j), calibrated thresholds T(l,h,i) (-inf where
  fewer than k off-diagonal candidates exist), keep iff s_max >= T, diagonal
  blocks always run.
* "Sglang Sparse Flash Attention", Description and I/O Contract:
  convert_vertical_slash_indexes -> block_count/block_offset (slash) and
  column_count/column_index (vertical); sparse attention over them.
* "Flash-Sparse-Attention (FSA)", Quickstart: NSA selected attention with
  per-token top-k key blocks of 64, cu_seqlens varlen packing.

Readings where the pages are silent are listed with each function.

Parity status: every function here is pinned by tests/test_oracle_pins.py
(dense brute force, library routines, closed forms, a hand-worked example).
The vertical/slash *reading* itself (aligned key blocks) is an assumption the
pages do not fix; the conversion is pinned only for that reading.
"""
from __future__ import annotations

import numpy as np

NEG_INF = -np.inf


def _f64(x) -> np.ndarray:
    """Exact fp64 values; a uint16 array is taken as bf16 bit patterns."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


# ----------------------------------------------------------------------------
# Core: softmax attention of some query rows over an explicit key set
# ----------------------------------------------------------------------------

def attend_keyset(qr, K, V, allowed, scale):
    """Softmax attention of rows ``qr`` (R, D) over keys K, V (N, D).

    ``allowed`` (R, N) bool marks which keys each row may see (None = all).
    Returns o (R, D) and natural-log lse (R,).  A row that sees no key gives
    o = 0, lse = -inf (Incremental_FlashAttention README, Usage 1: the empty
    table is a neutral partial)."""
    qr, K, V = _f64(qr), _f64(K), _f64(V)
    R = qr.shape[0]
    o = np.zeros((R, V.shape[1]))
    lse = np.full(R, NEG_INF)
    if K.shape[0] == 0 or R == 0:
        return o, lse
    s = scale * (qr @ K.T)
    if allowed is not None:
        s = np.where(allowed, s, NEG_INF)
    m = s.max(axis=1)
    live = np.isfinite(m)
    if not live.any():
        return o, lse
    w = np.exp(s[live] - m[live, None])
    l = w.sum(axis=1)
    o[live] = (w @ V) / l[:, None]
    lse[live] = m[live] + np.log(l)
    return o, lse


def _keys_of_blocks(blocks, kv_block, Sk):
    blocks = np.unique(np.asarray(blocks, dtype=np.int64))
    blocks = blocks[blocks >= 0]
    if blocks.size == 0:
        return np.zeros(0, dtype=np.int64)
    keys = (blocks[:, None] * kv_block + np.arange(kv_block)[None, :]).reshape(-1)
    return keys[keys < Sk]


# ----------------------------------------------------------------------------
# O1: block-table attention
# ----------------------------------------------------------------------------

def attend_block_table(q, k, v, table, q_block, kv_block, causal, scale, rows=None):
    """Attention of each query row over the K/V blocks its table row lists.

    q (B, Sq, Hq, D); k, v (B, Sk, Hkv, D); table int [B, Hkv, nQB, nmax].
    Row r of head h uses table[b, h // G, r // q_block, :]; entries < 0 are
    padding; repeated entries count once (a set).  Block j covers keys
    [j*kv_block, (j+1)*kv_block) clipped to Sk.  causal: key kk is visible to
    row r iff kk <= r + (Sk - Sq) (bottom-right alignment; the pages are
    silent, all workloads have Sq == Sk or Sq == 1).

    ``rows``: None (all rows) or a callable (b, h) -> sorted row indices.
    Returns o (B, Sq, Hq, D) and lse (B, Hq, Sq); rows not computed are NaN.
    """
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    o = np.full((B, Sq, Hq, D), np.nan)
    lse = np.full((B, Hq, Sq), np.nan)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            rr = np.arange(Sq) if rows is None else np.asarray(rows(b, h))
            if rr.size == 0:
                continue
            Kg, Vg = k[b, :, g, :], v[b, :, g, :]
            for qb in np.unique(rr // q_block):
                r = rr[rr // q_block == qb]
                keys = _keys_of_blocks(table[b, g, qb], kv_block, Sk)
                allowed = None
                if causal:
                    allowed = keys[None, :] <= (r[:, None] + (Sk - Sq))
                oo, ll = attend_keyset(q[b, r, h, :], Kg[keys], Vg[keys], allowed, scale)
                o[b, r, h, :] = oo
                lse[b, h, r] = ll
    return o, lse


# ----------------------------------------------------------------------------
# O2: dense brute force with an element mask (tiny inputs only)
# ----------------------------------------------------------------------------

def element_mask_from_table(Sq, Sk, Hq, Hkv, table_b, q_block, kv_block, causal):
    """bool [Hq, Sq, Sk] built one element at a time from one batch's table."""
    G = Hq // Hkv
    mask = np.zeros((Hq, Sq, Sk), dtype=bool)
    for h in range(Hq):
        for r in range(Sq):
            listed = set(int(j) for j in table_b[h // G, r // q_block] if j >= 0)
            for kk in range(Sk):
                ok = (kk // kv_block) in listed
                if causal and kk > r + (Sk - Sq):
                    ok = False
                mask[h, r, kk] = ok
    return mask


def attend_dense_masked(q, k, v, mask, scale):
    """Dense softmax attention over all Sk keys with an element mask.

    q (Sq, Hq, D), k/v (Sk, Hkv, D), mask bool [Hq, Sq, Sk].  Uses an explicit
    sum of exponentials per row (no shared helper with attend_keyset)."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    Sq, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    o = np.zeros((Sq, Hq, D))
    lse = np.full((Hq, Sq), NEG_INF)
    for h in range(Hq):
        s = scale * (q[:, h, :] @ k[:, h // G, :].T)
        for r in range(Sq):
            vis = np.nonzero(mask[h, r])[0]
            if vis.size == 0:
                continue
            row = s[r, vis]
            top = row.max()
            e = np.exp(row - top)
            tot = e.sum()
            o[r, h] = (e[:, None] * v[vis, h // G, :]).sum(axis=0) / tot
            lse[h, r] = top + np.log(tot)
    return o, lse


# ----------------------------------------------------------------------------
# O3: LSE combine of partial results over disjoint key sets
# ----------------------------------------------------------------------------

def combine(o_parts, lse_parts):
    """Merge P partials (o_p, lse_p) into (o, lse).

    o_parts (P, ..., D), lse_parts (P, ...).  M = max_p lse_p;
    w_p = exp(lse_p - M); lse = M + ln sum w_p; o = sum w_p o_p / sum w_p.
    If every partial is empty (lse = -inf) the result is (0, -inf)."""
    o_parts, lse_parts = _f64(o_parts), _f64(lse_parts)
    M = lse_parts.max(axis=0)
    live = np.isfinite(M)
    Ms = np.where(live, M, 0.0)
    w = np.where(np.isfinite(lse_parts), np.exp(lse_parts - Ms[None]), 0.0)
    wsum = w.sum(axis=0)
    safe = np.where(live, wsum, 1.0)
    o = (w[..., None] * np.nan_to_num(o_parts)).sum(axis=0) / safe[..., None]
    o = np.where(live[..., None], o, 0.0)
    lse = np.where(live, Ms + np.log(safe), NEG_INF)
    return o, lse


def combine_bshd(o_parts, lse_parts):
    """combine() for partials in the attention layouts: o_parts
    (P, B, Sq, Hq, D) and lse_parts (P, B, Hq, Sq); returns o (B, Sq, Hq, D),
    lse (B, Hq, Sq)."""
    o, lse = combine(o_parts, np.swapaxes(_f64(lse_parts), -1, -2))
    return o, np.swapaxes(lse, -1, -2)


def speculative_sparse(q, k_spec, v_spec, causal_spec, k, v, table, kv_block, scale):
    """Two-pass decode: dense attention over (k_spec, v_spec) with optional
    causal mask, sparse attention over the table's (missed) blocks of (k, v)
    with no mask, then the LSE combine (Incremental_FlashAttention README,
    Usage 2).  table int [B, Hkv, 1, nmax] (one q-block covers all Sq rows)."""
    B, Sq, Hq, D = q.shape
    S_spec = k_spec.shape[1]
    Hkv = k.shape[2]
    full = np.zeros((B, Hkv, 1, 1), dtype=np.int64)
    oa, la = attend_block_table(q, k_spec, v_spec, full, max(Sq, 1), S_spec,
                                causal_spec, scale)
    ob, lb = attend_block_table(q, k, v, table, max(Sq, 1), kv_block, False, scale)
    return combine_bshd(np.stack([oa, ob]), np.stack([la, lb]))


# ----------------------------------------------------------------------------
# O4: BSFA per-block max, calibrated threshold, gate
# ----------------------------------------------------------------------------

def block_max_head(qh, kh, block, scale, i_list=None):
    """s_max[i, j] = max over rows r of q-block i and keys c of k-block j of
    scale * q_r.k_c, for one head: qh (L, D), kh (L, D), causal (c <= r).
    Only candidates j <= i are evaluated; the rest are -inf.  (BSFA, Figure
    2a: per-block maxima computed exactly inside the attention tile, where
    the causal mask hides c > r; this only matters on the diagonal block,
    which is always kept.)"""
    qh, kh = _f64(qh), _f64(kh)
    L = qh.shape[0]
    n = -(-L // block)
    i_list = range(n) if i_list is None else i_list
    out = np.full((n, n), NEG_INF)
    for i in i_list:
        r0, r1 = i * block, min((i + 1) * block, L)
        kend = min((i + 1) * block, L)
        s = scale * (qh[r0:r1] @ kh[:kend].T)          # (rows, keys <= end of block i)
        s = np.where(np.arange(kend)[None, :] <= np.arange(r0, r1)[:, None], s, NEG_INF)
        pad = (i + 1) * block - kend                   # ragged last key block
        if pad:
            s = np.concatenate([s, np.full((s.shape[0], pad), NEG_INF)], axis=1)
        out[i, :i + 1] = s.reshape(s.shape[0], i + 1, block).max(axis=(0, 2))
    return out


def calibrate_thresholds(smax, k_top):
    """T[h, i] = k-th largest off-diagonal block max {s_max[h,i,j] : j < i}
    (with multiplicity); -inf when fewer than k candidates exist (BSFA,
    Figure 2a).  smax (Hq, n, n)."""
    Hq, n, _ = smax.shape
    T = np.full((Hq, n), NEG_INF)
    for h in range(Hq):
        for i in range(n):
            if i < k_top:
                continue
            cand = np.sort(smax[h, i, :i])[::-1]
            T[h, i] = cand[k_top - 1]
    return T


def gate_keep(smax, T):
    """keep[h, i, j] for causal candidates j <= i: the diagonal always runs,
    an off-diagonal block runs iff s_max >= T[h, i] (BSFA, Figure 2b)."""
    Hq, n, _ = smax.shape
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    cand = (j <= i)[None]
    keep = (smax >= T[:, :, None]) | (j == i)[None]
    return keep & cand


def attend_gated(q, k, v, T, block, scale, rows=None, return_keep=False):
    """Gated causal attention (BSFA): for each head h and q-block i, attend
    the kept key blocks with the causal element mask.  q (B, L, Hq, D),
    k/v (B, L, Hkv, D), T (Hq, nQB) (compared in fp64 against the given
    values).  ``rows``: None or callable (b, h) -> rows (whole q-blocks are
    evaluated for the gate either way).  Returns o, lse and, optionally, a
    dict {(b, h, i): (smax_row (i+1,), keep_row (i+1,))} for evaluated i."""
    B, L, Hq, D = q.shape
    Hkv = k.shape[2]
    G = Hq // Hkv
    n = -(-L // block)
    T = _f64(T)
    o = np.full((B, L, Hq, D), np.nan)
    lse = np.full((B, Hq, L), np.nan)
    info = {}
    for b in range(B):
        for h in range(Hq):
            g = h // G
            rr = np.arange(L) if rows is None else np.asarray(rows(b, h))
            qh, kh = _f64(q[b, :, h, :]), _f64(k[b, :, g, :])
            for i in np.unique(rr // block):
                r = rr[rr // block == i]
                sm = block_max_head(qh, kh, block, scale, [i])[i, :i + 1]
                keep = (sm >= T[h, i]) | (np.arange(i + 1) == i)
                keys = _keys_of_blocks(np.nonzero(keep)[0], block, L)
                allowed = keys[None, :] <= r[:, None]
                oo, ll = attend_keyset(q[b, r, h, :], k[b, keys, g, :], v[b, keys, g, :],
                                       allowed, scale)
                o[b, r, h, :] = oo
                lse[b, h, r] = ll
                info[(b, h, int(i))] = (sm, keep)
    if return_keep:
        return o, lse, info
    return o, lse


def kept_density_closed_form(n, k_top):
    """Kept fraction of causal tiles when exactly min(i, k) off-diagonal
    blocks pass in row i plus the diagonal: sum_i (min(i,k)+1) / (n(n+1)/2)."""
    kept = sum(min(i, k_top) + 1 for i in range(n))
    return kept / (n * (n + 1) / 2)


# ----------------------------------------------------------------------------
# O5: vertical/slash index conversion and attention
# ----------------------------------------------------------------------------

def convert_vertical_slash(q_seqlens, kv_seqlens, vertical, slash, context_size,
                           block_M, block_N, causal=True, qblocks=None, v_count=None,
                           s_count=None):
    """Per (b, h, q-block i), rows [m0, m1) with m1 = min(m0 + BM, q_len):

    * a slash offset s is the diagonal key = row + (kv_len - q_len) - s; over
      the block's rows it covers keys [m0+d-s, m1-1+d-s] clipped to
      [0, kv_len); U_i = union of these intervals;
    * block_offset = ascending BN-aligned offsets j*BN of every key block that
      meets U_i, block_count = their number;
    * column_index = ascending vertical columns v < kv_len (and, if causal,
      v <= m1-1+d) that lie in no listed block, column_count = their number.
    Entries past the counts are 0.  (Sglang Sparse Flash Attention, I/O
    contract; the aligned-block reading is an assumption.)  ``qblocks``:
    None (every q-block) or the q-block indices to convert; the others are
    left at count 0.  ``v_count`` / ``s_count``: None, or per-head numbers
    of entries in use (convert_vertical_slash_indexes_mergehead: head h reads
    only the first v_count[h] / s_count[h] entries of its rows)."""
    B, H, nnz_v = vertical.shape
    nnz_s = slash.shape[2]
    nqb = -(-context_size // block_M)
    bc = np.zeros((B, H, nqb), dtype=np.int32)
    bo = np.zeros((B, H, nqb, nnz_s), dtype=np.int32)
    cc = np.zeros((B, H, nqb), dtype=np.int32)
    ci = np.zeros((B, H, nqb, nnz_v), dtype=np.int32)
    for b in range(B):
        ql, kl = int(q_seqlens[b]), int(kv_seqlens[b])
        d = kl - ql
        nkb = -(-kl // block_N)
        for h in range(H):
            ns = nnz_s if s_count is None else min(max(int(s_count[h]), 0), nnz_s)
            nv = nnz_v if v_count is None else min(max(int(v_count[h]), 0), nnz_v)
            s = slash[b, h, :ns].astype(np.int64)
            vv = vertical[b, h, :nv].astype(np.int64)
            for i in (range(nqb) if qblocks is None else qblocks):
                m0 = i * block_M
                if m0 >= ql:
                    continue
                m1 = min(m0 + block_M, ql)
                lo = np.maximum(m0 + d - s, 0)
                hi = np.minimum(m1 - 1 + d - s, kl - 1)
                ok = hi >= lo
                hit = np.zeros(nkb, dtype=bool)
                for a, z in zip(lo[ok], hi[ok]):
                    hit[a // block_N:z // block_N + 1] = True
                blocks = np.nonzero(hit)[0]
                bc[b, h, i] = blocks.size
                bo[b, h, i, :blocks.size] = blocks * block_N
                cols = vv[(vv >= 0) & (vv < kl)]
                if causal:
                    cols = cols[cols <= m1 - 1 + d]
                cols = cols[~hit[cols // block_N]]
                cols = np.unique(cols)
                cc[b, h, i] = cols.size
                ci[b, h, i, :cols.size] = cols
    return bc, bo, cc, ci


def attend_vertical_slash(q, k, v, block_count, block_offset, column_count,
                          column_index, block_M, block_N, causal, scale, rows=None):
    """Row r of q-block i attends keys in the listed blocks
    [off, off+BN) and the listed columns, clipped to Sk, with the causal
    element mask (bottom-right).  Shapes as in attend_block_table."""
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    o = np.full((B, Sq, Hq, D), np.nan)
    lse = np.full((B, Hq, Sq), np.nan)
    for b in range(B):
        for h in range(Hq):
            g = h // G
            rr = np.arange(Sq) if rows is None else np.asarray(rows(b, h))
            for i in np.unique(rr // block_M):
                r = rr[rr // block_M == i]
                offs = block_offset[b, h, i, :block_count[b, h, i]].astype(np.int64)
                bk = (offs[:, None] + np.arange(block_N)[None, :]).reshape(-1)
                cols = column_index[b, h, i, :column_count[b, h, i]].astype(np.int64)
                keys = np.unique(np.concatenate([bk, cols]))
                keys = keys[(keys >= 0) & (keys < Sk)]
                allowed = None
                if causal:
                    allowed = keys[None, :] <= (r[:, None] + (Sk - Sq))
                oo, ll = attend_keyset(q[b, r, h, :], k[b, keys, g, :], v[b, keys, g, :],
                                       allowed, scale)
                o[b, r, h, :] = oo
                lse[b, h, r] = ll
    return o, lse


# ----------------------------------------------------------------------------
# Causal sliding window (NSA's window branch, Flash-Sparse-Attention Quickstart)
# ----------------------------------------------------------------------------

def attend_window(q, k, v, window, scale, rows=None):
    """Row r attends the keys r + (Sk - Sq) - window < key <= r + (Sk - Sq)
    (bottom-right causal window of ``window`` keys ending at the row's own
    position).  Shapes and ``rows`` as in attend_block_table."""
    B, Sq, Hq, D = q.shape
    Sk, Hkv = k.shape[1], k.shape[2]
    G = Hq // Hkv
    off = Sk - Sq
    o = np.full((B, Sq, Hq, D), np.nan)
    lse = np.full((B, Hq, Sq), np.nan)
    for b in range(B):
        for h in range(Hq):
            rr = np.arange(Sq) if rows is None else np.asarray(rows(b, h))
            for r in rr:
                hi = r + off                       # last visible key
                keys = np.arange(max(0, hi - window + 1), min(Sk, hi + 1))
                oo, ll = attend_keyset(q[b, r:r + 1, h, :], k[b, keys, h // G, :],
                                       v[b, keys, h // G, :], None, scale)
                o[b, r, h, :] = oo[0]
                lse[b, h, r] = ll[0]
    return o, lse


def attend_window_varlen(q, k, v, cu_q, cu_k, window, scale):
    """attend_window on each packed sequence."""
    return _varlen_apply(lambda qs, ks, vs, s: attend_window(qs, ks, vs, window, scale),
                         q, k, v, cu_q, cu_k)


# ----------------------------------------------------------------------------
# Varlen packing (cu_seqlens): each sequence on its own
# ----------------------------------------------------------------------------

def _varlen_apply(fn, q, k, v, cu_q, cu_k):
    """Run fn(q_s, k_s, v_s, s) -> (o (1, Lq, Hq, D), lse (1, Hq, Lq)) on
    every packed sequence s and pack the results as o (Tq, Hq, D), lse
    (Hq, Tq) (Flash-Sparse-Attention Quickstart; Sglang sparse_attn_varlen_func:
    cu_seqlens_q / cu_seqlens_k give each sequence's rows)."""
    cu_q, cu_k = np.asarray(cu_q, dtype=np.int64), np.asarray(cu_k, dtype=np.int64)
    Tq, Hq, D = q.shape
    o = np.full((Tq, Hq, D), np.nan)
    lse = np.full((Hq, Tq), np.nan)
    for s in range(len(cu_q) - 1):
        a, z = cu_q[s], cu_q[s + 1]
        ka, kz = cu_k[s], cu_k[s + 1]
        if z == a:
            continue
        oo, ll = fn(q[None, a:z], k[None, ka:kz], v[None, ka:kz], s)
        o[a:z] = oo[0]
        lse[:, a:z] = ll[0]
    return o, lse


def attend_block_table_varlen(q, k, v, cu_q, cu_k, table, q_block, kv_block, causal, scale):
    """attend_block_table on each packed sequence: table[s] is its
    [Hkv, nQB, nmax] table of sequence-local blocks; causal is bottom-right
    within the sequence."""
    return _varlen_apply(lambda qs, ks, vs, s: attend_block_table(
        qs, ks, vs, table[s:s + 1], q_block, kv_block, causal, scale), q, k, v, cu_q, cu_k)


def attend_vertical_slash_varlen(q, k, v, cu_q, cu_k, block_count, block_offset, column_count,
                                 column_index, block_M, block_N, causal, scale):
    """attend_vertical_slash on each packed sequence with its converted lists
    (index arrays [nseq, Hq, nQB, nnz], sequence-local offsets and columns)."""
    def one(qs, ks, vs, s):
        sl = slice(s, s + 1)
        return attend_vertical_slash(qs, ks, vs, block_count[sl], block_offset[sl],
                                     column_count[sl], column_index[sl], block_M, block_N,
                                     causal, scale)
    return _varlen_apply(one, q, k, v, cu_q, cu_k)


# ----------------------------------------------------------------------------
# O6: NSA selected attention over varlen-packed sequences
# ----------------------------------------------------------------------------

def attend_selected_varlen(q, k, v, cu_seqlens, sel, block, causal, scale, rows=None):
    """Token t (local index tl in its sequence) of head h attends the keys of
    its selected blocks sel[t, h // G, :] (>= 0; sequence-local block
    indices of ``block`` keys), clipped to the sequence and, if causal, to
    keys <= tl.  q (T, Hq, D), k/v (T, Hkv, D) packed by cu_seqlens.
    ``rows``: None or callable (h) -> global token indices.
    Returns o (T, Hq, D), lse (Hq, T); rows not computed are NaN."""
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    G = Hq // Hkv
    cu = np.asarray(cu_seqlens, dtype=np.int64)
    o = np.full((T, Hq, D), np.nan)
    lse = np.full((Hq, T), np.nan)
    for h in range(Hq):
        g = h // G
        tt = np.arange(T) if rows is None else np.asarray(rows(h))
        for t in tt:
            s = np.searchsorted(cu, t, side="right") - 1
            base, L = cu[s], cu[s + 1] - cu[s]
            tl = t - base
            keys = _keys_of_blocks(sel[t, g], block, L)
            if causal:
                keys = keys[keys <= tl]
            oo, ll = attend_keyset(q[t:t + 1, h, :], k[base + keys, g, :],
                                   v[base + keys, g, :], None, scale)
            o[t, h] = oo[0]
            lse[h, t] = ll[0]
    return o, lse
