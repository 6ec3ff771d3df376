"""Pins for the fp64 oracle against things other than itself: library
routines (torch SDPA in fp64, scipy logsumexp, heapq), element-by-element
brute force on tiny inputs, closed forms and a hand-worked example."""
import heapq
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(rng, *shape):
    return rng.standard_normal(shape)


def _sdpa_dense(q, k, v, scale, causal_mask=None):
    """Library reference: torch SDPA in fp64 on CPU over all keys.
    q (Sq, Hq, D), k/v (Sk, Hkv, D); GQA by repeating kv heads."""
    Hq, Hkv = q.shape[1], k.shape[1]
    G = Hq // Hkv
    qt = torch.from_numpy(q).permute(1, 0, 2)[None]
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(G, 0)[None]
    mask = None if causal_mask is None else torch.from_numpy(causal_mask)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    return o[0].permute(1, 0, 2).numpy()


# ---------------------------------------------------------------- O1 vs library

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("G", [1, 4])
def test_full_table_equals_dense_sdpa(causal, G):
    rng = np.random.default_rng(0)
    B, Sq, Sk, Hkv, D, bs = 2, 70, 96, 2, 16, 16
    Hq = Hkv * G
    q, k, v = _rand(rng, B, Sq, Hq, D), _rand(rng, B, Sk, Hkv, D), _rand(rng, B, Sk, Hkv, D)
    nkb = Sk // bs
    table = np.broadcast_to(np.arange(nkb, dtype=np.int32), (B, Hkv, 1, nkb))
    scale = 0.3
    o, lse = oracle.attend_block_table(q, k, v, table, Sq, bs, causal, scale)
    for b in range(B):
        cm = None
        if causal:
            cm = np.arange(Sk)[None, :] <= np.arange(Sq)[:, None] + (Sk - Sq)
        ref = _sdpa_dense(q[b], k[b], v[b], scale, cm)
        np.testing.assert_allclose(o[b], ref, rtol=0, atol=1e-12)
        for h in range(Hq):
            s = scale * q[b, :, h, :] @ k[b, :, h // G, :].T
            if causal:
                s = np.where(cm, s, -np.inf)
            np.testing.assert_allclose(lse[b, h], logsumexp(s, axis=1), rtol=0, atol=1e-12)


# ---------------------------------------------------------------- O1 vs O2 brute force

@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("shape", [
    # B, Sq, Sk, Hq, Hkv, q_block, kv_block, nmax
    (1, 40, 40, 2, 2, 8, 8, 3),
    (2, 33, 50, 4, 2, 16, 8, 4),      # ragged Sk tail, Sq != Sk, GQA
    (1, 24, 64, 2, 1, 24, 16, 5),
])
def test_block_table_vs_elementwise(causal, shape):
    B, Sq, Sk, Hq, Hkv, qbs, kbs, nmax = shape
    rng = np.random.default_rng(hash(shape) % 2**32)
    D = 8
    q, k, v = _rand(rng, B, Sq, Hq, D), _rand(rng, B, Sk, Hkv, D), _rand(rng, B, Sk, Hkv, D)
    nqb, nkb = -(-Sq // qbs), -(-Sk // kbs)
    table = rng.integers(-1, nkb, size=(B, Hkv, nqb, nmax)).astype(np.int32)
    table[..., -1] = table[..., 0]          # a duplicate entry counts once
    o, lse = oracle.attend_block_table(q, k, v, table, qbs, kbs, causal, 0.5)
    for b in range(B):
        mask = oracle.element_mask_from_table(Sq, Sk, Hq, Hkv, table[b], qbs, kbs, causal)
        ob, lb = oracle.attend_dense_masked(q[b], k[b], v[b], mask, 0.5)
        np.testing.assert_allclose(o[b], ob, rtol=0, atol=1e-12)
        np.testing.assert_array_equal(np.isneginf(lse[b]), np.isneginf(lb))
        fin = np.isfinite(lb)
        np.testing.assert_allclose(lse[b][fin], lb[fin], rtol=0, atol=1e-12)


def test_empty_table_is_neutral():
    rng = np.random.default_rng(1)
    q, k, v = _rand(rng, 1, 5, 2, 8), _rand(rng, 1, 32, 2, 8), _rand(rng, 1, 32, 2, 8)
    table = np.full((1, 2, 1, 4), -1, dtype=np.int32)
    o, lse = oracle.attend_block_table(q, k, v, table, 5, 8, False, 1.0)
    assert np.all(o == 0) and np.all(np.isneginf(lse))


# ---------------------------------------------------------------- O3 combine

@pytest.mark.parametrize("n_parts", [2, 3, 4])
def test_combine_identity_random_disjoint_splits(n_parts):
    rng = np.random.default_rng(10 + n_parts)
    B, Sq, Sk, Hq, Hkv, bs = 2, 16, 128, 4, 2, 16
    D = 8
    q, k, v = _rand(rng, B, Sq, Hq, D), _rand(rng, B, Sk, Hkv, D), _rand(rng, B, Sk, Hkv, D)
    nkb = Sk // bs
    for trial in range(5):
        blocks = rng.permutation(nkb)[: rng.integers(1, nkb + 1)]
        cut = np.sort(rng.integers(0, len(blocks) + 1, size=n_parts - 1))
        parts = np.split(blocks, cut)            # some parts may be empty
        union_tab = np.full((B, Hkv, 1, nkb), -1, dtype=np.int32)
        union_tab[..., :len(blocks)] = blocks
        ou, lu = oracle.attend_block_table(q, k, v, union_tab, Sq, bs, False, 0.7)
        os_, ls_ = [], []
        for p in parts:
            t = np.full((B, Hkv, 1, nkb), -1, dtype=np.int32)
            t[..., :len(p)] = p
            o, l = oracle.attend_block_table(q, k, v, t, Sq, bs, False, 0.7)
            os_.append(o)
            ls_.append(l)
        oc, lc = oracle.combine_bshd(np.stack(os_), np.stack(ls_))
        np.testing.assert_allclose(oc, ou, rtol=0, atol=1e-12)
        np.testing.assert_allclose(lc, lu, rtol=0, atol=1e-12)


def test_combine_all_empty_and_one_empty():
    o = np.ones((3, 2, 4))
    lse = np.full((3, 2), -np.inf)
    oc, lc = oracle.combine(o, lse)
    assert np.all(oc == 0) and np.all(np.isneginf(lc))
    lse2 = lse.copy()
    lse2[1] = [0.5, -1.0]
    oc, lc = oracle.combine(o * np.arange(1, 4)[:, None, None], lse2)
    np.testing.assert_allclose(oc, 2.0, atol=1e-15)
    np.testing.assert_allclose(lc, [0.5, -1.0], atol=1e-15)


def test_hand_worked_two_block_example():
    g = json.load(open(os.path.join(GOLDEN, "hand_two_block.json")))
    q = np.array(g["q"])[None, :, None, :]            # (1, 1, 1, 2)
    k = np.array(g["k"])[None, :, None, :]
    v = np.array(g["v"])[None, :, None, :]
    bs = g["kv_block"]

    def run(blocks):
        t = np.array(blocks, dtype=np.int32).reshape(1, 1, 1, -1)
        o, l = oracle.attend_block_table(q, k, v, t, 1, bs, False, 1.0)
        return o[0, 0, 0], l[0, 0, 0]

    for key, blocks in (("A_only", [0]), ("B_only", [1]), ("union", [0, 1])):
        o, l = run(blocks)
        np.testing.assert_allclose(o, g[key]["o"], atol=1e-14)
        assert abs(l - g[key]["lse"]) < 1e-14
    oa, la = run([0])
    ob, lb = run([1])
    oc, lc = oracle.combine(np.stack([oa, ob]), np.array([la, lb]))
    np.testing.assert_allclose(oc, g["union"]["o"], atol=1e-14)
    assert abs(lc - g["union"]["lse"]) < 1e-14
    # Gate: q-block 1's diagonal is A (always runs); its off-diagonal is B.
    sm = np.full((1, 2, 2), -np.inf)
    sm[0, 1, 0] = g["gate"]["s_max_B"]
    sm[0, 1, 1] = math.log(3.0)
    for T, expect in ((g["gate"]["T_skip"], False), (g["gate"]["T_keep"], True)):
        keep = oracle.gate_keep(sm, np.array([[-np.inf, T]]))
        assert bool(keep[0, 1, 1]) is True
        assert bool(keep[0, 1, 0]) is expect


# ---------------------------------------------------------------- O4 block max / gate

def test_block_max_vs_elementwise():
    rng = np.random.default_rng(3)
    L, D, bs = 45, 6, 8                      # ragged last block
    qh, kh = _rand(rng, L, D), _rand(rng, L, D)
    sm = oracle.block_max_head(qh, kh, bs, 0.4)
    n = -(-L // bs)
    for i in range(n):
        for j in range(n):
            if j > i:
                assert sm[i, j] == -np.inf
                continue
            best = -np.inf
            for r in range(i * bs, min((i + 1) * bs, L)):
                for c in range(j * bs, min((j + 1) * bs, L)):
                    if c <= r:
                        best = max(best, 0.4 * float(np.dot(qh[r], kh[c])))
            assert abs(sm[i, j] - best) < 1e-12


def test_calibration_kth_largest_with_ties():
    rng = np.random.default_rng(4)
    n, k = 40, 5
    sm = np.round(rng.standard_normal((2, n, n)), 1)   # many ties
    T = oracle.calibrate_thresholds(sm, k)
    for h in range(2):
        for i in range(n):
            if i < k:
                assert T[h, i] == -np.inf
            else:
                assert T[h, i] == heapq.nlargest(k, list(sm[h, i, :i]))[-1]


def test_gate_density_closed_form_matches_bsfa_table6():
    """With T calibrated on the same block maxima (distinct values), exactly
    min(i, k) off-diagonal blocks pass in row i; at n = 512 tiles (32K tokens
    of 64), k = 64 the kept fraction of causal tiles is 31200/131328 = 0.2376,
    BSFA Table 6's predicted density 0.24 at 32K, k = 64."""
    rng = np.random.default_rng(5)
    n, k = 512, 64
    sm = rng.standard_normal((1, n, n))
    T = oracle.calibrate_thresholds(sm, k)
    keep = oracle.gate_keep(sm, T)
    dens = keep.sum() / (n * (n + 1) / 2)
    assert keep.sum() == 31200
    assert dens == pytest.approx(oracle.kept_density_closed_form(n, k), abs=1e-15)
    assert abs(dens - 0.24) < 0.005


def test_gated_attention_vs_elementwise():
    rng = np.random.default_rng(6)
    B, L, Hq, Hkv, D, bs = 1, 40, 4, 2, 8, 8
    q, k, v = _rand(rng, B, L, Hq, D), _rand(rng, B, L, Hkv, D), _rand(rng, B, L, Hkv, D)
    n = L // bs
    T = rng.uniform(0.0, 1.5, size=(Hq, n))
    T[:, :2] = -np.inf
    o, lse, info = oracle.attend_gated(q, k, v, T, bs, 0.5, return_keep=True)
    G = Hq // Hkv
    mask = np.zeros((Hq, L, L), dtype=bool)
    for h in range(Hq):
        sm = oracle.block_max_head(q[0, :, h], k[0, :, h // G], bs, 0.5)
        for r in range(L):
            i = r // bs
            for c in range(r + 1):
                j = c // bs
                mask[h, r, c] = (j == i) or (sm[i, j] >= T[h, i])
        for i in range(n):
            np.testing.assert_array_equal(info[(0, h, i)][1],
                                          [(j == i) or sm[i, j] >= T[h, i] for j in range(i + 1)])
    ob, lb = oracle.attend_dense_masked(q[0], k[0], v[0], mask, 0.5)
    np.testing.assert_allclose(o[0], ob, atol=1e-12)
    np.testing.assert_allclose(lse[0], lb, atol=1e-12)


# ---------------------------------------------------------------- O5 vertical / slash

def _vs_elementwise(q_len, kv_len, vert, slash, BM, BN, causal):
    """Per-row sets: the slash keys of row r are r + d - s for every offset s
    (inside [0, kv_len)); a block is listed iff some row of the q-block has a
    slash key in it; a column is listed iff it is visible and in no listed block."""
    d = kv_len - q_len
    nqb = -(-q_len // BM)
    out = []
    for i in range(nqb):
        rows = range(i * BM, min((i + 1) * BM, q_len))
        blocks = set()
        for r in rows:
            for s in slash:
                key = r + d - int(s)
                if 0 <= key < kv_len:
                    blocks.add(key // BN)
        m1 = max(rows) + 1
        cols = sorted(set(int(c) for c in vert
                          if 0 <= c < kv_len and (not causal or c <= m1 - 1 + d)
                          and (c // BN) not in blocks))
        out.append((sorted(blocks), cols))
    return out


@pytest.mark.parametrize("q_len,kv_len,BM,BN", [(150, 150, 16, 16), (100, 130, 32, 16),
                                                 (64, 64, 64, 64)])
def test_vertical_slash_convert_vs_elementwise(q_len, kv_len, BM, BN):
    rng = np.random.default_rng(q_len + kv_len)
    H, nv, ns = 2, 12, 9
    vert = np.stack([np.sort(rng.choice(kv_len, nv, replace=False)) for _ in range(H)])[None]
    slash = np.stack([np.sort(rng.choice(kv_len, ns, replace=False)) for _ in range(H)])[None]
    bc, bo, cc, ci = oracle.convert_vertical_slash(
        np.array([q_len]), np.array([kv_len]), vert.astype(np.int32), slash.astype(np.int32),
        q_len, BM, BN, True)
    for h in range(H):
        ref = _vs_elementwise(q_len, kv_len, vert[0, h], slash[0, h], BM, BN, True)
        for i, (blocks, cols) in enumerate(ref):
            assert list(bo[0, h, i, :bc[0, h, i]]) == [b * BN for b in blocks]
            assert list(ci[0, h, i, :cc[0, h, i]]) == cols
            assert np.all(bo[0, h, i, bc[0, h, i]:] == 0)


def test_vertical_slash_attention_vs_elementwise():
    rng = np.random.default_rng(8)
    L, H, D, BM = 96, 2, 8, 16
    q, k, v = _rand(rng, 1, L, H, D), _rand(rng, 1, L, H, D), _rand(rng, 1, L, H, D)
    vert = np.stack([np.sort(rng.choice(L, 10, replace=False)) for _ in range(H)])[None]
    slash = np.stack([np.sort(rng.choice(L, 4, replace=False)) for _ in range(H)])[None]
    bc, bo, cc, ci = oracle.convert_vertical_slash(np.array([L]), np.array([L]),
                                                   vert, slash, L, BM, BM, True)
    o, lse = oracle.attend_vertical_slash(q, k, v, bc, bo, cc, ci, BM, BM, True, 0.5)
    mask = np.zeros((H, L, L), dtype=bool)
    for h in range(H):
        for r in range(L):
            i = r // BM
            blocks = set(int(x) // BM for x in bo[0, h, i, :bc[0, h, i]])
            cols = set(int(x) for x in ci[0, h, i, :cc[0, h, i]])
            for c in range(r + 1):
                mask[h, r, c] = (c // BM) in blocks or c in cols
    ob, lb = oracle.attend_dense_masked(q[0], k[0], v[0], mask, 0.5)
    np.testing.assert_allclose(o[0], ob, atol=1e-12)
    np.testing.assert_allclose(lse[0], lb, atol=1e-12)


# ---------------------------------------------------------------- O6 NSA selected

def test_nsa_selection_invariants():
    seqlens = (700, 300)
    sel = W.nsa_selection(np.random.default_rng(0), seqlens, H=3, block=16, topk=16)
    base = 0
    for L in seqlens:
        for tl in range(L):
            c = tl // 16
            for h in range(3):
                row = sel[base + tl, h]
                valid = row[row >= 0]
                assert len(set(valid.tolist())) == len(valid)
                assert np.all(valid <= c)
                assert 0 in valid and c in valid and (c < 1 or c - 1 in valid or c - 1 == 0)
                expect = min(16, 1 + (1 if c >= 1 else 0) + (1 if c >= 2 else 0) + max(c - 2, 0))
                assert len(valid) == expect
                assert np.all(row[len(valid):] == -1)
        base += L


def test_nsa_attention_vs_elementwise():
    rng = np.random.default_rng(9)
    seqlens = (70, 45)
    T, H, D, bs = sum(seqlens), 2, 8, 8
    q, k, v = _rand(rng, T, H, D), _rand(rng, T, H, D), _rand(rng, T, H, D)
    sel = W.nsa_selection(np.random.default_rng(1), seqlens, H, block=bs, topk=5)
    cu = np.array([0, seqlens[0], T])
    o, lse = oracle.attend_selected_varlen(q, k, v, cu, sel, bs, True, 0.5)
    for s in range(2):
        b0, L = cu[s], cu[s + 1] - cu[s]
        mask = np.zeros((H, L, L), dtype=bool)
        for h in range(H):
            for r in range(L):
                picked = set(int(x) for x in sel[b0 + r, h] if x >= 0)
                for c in range(r + 1):
                    mask[h, r, c] = (c // bs) in picked
        ob, lb = oracle.attend_dense_masked(q[b0:b0 + L], k[b0:b0 + L], v[b0:b0 + L], mask, 0.5)
        np.testing.assert_allclose(o[b0:b0 + L], ob, atol=1e-12)
        np.testing.assert_allclose(lse[:, b0:b0 + L], lb, atol=1e-12)


# ---------------------------------------------------------------- speculative decode

@pytest.mark.parametrize("Sq,causal_spec", [(1, True), (2, True), (2, False)])
def test_speculative_sparse_equals_union_sdpa(Sq, causal_spec):
    rng = np.random.default_rng(11)
    B, Hq, Hkv, Lk, D, bs, spec = 2, 4, 2, 256, 8, 32, 64
    q, k, v = _rand(rng, B, Sq, Hq, D), _rand(rng, B, Lk, Hkv, D), _rand(rng, B, Lk, Hkv, D)
    n_rest = (Lk - spec) // bs
    table = np.stack([np.stack([rng.choice(n_rest, 3, replace=False) for _ in range(Hkv)])
                      for _ in range(B)])[:, :, None, :].astype(np.int32)
    o, lse = oracle.speculative_sparse(q, k[:, Lk - spec:], v[:, Lk - spec:], causal_spec,
                                       k, v, table, bs, 0.5)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            keys_b = set()
            for j in table[b, h // G, 0]:
                keys_b.update(range(j * bs, (j + 1) * bs))
            mask = np.zeros((Sq, Lk), dtype=bool)
            for r in range(Sq):
                for c in range(Lk):
                    in_spec = c >= Lk - spec and (not causal_spec or c - (Lk - spec) <= r + spec - Sq)
                    mask[r, c] = in_spec or c in keys_b
            ref = _sdpa_dense(q[b][:, h:h + 1], k[b][:, h // G:h // G + 1], v[b][:, h // G:h // G + 1],
                              0.5, mask)
            np.testing.assert_allclose(o[b, :, h], ref[:, 0], atol=1e-12)


# ---------------------------------------------------------------- generator rounding

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(12)
    x = (rng.standard_normal(10000) * 10 ** rng.uniform(-3, 3, 10000)).astype(np.float32)
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -0.0, 65504.0]     # ties to even
    ours = W.bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)


# ---------------------------------------------------------------- stored thresholds

def test_stored_gated_thresholds_recompute_on_two_heads():
    """tests/golden/gated_T_seed101.npy was written by oracle/make_golden.py;
    recompute two heads from the seed-101 calibration data and compare."""
    T = np.load(os.path.join(GOLDEN, "gated_T_seed101.npy"))
    assert T.shape == (32, 512) and T.dtype == np.float32
    assert np.all(np.isneginf(T[:, :64])) and np.all(np.isfinite(T[:, 64:]))
    wl = W.make_gated(seed=101)
    for h in (0, 29):
        sm = oracle.block_max_head(wl.q[0, :, h, :], wl.k[0, :, h // 4, :], 64, wl.scale)
        ref = oracle.calibrate_thresholds(sm[None], 64)[0].astype(np.float32)
        np.testing.assert_array_equal(T[h], ref)


# ---------------------------------------------------------------- varlen packing and mergehead

def test_varlen_block_table_vs_elementwise_per_sequence():
    """Packed sequences of different lengths: each sequence's rows equal the
    element-wise brute force on that sequence alone (bottom-right causal
    inside the sequence), and rows never see another sequence's keys."""
    rng = np.random.default_rng(61)
    D, Hq, Hkv, qbs, kbs, nmax = 8, 4, 2, 16, 8, 5
    lq, lk = [20, 7, 33], [20, 15, 40]
    cu_q, cu_k = np.concatenate([[0], np.cumsum(lq)]), np.concatenate([[0], np.cumsum(lk)])
    q, k, v = _rand(rng, cu_q[-1], Hq, D), _rand(rng, cu_k[-1], Hkv, D), _rand(rng, cu_k[-1], Hkv, D)
    nqb, nkb = -(-max(lq) // qbs), -(-max(lk) // kbs)
    table = rng.integers(-1, nkb, size=(3, Hkv, nqb, nmax)).astype(np.int32)
    for causal in (False, True):
        o, lse = oracle.attend_block_table_varlen(q, k, v, cu_q, cu_k, table, qbs, kbs, causal, 0.5)
        for s in range(3):
            a, z, ka, kz = cu_q[s], cu_q[s + 1], cu_k[s], cu_k[s + 1]
            mask = oracle.element_mask_from_table(lq[s], lk[s], Hq, Hkv, table[s], qbs, kbs, causal)
            ob, lb = oracle.attend_dense_masked(q[a:z], k[ka:kz], v[ka:kz], mask, 0.5)
            np.testing.assert_allclose(o[a:z], ob, rtol=0, atol=1e-12)
            ls = lse[:, a:z]
            np.testing.assert_array_equal(np.isneginf(ls), np.isneginf(lb))
            fin = np.isfinite(lb)
            np.testing.assert_allclose(ls[fin], lb[fin], rtol=0, atol=1e-12)


def test_varlen_vertical_slash_equal_lengths_equal_batched():
    """Two packed sequences of one length give the batched (B = 2) result."""
    rng = np.random.default_rng(62)
    L, H, D, BM = 64, 2, 8, 16
    q, k, v = _rand(rng, 2, L, H, D), _rand(rng, 2, L, H, D), _rand(rng, 2, L, H, D)
    vert = np.stack([np.stack([np.sort(rng.choice(L, 6, replace=False)) for _ in range(H)])
                     for _ in range(2)]).astype(np.int32)
    slash = np.stack([np.stack([np.sort(rng.choice(L, 5, replace=False)) for _ in range(H)])
                      for _ in range(2)]).astype(np.int32)
    lists = oracle.convert_vertical_slash([L, L], [L, L], vert, slash, L, BM, BM, True)
    ob, lb = oracle.attend_vertical_slash(q, k, v, *lists, BM, BM, True, 0.5)
    cu = np.array([0, L, 2 * L])
    ov, lv = oracle.attend_vertical_slash_varlen(q.reshape(2 * L, H, D), k.reshape(2 * L, H, D),
                                                 v.reshape(2 * L, H, D), cu, cu, *lists, BM, BM,
                                                 True, 0.5)
    np.testing.assert_array_equal(ov, ob.reshape(2 * L, H, D))
    np.testing.assert_array_equal(lv, np.concatenate([lb[0], lb[1]], axis=1))


def test_mergehead_counts_truncate_each_head():
    """Per-head counts: head h's lists equal the element-wise sets of its
    first v_count[h] vertical and s_count[h] slash entries; full counts give
    the plain conversion."""
    rng = np.random.default_rng(63)
    q_len = kv_len = 120
    H, nv, ns, BM = 3, 12, 9, 16
    vert = np.stack([np.sort(rng.choice(kv_len, nv, replace=False)) for _ in range(H)])[None]
    slash = np.stack([np.sort(rng.choice(kv_len, ns, replace=False)) for _ in range(H)])[None]
    vert, slash = vert.astype(np.int32), slash.astype(np.int32)
    vc, sc = np.array([12, 5, 0]), np.array([2, 9, 4])
    bc, bo, cc, ci = oracle.convert_vertical_slash([q_len], [kv_len], vert, slash, q_len, BM, BM,
                                                   True, v_count=vc, s_count=sc)
    for h in range(H):
        ref = _vs_elementwise(q_len, kv_len, vert[0, h, :vc[h]], slash[0, h, :sc[h]], BM, BM, True)
        for i, (blocks, cols) in enumerate(ref):
            assert list(bo[0, h, i, :bc[0, h, i]]) == [b * BM for b in blocks]
            assert list(ci[0, h, i, :cc[0, h, i]]) == cols
    full = oracle.convert_vertical_slash([q_len], [kv_len], vert, slash, q_len, BM, BM, True,
                                         v_count=[nv] * H, s_count=[ns] * H)
    plain = oracle.convert_vertical_slash([q_len], [kv_len], vert, slash, q_len, BM, BM, True)
    for a, b in zip(full, plain):
        np.testing.assert_array_equal(a, b)


def test_window_vs_elementwise_and_full_window_equals_causal():
    rng = np.random.default_rng(64)
    B, Sq, Sk, Hq, Hkv, D = 1, 30, 45, 4, 2, 8
    q, k, v = _rand(rng, B, Sq, Hq, D), _rand(rng, B, Sk, Hkv, D), _rand(rng, B, Sk, Hkv, D)
    w = 7
    o, lse = oracle.attend_window(q, k, v, w, 0.5)
    mask = np.zeros((Hq, Sq, Sk), dtype=bool)
    for h in range(Hq):
        for r in range(Sq):
            for c in range(Sk):
                mask[h, r, c] = (r + (Sk - Sq) - w) < c <= r + (Sk - Sq)
    ob, lb = oracle.attend_dense_masked(q[0], k[0], v[0], mask, 0.5)
    np.testing.assert_allclose(o[0], ob, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0], lb, rtol=0, atol=1e-12)
    # a window as long as the keys is plain causal attention
    ow, lw = oracle.attend_window(q, k, v, Sk, 0.5)
    full = np.broadcast_to(np.arange(Sk // 5, dtype=np.int32), (B, Hkv, 1, Sk // 5))
    oc, lc = oracle.attend_block_table(q, k, v, full, Sq, 5, True, 0.5)
    np.testing.assert_allclose(ow, oc, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lw, lc, rtol=0, atol=1e-12)
