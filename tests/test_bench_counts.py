"""The algorithmic work behind every number bench.py reports, checked
against brute-force counts on small inputs (CPU).

bench.py divides by these counts: kept K/V bytes for the decode GB/s, and
exact visible (row, key) pairs for the prefill TFLOP/s.  Each count is
recomputed here element by element from the same tables, masks and lists."""
import importlib.util
import os

import numpy as np

import oracle
import workloads as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench", os.path.join(ROOT, "bench.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def test_decode_bytes_count_every_kept_key_once():
    bm = _bench()
    wl = W.make_spec_decode(B=2, Hq=8, Hkv=2, Lq=1, Lk=1000, block=128, spec_len=200,
                            n_missed=3, seed=5, table_seed=6)
    total, kv = bm.decode_bytes(wl)
    t = wl.meta["table"]
    keys = 0
    for b in range(2):
        for g in range(2):
            seen = np.zeros(1000, dtype=bool)
            for j in t[b, g, 0]:
                if j >= 0:
                    seen[j * 128:min((j + 1) * 128, 1000)] = True
            keys += 200 + int(seen.sum())      # the spec range, then the listed blocks
    assert kv == keys * 128 * 2 * 2             # K and V rows, bf16
    assert total == kv + 2 * 2 * 1 * 8 * 128 * 2 + 2 * 8 * 1 * 4 + t.size * 4


def test_gated_flops_match_pair_counts_of_the_keep_mask():
    bm = _bench()
    rng = np.random.default_rng(3)
    L, H, blk = 640, 3, 64
    n = L // blk
    keep = np.zeros((1, H, n, n), dtype=np.uint8)
    for h in range(H):
        for i in range(n):
            keep[0, h, i, :i + 1] = rng.random(i + 1) < 0.4
            keep[0, h, i, i] = 1
    flops, n_qk, n_pv = bm.gated_flops(keep, L, H)
    r = np.arange(L)
    causal = r[None, :] <= r[:, None]             # [row, key]
    qk = H * int(causal.sum())
    pv = 0
    for h in range(H):
        kept = np.kron(keep[0, h].astype(bool), np.ones((blk, blk), dtype=bool))
        pv += int((kept & causal).sum())
    assert (n_qk, n_pv) == (qk, pv)
    assert flops == 2 * 128 * (qk + pv)


def test_vertical_slash_flops_match_visible_pairs():
    bm = _bench()
    L, H = 1024, 2
    vert, slash = W.vertical_slash_indices(np.random.default_rng(11), 1, H, L, 80, 120)
    bc, bo, cc, ci = oracle.convert_vertical_slash([L], [L], vert, slash, L, 64, 64, True)
    flops, pairs = bm.vs_flops(bc, bo, cc, ci, L)
    count = 0
    r = np.arange(L)
    for h in range(H):
        for i in range(L // 64):
            rows = r[i * 64:(i + 1) * 64]
            keys = set()
            for off in bo[0, h, i, :bc[0, h, i]]:
                keys.update(range(off, min(off + 64, L)))
            keys.update(int(c) for c in ci[0, h, i, :cc[0, h, i]])
            kk = np.array(sorted(keys), dtype=np.int64)
            count += int((kk[None, :] <= rows[:, None]).sum())
    assert pairs == count
    assert flops == 4 * 128 * count


def test_nsa_pairs_match_visible_pairs():
    bm = _bench()
    wl = W.make_nsa_varlen(seqlens=(300, 130), H=2, seed=9, table_seed=19)
    cu, sel = wl.meta["cu_seqlens"], wl.meta["sel"]
    count = 0
    for s in range(len(cu) - 1):
        for t in range(cu[s], cu[s + 1]):
            tl = t - cu[s]
            for g in range(sel.shape[1]):
                for j in sel[t, g]:
                    if j >= 0:
                        count += max(0, min(64, tl - 64 * int(j) + 1))
    assert bm.nsa_pairs(wl) == count


def test_oracle_samples_beside_the_prefill_numbers():
    """The bench's oracle-on-a-sample lines run on small workloads and report
    a positive rate with a consistent extrapolation."""
    bm = _bench()
    wl = W.make_gated(B=1, Hq=4, Hkv=1, L=1024, seed=12)
    sm = np.stack([oracle.block_max_head(wl.q[0, :, h], wl.k[0, :, 0], 64, wl.scale)
                   for h in range(4)])
    T = oracle.calibrate_thresholds(sm, 4).astype(np.float32)
    g = bm.oracle_sample_gated(wl, T, full_flops=10 ** 12)
    wv = W.make_vertical_slash(B=1, H=2, L=1024, nnz_v=80, nnz_s=120, seed=13, table_seed=14)
    v = bm.oracle_sample_vs(wv, full_flops=10 ** 12)
    wn = W.make_nsa_varlen(seqlens=(700, 300), H=2, seed=15, table_seed=16)
    n = bm.oracle_sample_nsa(wn, full_flops=10 ** 12, n_tok=64)
    for line in (g, v, n):
        assert line["kind"] == "oracle" and line["value"] > 0 and line["sample_seconds"] > 0
        assert line["extrapolated_full_seconds"] > line["sample_seconds"]
    c = bm.oracle_sample_vs_convert(wv, n_qb=4)
    assert c["extrapolated_full_seconds"] >= c["sample_seconds"] > 0


def test_oracle_sample_flops_match_element_counts():
    """The FLOPs each oracle sample line divides by, against element-by-element
    counts of the pairs that sample evaluates."""
    bm = _bench()
    # gated: q-block i of one head; QK over every causal key, PV over kept blocks
    rng = np.random.default_rng(21)
    L, i = 640, 9
    keep = rng.random(i + 1) < 0.5
    keep[i] = True
    r = np.arange(i * 64, (i + 1) * 64)
    qk = int((np.arange(L)[None, :] <= r[:, None]).sum())
    kept_keys = np.concatenate([np.arange(j * 64, (j + 1) * 64) for j in np.nonzero(keep)[0]])
    pv = int((kept_keys[None, :] <= r[:, None]).sum())
    assert bm.gated_sample_flops(i, keep) == 2 * 128 * (qk + pv)
    # vertical/slash: visible pairs of one q-block under converted lists
    L = 1024
    vert, slash = W.vertical_slash_indices(np.random.default_rng(22), 1, 1, L, 80, 120)
    bc, bo, cc, ci = oracle.convert_vertical_slash([L], [L], vert, slash, L, 64, 64, True)
    for i in (3, 15):
        rows = np.arange(i * 64, (i + 1) * 64)
        keys = set()
        for off in bo[0, 0, i, :bc[0, 0, i]]:
            keys.update(range(off, min(off + 64, L)))
        keys.update(int(c) for c in ci[0, 0, i, :cc[0, 0, i]])
        kk = np.array(sorted(keys))
        assert bm.vs_sample_pairs(bc, bo, cc, ci, i, L) == int((kk[None, :] <= rows[:, None]).sum())
    # NSA: visible pairs of head 0 over chosen tokens of sequence 0
    wl = W.make_nsa_varlen(seqlens=(500, 100), H=2, seed=23, table_seed=24)
    cu, sel = wl.meta["cu_seqlens"], wl.meta["sel"]
    toks = np.arange(400, 500)
    count = 0
    for t in toks:
        for j in sel[t, 0]:
            if j >= 0:
                count += max(0, min(64, t - 64 * int(j) + 1))
    assert bm.nsa_sample_pairs(cu, sel, toks) == count
