"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on
the same seeded inputs.  Tolerances: o max-abs <= 2e-2, lse max-abs <= 1e-3
(bf16 inputs, fp32 accumulation); integer outputs bit-exact; gate keep bits
bit-exact except blocks with |s_max - T| < 1e-3, which are reported."""
import math

import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu

O_TOL, LSE_TOL = 2e-2, 1e-3


@pytest.fixture(scope="module")
def sb():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import block_sparse_flashattention_sbfa_b200 as m
    return m


def dev(bits):
    return W.to_torch_bf16(bits, "cuda")


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what=""):
    """Element-wise comparison on every row the oracle computed."""
    o = o_gpu.float().cpu().numpy().astype(np.float64)
    lse = lse_gpu.float().cpu().numpy().astype(np.float64)
    rows = ~np.isnan(lse_ref)
    orow = ~np.isnan(o_ref[..., 0])
    assert orow.sum() > 0
    err_o = np.abs(o[orow] - o_ref[orow]).max()
    lr, lg = lse_ref[rows], lse[rows]
    inf_ref = np.isneginf(lr)
    assert np.array_equal(inf_ref, np.isneginf(lg)), f"{what}: -inf pattern of lse differs"
    err_l = np.abs(lg[~inf_ref] - lr[~inf_ref]).max() if (~inf_ref).any() else 0.0
    print(f"{what}: o max-abs {err_o:.3e}, lse max-abs {err_l:.3e}, rows {rows.sum()}")
    assert err_o <= O_TOL, f"{what}: o max-abs {err_o}"
    assert err_l <= LSE_TOL, f"{what}: lse max-abs {err_l}"


def sampled_rows(n_rows, block, seed, n=4):
    rng = np.random.default_rng(seed)
    nqb = -(-n_rows // block)
    qbs = W.sample_qblocks(rng, nqb, n)
    return np.concatenate([np.arange(b * block, min((b + 1) * block, n_rows)) for b in qbs])


# ------------------------------------------------------------------ block table

def test_block_table_tiny_workload(sb):
    """B=1, H=2, Lq=256, Lk=1024, bs=64, non-causal, diagonal + 7 random blocks;
    plus the LSE combine of the two disjoint halves of every table row."""
    wl = W.make_block_table()
    tab = wl.meta["table"]
    q, k, v = dev(wl.q), dev(wl.k), dev(wl.v)
    t = torch.from_numpy(tab).cuda()
    st = sb.new_status("cuda")
    o, lse = sb.fwd(q, k, v, t, 64, 64, causal=False, status=st)
    sb.check_status(st)
    ro, rl = oracle.attend_block_table(wl.q, wl.k, wl.v, tab, 64, 64, False, wl.scale)
    compare(o, lse, ro, rl, "block table")
    # halves -> combine
    oa, la = sb.fwd(q, k, v, t[..., :4], 64, 64)
    ob, lb = sb.fwd(q, k, v, t[..., 4:], 64, 64)
    oc, lc = sb.combine(torch.stack([oa.float(), ob.float()]), torch.stack([la, lb]))
    compare(oc, lc, ro, rl, "combine of halves")
    # per-entry partials -> combine
    op, lp = sb.fwd_partials(q, k, v, t, 64, 64)
    oc2, lc2 = sb.combine(op, lp)
    compare(oc2, lc2, ro, rl, "combine of 8 partials")
    ro0, rl0 = oracle.attend_block_table(wl.q, wl.k, wl.v, tab[..., 3:4], 64, 64, False, wl.scale)
    compare(op[3], lp[3], ro0, rl0, "partial 3")


@pytest.mark.parametrize("G,causal,q_block,kv_block", [(1, True, 64, 64), (2, True, 128, 128),
                                                        (4, False, 64, 256), (8, True, 192, 64)])
def test_block_table_ragged_gqa(sb, G, causal, q_block, kv_block):
    rng = np.random.default_rng(100 + G)
    B, Sq, Sk, Hkv = 2, 333, 1000, 2
    Hq = Hkv * G
    q = W.normal_bf16(rng, (B, Sq, Hq, 128))
    k = W.normal_bf16(rng, (B, Sk, Hkv, 128))
    v = W.normal_bf16(rng, (B, Sk, Hkv, 128))
    nqb, nkb = -(-Sq // q_block), -(-Sk // kv_block)
    tab = rng.integers(-1, nkb, size=(B, Hkv, nqb, 6)).astype(np.int32)
    tab[..., 5] = tab[..., 0]                # duplicate entry counts once
    tab[0, 0, 0, :] = -1                     # an empty row: o = 0, lse = -inf
    o, lse = sb.fwd(dev(q), dev(k), dev(v), torch.from_numpy(tab).cuda(), q_block, kv_block,
                    causal=causal)
    ro, rl = oracle.attend_block_table(q, k, v, tab, q_block, kv_block, causal, W.default_scale())
    compare(o, lse, ro, rl, f"ragged G={G}")


def test_block_table_1d_broadcast_and_dense(sb):
    rng = np.random.default_rng(7)
    B, S, H = 1, 512, 4
    q, k, v = (W.normal_bf16(rng, (B, S, H, 128)) for _ in range(3))
    full = torch.arange(S // 64, dtype=torch.int32, device="cuda")
    o1, l1 = sb.fwd(dev(q), dev(k), dev(v), full, 64, 64, causal=True)
    o2, l2 = sb.fwd_dense(dev(q), dev(k), dev(v), causal=True)
    tab = np.broadcast_to(np.arange(S // 64, dtype=np.int32), (B, H, 1, S // 64))
    ro, rl = oracle.attend_block_table(q, k, v, tab, S, 64, True, W.default_scale())
    compare(o1, l1, ro, rl, "1-D table")
    compare(o2, l2, ro, rl, "dense")


# ------------------------------------------------------------------ decode

def _spec_case(B, Hq, Hkv, Sq, Lk, bs, spec, n_missed, seed):
    wl = W.make_spec_decode(B=B, Hq=Hq, Hkv=Hkv, Lq=Sq, Lk=Lk, block=bs, spec_len=spec,
                            n_missed=n_missed, seed=seed, table_seed=seed + 1000)
    return wl


@pytest.mark.parametrize("Sq,causal_spec", [(1, True), (2, True), (4, False)])
def test_speculative_sparse_small(sb, Sq, causal_spec):
    wl = _spec_case(2, 8, 2, Sq, 4096, 128, 512, 6, 20 + Sq)
    t = wl.meta["table"]
    s0 = wl.meta["spec_begin"]
    q, k, v = dev(wl.q), dev(wl.k), dev(wl.v)
    tab = torch.from_numpy(t).cuda()
    st = sb.new_status("cuda")
    o, lse = sb.speculative_sparse(q, k[:, s0:], v[:, s0:], causal_spec, k, v, tab, 128,
                                   status=st)
    sb.check_status(st)
    ro, rl = oracle.speculative_sparse(wl.q, wl.k[:, s0:], wl.v[:, s0:], causal_spec, wl.k,
                                       wl.v, t, 128, wl.scale)
    compare(o, lse, ro, rl, f"spec fused Sq={Sq}")
    # three-call path: dense pass A, sparse pass B, combine
    oa, la = sb.fwd_dense(q, k[:, s0:], v[:, s0:], causal=causal_spec)
    ob, lb = sb.fwd(q, k, v, tab, max(Sq, 1), 128, causal=False)
    oc, lc = sb.combine(torch.stack([oa.float(), ob.float()]), torch.stack([la, lb]))
    compare(oc, lc, ro, rl, f"spec 3-call Sq={Sq}")


def test_speculative_sparse_full_workload(sb):
    """B=8, Hq=32, Hkv=8, Lk=32768, bs=128: dense last 2048 + 32 missed blocks;
    every (b, h) row checked against attention over the union."""
    wl = W.make_spec_decode()
    t = wl.meta["table"]
    s0 = wl.meta["spec_begin"]
    q, k, v = dev(wl.q), dev(wl.k), dev(wl.v)
    tab = torch.from_numpy(t).cuda()
    ws = sb.decode_workspace(8, 8, 1, 32, "cuda")
    for rep in range(2):       # the workspace's counters must come back to zero
        o, lse = sb.speculative_sparse(q, k[:, s0:], v[:, s0:], True, k, v, tab, 128, ws=ws)
    torch.cuda.synchronize()
    union = np.concatenate([t, np.broadcast_to(np.arange(s0 // 128, 256, dtype=np.int32),
                                               (8, 8, 1, 16))], axis=-1)
    ro, rl = oracle.attend_block_table(wl.q, wl.k, wl.v, union, 1, 128, False, wl.scale)
    compare(o, lse, ro, rl, "spec decode full")


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Lk,bs,spec,nmax", [
    (1, 16, 1, 1, 8192, 256, 1000, 12),   # one pair spread over every CTA, 16 rows
    (3, 4, 2, 2, 1000, 16, 100, 9),       # kv_block 16, ragged last block
    (2, 8, 4, 1, 3000, 32, 1, 40),        # a one-key spec pass, many short blocks
    (4, 4, 4, 4, 5000, 64, 777, 5),       # G = 1, Sq = 4
])
def test_speculative_sparse_edge_cases(sb, B, Hq, Hkv, Sq, Lk, bs, spec, nmax):
    """Padding entries (-1) scattered through the table, one (b, kv-head) row
    with only padding, a spec range that is not a multiple of 64 keys and a
    key length that is not a multiple of the block size; the same workspace
    is used twice in a row."""
    rng = np.random.default_rng(B * 1000 + bs)
    q = W.normal_bf16(rng, (B, Sq, Hq, 128))
    k = W.normal_bf16(rng, (B, Lk, Hkv, 128))
    v = W.normal_bf16(rng, (B, Lk, Hkv, 128))
    ks, vs = k[:, Lk - spec:], v[:, Lk - spec:]
    nkb = -(-Lk // bs)
    tab = np.full((B, Hkv, 1, nmax), -1, dtype=np.int32)
    for b in range(B):
        for g in range(Hkv):
            if b == B - 1 and g == 0:
                continue                      # this row keeps only padding
            sel = rng.choice(nkb, size=min(nmax, nkb), replace=False)
            keep = rng.random(sel.size) < 0.8
            tab[b, g, 0, :keep.sum()] = sel[keep]
            rng.shuffle(tab[b, g, 0])
    ws = sb.decode_workspace(B, Hkv, Sq, Hq, "cuda")
    st = sb.new_status("cuda")
    for _ in range(2):
        o, lse = sb.speculative_sparse(dev(q), dev(ks), dev(vs), True, dev(k), dev(v),
                                       torch.from_numpy(tab).cuda(), bs, ws=ws, status=st)
    sb.check_status(st)
    ro, rl = oracle.speculative_sparse(q, ks, vs, True, k, v, tab, bs, W.default_scale())
    compare(o, lse, ro, rl, f"spec edge B={B} G={Hq // Hkv} Sq={Sq} bs={bs}")


@pytest.mark.parametrize("Sq,G,causal", [(1, 4, False), (4, 4, False), (2, 8, False),
                                          (16, 1, False), (1, 8, True), (4, 4, True)])
def test_block_table_short_queries(sb, Sq, G, causal):
    """Query blocks of <= 16 rows (Sq x G): padding, an all-padding row and a
    ragged key length.  Non-causal calls and Sq = 1 run on the split-KV
    kernel; causal calls with Sq > 1 on the tiled kernel, which applies the
    bottom-right causal mask."""
    rng = np.random.default_rng(300 + 10 * Sq + G)
    B, Hkv, Sk, bs, nmax = 3, 2, 1500, 64, 10
    Hq = Hkv * G
    q = W.normal_bf16(rng, (B, Sq, Hq, 128))
    k = W.normal_bf16(rng, (B, Sk, Hkv, 128))
    v = W.normal_bf16(rng, (B, Sk, Hkv, 128))
    nkb = -(-Sk // bs)
    tab = np.full((B, Hkv, 1, nmax), -1, dtype=np.int32)
    for b in range(B):
        for g in range(Hkv):
            blocks = rng.choice(nkb, size=nmax - 3, replace=False)
            tab[b, g, 0, rng.choice(nmax, size=nmax - 3, replace=False)] = blocks
    tab[1, 0, 0, :] = -1
    tab[1, 0, 0, 0] = nkb - 1                   # the last (ragged) block: causal cuts it
    tab[2, 0, 0, :] = -1                        # only padding: o = 0, lse = -inf
    o, lse = sb.fwd(dev(q), dev(k), dev(v), torch.from_numpy(tab).cuda(), max(Sq, 1), bs,
                    causal=causal)
    ro, rl = oracle.attend_block_table(q, k, v, tab, max(Sq, 1), bs, causal, W.default_scale())
    compare(o, lse, ro, rl, f"short queries Sq={Sq} G={G} causal={causal}")


def test_repeated_blocks_count_once_on_split_kv(sb):
    """A table row that lists a block more than once counts it once in
    sbfa_fwd whichever kernel serves the call: with one query position it
    runs on the split-KV kernel, with 64 on the tiled one; both against the
    oracle's set reading of a table row."""
    rng = np.random.default_rng(311)
    B, Hq, Hkv, Sk, bs, nmax = 2, 8, 2, 2000, 64, 12
    nkb = -(-Sk // bs)
    tab = np.full((B, Hkv, 1, nmax), -1, dtype=np.int32)
    for b in range(B):
        for g in range(Hkv):
            first = rng.choice(nkb, size=7, replace=False)
            row = np.concatenate([first, rng.choice(first, size=3), [-1, -1]])
            rng.shuffle(row)
            tab[b, g, 0] = row
    assert any(len(set(r[r >= 0])) < (r >= 0).sum() for r in tab.reshape(-1, nmax))
    k = W.normal_bf16(rng, (B, Sk, Hkv, 128))
    v = W.normal_bf16(rng, (B, Sk, Hkv, 128))
    td = torch.from_numpy(tab).cuda()
    for Sq in (1, 64):
        q = W.normal_bf16(rng, (B, Sq, Hq, 128))
        st = sb.new_status("cuda")
        o, lse = sb.fwd(dev(q), dev(k), dev(v), td, Sq, bs, causal=False, status=st)
        sb.check_status(st)
        ro, rl = oracle.attend_block_table(q, k, v, tab, Sq, bs, False, W.default_scale())
        compare(o, lse, ro, rl, f"repeats, sbfa_fwd Sq={Sq}")


def test_paged_kv_decode(sb):
    """A paged KV cache through the same entry point: one physical pool of
    pages shared by every sequence (k/v views with batch stride 0), each
    (sequence, kv-head) row of the table listing the physical pages of its
    missed blocks (kv_block = page size), pages shared between sequences
    allowed.  Checked against attention over the union of the spec range
    and the listed pages."""
    rng = np.random.default_rng(91)
    B, Hq, Hkv, page, n_pages, spec, nmax = 4, 16, 4, 128, 40, 300, 12
    pool_k = W.normal_bf16(rng, (1, n_pages * page, Hkv, 128))
    pool_v = W.normal_bf16(rng, (1, n_pages * page, Hkv, 128))
    q = W.normal_bf16(rng, (B, 1, Hq, 128))
    ks = W.normal_bf16(rng, (B, spec, Hkv, 128))
    vs = W.normal_bf16(rng, (B, spec, Hkv, 128))
    tab = np.stack([np.stack([rng.choice(n_pages, size=nmax, replace=False)
                              for _ in range(Hkv)]) for _ in range(B)])[:, :, None, :]
    tab = tab.astype(np.int32)
    tab[3, 1, 0, 5:] = -1                      # a shorter page list
    kd = dev(pool_k).expand(B, -1, -1, -1)     # batch stride 0: every sequence reads the pool
    vd = dev(pool_v).expand(B, -1, -1, -1)
    assert kd.stride(0) == 0
    st = sb.new_status("cuda")
    o, lse = sb.speculative_sparse(dev(q), dev(ks), dev(vs), True, kd, vd,
                                   torch.from_numpy(tab).cuda(), page, status=st)
    sb.check_status(st)
    kl = np.broadcast_to(pool_k, (B,) + pool_k.shape[1:])
    vl = np.broadcast_to(pool_v, (B,) + pool_v.shape[1:])
    ro, rl = oracle.speculative_sparse(q, ks, vs, True, kl, vl, tab, page, W.default_scale())
    compare(o, lse, ro, rl, "paged kv decode")


# ------------------------------------------------------------------ gated

def _gated_small(L=1024, Hq=8, Hkv=2, k_top=4):
    wl = W.make_gated(B=1, Hq=Hq, Hkv=Hkv, L=L, seed=30)
    cal = W.make_gated(B=1, Hq=Hq, Hkv=Hkv, L=L, seed=31)
    G = Hq // Hkv
    sm = np.stack([oracle.block_max_head(cal.q[0, :, h], cal.k[0, :, h // G], 64, cal.scale)
                   for h in range(Hq)])
    T = oracle.calibrate_thresholds(sm, k_top).astype(np.float32)
    return wl, T


def _check_keep(info, smax_g, keep_g, T, what):
    """Keep bits bit-exact except blocks whose s_max is within 1e-3 of T,
    which are reported.  Returns the (b, h, i) q-blocks that hold such a
    near-threshold flip."""
    n_diff = n_near = n_tot = 0
    max_sm_err = 0.0
    flipped = []
    for (b, h, i), (sm_ref, keep_ref) in info.items():
        kg = keep_g[b, h, i, :i + 1].astype(bool)
        sg = smax_g[b, h, i, :i + 1]
        max_sm_err = max(max_sm_err, np.abs(sg - sm_ref).max())
        near = np.abs(sm_ref - T[h, i]) < 1e-3
        diff = kg != keep_ref
        n_near += int((diff & near).sum())
        n_diff += int((diff & ~near).sum())
        n_tot += i + 1
        if (diff & near).any():
            flipped.append((b, h, i))
            print(f"{what}: near-threshold flip at b={b} h={h} i={i}, blocks "
                  f"{np.nonzero(diff & near)[0].tolist()}")
    print(f"{what}: {n_tot} blocks, keep mismatches {n_diff}, near-threshold flips {n_near}, "
          f"s_max max-abs {max_sm_err:.2e}")
    assert n_diff == 0
    assert max_sm_err < 1e-3
    return flipped


def _regate(wl, keep_g, flipped, ro, rl, block=64):
    """For a q-block whose keep row differs from the oracle's only by
    near-threshold flips, the oracle's output rows are recomputed over the
    blocks the GPU kept, so that every sampled row is still compared."""
    L = wl.q.shape[1]
    G = wl.q.shape[2] // wl.k.shape[2]
    for (b, h, i) in flipped:
        kept = np.nonzero(keep_g[b, h, i, :i + 1])[0]
        keys = (kept[:, None] * block + np.arange(block)[None, :]).reshape(-1)
        keys = keys[keys < L]
        r = np.arange(i * block, min((i + 1) * block, L))
        oo, ll = oracle.attend_keyset(wl.q[b, r, h, :], wl.k[b, keys, h // G, :],
                                      wl.v[b, keys, h // G, :], keys[None, :] <= r[:, None],
                                      wl.scale)
        ro[b, r, h, :] = oo
        rl[b, h, r] = ll


def test_gated_small_all_rows(sb):
    wl, T = _gated_small()
    q, k, v = dev(wl.q), dev(wl.k), dev(wl.v)
    n = T.shape[1]
    smax = torch.full((1, 8, n, n), float("nan"), device="cuda")
    keep = torch.full((1, 8, n, n), 255, dtype=torch.uint8, device="cuda")
    o, lse = sb.fwd_gated(q, k, v, torch.from_numpy(T).cuda(), smax_out=smax, keep_out=keep)
    ro, rl, info = oracle.attend_gated(wl.q, wl.k, wl.v, T, 64, wl.scale, return_keep=True)
    kept = keep.cpu().numpy()
    flipped = _check_keep(info, smax.cpu().numpy(), kept, T, "gated small")
    _regate(wl, kept, flipped, ro, rl)
    compare(o, lse, ro, rl, "gated small")
    assert np.all(kept[0][:, np.triu_indices(n, 1)[0], np.triu_indices(n, 1)[1]] == 255)


@pytest.mark.parametrize("Hq,Hkv", [(4, 4), (4, 2)])
def test_gated_group_sizes(sb, Hq, Hkv):
    """Unit shapes other than one GQA group of 4 at one q-block: G = 1 (four
    consecutive q-blocks of one head, each segment with its own diagonal)
    and G = 2 (two heads at two q-blocks).  Keep bits exact, all rows."""
    wl, T = _gated_small(Hq=Hq, Hkv=Hkv, k_top=3)
    q, k, v = dev(wl.q), dev(wl.k), dev(wl.v)
    n = T.shape[1]
    smax = torch.full((1, Hq, n, n), float("nan"), device="cuda")
    keep = torch.full((1, Hq, n, n), 255, dtype=torch.uint8, device="cuda")
    o, lse = sb.fwd_gated(q, k, v, torch.from_numpy(T).cuda(), smax_out=smax, keep_out=keep)
    ro, rl, info = oracle.attend_gated(wl.q, wl.k, wl.v, T, 64, wl.scale, return_keep=True)
    kept = keep.cpu().numpy()
    flipped = _check_keep(info, smax.cpu().numpy(), kept, T, f"gated Hq={Hq} Hkv={Hkv}")
    _regate(wl, kept, flipped, ro, rl)
    compare(o, lse, ro, rl, f"gated Hq={Hq} Hkv={Hkv}")


@pytest.mark.parametrize("L", [1000, 1090])
def test_gated_ragged_length(sb, L):
    """A sequence length that is not a multiple of 64: the last q-block and
    the last key block are partial (all rows checked)."""
    wl, T = _gated_small(L=L, Hq=8, Hkv=2, k_top=3)
    n = T.shape[1]
    smax = torch.full((1, 8, n, n), float("nan"), device="cuda")
    keep = torch.full((1, 8, n, n), 255, dtype=torch.uint8, device="cuda")
    st = sb.new_status("cuda")
    o, lse = sb.fwd_gated(dev(wl.q), dev(wl.k), dev(wl.v), torch.from_numpy(T).cuda(),
                          smax_out=smax, keep_out=keep, status=st)
    sb.check_status(st)
    ro, rl, info = oracle.attend_gated(wl.q, wl.k, wl.v, T, 64, wl.scale, return_keep=True)
    kept = keep.cpu().numpy()
    flipped = _check_keep(info, smax.cpu().numpy(), kept, T, f"gated L={L}")
    _regate(wl, kept, flipped, ro, rl)
    compare(o, lse, ro, rl, f"gated L={L}")


def test_gated_full_workload_sampled(sb):
    """Llama-3.1-8B shape, L=32768, 64x64 tiles, T from the stored seed-101
    calibration; 4 whole q-blocks (256 rows) per head checked."""
    import os
    T = np.load(os.path.join(os.path.dirname(__file__), "golden", "gated_T_seed101.npy"))
    wl = W.make_gated()
    q, k, v = dev(wl.q), dev(wl.k), dev(wl.v)
    n = 512
    smax = torch.empty((1, 32, n, n), device="cuda")
    keep = torch.empty((1, 32, n, n), dtype=torch.uint8, device="cuda")
    o, lse = sb.fwd_gated(q, k, v, torch.from_numpy(T).cuda(), smax_out=smax, keep_out=keep)
    torch.cuda.synchronize()
    rows = {h: sampled_rows(32768, 64, 500 + h) for h in range(32)}
    ro, rl, info = oracle.attend_gated(wl.q, wl.k, wl.v, T, 64, wl.scale,
                                       rows=lambda b, h: rows[h], return_keep=True)
    kp = keep.cpu().numpy()
    flipped = _check_keep(info, smax.cpu().numpy(), kp, T, "gated full")
    dens = sum(int(kp[0, h, i, :i + 1].sum()) for (_, h, i) in info) / \
        sum(i + 1 for (_, _, i) in info)
    print(f"gated full: kept density on the sampled q-blocks {dens:.3f}")
    _regate(wl, kp, flipped, ro, rl)
    compare(o, lse, ro, rl, "gated full")


def test_calibrate_thresholds_exact(sb):
    """GPU calibration (k-th largest off-diagonal block maximum per q-block)
    on the block maxima the gated kernel writes, bit for bit against the
    oracle's selection on the same values; ties counted with multiplicity on
    a small-integer matrix; and within 1e-3 of thresholds built from the
    oracle's own fp64 block maxima."""
    cal = W.make_gated(B=1, Hq=8, Hkv=2, L=2048, seed=31)
    n = 2048 // 64
    smax = torch.empty((1, 8, n, n), device="cuda")
    sb.fwd_gated(dev(cal.q), dev(cal.k), dev(cal.v),
                 torch.full((8, n), -float("inf"), device="cuda"), smax_out=smax)
    sm = smax.cpu().numpy()[0].astype(np.float64)
    for k_top in (1, 4, 16, n):
        Tg = sb.calibrate_thresholds(smax, k_top).cpu().numpy()[0].astype(np.float64)
        assert np.array_equal(Tg, oracle.calibrate_thresholds(sm, k_top)), k_top
    ties = torch.randint(-3, 4, (2, 3, 40, 40), device="cuda").float()
    Tt = sb.calibrate_thresholds(ties.contiguous(), 5).cpu().numpy().astype(np.float64)
    for b in range(2):
        assert np.array_equal(Tt[b], oracle.calibrate_thresholds(ties[b].cpu().numpy().astype(np.float64), 5))
    G = 4
    ref = np.stack([oracle.block_max_head(cal.q[0, :, h], cal.k[0, :, h // G], 64, cal.scale)
                    for h in range(8)])
    Tr = oracle.calibrate_thresholds(ref, 4)
    Tg = sb.calibrate_thresholds(smax, 4).cpu().numpy()[0].astype(np.float64)
    fin = np.isfinite(Tr)
    assert np.array_equal(fin, np.isfinite(Tg))
    err = np.abs(Tg[fin] - Tr[fin]).max()
    print(f"calibration: T max-abs vs fp64 block maxima {err:.2e}")
    assert err < 1e-3


# ------------------------------------------------------------------ vertical-slash

def _vs_small(L=2048, H=4, nnz_v=64, nnz_s=160, seed=40):
    return W.make_vertical_slash(B=1, H=H, L=L, nnz_v=nnz_v, nnz_s=nnz_s, seed=seed,
                                 table_seed=seed + 1000)


def test_vertical_slash_small(sb):
    wl = _vs_small()
    L, H = wl.q.shape[1], wl.q.shape[2]
    vert, slash = wl.meta["vertical"], wl.meta["slash"]
    sl = torch.tensor([L], dtype=torch.int32, device="cuda")
    bc, bo, cc, ci = sb.convert_vertical_slash(sl, sl, torch.from_numpy(vert).cuda(),
                                               torch.from_numpy(slash).cuda(), L)
    rbc, rbo, rcc, rci = oracle.convert_vertical_slash([L], [L], vert, slash, L, 64, 64, True)
    bc, bo, cc, ci = (x.cpu().numpy() for x in (bc, bo, cc, ci))
    assert np.array_equal(bc, rbc) and np.array_equal(cc, rcc)
    for idx in np.ndindex(bc.shape):
        assert np.array_equal(bo[idx][:bc[idx]], rbo[idx][:rbc[idx]])
        assert np.array_equal(ci[idx][:cc[idx]], rci[idx][:rcc[idx]])
    print(f"vs small: mean blocks {bc.mean():.1f}, mean columns {cc.mean():.2f}")
    o, lse = sb.fwd_vertical_slash(dev(wl.q), dev(wl.k), dev(wl.v), *(torch.from_numpy(x).cuda()
                                   for x in (rbc, rbo, rcc, rci)), causal=True)
    ro, rl = oracle.attend_vertical_slash(wl.q, wl.k, wl.v, rbc, rbo, rcc, rci, 64, 64, True,
                                          wl.scale)
    compare(o, lse, ro, rl, "vs small")


def test_vertical_slash_gqa(sb):
    """Per-query-head lists over shared kv heads (Hq = 8, Hkv = 2): the
    unit is one GQA group at one q-block, each segment with its own lists."""
    wl = _vs_small(L=1536, H=8, nnz_v=96, nnz_s=120, seed=45)
    L = wl.q.shape[1]
    rng = np.random.default_rng(1045)
    k = W.normal_bf16(rng, (1, L, 2, 128))
    v = W.normal_bf16(rng, (1, L, 2, 128))
    vert, slash = wl.meta["vertical"], wl.meta["slash"]
    sl = torch.tensor([L], dtype=torch.int32, device="cuda")
    bc, bo, cc, ci = sb.convert_vertical_slash(sl, sl, torch.from_numpy(vert).cuda(),
                                               torch.from_numpy(slash).cuda(), L)
    o, lse = sb.fwd_vertical_slash(dev(wl.q), dev(k), dev(v), bc, bo, cc, ci, causal=True)
    rbc, rbo, rcc, rci = oracle.convert_vertical_slash([L], [L], vert, slash, L, 64, 64, True)
    ro, rl = oracle.attend_vertical_slash(wl.q, k, v, rbc, rbo, rcc, rci, 64, 64, True, wl.scale)
    compare(o, lse, ro, rl, "vertical/slash gqa")


def test_vertical_slash_columns_heavy(sb):
    """Few slash lines, many vertical columns: most keys come from the column
    gather path."""
    wl = _vs_small(L=1536, H=2, nnz_v=400, nnz_s=64, seed=41)
    L = wl.q.shape[1]
    vert, slash = wl.meta["vertical"], wl.meta["slash"]
    rbc, rbo, rcc, rci = oracle.convert_vertical_slash([L], [L], vert, slash, L, 64, 64, True)
    assert rcc.max() > 64
    o, lse = sb.fwd_vertical_slash(dev(wl.q), dev(wl.k), dev(wl.v), *(torch.from_numpy(x).cuda()
                                   for x in (rbc, rbo, rcc, rci)), causal=True)
    ro, rl = oracle.attend_vertical_slash(wl.q, wl.k, wl.v, rbc, rbo, rcc, rci, 64, 64, True,
                                          wl.scale)
    compare(o, lse, ro, rl, "vs columns")


def test_vertical_slash_full_workload_sampled(sb):
    """L=131072, H=32, 1000 vertical columns and 6000 slash offsets per head,
    64 x 64 blocks, causal.  On every one of the 32 heads, 4 whole seeded
    q-blocks (256 rows, always including the last): the GPU's converted lists
    match the oracle's bit for bit, and the attention rows match the
    oracle's."""
    wl = W.make_vertical_slash()
    L, H = wl.q.shape[1], wl.q.shape[2]
    vert, slash = wl.meta["vertical"], wl.meta["slash"]
    sl = torch.tensor([L], dtype=torch.int32, device="cuda")
    bc, bo, cc, ci = sb.convert_vertical_slash(sl, sl, torch.from_numpy(vert).cuda(),
                                               torch.from_numpy(slash).cuda(), L)
    o, lse = sb.fwd_vertical_slash(dev(wl.q), dev(wl.k), dev(wl.v), bc, bo, cc, ci, causal=True)
    torch.cuda.synchronize()
    n_rows = n_lists = 0
    err_o = err_l = 0.0
    for h in range(H):
        qbs = W.sample_qblocks(np.random.default_rng(700 + h), L // 64)
        rbc, rbo, rcc, rci = oracle.convert_vertical_slash([L], [L], vert[:, h:h + 1],
                                                           slash[:, h:h + 1], L, 64, 64, True,
                                                           qblocks=qbs)
        qi = torch.from_numpy(qbs).cuda()
        gbc, gcc = (x[0, h].index_select(0, qi).cpu().numpy() for x in (bc, cc))
        gbo, gci = (x[0, h].index_select(0, qi).cpu().numpy() for x in (bo, ci))
        for j, i in enumerate(qbs):
            assert gbc[j] == rbc[0, 0, i] and gcc[j] == rcc[0, 0, i], (h, i)
            assert np.array_equal(gbo[j][:gbc[j]], rbo[0, 0, i][:rbc[0, 0, i]]), (h, i)
            assert np.array_equal(gci[j][:gcc[j]], rci[0, 0, i][:rcc[0, 0, i]]), (h, i)
            n_lists += 1
        rows = np.concatenate([np.arange(i * 64, (i + 1) * 64) for i in qbs])
        ro, rl = oracle.attend_vertical_slash(wl.q[:, :, h:h + 1], wl.k[:, :, h:h + 1],
                                              wl.v[:, :, h:h + 1], rbc, rbo, rcc, rci, 64, 64,
                                              True, wl.scale, rows=lambda b, j: rows)
        ri = torch.from_numpy(rows).cuda()
        og = o[0, :, h].index_select(0, ri).float().cpu().numpy()
        lg = lse[0, h].index_select(0, ri).cpu().numpy()
        assert np.isfinite(lg).all()
        err_o = max(err_o, np.abs(og - ro[0, rows, 0]).max())
        err_l = max(err_l, np.abs(lg - rl[0, 0, rows]).max())
        n_rows += rows.size
    print(f"vs full: {n_lists} converted q-blocks exact, {n_rows} rows on {H} heads, "
          f"o max-abs {err_o:.3e}, lse max-abs {err_l:.3e}")
    assert err_o <= O_TOL and err_l <= LSE_TOL


def test_vertical_slash_ragged_length(sb):
    """L = 1500 (partial last q-block and key block), all rows checked."""
    wl = _vs_small(L=1500, H=2, nnz_v=80, nnz_s=120, seed=42)
    L = wl.q.shape[1]
    vert, slash = wl.meta["vertical"], wl.meta["slash"]
    sl = torch.tensor([L], dtype=torch.int32, device="cuda")
    bc, bo, cc, ci = sb.convert_vertical_slash(sl, sl, torch.from_numpy(vert).cuda(),
                                               torch.from_numpy(slash).cuda(), L)
    rbc, rbo, rcc, rci = oracle.convert_vertical_slash([L], [L], vert, slash, L, 64, 64, True)
    _check_lists((bc, bo, cc, ci), (rbc, rbo, rcc, rci))
    st = sb.new_status("cuda")
    o, lse = sb.fwd_vertical_slash(dev(wl.q), dev(wl.k), dev(wl.v), bc, bo, cc, ci, causal=True,
                                   status=st)
    sb.check_status(st)
    ro, rl = oracle.attend_vertical_slash(wl.q, wl.k, wl.v, rbc, rbo, rcc, rci, 64, 64, True,
                                          wl.scale)
    compare(o, lse, ro, rl, "vs L=1500")


def test_vertical_slash_batch2_short_queries(sb):
    """B = 2 with q_len = 700 < kv_len = 1000 (bottom-right causal alignment:
    slash offsets and the causal limit are shifted by kv_len - q_len)."""
    rng = np.random.default_rng(43)
    B, H, Sq, Sk = 2, 2, 700, 1000
    q = W.normal_bf16(rng, (B, Sq, H, 128))
    k = W.normal_bf16(rng, (B, Sk, H, 128))
    v = W.normal_bf16(rng, (B, Sk, H, 128))
    vert, slash = W.vertical_slash_indices(np.random.default_rng(1043), B, H, Sk, 70, 90)
    qs = torch.tensor([Sq] * B, dtype=torch.int32, device="cuda")
    ks = torch.tensor([Sk] * B, dtype=torch.int32, device="cuda")
    bc, bo, cc, ci = sb.convert_vertical_slash(qs, ks, torch.from_numpy(vert).cuda(),
                                               torch.from_numpy(slash).cuda(), Sq)
    rbc, rbo, rcc, rci = oracle.convert_vertical_slash([Sq] * B, [Sk] * B, vert, slash, Sq, 64,
                                                       64, True)
    _check_lists((bc, bo, cc, ci), (rbc, rbo, rcc, rci))
    o, lse = sb.fwd_vertical_slash(dev(q), dev(k), dev(v), bc, bo, cc, ci, causal=True)
    ro, rl = oracle.attend_vertical_slash(q, k, v, rbc, rbo, rcc, rci, 64, 64, True,
                                          W.default_scale())
    compare(o, lse, ro, rl, "vs B=2 Sq<Sk")


def _check_lists(gpu, ref):
    bc, bo, cc, ci = (x.cpu().numpy() for x in gpu)
    rbc, rbo, rcc, rci = ref
    assert np.array_equal(bc, rbc) and np.array_equal(cc, rcc)
    for idx in np.ndindex(bc.shape):
        assert np.array_equal(bo[idx][:bc[idx]], rbo[idx][:rbc[idx]])
        assert np.array_equal(ci[idx][:cc[idx]], rci[idx][:rcc[idx]])


# ------------------------------------------------------------------ NSA selected (varlen)

def _nsa_case(seqlens, H, seed):
    return W.make_nsa_varlen(seqlens=seqlens, H=H, seed=seed, table_seed=seed + 1000)


@pytest.mark.parametrize("seqlens", [(700, 300), (1000, 64, 5)])
def test_nsa_varlen_small_all_tokens(sb, seqlens):
    wl = _nsa_case(seqlens, 2, 60 + len(seqlens))
    cu, sel = wl.meta["cu_seqlens"], wl.meta["sel"]
    q, k, v = (dev(x)[0] for x in (wl.q, wl.k, wl.v))
    st = sb.new_status("cuda")
    o, lse = sb.fwd_varlen_selected(q, k, v, torch.from_numpy(cu).cuda(), max(seqlens),
                                    torch.from_numpy(sel).cuda(), status=st)
    sb.check_status(st)
    ro, rl = oracle.attend_selected_varlen(wl.q[0], wl.k[0], wl.v[0], cu, sel, 64, True, wl.scale)
    compare(o[None], lse[None], ro[None], rl[None], f"nsa small {seqlens}")


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (16, 1)])
def test_nsa_varlen_gqa(sb, Hq, Hkv):
    """Query heads sharing a kv head's selection (G = Hq / Hkv rows of a
    unit per list entry): every token and head against the oracle."""
    seqlens = (700, 300, 130)
    rng = np.random.default_rng(70 + Hq)
    total = sum(seqlens)
    q = W.normal_bf16(rng, (total, Hq, 128))
    k = W.normal_bf16(rng, (total, Hkv, 128))
    v = W.normal_bf16(rng, (total, Hkv, 128))
    cu = np.concatenate([[0], np.cumsum(seqlens)]).astype(np.int32)
    sel = W.nsa_selection(np.random.default_rng(1070 + Hq), seqlens, Hkv, 64, 16)
    st = sb.new_status("cuda")
    o, lse = sb.fwd_varlen_selected(dev(q), dev(k), dev(v), torch.from_numpy(cu).cuda(),
                                    max(seqlens), torch.from_numpy(sel).cuda(), status=st)
    sb.check_status(st)
    ro, rl = oracle.attend_selected_varlen(q, k, v, cu, sel, 64, True, W.default_scale())
    compare(o[None], lse[None], ro[None], rl[None], f"nsa gqa Hq={Hq} Hkv={Hkv}")


def test_nsa_varlen_large_key_space(sb):
    """max_seqlen far above the real lengths makes the (kv head, block) key
    space too large for the shared-memory histograms: the inverted index is
    built by the per-entry global-atomic kernels instead."""
    seqlens = (600, 450)
    wl = _nsa_case(seqlens, 2, 77)
    cu, sel = wl.meta["cu_seqlens"], wl.meta["sel"]
    q, k, v = (dev(x)[0] for x in (wl.q, wl.k, wl.v))
    max_seqlen = 600000                      # 2 heads x 2 sequences x 9375 blocks
    st = sb.new_status("cuda")
    o, lse = sb.fwd_varlen_selected(q, k, v, torch.from_numpy(cu).cuda(), max_seqlen,
                                    torch.from_numpy(sel).cuda(), status=st)
    sb.check_status(st)
    ro, rl = oracle.attend_selected_varlen(wl.q[0], wl.k[0], wl.v[0], cu, sel, 64, True, wl.scale)
    compare(o[None], lse[None], ro[None], rl[None], "nsa large key space")


def test_nsa_varlen_full_workload_sampled(sb):
    """cu_seqlens [0, 65536, 98304], Hq=Hkv=4, top-16 blocks of 64; 4 whole
    64-token blocks (256 tokens) per head checked, incl. each sequence's last."""
    wl = W.make_nsa_varlen()
    cu, sel = wl.meta["cu_seqlens"], wl.meta["sel"]
    q, k, v = (dev(x)[0] for x in (wl.q, wl.k, wl.v))
    ws = sb.varlen_selected_workspace(2, 98304, 65536, 4, 4, 16, "cuda")
    for _ in range(2):
        o, lse = sb.fwd_varlen_selected(q, k, v, torch.from_numpy(cu).cuda(), 65536,
                                        torch.from_numpy(sel).cuda(), ws=ws)
    torch.cuda.synchronize()
    rows = {h: np.concatenate([sampled_rows(65536, 64, 700 + h, n=2),
                               65536 + sampled_rows(32768, 64, 800 + h, n=2)]) for h in range(4)}
    ro, rl = oracle.attend_selected_varlen(wl.q[0], wl.k[0], wl.v[0], cu, sel, 64, True,
                                           wl.scale, rows=lambda h: rows[h])
    compare(o[None], lse[None], ro[None], rl[None], "nsa full")


# ------------------------------------------------------------------ varlen (cu_seqlens)

def _cu(lens):
    return np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)


@pytest.mark.parametrize("causal,q_block,kv_block,G", [(True, 64, 128, 4), (False, 128, 64, 1),
                                                        (True, 192, 256, 2)])
def test_fwd_varlen_ragged_sequences(sb, causal, q_block, kv_block, G):
    """Three packed sequences of different lengths (q_len <= k_len, not
    multiples of 64), per-sequence tables of sequence-local blocks with
    padding and a repeat, against the oracle on each sequence alone."""
    rng = np.random.default_rng(600 + q_block + G)
    lq, lk = [300, 64, 777], [300, 200, 900]
    Hkv, nmax = 2, 7
    Hq = Hkv * G
    cu_q, cu_k = _cu(lq), _cu(lk)
    q = W.normal_bf16(rng, (int(cu_q[-1]), Hq, 128))
    k = W.normal_bf16(rng, (int(cu_k[-1]), Hkv, 128))
    v = W.normal_bf16(rng, (int(cu_k[-1]), Hkv, 128))
    nqb = -(-max(lq) // q_block)
    tab = np.full((3, Hkv, nqb, nmax), -1, np.int32)
    for s in range(3):
        nkb = -(-lk[s] // kv_block)
        for g in range(Hkv):
            for i in range(-(-lq[s] // q_block)):
                m = min(nmax - 1, nkb)
                tab[s, g, i, :m] = rng.choice(nkb, size=m, replace=False)
    tab[2, 1, 0, -1] = tab[2, 1, 0, 0]        # a repeat counts once
    st = sb.new_status("cuda")
    o, lse = sb.fwd_varlen(dev(q), dev(k), dev(v), torch.from_numpy(cu_q).cuda(),
                           torch.from_numpy(cu_k).cuda(), max(lq), max(lk),
                           torch.from_numpy(tab).cuda(), q_block, kv_block, causal=causal,
                           status=st)
    sb.check_status(st)
    ro, rl = oracle.attend_block_table_varlen(q, k, v, cu_q, cu_k, tab, q_block, kv_block,
                                              causal, W.default_scale())
    compare(o[None], lse[None], ro[None], rl[None], f"varlen table causal={causal} G={G}")


def test_vertical_slash_varlen(sb):
    """sparse_attn_varlen_func: three packed sequences (q_len <= kv_len),
    lists converted per sequence on the GPU (bit-exact against the oracle),
    then attention over them."""
    rng = np.random.default_rng(610)
    lq, lk = [500, 130, 900], [500, 300, 900]
    H, nnz_v, nnz_s = 4, 80, 100
    cu_q, cu_k = _cu(lq), _cu(lk)
    q = W.normal_bf16(rng, (int(cu_q[-1]), H, 128))
    k = W.normal_bf16(rng, (int(cu_k[-1]), H, 128))
    v = W.normal_bf16(rng, (int(cu_k[-1]), H, 128))
    irng = np.random.default_rng(1610)
    lists = [W.vertical_slash_indices(irng, 1, H, L, nnz_v, nnz_s) for L in lk]
    vert = np.concatenate([x[0] for x in lists])
    slash = np.concatenate([x[1] for x in lists])
    qs = torch.tensor(lq, dtype=torch.int32, device="cuda")
    ks = torch.tensor(lk, dtype=torch.int32, device="cuda")
    g = sb.convert_vertical_slash(qs, ks, torch.from_numpy(vert).cuda(),
                                  torch.from_numpy(slash).cuda(), max(lq))
    ref = oracle.convert_vertical_slash(lq, lk, vert, slash, max(lq), 64, 64, True)
    _check_lists(g, ref)
    st = sb.new_status("cuda")
    o, lse = sb.fwd_vertical_slash_varlen(dev(q), dev(k), dev(v), torch.from_numpy(cu_q).cuda(),
                                          torch.from_numpy(cu_k).cuda(), max(lq), max(lk), *g,
                                          causal=True, status=st)
    sb.check_status(st)
    ro, rl = oracle.attend_vertical_slash_varlen(q, k, v, cu_q, cu_k, *ref, 64, 64, True,
                                                 W.default_scale())
    compare(o[None], lse[None], ro[None], rl[None], "vs varlen")


def test_convert_vertical_slash_mergehead(sb):
    """Per-head entry counts (convert_vertical_slash_indexes_mergehead):
    lists bit-exact against the oracle, then attention over them."""
    wl = _vs_small(L=2048, H=4, nnz_v=120, nnz_s=160, seed=44)
    L = wl.q.shape[1]
    vert, slash = wl.meta["vertical"], wl.meta["slash"]
    vc = np.array([120, 70, 64, 0], dtype=np.int32)
    sc = np.array([160, 64, 100, 5], dtype=np.int32)
    sl = torch.tensor([L], dtype=torch.int32, device="cuda")
    g = sb.convert_vertical_slash_mergehead(sl, sl, torch.from_numpy(vert).cuda(),
                                            torch.from_numpy(slash).cuda(),
                                            torch.from_numpy(vc).cuda(),
                                            torch.from_numpy(sc).cuda(), L)
    ref = oracle.convert_vertical_slash([L], [L], vert, slash, L, 64, 64, True, v_count=vc,
                                        s_count=sc)
    _check_lists(g, ref)
    o, lse = sb.fwd_vertical_slash(dev(wl.q), dev(wl.k), dev(wl.v), *g, causal=True)
    ro, rl = oracle.attend_vertical_slash(wl.q, wl.k, wl.v, *ref, 64, 64, True, wl.scale)
    compare(o, lse, ro, rl, "vs mergehead")


# ------------------------------------------------------------------ sliding window, small blocks

@pytest.mark.parametrize("Sq,Sk,window,G", [(2048, 2048, 512, 4), (700, 1000, 100, 1)])
def test_sliding_window(sb, Sq, Sk, window, G):
    """NSA's window branch (window 512 in the FSA Quickstart), and a window
    that is not a multiple of 64 with q_len < kv_len; all rows checked."""
    rng = np.random.default_rng(620 + window)
    Hkv = 2
    q = W.normal_bf16(rng, (1, Sq, Hkv * G, 128))
    k = W.normal_bf16(rng, (1, Sk, Hkv, 128))
    v = W.normal_bf16(rng, (1, Sk, Hkv, 128))
    st = sb.new_status("cuda")
    o, lse = sb.fwd_window(dev(q), dev(k), dev(v), window, status=st)
    sb.check_status(st)
    ro, rl = oracle.attend_window(q, k, v, window, W.default_scale())
    compare(o, lse, ro, rl, f"window {window} Sq={Sq} Sk={Sk}")


def test_sliding_window_varlen(sb):
    rng = np.random.default_rng(630)
    lq, lk = [900, 64, 1300], [900, 300, 1300]
    Hq, Hkv = 4, 2
    cu_q, cu_k = _cu(lq), _cu(lk)
    q = W.normal_bf16(rng, (int(cu_q[-1]), Hq, 128))
    k = W.normal_bf16(rng, (int(cu_k[-1]), Hkv, 128))
    v = W.normal_bf16(rng, (int(cu_k[-1]), Hkv, 128))
    o, lse = sb.fwd_window_varlen(dev(q), dev(k), dev(v), torch.from_numpy(cu_q).cuda(),
                                  torch.from_numpy(cu_k).cuda(), max(lq), max(lk), 512)
    ro, rl = oracle.attend_window_varlen(q, k, v, cu_q, cu_k, 512, W.default_scale())
    compare(o[None], lse[None], ro[None], rl[None], "window varlen")


@pytest.mark.parametrize("kv_block,causal", [(16, True), (32, False), (16, False), (32, True)])
def test_block_table_small_blocks_tiled(sb, kv_block, causal):
    """Table blocks of 16 and 32 keys (README: block_size in {16, 32, 64,
    128, 256} at hdim 128) on the tiled kernel, Sq = Sk = 2048, GQA 4, with
    padding and a repeat."""
    rng = np.random.default_rng(640 + kv_block + causal)
    S, Hkv, G, nmax = 2048, 2, 4, 40
    q = W.normal_bf16(rng, (1, S, Hkv * G, 128))
    k = W.normal_bf16(rng, (1, S, Hkv, 128))
    v = W.normal_bf16(rng, (1, S, Hkv, 128))
    nkb = S // kv_block
    tab = np.stack([np.stack([rng.choice(nkb, size=nmax, replace=False) for _ in range(S // 64)])
                    for _ in range(Hkv)])[None].astype(np.int32)
    tab[..., -3:] = -1
    tab[..., -4] = tab[..., 0]
    st = sb.new_status("cuda")
    o, lse = sb.fwd(dev(q), dev(k), dev(v), torch.from_numpy(tab).cuda(), 64, kv_block,
                    causal=causal, status=st)
    sb.check_status(st)
    ro, rl = oracle.attend_block_table(q, k, v, tab, 64, kv_block, causal, W.default_scale())
    compare(o, lse, ro, rl, f"kv_block {kv_block} causal={causal}")
