"""Failure paths on the GPU, in the forms that leave the context usable.

* Bad indices: table, vertical/slash and selection entries that name keys
  outside the sequence are skipped by the kernels and reported through the
  device status word (SBFA_ERR_DEVICE from sbfa_check_status); the results
  over the valid entries still match the oracle, which drops keys past the
  end of the sequence by definition.
* Wait limit: with the bounded-wait limit set to 100 ns, waits inside the
  pipelined kernels run out; the CTAs drain their copies and tensor-core
  operations, stop, and report SBFA_ERR_TIMEOUT.  A normal call on the same
  stream afterwards must still be correct.
"""
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


def compare(o_gpu, lse_gpu, o_ref, lse_ref, what):
    o = o_gpu.float().cpu().numpy().astype(np.float64)
    lse = lse_gpu.float().cpu().numpy().astype(np.float64)
    rows = ~np.isnan(lse_ref)
    err_o = np.abs(o[~np.isnan(o_ref)] - o_ref[~np.isnan(o_ref)]).max()
    lr, lg = lse_ref[rows], lse[rows]
    fin = np.isfinite(lr)
    assert np.array_equal(fin, np.isfinite(lg)), what
    err_l = np.abs(lg[fin] - lr[fin]).max() if fin.any() else 0.0
    print(f"{what}: o max-abs {err_o:.3e}, lse max-abs {err_l:.3e}")
    assert err_o <= O_TOL and err_l <= LSE_TOL, what


def expect_code(sb, st, code):
    with pytest.raises(sb.SbfaError) as e:
        sb.check_status(st)
    assert e.value.code == code, str(e.value)
    print(f"status: {e.value}")


# ------------------------------------------------------------------ bad indices

@pytest.mark.parametrize("Sq,causal", [(256, True), (1, False)])
def test_bad_table_entries_are_skipped_and_reported(sb, Sq, causal):
    """Entries >= ceil(Sk / kv_block) in a block table: the tiled kernel
    (Sq = 256) and the split-KV kernel (Sq = 1)."""
    rng = np.random.default_rng(501)
    B, Hq, Hkv, Sk, bs, nmax = 2, 8, 2, 1000, 64, 6
    q = W.normal_bf16(rng, (B, Sq, Hq, 128))
    k = W.normal_bf16(rng, (B, Sk, Hkv, 128))
    v = W.normal_bf16(rng, (B, Sk, Hkv, 128))
    nkb = -(-Sk // bs)
    nqb = -(-Sq // 64)
    tab = np.stack([np.stack([np.stack([rng.choice(nkb, size=nmax, replace=False)
                                        for _ in range(nqb)]) for _ in range(Hkv)])
                    for _ in range(B)]).astype(np.int32)
    tab[0, 0, 0, 1] = nkb            # one past the end
    tab[1, 1, -1, 3] = nkb + 1000
    st = sb.new_status("cuda")
    o, lse = sb.fwd(dev(q), dev(k), dev(v), torch.from_numpy(tab).cuda(), 64 if Sq > 1 else 1,
                    bs, causal=causal, status=st)
    expect_code(sb, st, sb.ERR_DEVICE)
    ro, rl = oracle.attend_block_table(q, k, v, tab, 64 if Sq > 1 else 1, bs, causal,
                                       W.default_scale())
    compare(o, lse, ro, rl, f"bad table entries Sq={Sq}")


def test_bad_vertical_slash_entries_are_skipped_and_reported(sb):
    """A block offset past the end of the keys and a column index past the
    end, appended to converted lists."""
    wl = W.make_vertical_slash(B=1, H=2, L=512, nnz_v=80, nnz_s=100, seed=502, table_seed=1502)
    L = wl.q.shape[1]
    bc, bo, cc, ci = oracle.convert_vertical_slash([L], [L], wl.meta["vertical"],
                                                   wl.meta["slash"], L, 64, 64, True)
    i = 5
    assert bc[0, 0, i] < bo.shape[-1] and cc[0, 1, i] < ci.shape[-1]
    bo[0, 0, i, bc[0, 0, i]] = L + 64
    bc[0, 0, i] += 1
    ci[0, 1, i, cc[0, 1, i]] = L + 3
    cc[0, 1, i] += 1
    st = sb.new_status("cuda")
    o, lse = sb.fwd_vertical_slash(dev(wl.q), dev(wl.k), dev(wl.v),
                                   *(torch.from_numpy(x).cuda() for x in (bc, bo, cc, ci)),
                                   causal=True, status=st)
    expect_code(sb, st, sb.ERR_DEVICE)
    ro, rl = oracle.attend_vertical_slash(wl.q, wl.k, wl.v, bc, bo, cc, ci, 64, 64, True,
                                          wl.scale)
    compare(o, lse, ro, rl, "bad vertical/slash entries")


def test_bad_selection_entries_are_skipped_and_reported(sb):
    """NSA selections naming a block past the end of their sequence."""
    wl = W.make_nsa_varlen(seqlens=(700, 300), H=2, seed=503, table_seed=1503)
    cu, sel = wl.meta["cu_seqlens"], wl.meta["sel"].copy()
    free = np.argwhere(sel < 0)
    pick = free[np.random.default_rng(5).choice(len(free), size=20, replace=False)]
    for t, g, c in pick:
        seq = 0 if t < cu[1] else 1
        sel[t, g, c] = -(-(cu[seq + 1] - cu[seq]) // 64) + int(c)   # >= blocks in the sequence
    q, k, v = (dev(x)[0] for x in (wl.q, wl.k, wl.v))
    st = sb.new_status("cuda")
    o, lse = sb.fwd_varlen_selected(q, k, v, torch.from_numpy(cu).cuda(), 700,
                                    torch.from_numpy(sel).cuda(), status=st)
    expect_code(sb, st, sb.ERR_DEVICE)
    ro, rl = oracle.attend_selected_varlen(wl.q[0], wl.k[0], wl.v[0], cu, sel, 64, True, wl.scale)
    compare(o[None], lse[None], ro[None], rl[None], "bad selection entries")


# ------------------------------------------------------------------ wait limit

def _short_limit_then_normal(sb, run, check):
    """run(status) under a 100 ns wait limit must report a timeout; with the
    default limit restored, run(status) again must pass check()."""
    st = sb.new_status("cuda")
    prev = sb.set_wait_limit_ns(100)
    try:
        run(st)
        expect_code(sb, st, sb.ERR_TIMEOUT)
    finally:
        sb.set_wait_limit_ns(prev)
    st2 = sb.new_status("cuda")
    out = run(st2)
    sb.check_status(st2)
    check(out)


def test_wait_limit_block_table(sb):
    rng = np.random.default_rng(511)
    B, S, Hq, Hkv = 1, 2048, 8, 2
    q = W.normal_bf16(rng, (B, S, Hq, 128))
    k = W.normal_bf16(rng, (B, S, Hkv, 128))
    v = W.normal_bf16(rng, (B, S, Hkv, 128))
    tab = np.broadcast_to(np.arange(S // 64, dtype=np.int32), (B, Hkv, S // 64, S // 64)).copy()
    qd, kd, vd, td = dev(q), dev(k), dev(v), torch.from_numpy(tab).cuda()

    def run(st):
        return sb.fwd(qd, kd, vd, td, 64, 64, causal=True, status=st)

    def check(out):
        rows = lambda b, h: np.arange(S - 64, S)  # noqa: E731
        ro, rl = oracle.attend_block_table(q, k, v, tab, 64, 64, True, W.default_scale(),
                                           rows=rows)
        compare(out[0], out[1], ro, rl, "after timeout: block table")

    _short_limit_then_normal(sb, run, check)


def test_wait_limit_gated(sb):
    L, Hq, Hkv = 2048, 8, 2
    wl = W.make_gated(B=1, Hq=Hq, Hkv=Hkv, L=L, seed=512)
    T = np.full((Hq, L // 64), -np.inf, dtype=np.float32)   # every block kept: no gate ties
    qd, kd, vd, Td = dev(wl.q), dev(wl.k), dev(wl.v), torch.from_numpy(T).cuda()

    def run(st):
        return sb.fwd_gated(qd, kd, vd, Td, status=st)

    def check(out):
        rows = lambda b, h: np.arange(L - 64, L)  # noqa: E731
        ro, rl = oracle.attend_gated(wl.q, wl.k, wl.v, T, 64, wl.scale, rows=rows)
        compare(out[0], out[1], ro, rl, "after timeout: gated")

    _short_limit_then_normal(sb, run, check)


def test_wait_limit_nsa(sb):
    wl = W.make_nsa_varlen(seqlens=(3000, 1000), H=2, seed=513, table_seed=1513)
    cu, sel = wl.meta["cu_seqlens"], wl.meta["sel"]
    q, k, v = (dev(x)[0] for x in (wl.q, wl.k, wl.v))
    cud, seld = torch.from_numpy(cu).cuda(), torch.from_numpy(sel).cuda()

    def run(st):
        return sb.fwd_varlen_selected(q, k, v, cud, 3000, seld, status=st)

    def check(out):
        toks = np.arange(2900, 3100)
        ro, rl = oracle.attend_selected_varlen(wl.q[0], wl.k[0], wl.v[0], cu, sel, 64, True,
                                               wl.scale, rows=lambda h: toks)
        compare(out[0][None], out[1][None], ro[None], rl[None], "after timeout: nsa")

    _short_limit_then_normal(sb, run, check)
