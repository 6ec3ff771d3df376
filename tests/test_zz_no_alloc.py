"""The allocation-free decode entry point (fixed scratch compiled into the
library, for callers that cannot call cudaMalloc) must give the results of
the workspace entry point, and match the fp64 oracle, on two calls in a row
(the second call reuses the scratch the first one left behind).  Collected
last on purpose."""
import numpy as np
import pytest
import torch

import oracle
import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sb():
    if not torch.cuda.is_available():
        pytest.skip("no GPU")
    import block_sparse_flashattention_sbfa_b200 as m
    return m


@pytest.mark.parametrize("shape", [dict(B=8, Hq=32, Hkv=8, Lq=1, Lk=32768),
                                   dict(B=3, Hq=8, Hkv=2, Lq=2, Lk=4096)])
def test_noalloc_matches_workspace_entry_point(sb, shape):
    wl = W.make_spec_decode(block=128, spec_len=512 if shape["Lk"] < 8192 else 2048,
                            n_missed=6 if shape["Lk"] < 8192 else 32, seed=90, table_seed=91,
                            **shape)
    s0 = wl.meta["spec_begin"]
    q, k, v = (W.to_torch_bf16(x, "cuda") for x in (wl.q, wl.k, wl.v))
    tab = torch.from_numpy(wl.meta["table"]).cuda()
    ref_o, ref_l = sb.speculative_sparse(q, k[:, s0:], v[:, s0:], True, k, v, tab, 128)
    oo, ol = oracle.speculative_sparse(wl.q, wl.k[:, s0:], wl.v[:, s0:], True, wl.k, wl.v,
                                       wl.meta["table"], 128, wl.scale)
    st = sb.new_status("cuda")
    out = torch.empty_like(q)
    lse = torch.empty_like(ref_l)
    for call in range(2):
        out.fill_(float("nan"))
        lse.fill_(float("nan"))
        sb.speculative_sparse_noalloc(q, k[:, s0:], v[:, s0:], True, k, v, tab, 128, out=out,
                                      lse=lse, status=st)
        sb.check_status(st)
        eo = (out.float() - ref_o.float()).abs().max().item()
        el = (lse - ref_l).abs().max().item()
        ro = np.abs(out.float().cpu().numpy() - oo).max()
        rl = np.abs(lse.cpu().numpy() - ol).max()
        print(f"no-alloc call {call}: vs workspace path o {eo:.2e} lse {el:.2e}; "
              f"vs oracle o {ro:.2e} lse {rl:.2e}")
        assert eo <= 2e-2 and el <= 1e-3
        assert ro <= 2e-2 and rl <= 1e-3


def test_noalloc_rejects_too_many_pairs(sb):
    q = torch.zeros(1, 1, 8, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(4097, 64, 1, 128, dtype=torch.bfloat16, device="cuda")[:1].expand(4097, -1, -1, -1)
    qq = q.expand(4097, -1, -1, -1)
    tab = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(sb.SbfaError, match="fixed scratch limit"):
        sb.speculative_sparse_noalloc(qq, k, k, True, k, k, tab, 64,
                                      out=torch.empty(4097, 1, 8, 128, dtype=torch.bfloat16,
                                                      device="cuda"))
