"""Rank-addressed dispatch and combine: every rank's S*K slots in a buffer of
its own (the layout of the exchange between GPUs), here R separate device
allocations on one GPU.  Results must equal the oracle and the single-buffer
calls bit for bit."""
import numpy as np
import pytest
import torch

import oracle
import parity
import token_dispatch_mep_b200 as mep
import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("name,S,H", [("tiny_r4_e16", 64, 128), ("r8_e64_h2048", 517, 2048),
                                      ("kimi_r64_e896_k16", 29, 1024), ("skew_r32_zipf1.5", 67, 264)])
@pytest.mark.parametrize("home_first", [False, True])
def test_ranked_matches_oracle_and_single_buffer(name, S, H, home_first):
    ora = oracle.get()
    wl = workloads.reduced(workloads.WORKLOADS[name], S=S, H=H)
    R, E, K, N, NK, SK = wl.R, wl.E, wl.K, wl.N, wl.NK, wl.SK
    idx, w = workloads.routing(wl)
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, DEV)
    (mep.mep_plan_home_first if home_first else mep.mep_plan)(s, torch.from_numpy(idx).to(DEV), plan)
    pl = (ora.plan_home_first if home_first else ora.plan)(R, S, E, K, idx)
    x = workloads.hidden(N, H, seed=1).to(DEV)
    y = workloads.expert_outputs(NK, H, seed=2).to(DEV)
    wd = torch.from_numpy(w).to(DEV)
    # R separate receive buffers, poisoned
    bufs = [torch.full((SK, H), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16) for _ in range(R)]
    table = mep.rank_pointer_table(bufs, s, H, DEV)
    mep.mep_dispatch_ranked(s, H, plan, x, table)
    ys = [y[r * SK:(r + 1) * SK].clone() for r in range(R)]
    ytab = mep.rank_pointer_table(ys, s, H, DEV)
    out_r = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_combine_ranked(s, H, plan, ytab, wd, out_r)
    # single-buffer reference calls
    buf = torch.empty((NK, H), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_dispatch(s, H, plan, x, buf)
    mep.mep_combine(s, H, plan, y, wd, out)
    assert mep.mep_read_status(plan) == 0
    assert torch.equal(torch.cat(bufs).view(torch.int16), buf.view(torch.int16))
    assert torch.equal(out_r.view(torch.int16), out.view(torch.int16))
    want = ora.dispatch(K, pl["src_pair"], _u16(x))
    assert np.array_equal(_u16(torch.cat(bufs)), want)
    ob, ex, ab = ora.combine(pl["slot"], w, _u16(y))
    parity.check_combine(_u16(out_r), ob, ex, ab, K, name)
