"""The bulk-copy (TMA engine) form of dispatch against the register form and
the oracle, through the C ABI: the same bytes in every slot, on every
workload at full size (long rows, where one or two pipelines fit a block,
included), with poisoned destination buffers and an out-of-range slot."""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_mep_b200 as mep
import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_bulk_dispatch_equals_register_dispatch(name):
    wl = workloads.WORKLOADS[name]
    s = mep.Shape(*wl.shape())
    idx, _ = workloads.routing(wl)
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    x = workloads.hidden(wl.N, wl.H, seed=1, device=DEV)
    ref = torch.empty((wl.NK, wl.H), dtype=torch.bfloat16, device=DEV)
    got = torch.full((wl.NK, wl.H), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    mep.mep_dispatch(s, wl.H, plan, x, ref)
    mep.mep_dispatch_bulk(s, wl.H, plan, x, got)
    assert mep.mep_read_status(plan) == 0
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


@pytest.mark.parametrize("H", [8, 136, 2048, 32768])
def test_bulk_dispatch_row_sizes_against_the_oracle(H):
    R, S, E, K = 4, 37, 16, 3
    rng = np.random.default_rng(H)
    idx = np.argsort(rng.random((R * S, E)), axis=1)[:, :K].astype(np.int32)
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    x = workloads.hidden(R * S, H, seed=3)
    got = torch.full((R * S * K, H), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    mep.mep_dispatch_bulk(s, H, plan, x.to(DEV), got)
    assert mep.mep_read_status(plan) == 0
    pl = oracle.get().plan(R, S, E, K, idx)
    assert np.array_equal(_u16(got), oracle.get().dispatch(K, pl["src_pair"], _u16(x)))


def test_bulk_dispatch_reports_a_bad_slot():
    R, S, E, K, H = 2, 16, 4, 2, 64
    s = mep.Shape(R, S, E, K)
    idx = np.zeros((R * S, K), dtype=np.int32)
    idx[:, 1] = 1
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    plan.slot[5, 1] = R * S * K          # one past the end: skipped, reported
    x = workloads.hidden(R * S, H, seed=2, device=DEV)
    buf = torch.zeros((R * S * K, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_dispatch_bulk(s, H, plan, x, buf)
    assert mep.mep_read_status(plan) == 5
