"""Replica weight prefetch on the GPU against the oracle (bit-exact copies),
through the C ABI, on every workload's plan."""
import numpy as np
import pytest
import torch

import oracle
import token_dispatch_mep_b200 as mep
import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def ora():
    return oracle.get()


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
@pytest.mark.parametrize("dtype,cols", [(torch.float32, 4100), (torch.bfloat16, 8 * 129)])
def test_prefetch_matches_oracle(ora, name, dtype, cols):
    wl = workloads.WORKLOADS[name]
    idx, _ = workloads.routing(wl)
    s = mep.Shape(*wl.shape())
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    g = torch.Generator(device=DEV)
    g.manual_seed(7)
    w_home = torch.randn((wl.E, cols), generator=g, device=DEV).to(dtype)
    w_rep = torch.full((wl.seg_rows, cols), -7.0, device=DEV).to(dtype)
    mep.mep_prefetch_replica_weights(s, plan, w_home, w_rep)
    assert mep.mep_read_status(plan) == 0
    h = plan.host()
    nr = h["num_replicas"]
    view = torch.int16 if dtype == torch.bfloat16 else torch.int32
    want = ora.prefetch_replicas(h, w_home.view(view).cpu().numpy())
    got = w_rep.view(view).cpu().numpy()
    assert np.array_equal(got[:nr], want)
    assert bool((w_rep[nr:] == -7.0).all())                 # rows past num_replicas untouched
    pl = ora.plan(*wl.shape(), idx)
    assert nr == pl["num_replicas"]


def test_prefetch_full_gradient_row_size(ora):
    """Rows the size of the bench workload's expert weights (3 x 2048 x 1024 fp32)."""
    wl = workloads.WORKLOADS["r8_e64_h2048"]
    idx, _ = workloads.routing(wl)
    s = mep.Shape(*wl.shape())
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    w_home = workloads.seg_grads(wl.E, wl.P, seed=8, device=DEV)
    w_rep = torch.zeros((wl.seg_rows, wl.P), dtype=torch.float32, device=DEV)
    mep.mep_prefetch_replica_weights(s, plan, w_home, w_rep)
    h = plan.host()
    nr = h["num_replicas"]
    experts = [int(h["seg"][h["replica_seg"][j]][0]) for j in range(nr)]
    for j, e in enumerate(experts):
        assert torch.equal(w_rep[j], w_home[e])
    assert mep.mep_read_status(plan) == 0
