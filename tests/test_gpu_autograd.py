"""Dispatch and combine inside torch autograd (token_dispatch_mep_b200.autograd):
the gradients autograd produces are exactly those of the explicit backward
calls (which are themselves checked against the oracle in
test_gpu_backward.py), for a chained dispatch -> expert -> combine step too."""
import numpy as np
import pytest
import torch

import token_dispatch_mep_b200 as mep
import workloads
from token_dispatch_mep_b200 import autograd as mag

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _bits(t):
    return t.detach().contiguous().view(torch.int16)


@pytest.mark.parametrize("name,S,H", [("r8_e64_h2048", 97, 256), ("kimi_r64_e896_k16", 9, 128)])
@pytest.mark.parametrize("home_first", [False, True])
def test_autograd_matches_explicit_backward(name, S, H, home_first):
    wl = workloads.reduced(workloads.WORKLOADS[name], S=S, H=H)
    R, E, K, N, NK = wl.R, wl.E, wl.K, wl.N, wl.NK
    idx, w = workloads.routing(wl)
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, DEV)
    (mep.mep_plan_home_first if home_first else mep.mep_plan)(s, torch.from_numpy(idx).to(DEV), plan)

    x = workloads.hidden(N, H, seed=1).to(DEV).requires_grad_()
    y = workloads.expert_outputs(NK, H, seed=2).to(DEV).view(R, S * K, H).requires_grad_()
    wt = torch.from_numpy(w).to(DEV).requires_grad_()
    gb = workloads.expert_outputs(NK, H, seed=3).to(DEV).view(R, S * K, H)
    go = workloads.hidden(N, H, seed=4).to(DEV)

    buf = mag.dispatch(x, plan)
    out = mag.combine(y, wt, plan)
    buf.backward(gb)
    out.backward(go)

    ref_buf = torch.empty_like(gb)
    mep.mep_dispatch(s, H, plan, x.detach(), ref_buf)
    ref_out = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_combine(s, H, plan, y.detach(), wt.detach(), ref_out)
    gx = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_dispatch_backward(s, H, plan, gb, gx)
    gy = torch.empty_like(gb)
    gw = torch.empty((N, K), dtype=torch.float32, device=DEV)
    mep.mep_combine_backward(s, H, plan, go, wt.detach(), y.detach(), gy, gw)
    assert mep.mep_read_status(plan) == 0

    assert torch.equal(_bits(buf), _bits(ref_buf))
    assert torch.equal(_bits(out), _bits(ref_out))
    assert torch.equal(_bits(x.grad), _bits(gx))
    assert torch.equal(_bits(y.grad), _bits(gy))
    assert torch.equal(wt.grad.view(torch.int32), gw.view(torch.int32))


def test_chained_step_backward():
    """dispatch -> an elementwise 'expert' -> combine, one backward pass: the
    input gradient is dispatch-backward of (2 x combine-backward's slot
    gradient), the weight gradient combine-backward's."""
    wl = workloads.reduced(workloads.WORKLOADS["skew_r32_zipf1.5"], S=21, H=64)
    R, S, E, K, H, N, NK = wl.R, wl.S, wl.E, wl.K, wl.H, wl.N, wl.NK
    idx, w = workloads.routing(wl)
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    x = workloads.hidden(N, H, seed=1).to(DEV).requires_grad_()
    wt = torch.from_numpy(w).to(DEV).requires_grad_()
    go = workloads.hidden(N, H, seed=4).to(DEV)

    buf = mag.dispatch(x, plan)
    y = buf * 2                               # exact in bf16
    out = mag.combine(y, wt, plan)
    out.backward(go)

    y_ref = torch.empty((R, S * K, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_dispatch(s, H, plan, x.detach(), y_ref)
    y_ref = y_ref * 2
    gy = torch.empty_like(y_ref)
    gw = torch.empty((N, K), dtype=torch.float32, device=DEV)
    mep.mep_combine_backward(s, H, plan, go, wt.detach(), y_ref, gy, gw)
    gx = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_dispatch_backward(s, H, plan, gy * 2, gx)
    assert mep.mep_read_status(plan) == 0
    assert torch.equal(_bits(x.grad), _bits(gx))
    assert torch.equal(wt.grad.view(torch.int32), gw.view(torch.int32))
    assert np.isfinite(wt.grad.cpu().numpy()).all()


def test_type_checks():
    s = mep.Shape(2, 4, 4, 2)
    with pytest.raises(TypeError):
        mag.dispatch(torch.zeros((8, 16), device=DEV), None)
    with pytest.raises(TypeError):
        mag.combine(torch.zeros((16, 16), dtype=torch.bfloat16, device=DEV),
                    torch.zeros((8, 2), dtype=torch.float64, device=DEV), None)
    del s
