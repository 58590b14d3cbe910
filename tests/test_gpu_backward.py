"""Backward of combine and dispatch on the GPU against the oracle, through the C ABI.

Tolerances (derived from the arithmetic):
  * grad_y = bf16(w * grad_out): the kernel rounds the exact product once
    (round-to-odd float32, then nearest-even bf16), so it must be bit-exact.
  * grad_w: each lane sums H/32 products with float32 FMAs, then a 5-level
    butterfly adds the lanes: |gpu - exact| <= (H/32 + 6) * 2^-24 * sum|terms|.
  * grad_x = bf16(sum_k grad_buf): same rule as the forward combine (1 bf16
    ulp unless cancellation makes the float32 bound exceed half an ulp).
"""
import numpy as np
import pytest
import torch

import oracle
import parity
import token_dispatch_mep_b200 as mep
import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def ora():
    return oracle.get()


def _u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def check_grad_w(gpu, exact, absum, H, what=""):
    tol = (H / 32 + 6) * 2.0 ** -24 * absum * (1 + 1e-9)
    err = np.abs(np.asarray(gpu, np.float64) - exact)
    assert np.all(err <= tol), f"grad_w {what}: {int((err > tol).sum())} out of tolerance"


def _backward(shape, H, idx, w, go, y, gb):
    s = mep.Shape(*shape)
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.as_tensor(idx).to(DEV), plan)
    grad_y = torch.empty((s.NK, H), dtype=torch.bfloat16, device=DEV)
    grad_y.view(torch.int16).fill_(-1)
    grad_w = torch.full((s.N, s.K), float("nan"), dtype=torch.float32, device=DEV)
    grad_x = torch.empty((s.N, H), dtype=torch.bfloat16, device=DEV)
    grad_x.view(torch.int16).fill_(-1)
    mep.mep_combine_backward(s, H, plan, go, torch.as_tensor(w).to(DEV), y, grad_y, grad_w)
    mep.mep_dispatch_backward(s, H, plan, gb, grad_x)
    assert mep.mep_read_status(plan) == 0
    return plan, grad_y, grad_w, grad_x


REDUCED = [("tiny_r4_e16", 64, None), ("r8_e64_h2048", 517, None), ("r16_e256_h7168", 33, None),
           ("kimi_r64_e896_k16", 41, None), ("skew_r32_zipf1.5", 67, 1032),
           ("skew_r32_adversarial", 67, 264)]


@pytest.mark.parametrize("name,S,H", REDUCED, ids=[r[0] for r in REDUCED])
def test_backward_every_element(ora, name, S, H):
    wl = workloads.reduced(workloads.WORKLOADS[name], S=S, H=H)
    R, E, K, H, N, NK = wl.R, wl.E, wl.K, wl.H, wl.N, wl.NK
    idx, w = workloads.routing(wl)
    go = workloads.hidden(N, H, seed=11)
    y = workloads.expert_outputs(NK, H, seed=12)
    gb = workloads.expert_outputs(NK, H, seed=13)
    plan, grad_y, grad_w, grad_x = _backward(wl.shape(), H, idx, w, go.to(DEV), y.to(DEV), gb.to(DEV))
    pl = ora.plan(R, S, E, K, idx)
    gy, _, gw, gwa = ora.combine_backward(pl["slot"], w, _u16(go), _u16(y))
    assert np.array_equal(_u16(grad_y), gy), "grad_y not bit-exact"
    check_grad_w(grad_w.cpu().numpy(), gw, gwa, H, name)
    gx, ex, ab = ora.dispatch_backward(pl["slot"], _u16(gb))
    parity.check_combine(_u16(grad_x), gx, ex, ab, K, name)


@pytest.mark.parametrize("name", ["r8_e64_h2048", "kimi_r64_e896_k16", "r16_e256_h7168",
                                  "skew_r32_zipf1.5"])
def test_backward_full_size_sampled(ora, name):
    wl = workloads.WORKLOADS[name]
    R, S, E, K, H, N, NK = wl.R, wl.S, wl.E, wl.K, wl.H, wl.N, wl.NK
    idx, w = workloads.routing(wl)
    go = workloads.hidden(N, H, seed=11, device=DEV)
    y = workloads.expert_outputs(NK, H, seed=12, device=DEV)
    gb = workloads.expert_outputs(NK, H, seed=13, device=DEV)
    plan, grad_y, grad_w, grad_x = _backward(wl.shape(), H, idx, w, go, y, gb)
    pl = ora.plan(R, S, E, K, idx)
    rng = np.random.default_rng(9)
    toks = np.unique(np.concatenate([np.arange(32), np.arange(N - 32, N), rng.integers(0, N, 96)]))
    sl = pl["slot"][toks]
    slt = torch.from_numpy(sl.reshape(-1)).to(DEV).long()
    tt = torch.from_numpy(toks).to(DEV).long()
    local = np.arange(sl.size, dtype=np.int32).reshape(sl.shape)
    gy, _, gw, gwa = ora.combine_backward(local, w[toks], _u16(go.index_select(0, tt)),
                                          _u16(y.index_select(0, slt)))
    assert np.array_equal(_u16(grad_y.index_select(0, slt)), gy)
    check_grad_w(grad_w.index_select(0, tt).cpu().numpy(), gw, gwa, H, name)
    gx, ex, ab = ora.dispatch_backward(local, _u16(gb.index_select(0, slt)))
    parity.check_combine(_u16(grad_x.index_select(0, tt)), gx, ex, ab, K, name)
    # every slot row of grad_y was written (no poison left)
    assert not bool((grad_y.view(torch.int16) == -1).all(dim=1).any())


def test_backward_reports_bad_slots(ora):
    R, S, E, K, H = 2, 16, 4, 2, 16
    rng = np.random.default_rng(1)
    idx = np.argsort(-rng.standard_normal((R * S, E)), axis=1)[:, :K].astype(np.int32)
    idx[5, 0] = 7                                          # out of range
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    z = lambda *shape: torch.zeros(shape, dtype=torch.bfloat16, device=DEV)
    mep.mep_combine_backward(s, H, plan, z(R * S, H), torch.ones(R * S, K, device=DEV),
                             z(R * S * K, H), z(R * S * K, H),
                             torch.zeros(R * S, K, device=DEV))
    mep.mep_dispatch_backward(s, H, plan, z(R * S * K, H), z(R * S, H))
    assert mep.mep_read_status(plan) == 5
