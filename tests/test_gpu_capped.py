"""The capped plan (at most B replica experts per rank) on the GPU against the
oracle, and the data movement driven by it (dispatch, combine,
replica-gradient reduce, replica weight prefetch), through the C ABI.

B follows the pages' two values ("Moonshot AI Open-Sources MoonEP, the Library
Used to Train the MoE Model Kimi K3", "Key facts about the release": B = E/R
for training, 3-4 for inference) and the edges B = 1, 2.  Every plan field and
the reported largest replica count per rank must equal the oracle's bit for
bit."""
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


def _capped(shape, B, idx):
    s = mep.Shape(*shape)
    plan = mep.Plan(s, DEV)
    mr = torch.full((1,), -7, dtype=torch.int32, device=DEV)
    mep.mep_plan_capped(s, B, torch.as_tensor(idx, dtype=torch.int32).to(DEV), plan, mr)
    assert mep.mep_read_status(plan) == 0
    return s, plan, int(mr.item())


def _check(plan, mr, pl, what):
    parity.check_plan(plan.host(), pl, what)
    assert mr == pl["max_rank_replicas"], (what, mr, pl["max_rank_replicas"])


REDUCED = [("tiny_r4_e16", 64, None, 100), ("r8_e64_h2048", 1031, 264, 4100),
           ("r16_e256_h7168", 65, 520, 1027), ("kimi_r64_e896_k16", 97, 136, 2052),
           ("skew_r32_uniform", 131, 256, 996), ("skew_r32_zipf1.5", 131, 264, 4096),
           ("skew_r32_adversarial", 131, 128, 8)]


@pytest.mark.parametrize("name,S,H,P", REDUCED, ids=[r[0] for r in REDUCED])
def test_capped_every_element(ora, name, S, H, P):
    wl = workloads.reduced(workloads.WORKLOADS[name], S=S, H=H, P=P)
    R, E, K, H, N, NK = wl.R, wl.E, wl.K, wl.H, wl.N, wl.NK
    idx, w = workloads.routing(wl)
    for B in (1, 2, 3, 4, E // R):
        s, plan, mr = _capped(wl.shape(), B, idx)
        _check(plan, mr, ora.plan_capped(R, S, E, K, B, idx), f"{name} B={B}")
    B = 4
    s, plan, mr = _capped(wl.shape(), B, idx)
    pl = ora.plan_capped(R, S, E, K, B, idx)
    x = workloads.hidden(N, H, seed=1)
    y = workloads.expert_outputs(NK, H, seed=2)
    G = workloads.seg_grads(wl.seg_rows, P, seed=3)
    buf = torch.empty((NK, H), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
    home = torch.empty((E, P), dtype=torch.float32, device=DEV)
    mep.mep_dispatch(s, H, plan, x.to(DEV), buf)
    mep.mep_combine(s, H, plan, y.to(DEV), torch.from_numpy(w).to(DEV), out)
    mep.mep_reduce_replica_grads(s, plan, P, G.to(DEV), home)
    w_home = workloads.seg_grads(E, 64, seed=4)
    w_rep = torch.zeros((wl.seg_rows, 64), dtype=torch.float32, device=DEV)
    mep.mep_prefetch_replica_weights(s, plan, w_home.to(DEV), w_rep)
    assert mep.mep_read_status(plan) == 0
    assert np.array_equal(_u16(buf), ora.dispatch(K, pl["src_pair"], _u16(x)))
    ob, ex, ab = ora.combine(pl["slot"], w, _u16(y))
    parity.check_combine(_u16(out), ob, ex, ab, K, name)
    hx, ha = ora.reduce(pl["expert_seg_ptr"], G.numpy())
    parity.check_reduce(home.cpu().numpy(), hx, ha, np.diff(pl["expert_seg_ptr"]), name)
    nr = pl["num_replicas"]
    assert np.array_equal(w_rep[:nr].cpu().numpy(), ora.prefetch_replicas(pl, w_home.numpy()))


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_capped_full_size_plan(ora, name):
    """Full size, B = E/R (training) and B = 4 (inference): the whole plan
    bit-exact, and the dispatch through it checked on every row."""
    wl = workloads.WORKLOADS[name]
    idx, _ = workloads.routing(wl)
    for B in (wl.E // wl.R, 4):
        s, plan, mr = _capped(wl.shape(), B, idx)
        pl = ora.plan_capped(*wl.shape(), B, idx)
        _check(plan, mr, pl, f"{name} B={B}")
    H = 64
    x = workloads.hidden(wl.N, H, seed=1, device=DEV)
    buf = torch.empty((wl.NK, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_dispatch(s, H, plan, x, buf)
    src_tok = torch.from_numpy(pl["src_pair"] // wl.K).to(DEV).long()
    assert torch.equal(buf.view(torch.int16), x.view(torch.int16).index_select(0, src_tok))
    assert mep.mep_read_status(plan) == 0


EDGE = [(1, 100, 8, 3), (4, 50, 4, 2), (2, 30, 6, 6), (8, 1, 16, 4), (3, 17, 12, 5),
        (16, 9, 32, 1), (2, 5, 1024, 16), (1024, 3, 1024, 2), (64, 40, 896, 16),
        (512, 4, 1024, 4)]


@pytest.mark.parametrize("R,S,E,K", EDGE)
@pytest.mark.parametrize("kind", ["random", "skewed", "dups", "one"])
def test_capped_edges(ora, R, S, E, K, kind):
    rng = np.random.default_rng(R * 1000 + S)
    N = R * S
    if kind == "dups":
        idx = rng.integers(0, E, size=(N, K)).astype(np.int32)
    elif kind == "one":
        idx = np.full((N, K), (E - 1) if E > 1 else 0, dtype=np.int32)
    else:
        lg = rng.standard_normal((N, E)) - (3.0 if kind == "skewed" else 0.0) * np.log(np.arange(1, E + 1))
        idx = np.argsort(-lg, axis=1, kind="stable")[:, :K].astype(np.int32)
    for B in (1, 3, max(1, E // R)):
        s, plan, mr = _capped((R, S, E, K), B, idx)
        _check(plan, mr, ora.plan_capped(R, S, E, K, B, idx), f"{(R, S, E, K)} {kind} B={B}")


def test_capped_workspace_reuse_across_kinds(ora):
    """One workspace serves the contiguous, home-first and capped plans in
    turn: each call leaves it ready for the next."""
    wl = workloads.reduced(workloads.WORKLOADS["kimi_r64_e896_k16"], S=97)
    idx, _ = workloads.routing(wl)
    s = mep.Shape(*wl.shape())
    plan = mep.Plan(s, DEV)
    idx_d = torch.from_numpy(idx).to(DEV)
    for _ in range(2):
        mep.mep_plan(s, idx_d, plan)
        parity.check_plan(plan.host(), ora.plan(*wl.shape(), idx), "contiguous")
        mr = mep.mep_plan_capped(s, 3, idx_d, plan)
        parity.check_plan(plan.host(), ora.plan_capped(*wl.shape(), 3, idx), "capped")
        assert int(mr.item()) == ora.plan_capped(*wl.shape(), 3, idx)["max_rank_replicas"]
        mep.mep_plan_home_first(s, idx_d, plan)
        parity.check_plan(plan.host(), ora.plan_home_first(*wl.shape(), idx), "home-first")
