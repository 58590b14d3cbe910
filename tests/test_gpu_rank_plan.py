"""One rank's share of the plan from the gathered per-rank histograms, on the
GPU, through the C ABI.

Every rank computes the same schedule from the current routing ("Moonshot AI
Open-Sources MoonEP, the Library Used to Train the MoE Model Kimi K3", "How
MoonEP works"); the only exchange the plan needs is the R x E matrix of
per-rank expert counts.  For every schedule (contiguous, home-first, capped)
each rank's call must reproduce the whole-range plan's tables bit for bit,
write exactly its own pairs' slots (and their src_pair entries), and leave
the other ranks' entries untouched."""
import numpy as np
import pytest
import torch

import oracle
import parity
import token_dispatch_mep_b200 as mep
import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
TABLES = ("counts", "expert_offset", "rank_seg_ptr", "expert_seg_ptr")


@pytest.fixture(scope="module")
def ora():
    return oracle.get()


def _whole(s, schedule, idx_d, B):
    plan = mep.Plan(s, DEV)
    mr = None
    if schedule == "contiguous":
        mep.mep_plan(s, idx_d, plan)
    elif schedule == "home_first":
        mep.mep_plan_home_first(s, idx_d, plan)
    else:
        mr = int(mep.mep_plan_capped(s, B, idx_d, plan).item())
    assert mep.mep_read_status(plan) == 0
    return plan.host(), mr


def _histograms(s, idx_d, scratch):
    rows = []
    for r in range(s.R):
        local = idx_d[r * s.S:(r + 1) * s.S].contiguous()
        rows.append(mep.mep_rank_histogram(s, local, plan=scratch))
    assert mep.mep_read_status(scratch) == 0
    return torch.stack(rows).contiguous()


def _check_share(got: dict, ref: dict, r: int, s, what: str):
    for k in TABLES:
        assert np.array_equal(got[k], ref[k]), (what, k)
    for k in ("num_seg", "num_replicas", "max_count"):
        assert got[k] == ref[k], (what, k)
    assert got["maxvio"] == ref["maxvio"], what
    ns, nr = ref["num_seg"], ref["num_replicas"]
    assert np.array_equal(got["seg"][:ns], ref["seg"][:ns]), what
    assert np.array_equal(got["rank_seg_idx"][:ns], ref["rank_seg_idx"][:ns]), what
    assert np.array_equal(got["replica_seg"][:nr], ref["replica_seg"][:nr]), what
    rows = slice(r * s.S, (r + 1) * s.S)
    assert np.array_equal(got["slot"][rows], ref["slot"][rows]), what
    others = np.ones(s.N, bool)
    others[rows] = False
    assert (got["slot"][others] == -1).all(), what               # not touched
    mine = ref["slot"][rows].reshape(-1)
    assert np.array_equal(got["src_pair"][mine], ref["src_pair"][mine]), what
    untouched = np.ones(s.NK, bool)
    untouched[mine] = False
    assert (got["src_pair"][untouched] == -1).all(), what


CASES = [("tiny_r4_e16", 64), ("r8_e64_h2048", 1031), ("r16_e256_h7168", 65),
         ("kimi_r64_e896_k16", 97), ("skew_r32_zipf1.5", 131), ("skew_r32_adversarial", 131),
         ("skew_r32_uniform", 40)]


@pytest.mark.parametrize("name,S", CASES, ids=[c[0] for c in CASES])
def test_rank_shares_equal_the_whole_plan(ora, name, S):
    wl = workloads.reduced(workloads.WORKLOADS[name], S=S)
    s = mep.Shape(*wl.shape())
    idx, _ = workloads.routing(wl)
    idx_d = torch.from_numpy(idx).to(DEV)
    scratch = mep.Plan(s, DEV)
    hist = _histograms(s, idx_d, scratch)
    want = np.stack([np.bincount(idx[r * S:(r + 1) * S].reshape(-1), minlength=wl.E)
                     for r in range(wl.R)])
    assert np.array_equal(hist.cpu().numpy(), want)              # bit-exact histograms
    for schedule, B in (("contiguous", 0), ("home_first", 0), ("capped", 4), ("capped", 1)):
        ref, ref_mr = _whole(s, schedule, idx_d, B)
        # the whole-range plan is the oracle's
        if schedule == "contiguous":
            parity.check_plan(ref, ora.plan(*wl.shape(), idx), name)
        for r in range(wl.R):
            plan = mep.Plan(s, DEV)
            plan.slot.fill_(-1)
            plan.src_pair.fill_(-1)
            local = idx_d[r * S:(r + 1) * S].contiguous()
            mr = mep.mep_plan_rank(s, schedule, r, local, hist, plan, B=B)
            assert mep.mep_read_status(plan) == 0
            _check_share(plan.host(), ref, r, s, f"{name} {schedule} B={B} rank {r}")
            if schedule == "capped":
                assert int(mr.item()) == ref_mr


def test_rank_row_must_match_the_rank_ids():
    """A gathered row that disagrees with the rank's own ids is reported
    (MEP_ERR_DEVICE_DATA), never trusted silently."""
    wl = workloads.reduced(workloads.WORKLOADS["r8_e64_h2048"], S=301)
    s = mep.Shape(*wl.shape())
    idx, _ = workloads.routing(wl)
    idx_d = torch.from_numpy(idx).to(DEV)
    scratch = mep.Plan(s, DEV)
    hist = _histograms(s, idx_d, scratch)
    bad = hist.clone()
    bad[3, 0] += 1
    bad[3, 1] -= 1
    plan = mep.Plan(s, DEV)
    mep.mep_plan_rank(s, "contiguous", 3, idx_d[3 * wl.S:4 * wl.S].contiguous(), bad, plan)
    assert mep.mep_read_status(plan) == 5
    mep.mep_plan_rank(s, "contiguous", 3, idx_d[3 * wl.S:4 * wl.S].contiguous(), hist, plan)
    assert mep.mep_read_status(plan) == 0


def test_histogram_reports_out_of_range_ids():
    s = mep.Shape(4, 50, 16, 2)
    local = torch.zeros((50, 2), dtype=torch.int32, device=DEV)
    local[7, 1] = 16
    scratch = mep.Plan(s, DEV)
    mep.mep_rank_histogram(s, local, plan=scratch)
    assert mep.mep_read_status(scratch) == 5
