"""Randomised parity (hypothesis, derandomised): small random shapes and
routings -- skewed, duplicate ids inside a token, everything on one expert,
ids at the edges of [0, E) -- through the C ABI on the GPU, against the
oracle: the contiguous, home-first and capped plans (B from 1 to 5) bit-exact,
dispatch, combine and reduce bit-exact, and one rank's token range of the rank-addressed
calls (dispatch, combine, and the home rank's share of the reduction)
equal to the whole-range results."""
import numpy as np
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
import parity
import token_dispatch_mep_b200 as mep
from token_dispatch_mep_b200 import ep

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
SETTINGS = settings(max_examples=60, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow, HealthCheck.function_scoped_fixture])


def _u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


@st.composite
def case(draw):
    R = draw(st.integers(1, 8))
    B = draw(st.integers(1, 6))
    E = R * B
    K = draw(st.integers(1, min(E, 16)))
    S = draw(st.integers(1, 90))
    H = 8 * draw(st.integers(1, 40))
    P = draw(st.integers(1, 70))
    kind = draw(st.sampled_from(["distinct", "dups", "one", "skew", "edges"]))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    rng = np.random.default_rng(seed)
    N = R * S
    if kind == "distinct":
        idx = np.argsort(-rng.standard_normal((N, E)), axis=1, kind="stable")[:, :K]
    elif kind == "skew":
        logits = rng.standard_normal((N, E)) - 3.0 * np.log(np.arange(1, E + 1))
        idx = np.argsort(-logits, axis=1, kind="stable")[:, :K]
    elif kind == "dups":
        idx = rng.integers(0, E, size=(N, K))
    elif kind == "edges":
        idx = rng.choice(np.array([0, E - 1]), size=(N, K))
    else:
        idx = np.full((N, K), int(rng.integers(0, E)))
    w = rng.standard_normal((N, K)).astype(np.float32)
    return R, S, E, K, H, P, np.ascontiguousarray(idx, dtype=np.int32), w, seed


@SETTINGS
@given(case())
def test_random_shapes_against_the_oracle(c):
    R, S, E, K, H, P, idx, w, seed = c
    B = E // R
    ora = oracle.get()
    N, NK, SK = R * S, R * S * K, S * K
    s = mep.Shape(R, S, E, K)
    gen = torch.Generator().manual_seed(seed)
    x = torch.randn((N, H), generator=gen).to(torch.bfloat16)
    y = torch.randn((NK, H), generator=gen).to(torch.bfloat16)
    G = torch.randn((E + R - 1, P), generator=gen)
    Bcap = 1 + seed % 5
    for home_first in (False, True, "capped"):
        plan = mep.Plan(s, DEV)
        idx_d = torch.from_numpy(idx).to(DEV)
        if home_first == "capped":
            mr = mep.mep_plan_capped(s, Bcap, idx_d, plan)
            pl = ora.plan_capped(R, S, E, K, Bcap, idx)
            assert int(mr.item()) == pl["max_rank_replicas"]
        elif home_first:
            mep.mep_plan_home_first(s, idx_d, plan)
            pl = ora.plan_home_first(R, S, E, K, idx)
        else:
            mep.mep_plan(s, idx_d, plan)
            pl = ora.plan(R, S, E, K, idx)
        buf = torch.empty((NK, H), dtype=torch.bfloat16, device=DEV)
        out = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
        home = torch.empty((E, P), dtype=torch.float32, device=DEV)
        mep.mep_dispatch(s, H, plan, x.to(DEV), buf)
        mep.mep_combine(s, H, plan, y.to(DEV), torch.from_numpy(w).to(DEV), out)
        mep.mep_reduce_replica_grads(s, plan, P, G.to(DEV), home)
        # one rank's share through the rank-addressed per-rank calls
        r = int(seed % R)
        bufs = [torch.full((SK, H), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
                for _ in range(R)]
        mep.mep_dispatch_ranked_tokens(s, H, plan, r * S, x[r * S:(r + 1) * S].to(DEV),
                                       mep.rank_pointer_table(bufs, s, H, DEV))
        out_r = torch.empty((S, H), dtype=torch.bfloat16, device=DEV)
        ys = [y[q * SK:(q + 1) * SK].to(DEV) for q in range(R)]
        ytab = mep.rank_pointer_table(ys, s, H, DEV)
        mep.mep_combine_ranked_tokens(s, H, plan, r * S, ytab,
                                      torch.from_numpy(w[r * S:(r + 1) * S].copy()).to(DEV), out_r)
        assert mep.mep_read_status(plan) == 0
        parity.check_plan(plan.host(), pl, f"fuzz hf={home_first}")
        if home_first is False:  # the counts-and-maxvio-only call on the same ids
            ws = torch.zeros(mep.mep_plan_workspace_bytes(s), dtype=torch.uint8, device=DEV)
            cnt = torch.empty(E, dtype=torch.int32, device=DEV)
            mc = torch.empty(1, dtype=torch.int32, device=DEV)
            mv = torch.empty(1, dtype=torch.float64, device=DEV)
            stt = torch.full((1,), 7, dtype=torch.int32, device=DEV)
            mep.mep_maxvio(s, torch.from_numpy(idx).to(DEV), cnt, mc, mv, stt, ws)
            c_o, m_o, v_o = ora.maxvio(R, S, E, K, idx)
            assert np.array_equal(cnt.cpu().numpy(), c_o)
            assert int(mc.item()) == m_o and float(mv.item()) == v_o and int(stt.item()) == 0
        assert np.array_equal(_u16(buf), ora.dispatch(K, pl["src_pair"], _u16(x)))
        ob, ex, ab = ora.combine(pl["slot"], w, _u16(y))
        parity.check_combine(_u16(out), ob, ex, ab, K, "fuzz")
        hexact, habs = ora.reduce(pl["expert_seg_ptr"], G.numpy())
        parity.check_reduce(home.cpu().numpy(), hexact, habs, np.diff(pl["expert_seg_ptr"]), "fuzz")
        assert torch.equal(out_r.view(torch.int16), out[r * S:(r + 1) * S].view(torch.int16))
        # the home rank r's share of the reduction, from per-rank gradient
        # buffers (P is often not a multiple of 4: the scalar path)
        ph = plan.host()
        rows = ep.max_local_segments(s)
        grads = []
        for q in range(R):
            gq = torch.zeros((rows, P), dtype=torch.float32, device=DEV)
            for j, (sidx, _, _, _) in enumerate(ep.local_segments(ph, q)):
                gq[j] = G[sidx].to(DEV)
            grads.append(gq)
        home_r = torch.empty((B, P), dtype=torch.float32, device=DEV)
        gtab = mep.pointer_table([g.data_ptr() for g in grads], DEV)
        mep.mep_reduce_replica_grads_ranked(s, plan, P, r, gtab, rows, home_r)
        assert mep.mep_read_status(plan) == 0
        assert torch.equal(home_r, home[r * B:(r + 1) * B])
        mine = np.unique(pl["slot"][r * S:(r + 1) * S].reshape(-1))
        flat = torch.cat(bufs)
        assert torch.equal(flat[torch.from_numpy(mine).to(DEV).long()].view(torch.int16),
                           buf[torch.from_numpy(mine).to(DEV).long()].view(torch.int16))
