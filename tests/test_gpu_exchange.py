"""One rank's share of the exchange, through the C ABI, on one GPU: the
token-range forms of rank-addressed dispatch and combine, and the
rank-addressed replica-gradient reduction of one home rank.  Every rank's
buffers are separate device allocations; each rank's call covers its own
tokens (or its own home experts).  The union over ranks must equal the
whole-range calls bit for bit and the oracle within the contract's
tolerances."""
import numpy as np
import pytest
import torch

import oracle
import parity
import token_dispatch_mep_b200 as mep
import workloads
from token_dispatch_mep_b200 import ep

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _poisoned(rows, H):
    return torch.full((rows, H), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16)


CASES = [("tiny_r4_e16", 64, 128, 40), ("r8_e64_h2048", 517, 2048, 1000),
         ("kimi_r64_e896_k16", 29, 1024, 64), ("skew_r32_zipf1.5", 67, 264, 36),
         ("skew_r32_adversarial", 33, 64, 20)]


@pytest.mark.parametrize("name,S,H,P", CASES, ids=[c[0] for c in CASES])
@pytest.mark.parametrize("home_first", [False, True], ids=["contiguous", "home_first"])
def test_per_rank_calls_equal_whole_calls(name, S, H, P, home_first):
    ora = oracle.get()
    wl = workloads.reduced(workloads.WORKLOADS[name], S=S, H=H, P=P)
    R, E, K, N, NK, SK = wl.R, wl.E, wl.K, wl.N, wl.NK, wl.SK
    idx, w = workloads.routing(wl)
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, DEV)
    (mep.mep_plan_home_first if home_first else mep.mep_plan)(s, torch.from_numpy(idx).to(DEV), plan)
    x = workloads.hidden(N, H, seed=1).to(DEV)
    y = workloads.expert_outputs(NK, H, seed=2).to(DEV)
    wd = torch.from_numpy(w).to(DEV)
    G = workloads.seg_grads(wl.seg_rows, P, seed=3).to(DEV)

    # whole-range calls on single buffers
    buf = torch.empty((NK, H), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
    home = torch.empty((E, P), dtype=torch.float32, device=DEV)
    mep.mep_dispatch(s, H, plan, x, buf)
    mep.mep_combine(s, H, plan, y, wd, out)
    mep.mep_reduce_replica_grads(s, plan, P, G, home)

    # per-rank calls: rank r sends / combines its own S tokens
    bufs = [_poisoned(SK, H) for _ in range(R)]
    btab = mep.rank_pointer_table(bufs, s, H, DEV)
    ys = [y[r * SK:(r + 1) * SK].clone() for r in range(R)]
    ytab = mep.rank_pointer_table(ys, s, H, DEV)
    outs = [_poisoned(S, H) for _ in range(R)]
    for r in range(R):
        mep.mep_dispatch_ranked_tokens(s, H, plan, r * S, x[r * S:(r + 1) * S], btab)
        mep.mep_combine_ranked_tokens(s, H, plan, r * S, ytab, wd[r * S:(r + 1) * S], outs[r])

    # per-rank segment gradients: rank r's row j = gradient of its j-th segment
    ph = plan.host()
    rows = ep.max_local_segments(s)
    grads = []
    for r in range(R):
        segs = ep.local_segments(ph, r)
        assert len(segs) <= rows
        g = torch.zeros((rows, P), dtype=torch.float32, device=DEV)
        for j, (sidx, _, _, _) in enumerate(segs):
            g[j] = G[sidx]
        grads.append(g)
    gtab = mep.pointer_table([g.data_ptr() for g in grads], DEV)
    B = E // R
    homes = [torch.full((B, P), float("nan"), dtype=torch.float32, device=DEV) for _ in range(R)]
    for r in range(R):
        mep.mep_reduce_replica_grads_ranked(s, plan, P, r, gtab, rows, homes[r])
    assert mep.mep_read_status(plan) == 0

    assert torch.equal(torch.cat(bufs).view(torch.int16), buf.view(torch.int16))
    assert torch.equal(torch.cat(outs).view(torch.int16), out.view(torch.int16))
    assert torch.equal(torch.cat(homes), home)          # same sums, same order
    # and against the oracle
    pl = (ora.plan_home_first if home_first else ora.plan)(R, S, E, K, idx)
    assert np.array_equal(_u16(torch.cat(bufs)), ora.dispatch(K, pl["src_pair"], _u16(x)))
    ob, ex, ab = ora.combine(pl["slot"], w, _u16(y))
    parity.check_combine(_u16(torch.cat(outs)), ob, ex, ab, K, name)
    hexact, habs = ora.reduce(pl["expert_seg_ptr"], G.cpu().numpy())
    nseg = np.diff(pl["expert_seg_ptr"])
    parity.check_reduce(torch.cat(homes).cpu().numpy(), hexact, habs, nseg, name)


def test_uneven_token_ranges_and_empty_range():
    """Any split of [0, N) into ranges, including empty ones, gives the
    whole-range result."""
    wl = workloads.reduced(workloads.WORKLOADS["r8_e64_h2048"], S=101, H=256)
    R, S, E, K, H, N, NK, SK = wl.R, wl.S, wl.E, wl.K, wl.H, wl.N, wl.NK, wl.SK
    idx, w = workloads.routing(wl)
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    x = workloads.hidden(N, H, seed=1).to(DEV)
    y = workloads.expert_outputs(NK, H, seed=2).to(DEV)
    wd = torch.from_numpy(w).to(DEV)
    bufs = [_poisoned(SK, H) for _ in range(R)]
    btab = mep.rank_pointer_table(bufs, s, H, DEV)
    ytab = mep.rank_pointer_table([y[r * SK:(r + 1) * SK] for r in range(R)], s, H, DEV)
    out = _poisoned(N, H)
    cuts = [0, 1, 1, 37, 300, 301, 512, N]
    for b, e in zip(cuts[:-1], cuts[1:]):
        mep.mep_dispatch_ranked_tokens(s, H, plan, b, x[b:e], btab, token_count=e - b)
        mep.mep_combine_ranked_tokens(s, H, plan, b, ytab, wd[b:e], out[b:e], token_count=e - b)
    ref_buf = torch.empty((NK, H), dtype=torch.bfloat16, device=DEV)
    ref_out = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_dispatch(s, H, plan, x, ref_buf)
    mep.mep_combine(s, H, plan, y, wd, ref_out)
    assert mep.mep_read_status(plan) == 0
    assert torch.equal(torch.cat(bufs).view(torch.int16), ref_buf.view(torch.int16))
    assert torch.equal(out.view(torch.int16), ref_out.view(torch.int16))


def test_missing_rank_buffers_are_reported_not_used():
    """A NULL or misaligned entry in a rank pointer array is detected on the
    device (MEP_ERR_DEVICE_DATA) and never dereferenced; the other ranks'
    rows are still written."""
    wl = workloads.reduced(workloads.WORKLOADS["tiny_r4_e16"], S=64, H=128, P=64)
    R, S, E, K, H, N, NK, SK, P = wl.R, wl.S, wl.E, wl.K, wl.H, wl.N, wl.NK, wl.SK, wl.P
    idx, w = workloads.routing(wl)
    s = mep.Shape(R, S, E, K)
    x = workloads.hidden(N, H, seed=1).to(DEV)
    wd = torch.from_numpy(w).to(DEV)
    for bad in (0, 2):        # NULL, then an address 2 bytes off alignment
        plan = mep.Plan(s, DEV)
        mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
        bufs = [_poisoned(SK, H) for _ in range(R)]
        ptrs = [b.data_ptr() for b in bufs]
        ptrs[1] = 0 if bad == 0 else ptrs[1] + bad
        tab = mep.pointer_table(ptrs, DEV)
        mep.mep_dispatch_ranked_tokens(s, H, plan, 0, x, tab)
        out = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
        mep.mep_combine_ranked_tokens(s, H, plan, 0, tab, wd, out)
        assert mep.mep_read_status(plan) == 5
        ref = torch.empty((NK, H), dtype=torch.bfloat16, device=DEV)
        mep.mep_dispatch(s, H, plan, x, ref)
        for r in (0, 2, 3):
            assert torch.equal(bufs[r].view(torch.int16), ref[r * SK:(r + 1) * SK].view(torch.int16))
        assert bool((bufs[1].view(torch.int16) == -1).all())
        # ranked reduce with a NULL gradient buffer for a rank that holds segments
        plan2 = mep.Plan(s, DEV)
        mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan2)
        ph = plan2.host()
        rows = ep.max_local_segments(s)
        grads = [torch.zeros((rows, P), device=DEV) for r in range(R)]
        gptr = [g.data_ptr() for g in grads]
        holder = int(ph["seg"][0][1])            # the rank holding segment 0 (expert 0)
        gptr[holder] = 0 if bad == 0 else gptr[holder] + bad
        home = torch.empty((E // R, P), device=DEV)
        mep.mep_reduce_replica_grads_ranked(s, plan2, P, 0, mep.pointer_table(gptr, DEV), rows,
                                            home)
        assert mep.mep_read_status(plan2) == 5
    # a gradient buffer declared too short for the rank's segments
    plan3 = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan3)
    ph3 = plan3.host()
    counts = [len(ep.local_segments(ph3, r)) for r in range(R)]
    short = max(1, min(c for c in counts if c > 0) - 1) if max(counts) > 1 else None
    if short is not None and any(c > short for c in counts):
        grads = [torch.zeros((max(counts), P), device=DEV) for r in range(R)]
        home = torch.empty((E // R, P), device=DEV)
        for hr in range(R):
            mep.mep_reduce_replica_grads_ranked(s, plan3, P, hr,
                                                mep.pointer_table([g.data_ptr() for g in grads], DEV),
                                                short, home)
        assert mep.mep_read_status(plan3) == 5


FULL = ["r8_e64_h2048", "r16_e256_h7168", "kimi_r64_e896_k16", "skew_r32_zipf1.5"]


@pytest.mark.parametrize("name", FULL)
def test_per_rank_calls_at_full_size_equal_the_single_buffer_calls(name):
    """At full size, in the configuration the bench times: every rank's
    token-range dispatch and combine through the rank pointer tables (rank
    buffers as slices of the single buffers) equal the single-buffer calls
    bit for bit, compared on the device (the single-buffer calls are checked
    against the oracle in test_gpu_parity)."""
    wl = workloads.WORKLOADS[name]
    R, S, E, K, H, N, NK = wl.R, wl.S, wl.E, wl.K, wl.H, wl.N, wl.NK
    SK = S * K
    s = mep.Shape(R, S, E, K)
    idx, w = workloads.routing(wl)
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    wd = torch.from_numpy(w).to(DEV)
    x = workloads.hidden(N, H, seed=1, device=DEV)
    buf = torch.empty((NK, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_dispatch(s, H, plan, x, buf)
    rbuf = torch.full((NK, H), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    btab = mep.rank_pointer_table([rbuf[r * SK:(r + 1) * SK] for r in range(R)], s, H, DEV)
    for r in range(R):
        mep.mep_dispatch_ranked_tokens(s, H, plan, r * S, x[r * S:(r + 1) * S], btab)
    assert mep.mep_read_status(plan) == 0
    assert torch.equal(rbuf.view(torch.int16), buf.view(torch.int16))
    del rbuf, btab, x
    y = buf  # expert outputs: the dispatched rows (identity experts)
    out = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_combine(s, H, plan, y, wd, out)
    rout = torch.full((N, H), -1, dtype=torch.int16, device=DEV).view(torch.bfloat16)
    ytab = mep.rank_pointer_table([y[r * SK:(r + 1) * SK] for r in range(R)], s, H, DEV)
    for r in range(R):
        mep.mep_combine_ranked_tokens(s, H, plan, r * S, ytab, wd[r * S:(r + 1) * S],
                                      rout[r * S:(r + 1) * S])
    assert mep.mep_read_status(plan) == 0
    assert torch.equal(rout.view(torch.int16), out.view(torch.int16))


@pytest.mark.parametrize("name", ["r8_e64_h2048", "kimi_r64_e896_k16", "skew_r32_adversarial"])
def test_home_rank_reductions_at_full_size_equal_the_single_buffer_reduce(name):
    """At full size: every home rank's reduction from per-rank gradient
    buffers (row j of rank q = q's j-th segment in slot order) equals the
    single-buffer reduction bit for bit, compared on the device."""
    wl = workloads.WORKLOADS[name]
    R, S, E, K, P = wl.R, wl.S, wl.E, wl.K, wl.P
    s = mep.Shape(R, S, E, K)
    idx, _ = workloads.routing(wl)
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    G = workloads.seg_grads(wl.seg_rows, P, seed=3, device=DEV)
    home = torch.empty((E, P), dtype=torch.float32, device=DEV)
    mep.mep_reduce_replica_grads(s, plan, P, G, home)
    ph = plan.host()
    # Each rank buffer holds exactly its own segments' rows (padding all 64
    # Kimi-shaped buffers to the busiest rank's ~540 rows would not fit one
    # GPU); the declared length is the largest, and the kernel reads only
    # rows of segments a rank lists.
    lists = [ep.local_segments(ph, q) for q in range(R)]
    rows = max(1, max(len(segs) for segs in lists))
    grads = []
    for segs in lists:
        gq = torch.empty((max(1, len(segs)), P), dtype=torch.float32, device=DEV)
        for j, (sidx, _, _, _) in enumerate(segs):
            gq[j] = G[sidx]
        grads.append(gq)
    del G
    gtab = mep.pointer_table([g.data_ptr() for g in grads], DEV)
    B = E // R
    rhome = torch.full((E, P), float("nan"), dtype=torch.float32, device=DEV)
    for q in range(R):
        mep.mep_reduce_replica_grads_ranked(s, plan, P, q, gtab, rows, rhome[q * B:(q + 1) * B])
    assert mep.mep_read_status(plan) == 0
    assert torch.equal(rhome.view(torch.int32), home.view(torch.int32))
