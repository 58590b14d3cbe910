"""CUDA path against the CPU oracle, through the C ABI (via the ctypes binding).

* Reduced sizes of every workload (ragged token counts, several plan tiles):
  every output element compared with the oracle.
* Full sizes of every workload, in the launch configuration the benchmark
  times: the whole plan bit-exact; every dispatched row checked on the device
  against the oracle's source token; every combine output and every
  home-gradient element against the oracle where the oracle runs in seconds
  (the tiny and R=8 E=64 H=2048 workloads), sampled tokens and columns
  elsewhere.
* Edge cases: one rank, one expert per rank, K = E, S = 1, minimum and maximum
  hidden sizes, ragged gradient rows, duplicate experts inside a token, empty
  experts, out-of-range expert ids, a grid barrier whose wait runs out,
  poisoned output buffers, workspace reuse across calls.
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


def _u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def run_path(shape, H, P, idx, w, x, y, G, poison=True):
    """Plan, dispatch, combine and reduce through the binding; returns the
    plan (host copy) and device outputs."""
    s = mep.Shape(*shape)
    plan = mep.Plan(s, DEV)
    idx_d = torch.as_tensor(idx, dtype=torch.int32).to(DEV).contiguous()
    w_d = torch.as_tensor(w, dtype=torch.float32).to(DEV).contiguous()
    buf = torch.empty((s.R, s.SK, H), dtype=torch.bfloat16, device=DEV)
    out = torch.empty((s.N, H), dtype=torch.bfloat16, device=DEV)
    if poison:
        buf.view(torch.int16).fill_(-1)
        out.view(torch.int16).fill_(-1)
    mep.mep_plan(s, idx_d, plan)
    mep.mep_dispatch(s, H, plan, x, buf)
    mep.mep_combine(s, H, plan, y, w_d, out)
    home = None
    if P:
        home = torch.full((s.E, P), float("nan"), dtype=torch.float32, device=DEV)
        mep.mep_reduce_replica_grads(s, plan, P, G, home)
    st = mep.mep_read_status(plan)
    assert st == 0, mep.mep_status_string(st)
    return plan, buf, out, home


def full_compare(ora, shape, H, P, idx, w, seed=0):
    R, S, E, K = shape
    N, NK = R * S, R * S * K
    x = workloads.hidden(N, H, seed=seed + 1)
    y = workloads.expert_outputs(NK, H, seed=seed + 2)
    G = workloads.seg_grads(E + R - 1, P, seed=seed + 3) if P else None
    plan, buf, out, home = run_path(shape, H, P, idx, w, x.to(DEV), y.to(DEV),
                                    G.to(DEV) if P else None)
    pl = ora.plan(R, S, E, K, idx)
    parity.check_plan(plan.host(), pl, str(shape))
    want_buf = ora.dispatch(K, pl["src_pair"], _u16(x))
    assert np.array_equal(_u16(buf).reshape(NK, H), want_buf)
    ob, exact, absum = ora.combine(pl["slot"], np.asarray(w, np.float32), _u16(y))
    stats = parity.check_combine(_u16(out), ob, exact, absum, K, str(shape))
    if P:
        hexact, habs = ora.reduce(pl["expert_seg_ptr"], G.numpy())
        parity.check_reduce(home.cpu().numpy(), hexact, habs, np.diff(pl["expert_seg_ptr"]), str(shape))
    return stats


# ------------------------------------------------------------ reduced sizes

REDUCED = [("tiny_r4_e16", 64, None, 100), ("r8_e64_h2048", 1031, None, 4100),
           ("r16_e256_h7168", 65, None, 1027), ("kimi_r64_e896_k16", 97, None, 2052),
           ("skew_r32_uniform", 131, None, 996), ("skew_r32_zipf1.5", 131, None, 4096),
           ("skew_r32_adversarial", 131, None, 8)]


@pytest.mark.parametrize("name,S,H,P", REDUCED, ids=[r[0] for r in REDUCED])
def test_reduced_every_element(ora, name, S, H, P):
    wl = workloads.reduced(workloads.WORKLOADS[name], S=S, H=H, P=P)
    idx, w = workloads.routing(wl)
    stats = full_compare(ora, wl.shape(), wl.H, wl.P, idx, w)
    assert stats["max_ulp"] == 0 and stats["bitexact"] == 1.0


# --------------------------------------------------------------- full sizes

def _combine_f64_bf16(y, w, slot):
    """sum_k w[g,k] * y[slot[g,k]] for a chunk of tokens, added in binary64 in
    k order (each product is exact, as in the oracle), then rounded once to
    bf16: round-to-odd to float32, then nearest-even to bf16 (Boldo and
    Melquiond: 16 extra bits make the two steps one correct rounding)."""
    acc = torch.zeros((w.shape[0], y.shape[1]), dtype=torch.float64, device=y.device)
    for k in range(w.shape[1]):
        acc = acc + w[:, k:k + 1].double() * y.index_select(0, slot[:, k]).double()
    f = acc.to(torch.float32)                                    # nearest-even
    over = f.double().abs() > acc.abs()
    fz = torch.where(over, torch.nextafter(f, torch.zeros_like(f)), f)   # toward zero
    bits = fz.view(torch.int32)
    bits = torch.where(fz.double() != acc, bits | 1, bits)              # sticky bit
    return bits.view(torch.float32).to(torch.bfloat16)


# Workloads whose every output element is compared at full size (the oracle
# runs them in seconds); the others are compared on samples.
EVERY_ELEMENT = ("tiny_r4_e16", "r8_e64_h2048")


@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_full_size(ora, name):
    wl = workloads.WORKLOADS[name]
    R, S, E, K, H, P = wl.R, wl.S, wl.E, wl.K, wl.H, wl.P
    N, NK = wl.N, wl.NK
    idx, w = workloads.routing(wl)
    x = workloads.hidden(N, H, seed=1, device=DEV)
    y = workloads.expert_outputs(NK, H, seed=2, device=DEV)
    G = workloads.seg_grads(wl.seg_rows, P, seed=3, device=DEV) if P else None
    plan, buf, out, home = run_path(wl.shape(), H, P, idx, w, x, y, G, poison=False)
    pl = ora.plan(R, S, E, K, idx)
    parity.check_plan(plan.host(), pl, name)
    # every dispatched row equals the oracle's source token row
    src_tok = torch.from_numpy(pl["src_pair"] // K).to(DEV).long()
    bufv = buf.view(NK, H).view(torch.int16)
    xv = x.view(torch.int16)
    step = max(1, (1 << 28) // (H * 2))
    for c0 in range(0, NK, step):
        c1 = min(NK, c0 + step)
        assert torch.equal(bufv[c0:c1], xv.index_select(0, src_tok[c0:c1])), (name, c0)
    del bufv
    if name in EVERY_ELEMENT:
        # every combine output and every home-gradient element, in chunks
        yh = None
        for t0 in range(0, N, 4096):
            t1 = min(N, t0 + 4096)
            sl = pl["slot"][t0:t1]
            yrows = _u16(y.view(NK, H).index_select(0, torch.from_numpy(sl.reshape(-1)).to(DEV).long()))
            ob, exact, absum = ora.combine(np.arange(sl.size, dtype=np.int32).reshape(sl.shape),
                                           w[t0:t1], yrows)
            parity.check_combine(_u16(out[t0:t1]), ob, exact, absum, K, f"{name} tokens {t0}..{t1}")
        if P:
            for c0 in range(0, P, 1 << 20):
                c1 = min(P, c0 + (1 << 20))
                hexact, habs = ora.reduce(pl["expert_seg_ptr"], G[:, c0:c1].cpu().numpy())
                parity.check_reduce(home[:, c0:c1].cpu().numpy(), hexact, habs,
                                    np.diff(pl["expert_seg_ptr"]), f"{name} columns {c0}..{c1}")
        return
    # every combine output against a float64 recomputation from the oracle's
    # slots, in chunks on the device (the oracle itself checks a sample below)
    wd = torch.from_numpy(np.asarray(w, np.float32)).to(DEV)
    slot_d = torch.from_numpy(pl["slot"].astype(np.int64)).to(DEV)
    yv = y.view(NK, H)
    step_t = max(1, (1 << 28) // (K * H * 8))
    for t0 in range(0, N, step_t):
        t1 = min(N, t0 + step_t)
        want = _combine_f64_bf16(yv, wd[t0:t1], slot_d[t0:t1])
        got = out[t0:t1].view(torch.int16)
        if not torch.equal(got, want.view(torch.int16)):
            bad = int((got != want.view(torch.int16)).sum())
            raise AssertionError(f"{name}: {bad} combine outputs differ from the float64 "
                                 f"recomputation in tokens {t0}..{t1}")
    # combine on sampled tokens
    rng = np.random.default_rng(5)
    toks = np.unique(np.concatenate([np.arange(64), np.arange(N - 64, N), rng.integers(0, N, 512)]))
    sl = pl["slot"][toks]                                   # [n, K] oracle slots
    yrows = _u16(y.view(NK, H).index_select(0, torch.from_numpy(sl.reshape(-1)).to(DEV).long()))
    ob, exact, absum = ora.combine(np.arange(sl.size, dtype=np.int32).reshape(sl.shape),
                                   w[toks], yrows)
    got = _u16(out.index_select(0, torch.from_numpy(toks).to(DEV).long()))
    parity.check_combine(got, ob, exact, absum, K, name)
    # replica-gradient reduce on sampled columns, every expert
    if P:
        cols = np.unique(np.concatenate([np.arange(256), np.arange(P - 256, P),
                                         rng.integers(0, P, 4096)]))
        ct = torch.from_numpy(cols).to(DEV).long()
        hexact, habs = ora.reduce(pl["expert_seg_ptr"], G.index_select(1, ct).cpu().numpy())
        parity.check_reduce(home.index_select(1, ct).cpu().numpy(), hexact, habs,
                            np.diff(pl["expert_seg_ptr"]), name)


# --------------------------------------------------------------- edge cases

EDGE = [
    # (R, S, E, K, H, P, routing)
    (1, 100, 8, 3, 64, 12, "random"),        # one rank: nothing is ever a replica
    (4, 50, 4, 2, 8, 5, "random"),           # one expert per rank, minimum H, ragged P
    (2, 30, 6, 6, 16, 1, "random"),          # K = E, P = 1
    (8, 1, 16, 4, 24, 7, "random"),          # one token per rank
    (3, 17, 12, 5, 296, 1023, "dups"),       # duplicate experts inside tokens
    (4, 64, 16, 16, 40, 64, "random"),       # K = 16 = E
    (16, 9, 32, 1, 128, 3, "one"),           # everything on one expert
    (2, 5, 1024, 16, 8, 4, "random"),        # E at its maximum
    (1024, 3, 1024, 2, 8, 4, "random"),      # R at its maximum
    (2, 7, 4, 2, 32768, 8, "random"),        # H at its maximum
]


def _edge_routing(R, S, E, K, kind, seed=0):
    rng = np.random.default_rng(seed)
    N = R * S
    if kind == "dups":
        idx = rng.integers(0, E, size=(N, K)).astype(np.int32)
    elif kind == "one":
        idx = np.full((N, K), 3 % E, dtype=np.int32)
    else:
        idx = np.argsort(-rng.standard_normal((N, E)), axis=1)[:, :K].astype(np.int32)
    w = rng.random((N, K)).astype(np.float32)
    return idx, w


@pytest.mark.parametrize("R,S,E,K,H,P,kind", EDGE)
def test_edge_cases(ora, R, S, E, K, H, P, kind):
    idx, w = _edge_routing(R, S, E, K, kind)
    full_compare(ora, (R, S, E, K), H, P, idx, w)


def test_roundrobin_and_adversarial_closed_forms():
    # round-robin: maxvio exactly 0, every expert home, E segments
    R, S, E, K = 8, 4096, 64, 6
    idx, _ = workloads.roundrobin_routing(R, S, E, K)
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    h = plan.host()
    assert h["maxvio"] == 0.0 and h["num_seg"] == E and h["num_replicas"] == 0
    # adversarial: maxvio 31, 32 segments, 31 replicas
    wl = workloads.WORKLOADS["skew_r32_adversarial"]
    idx, _ = workloads.routing(wl)
    s = mep.Shape(*wl.shape())
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    h = plan.host()
    assert h["maxvio"] == 31.0 and h["num_seg"] == 32 and h["num_replicas"] == 31
    assert h["seg"][:32].tolist() == [[e, 4 * e + j, 0, 32768] for e in range(8) for j in range(4)]


def test_maxvio_call(ora):
    # tiny: one block; r8: the one-barrier (small tile matrix) form; the
    # others: two barriers
    for name in ("tiny_r4_e16", "r8_e64_h2048", "kimi_r64_e896_k16", "skew_r32_zipf1.5"):
        wl = workloads.WORKLOADS[name]
        idx, _ = workloads.routing(wl)
        s = mep.Shape(*wl.shape())
        ws = torch.zeros(mep.mep_plan_workspace_bytes(s), dtype=torch.uint8, device=DEV)
        counts = torch.empty(wl.E, dtype=torch.int32, device=DEV)
        mc = torch.empty(1, dtype=torch.int32, device=DEV)
        mv = torch.empty(1, dtype=torch.float64, device=DEV)
        st = torch.full((1,), 7, dtype=torch.int32, device=DEV)
        mep.mep_maxvio(s, torch.from_numpy(idx).to(DEV), counts, mc, mv, st, ws)
        c, m, v = ora.maxvio(*wl.shape(), idx)
        assert np.array_equal(counts.cpu().numpy(), c)
        assert int(mc.item()) == m and float(mv.item()) == v and int(st.item()) == 0


def test_out_of_range_ids_reported_not_fatal(ora):
    R, S, E, K, H = 4, 40, 8, 2, 16
    idx, w = _edge_routing(R, S, E, K, "random")
    bad = idx.copy()
    bad[3, 1] = E
    bad[77, 0] = -1
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(bad).to(DEV), plan)
    assert mep.mep_read_status(plan) == 5
    x = torch.randn(R * S, H, device=DEV).to(torch.bfloat16)
    buf = torch.zeros(R, S * K, H, dtype=torch.bfloat16, device=DEV)
    out = torch.zeros(R * S, H, dtype=torch.bfloat16, device=DEV)
    mep.mep_dispatch(s, H, plan, x, buf)
    mep.mep_combine(s, H, plan, buf, torch.from_numpy(w).to(DEV), out)
    assert mep.mep_read_status(plan) == 5
    # a clean plan clears the status and is right again
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    assert mep.mep_read_status(plan) == 0
    parity.check_plan(plan.host(), ora.plan(R, S, E, K, idx))


def test_barrier_wait_runs_out_and_recovers(ora):
    """A grid barrier whose arrival count is poisoned (a large negative value,
    so it can never reach its target) never opens: every block gives up after
    the wait limit, the status says MEP_ERR_TIMEOUT, and the context stays
    usable."""
    R, S, E, K = 8, 4096, 64, 6
    idx, _ = _edge_routing(R, S, E, K, "random")
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, DEV)
    old = mep.mep_get_wait_limit_ns()
    try:
        plan.workspace[:4].view(torch.int32).fill_(-(1 << 31))
        mep.mep_set_wait_limit_ns(2_000_000)
        mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
        assert mep.mep_read_status(plan) == 6
    finally:
        mep.mep_set_wait_limit_ns(old)
    plan.reset_workspace()
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    assert mep.mep_read_status(plan) == 0
    parity.check_plan(plan.host(), ora.plan(R, S, E, K, idx))


def test_workspace_reuse_and_shape_changes(ora):
    shapes = [(8, 512, 64, 6), (4, 300, 896 // 4 * 4, 16), (8, 512, 64, 6), (2, 9, 16, 2)]
    plans = {}
    for i, (R, S, E, K) in enumerate(shapes):
        idx, _ = _edge_routing(R, S, E, K, "random", seed=i)
        s = mep.Shape(R, S, E, K)
        plan = plans.setdefault((R, S, E, K), mep.Plan(s, DEV))
        mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
        parity.check_plan(plan.host(), ora.plan(R, S, E, K, idx), str((R, S, E, K)))


def test_host_errors_on_device_tensors():
    R, S, E, K, H = 2, 8, 4, 2, 16
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, DEV)
    idx, _ = _edge_routing(R, S, E, K, "random")
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    x = torch.zeros(R * S * H + 8, dtype=torch.bfloat16, device=DEV)
    buf = torch.zeros(R * S * K * H, dtype=torch.bfloat16, device=DEV)
    with pytest.raises(mep.MepError) as e:
        mep.mep_dispatch(s, H, plan, x[1:], buf)          # 2-byte offset
    assert e.value.code == 2
    with pytest.raises(ValueError):
        mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan, workspace=plan.workspace[:64])
    with pytest.raises(ValueError):
        mep.mep_dispatch(s, H, plan, x[: R * S * H - 8], buf)   # too small
