"""Property-based pins of the oracle (hypothesis): on random small shapes and
routings -- skewed, duplicated ids inside a token, all ids on one expert --
the oracle's contiguous plan equals Python's sorted() over (expert, g, k),
its home-first and capped plans equal the queue simulations of their
schedules, all keep
the invariants that fix them (every rank exactly S*K slots, each pair placed
once, runs of one expert, segment bound), and combine / reduce equal exact
rational sums.  CPU only; a bounded number of examples keeps it to seconds."""
from fractions import Fraction

import numpy as np
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import oracle
import oracle_pins as pins

ORA = oracle.get()
SETTINGS = settings(max_examples=120, deadline=None, derandomize=True,
                    suppress_health_check=[HealthCheck.too_slow])


@st.composite
def routed(draw):
    R = draw(st.integers(1, 6))
    B = draw(st.integers(1, 5))          # experts per rank
    E = R * B
    K = draw(st.integers(1, min(E, 6)))
    S = draw(st.integers(1, 12))
    kind = draw(st.sampled_from(["distinct", "dups", "one", "skew"]))
    seed = draw(st.integers(0, 2 ** 31 - 1))
    rng = np.random.default_rng(seed)
    N = R * S
    if kind == "distinct":
        idx = np.argsort(-rng.standard_normal((N, E)), axis=1, kind="stable")[:, :K]
    elif kind == "skew":
        logits = rng.standard_normal((N, E)) - 2.5 * np.log(np.arange(1, E + 1))
        idx = np.argsort(-logits, axis=1, kind="stable")[:, :K]
    elif kind == "dups":
        idx = rng.integers(0, E, size=(N, K))
    else:
        idx = np.full((N, K), int(rng.integers(0, E)))
    return R, S, E, K, np.ascontiguousarray(idx, dtype=np.int32)


@SETTINGS
@given(routed())
def test_contiguous_plan_is_the_sorted_cut(case):
    R, S, E, K, idx = case
    pl = ORA.plan(R, S, E, K, idx)
    ref = pins.brute_plan(R, S, E, K, idx)
    pins._check_plan_equal(pl, ref, R, E)
    pins.check_plan_invariants(pl, R, S, E, K, idx)
    exact = ref["maxvio"]
    assert abs(Fraction(pl["maxvio"]) - exact) <= Fraction(2, 2 ** 52) * max(1, abs(exact))


@SETTINGS
@given(routed())
def test_home_first_plan_is_the_queue_simulation(case):
    R, S, E, K, idx = case
    pl = ORA.plan_home_first(R, S, E, K, idx)
    pins._check_hf_equal(pl, pins.brute_home_first(R, S, E, K, idx))
    pins.check_home_first_invariants(pl, R, S, E, K, idx)
    # (Fewer replicas than the contiguous cut is typical, not a theorem: with
    # R=4, S=4, E=12, K=1 a routing exists where home-first makes 2 and the
    # contiguous cut 1, so no such bound is asserted here.)


@SETTINGS
@given(routed(), st.integers(1, 8))
def test_capped_plan_is_the_queue_simulation(case, B):
    R, S, E, K, idx = case
    pl = ORA.plan_capped(R, S, E, K, B, idx)
    pins._check_capped_equal(pl, pins.brute_capped(R, S, E, K, B, idx), str((R, S, E, K, B)))
    pins.check_capped_invariants(pl, R, S, E, K, B, idx)


@SETTINGS
@given(routed(), st.integers(1, 8))
def test_capped_items_and_rooms_number_at_most_E(case, B):
    """The capped schedule's items (experts that overflow their home rank)
    and rooms (ranks with spare room after their home fill) number at most E
    together: an overflowing expert's home rank is full, so items come from
    full ranks (E/R experts each) and rooms are the other ranks.  The GPU
    builder sorts them with one key per thread of a 1024-thread block and
    relies on this bound (E <= 1024)."""
    R, S, E, K, idx = case
    pl = ORA.plan_capped(R, S, E, K, B, idx)
    C, Bh = S * K, E // R
    counts = np.bincount(idx.ravel(), minlength=E)
    seg = pl["seg"][:pl["num_seg"]]
    items = {int(e) for e, r, _, _ in seg if r != e // Bh}   # experts with a replica piece
    home_load = counts.reshape(R, Bh).sum(axis=1)
    rooms = int((home_load < C).sum())
    assert len(items) + rooms <= E
    full = int((home_load >= C).sum())
    assert len(items) <= Bh * full


@SETTINGS
@given(routed(), st.integers(1, 5), st.integers(0, 2 ** 31 - 1))
def test_combine_and_reduce_are_exact_sums(case, P, seed):
    R, S, E, K, idx = case
    rng = np.random.default_rng(seed)
    pl = ORA.plan(R, S, E, K, idx)
    N, H = R * S, 8
    w = rng.standard_normal((N, K)).astype(np.float32)
    y = pins._bf16_rows(ORA, rng, N * K, H)
    _, exact, _ = ORA.combine(pl["slot"], w, y)
    yv = ((y.astype(np.uint32) << 16).view(np.float32)).astype(np.float64)
    for g in range(N):
        for h in range(H):
            want = sum(Fraction(float(w[g, k])) * Fraction(float(yv[pl["slot"][g, k], h]))
                       for k in range(K))
            assert Fraction(float(exact[g, h])) == want or \
                abs(Fraction(float(exact[g, h])) - want) <= abs(want) * Fraction(1, 2 ** 50)
    G = rng.standard_normal((E + R - 1, P)).astype(np.float32)
    hexact, _ = ORA.reduce(pl["expert_seg_ptr"], G)
    ptr = pl["expert_seg_ptr"]
    for e in range(E):
        for c in range(P):
            want = sum(Fraction(float(G[s, c])) for s in range(ptr[e], ptr[e + 1]))
            assert abs(Fraction(float(hexact[e, c])) - want) <= abs(want) * Fraction(1, 2 ** 50)
