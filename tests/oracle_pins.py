"""Pins for the CPU oracle: checks against things other than the oracle itself.

Each ``pin_*`` takes an ``oracle.Oracle`` instance and raises AssertionError on
a mismatch.  The pins rest on
  * hand-derived worked examples (``tests/golden/``), built from the
    definitions on the MoonEP pages;
  * brute force on tiny inputs with independent Python code (``sorted`` for
    the schedule, ``fractions.Fraction`` for exact sums and rounding, a search
    over the whole bf16 grid for rounding);
  * closed forms (round-robin routing gives maxvio = 0 and no replicas;
    adversarial routing gives maxvio = 31 and 31 replicas at the skew shape);
  * invariants the pages fix (exactly S*K slots per rank, every (token,k)
    placed once, slots in expert order, counts sum to R*S*K);
  * a library routine (torch's float32 -> bf16 conversion).
They are kept in one module so ``test_oracle_mutants.py`` can rerun the whole
set against oracles with planted mistakes.
"""
from __future__ import annotations

import bisect
import json
import math
import os
import struct
from collections import Counter
from fractions import Fraction

import numpy as np

import oracle as oracle_mod

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def load_golden(name: str) -> dict:
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# ---------------------------------------------------------------- bf16 helpers

def _bits_to_f32(b: int) -> float:
    return struct.unpack("<f", struct.pack("<I", (b & 0xFFFF) << 16))[0]


def _bf16_grid():
    """All finite non-negative bf16 values with their bit patterns, sorted."""
    vals = []
    for b in range(0x0000, 0x7F80):
        vals.append((_bits_to_f32(b), b))
    vals.sort()
    return [v for v, _ in vals], [b for _, b in vals]


_GRID = None


def bf16_round_by_search(d: float) -> int:
    """Nearest bf16 to ``d`` by bracketing it in the sorted grid and comparing
    exact rational distances; ties go to the even bit pattern."""
    global _GRID
    if _GRID is None:
        _GRID = _bf16_grid()
    vals, bits = _GRID
    sign = 0x8000 if math.copysign(1.0, d) < 0 else 0
    a = abs(d)
    big = vals[-1]
    half_next = Fraction(big) + (Fraction(2) ** 128 - Fraction(big)) / 2
    if Fraction(a) >= half_next:
        return sign | 0x7F80
    i = bisect.bisect_left(vals, a)
    if i < len(vals) and vals[i] == a:
        return sign | bits[i]
    lo, hi = vals[i - 1], (vals[i] if i < len(vals) else 2.0 ** 128)
    dlo, dhi = Fraction(a) - Fraction(lo), Fraction(hi) - Fraction(a)
    if dlo < dhi:
        return sign | bits[i - 1]
    if dhi < dlo:
        return sign | (bits[i] if i < len(vals) else 0x7F80)
    blo = bits[i - 1]
    bhi = bits[i] if i < len(vals) else 0x7F80
    return sign | (blo if blo % 2 == 0 else bhi)


def pin_bf16_widen(ora):
    """Every non-NaN bf16 pattern widens to the float32 with the same upper
    half and narrows back to itself."""
    for b in list(range(0, 0x7F81)) + list(range(0x8000, 0xFF81)):
        f = ora.bf16_to_f32(b)
        assert struct.unpack("<I", struct.pack("<f", f))[0] == b << 16, hex(b)
        assert ora.f64_to_bf16(f) == b, hex(b)


def pin_bf16_rounding(ora):
    """Round-to-nearest-even against a grid search, a library conversion and
    hand-picked ties, subnormals and overflow."""
    one = 1.0
    cases = [
        (one + 2.0 ** -8, 0x3F80),            # tie between 1 and 1+2^-7 -> even (1)
        (one + 3 * 2.0 ** -8, 0x3F82),        # tie -> even (1 + 2^-6)
        (one + 2.0 ** -8 + 2.0 ** -30, 0x3F81),  # just above the tie
        (-(one + 2.0 ** -8), 0xBF80),
        (2.0 ** -133, 0x0001),                # smallest subnormal
        (2.0 ** -134, 0x0000),                # tie with zero -> even (0)
        (3 * 2.0 ** -134, 0x0002),            # tie 1.5 units -> 2 units
        (255 * 2.0 ** 120, 0x7F7F),           # largest finite
        (255.5 * 2.0 ** 120, 0x7F80),         # tie past the largest finite -> inf
        (255.49 * 2.0 ** 120, 0x7F7F),
        (math.inf, 0x7F80), (-math.inf, 0xFF80), (0.0, 0x0000), (-0.0, 0x8000),
    ]
    for d, want in cases:
        assert ora.f64_to_bf16(d) == want, (d, hex(ora.f64_to_bf16(d)), hex(want))
    assert ora.f64_to_bf16(math.nan) & 0x7FFF > 0x7F80
    rng = np.random.default_rng(1234)
    ds = np.concatenate([rng.standard_normal(600) * 10.0 ** rng.integers(-8, 8, 600),
                         rng.standard_normal(100) * 2.0 ** -128])
    for d in ds:
        assert ora.f64_to_bf16(float(d)) == bf16_round_by_search(float(d)), d
    import torch
    f32 = rng.standard_normal(4000).astype(np.float32) * np.float32(37.0)
    lib = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().astype(np.uint16)
    mine = np.array([ora.f64_to_bf16(float(v)) for v in f32], dtype=np.uint16)
    assert np.array_equal(lib, mine)


# --------------------------------------------------------- plan brute force

def brute_plan(R, S, E, K, idx):
    """The schedule written out as Python's sorted() over (expert, g, k)."""
    idx = np.asarray(idx).reshape(R * S, K)
    N, SK = R * S, S * K
    pairs = sorted((int(idx[g, k]), g, k) for g in range(N) for k in range(K))
    slot = np.zeros((N, K), np.int64)
    src = np.zeros(N * K, np.int64)
    for p, (e, g, k) in enumerate(pairs):
        slot[g, k] = p
        src[p] = g * K + k
    runs = []
    for p, (e, g, k) in enumerate(pairs):
        key = (p // SK, e)
        if runs and runs[-1][0] == key:
            runs[-1][2] += 1
        else:
            runs.append([key, p % SK, 1])
    seg = [(e, r, start, cnt) for (r, e), start, cnt in runs]
    B = E // R
    cnt = Counter(e for e, _, _ in pairs)
    counts = [cnt.get(e, 0) for e in range(E)]
    return dict(
        counts=counts,
        slot=slot, src_pair=src, seg=seg,
        replica_seg=[i for i, s in enumerate(seg) if s[1] != s[0] // B],
        rank_seg_ptr=[next((i for i, s in enumerate(seg) if s[1] >= r), len(seg)) for r in range(R + 1)],
        expert_seg_ptr=[next((i for i, s in enumerate(seg) if s[0] >= e), len(seg)) for e in range(E + 1)],
        maxvio=Fraction(max(counts) * E, N * K) - 1,
    )


def _check_plan_equal(pl, ref, R, E):
    ns = pl["num_seg"]
    assert list(pl["counts"]) == ref["counts"]
    assert np.array_equal(pl["slot"], ref["slot"])
    assert np.array_equal(pl["src_pair"], ref["src_pair"])
    assert ns == len(ref["seg"])
    assert [tuple(s) for s in pl["seg"][:ns].tolist()] == [tuple(s) for s in ref["seg"]]
    assert pl["num_replicas"] == len(ref["replica_seg"])
    assert list(pl["replica_seg"][:pl["num_replicas"]]) == ref["replica_seg"]
    assert list(pl["rank_seg_ptr"]) == ref["rank_seg_ptr"]
    assert list(pl["expert_seg_ptr"]) == ref["expert_seg_ptr"]


def _random_idx(rng, R, S, E, K, distinct=True, skew=0.0):
    N = R * S
    if distinct:
        logits = rng.standard_normal((N, E)) - skew * np.log(np.arange(1, E + 1))
        return np.argsort(-logits, axis=1, kind="stable")[:, :K].astype(np.int32)
    return rng.integers(0, E, size=(N, K)).astype(np.int32)


SMALL_SHAPES = [(1, 1, 1, 1), (1, 5, 3, 2), (2, 3, 4, 2), (4, 7, 8, 3), (3, 9, 6, 6),
                (4, 16, 16, 2), (8, 5, 16, 4), (2, 33, 10, 5), (5, 4, 20, 7)]


def pin_plan_bruteforce(ora):
    rng = np.random.default_rng(7)
    for (R, S, E, K) in SMALL_SHAPES:
        for distinct, skew in ((True, 0.0), (True, 2.0), (False, 0.0)):
            idx = _random_idx(rng, R, S, E, K, distinct, skew)
            pl = ora.plan(R, S, E, K, idx)
            ref = brute_plan(R, S, E, K, idx)
            _check_plan_equal(pl, ref, R, E)
            exact = ref["maxvio"]
            assert abs(Fraction(pl["maxvio"]) - exact) <= Fraction(2, 2 ** 52) * max(1, abs(exact))
            assert pl["max_count"] == max(ref["counts"])
            c, m, v = ora.maxvio(R, S, E, K, idx)
            assert list(c) == ref["counts"] and m == pl["max_count"] and v == pl["maxvio"]


def pin_plan_golden(ora):
    for name in ("example_a.json", "example_b.json"):
        gd = load_golden(name)
        R, S, E, K = gd["R"], gd["S"], gd["E"], gd["K"]
        pl = ora.plan(R, S, E, K, np.array(gd["idx"], np.int32))
        assert list(pl["counts"]) == gd["counts"]
        assert pl["max_count"] == gd["max_count"]
        assert pl["maxvio"] == gd["maxvio"]
        assert list(pl["expert_offset"]) == gd["expert_offset"]
        assert pl["slot"].tolist() == gd["slot"]
        assert list(pl["src_pair"]) == gd["src_pair"]
        assert pl["num_seg"] == len(gd["segments"])
        assert pl["seg"][:pl["num_seg"]].tolist() == gd["segments"]
        assert list(pl["replica_seg"][:pl["num_replicas"]]) == gd["replica_seg"]
        assert list(pl["rank_seg_ptr"]) == gd["rank_seg_ptr"]
        assert list(pl["expert_seg_ptr"]) == gd["expert_seg_ptr"]


def check_plan_invariants(pl, R, S, E, K, idx):
    """Properties the pages fix, valid at any size."""
    idx = np.asarray(idx).reshape(-1)
    NK, SK = R * S * K, S * K
    slot = np.asarray(pl["slot"]).reshape(-1).astype(np.int64)
    src = np.asarray(pl["src_pair"]).astype(np.int64)
    counts = np.asarray(pl["counts"])
    assert counts.sum() == NK
    assert np.array_equal(np.bincount(idx, minlength=E), counts)
    # every (token, k) placed exactly once: slot is a bijection, src its inverse
    assert np.array_equal(np.sort(slot), np.arange(NK))
    assert np.array_equal(src[slot], np.arange(NK))
    # expert order, and (g, k) order inside an expert (stability)
    e_of_p = idx[src]
    assert np.all(np.diff(e_of_p) >= 0)
    same = np.diff(e_of_p) == 0
    assert np.all(np.diff(src)[same] > 0)
    # segments tile every rank with exactly S*K slots and match the slot experts
    ns = pl["num_seg"]
    seg = np.asarray(pl["seg"])[:ns]
    per_rank = np.bincount(seg[:, 1], weights=seg[:, 3], minlength=R)
    assert np.array_equal(per_rank, np.full(R, SK))
    p0 = seg[:, 1].astype(np.int64) * SK + seg[:, 2]
    assert np.array_equal(p0[1:], p0[:-1] + seg[:-1, 3]) and p0[0] == 0
    assert np.array_equal(e_of_p[p0], seg[:, 0])
    assert np.array_equal(e_of_p[p0 + seg[:, 3] - 1], seg[:, 0])
    nz = int((counts > 0).sum())
    assert nz <= ns <= nz + R - 1
    B = E // R
    rep = np.nonzero(seg[:, 1] != seg[:, 0] // B)[0]
    assert pl["num_replicas"] == rep.size
    assert np.array_equal(np.asarray(pl["replica_seg"])[:rep.size], rep)


def pin_plan_invariants(ora):
    import workloads
    for name, S in (("kimi_r64_e896_k16", 37), ("skew_r32_zipf1.5", 61),
                    ("r16_e256_h7168", 45), ("tiny_r4_e16", 64)):
        wl = workloads.reduced(workloads.WORKLOADS[name], S=S)
        idx, _ = workloads.routing(wl)
        pl = ora.plan(wl.R, wl.S, wl.E, wl.K, idx)
        check_plan_invariants(pl, wl.R, wl.S, wl.E, wl.K, idx)


def pin_closed_forms(ora):
    import workloads
    # Round-robin routing: T_e = R*S*K/E for all e -> maxvio = 0 ("zero means
    # perfect balance"); every rank boundary is an expert boundary, so every
    # expert sits whole on its home rank: E segments, no replica.
    for (R, S, E, K) in [(4, 64, 16, 2), (8, 4096, 64, 6), (16, 8192, 256, 8),
                         (64, 56, 896, 16), (32, 4096, 256, 8), (2, 3, 6, 4)]:
        idx, _ = workloads.roundrobin_routing(R, S, E, K)
        c, m, v = ora.maxvio(R, S, E, K, idx)
        assert v == 0.0 and m == R * S * K // E and np.all(c == m)
        if R * S * K <= 2_200_000:
            pl = ora.plan(R, S, E, K, idx)
            assert pl["num_seg"] == E and pl["num_replicas"] == 0
            T = R * S * K // E
            B = E // R
            want = [(e, e // B, (e % B) * T, T) for e in range(E)]
            assert [tuple(s) for s in pl["seg"][:E].tolist()] == want
            assert list(pl["rank_seg_ptr"]) == [r * B for r in range(R + 1)]
    # Adversarial routing at the skew shape: every token picks experts 0..7.
    # T_0..7 = 131072, maxvio = 131072 / 4096 - 1 = 31; expert e fills ranks
    # 4e..4e+3; home(e) = 0 for e < 8, so 31 of the 32 segments are replicas.
    R, S, E, K = 32, 4096, 256, 8
    rng = np.random.default_rng(0)
    idx = np.argsort(-rng.standard_normal((R * S, K)), axis=1).astype(np.int32)
    pl = ora.plan(R, S, E, K, idx)
    assert pl["maxvio"] == 31.0 and pl["max_count"] == 131072
    assert pl["num_seg"] == 32 and pl["num_replicas"] == 31
    want = [(e, 4 * e + j, 0, 32768) for e in range(8) for j in range(4)]
    assert [tuple(s) for s in pl["seg"][:32].tolist()] == want
    assert list(pl["expert_seg_ptr"]) == [4 * e for e in range(9)] + [32] * (E - 8)
    # One expert takes everything (K = 1): maxvio = E - 1.
    idx = np.zeros((4 * 5, 1), np.int32)
    c, m, v = ora.maxvio(4, 5, 8, 1, idx)
    assert v == 7.0 and m == 20


def pin_errors(ora):
    idx = np.zeros((4, 2), np.int32)
    for shape in [(2, 2, 3, 2), (0, 2, 4, 2), (2, 0, 4, 2), (2, 2, 4, 5), (2, 2, 4, 0)]:
        try:
            ora.plan(*shape, idx)
        except oracle_mod.OracleError as e:
            assert e.code == oracle_mod.ERR_ARG
        else:
            raise AssertionError(f"shape {shape} accepted")
    for bad in (-1, 4, 1 << 30):
        idx2 = idx.copy()
        idx2[3, 1] = bad
        try:
            ora.plan(2, 2, 4, 2, idx2)
        except oracle_mod.OracleError as e:
            assert e.code == oracle_mod.ERR_DATA
        else:
            raise AssertionError("bad id accepted")


# ------------------------------------------------------------ data movement

def pin_dispatch(ora):
    rng = np.random.default_rng(11)
    for (R, S, E, K) in [(2, 3, 4, 2), (4, 16, 16, 2), (3, 5, 6, 6)]:
        H = 8
        idx = _random_idx(rng, R, S, E, K)
        ref = brute_plan(R, S, E, K, idx)
        x = rng.integers(0, 1 << 16, size=(R * S, H), dtype=np.uint16)
        buf = ora.dispatch(K, ref["src_pair"].astype(np.int32), x)
        for g in range(R * S):
            for k in range(K):
                assert np.array_equal(buf[ref["slot"][g, k]], x[g])
        # each token row appears exactly K times
        rows = Counter(bytes(r) for r in buf)
        assert all(rows[bytes(x[g])] >= K for g in range(R * S))


def pin_combine(ora):
    rng = np.random.default_rng(5)
    # (a) golden example A with y[p,:] = p+1 and w = [0.75, 0.25]
    gd = load_golden("example_a.json")
    slot = np.array(gd["slot"], np.int32)
    w = np.array(gd["combine_w"], np.float32)
    y = np.array([[ora.f64_to_bf16(p + 1.0)] * 8 for p in range(8)], np.uint16)
    out, exact, _ = ora.combine(slot, w, y)
    assert np.array_equal(exact[:, 0], np.array(gd["combine_out"]))
    assert all(ora.bf16_to_f32(b) == v for b, v in zip(out[:, 0], gd["combine_out"]))
    # (b) one-hot weights pick one expert output exactly, for every k
    n, K, H, rows = 6, 5, 16, 30
    y = rng.integers(0, 0x7F00, size=(rows, H), dtype=np.uint16)
    slot = rng.integers(0, rows, size=(n, K)).astype(np.int32)
    for kstar in range(K):
        w = np.zeros((n, K), np.float32)
        w[:, kstar] = 1.0
        out, _, _ = ora.combine(slot, w, y)
        assert np.array_equal(out, y[slot[:, kstar]])
    # (c) exact rational sums, rounded by grid search
    for K in (1, 2, 6, 16):
        n, H, rows = 5, 8, 40
        y = np.array([[ora.f64_to_bf16(float(v)) for v in r]
                      for r in rng.standard_normal((rows, H))], np.uint16)
        slot = rng.integers(0, rows, size=(n, K)).astype(np.int32)
        w = rng.random((n, K)).astype(np.float32)
        out, exact, absum = ora.combine(slot, w, y)
        for g in range(n):
            for h in range(H):
                terms = [Fraction(float(w[g, k])) * Fraction(_bits_to_f32(int(y[slot[g, k], h])))
                         for k in range(K)]
                v = sum(terms, Fraction(0))
                assert abs(Fraction(exact[g, h]) - v) <= Fraction(K, 2 ** 52) * sum(abs(t) for t in terms)
                assert out[g, h] == bf16_round_by_search(float(exact[g, h]))
                assert abs(absum[g, h] - float(sum(abs(t) for t in terms))) <= 1e-12 * absum[g, h]


def pin_reduce(ora):
    # (a) golden example B with G[s,:] = 10^s
    gd = load_golden("example_b.json")
    G = np.array([[10.0 ** s] * 3 for s in range(3)], np.float32)
    home, _ = ora.reduce(np.array(gd["expert_seg_ptr"], np.int32), G)
    assert np.array_equal(home[:, 0], np.array(gd["home"]))
    # (b) G[s,:] = s + 1: home[e] = sum of (s+1) over e's segments, 0 if none
    ptr = np.array([0, 3, 3, 4, 9, 9], np.int32)          # expert 1 and 4 empty
    P = 7
    G = np.repeat(np.arange(1, 11, dtype=np.float32)[:, None], P, axis=1)
    home, absum = ora.reduce(ptr, G)
    want = [sum(range(ptr[e] + 1, ptr[e + 1] + 1)) for e in range(5)]
    assert np.array_equal(home, np.repeat(np.array(want, np.float64)[:, None], P, axis=1))
    assert np.array_equal(absum, home)
    # (c) random values against exact rational sums
    rng = np.random.default_rng(3)
    ptr = np.array([0, 2, 2, 7, 8], np.int32)
    G = (rng.standard_normal((9, 11)) * 100).astype(np.float32)
    home, _ = ora.reduce(ptr, G)
    for e in range(4):
        for i in range(11):
            v = sum((Fraction(float(G[s, i])) for s in range(ptr[e], ptr[e + 1])), Fraction(0))
            assert abs(Fraction(home[e, i]) - v) <= Fraction(8, 2 ** 52) * max(1, abs(v))


# ------------------------------------------------------------- backward

def _bf16_rows(ora, rng, rows, H, scale=1.0):
    return np.array([[ora.f64_to_bf16(float(v)) for v in r]
                     for r in rng.standard_normal((rows, H)) * scale], np.uint16)


def _perm_slots(rng, n, K):
    """A slot table like a plan's: every row of a [n*K, H] buffer used once."""
    return rng.permutation(n * K).astype(np.int32).reshape(n, K)


def pin_combine_backward(ora):
    rng = np.random.default_rng(21)
    for K in (1, 2, 5, 16):
        n, H = 4, 8
        slot = _perm_slots(rng, n, K)
        w = rng.random((n, K)).astype(np.float32)
        y = _bf16_rows(ora, rng, n * K, H)
        go = _bf16_rows(ora, rng, n, H)
        gy, gye, gw, gwa = ora.combine_backward(slot, w, go, y)
        F = lambda b: Fraction(_bits_to_f32(int(b)))
        # adjoint: <combine(y), go> == <y, grad_y>, exactly
        lhs = sum((F(go[g, h]) * Fraction(float(w[g, k])) * F(y[slot[g, k], h])
                   for g in range(n) for h in range(H) for k in range(K)), Fraction(0))
        rhs = sum((F(y[p, h]) * Fraction(gye[p, h]) for p in range(n * K) for h in range(H)),
                  Fraction(0))
        assert lhs == rhs, (K, float(lhs), float(rhs))
        for g in range(n):
            for k in range(K):
                p = slot[g, k]
                for h in range(H):
                    want = Fraction(float(w[g, k])) * F(go[g, h])
                    assert Fraction(gye[p, h]) == want
                    assert gy[p, h] == bf16_round_by_search(float(want))
                dot = sum((F(go[g, h]) * F(y[p, h]) for h in range(H)), Fraction(0))
                assert abs(Fraction(gw[g, k]) - dot) <= Fraction(H, 2 ** 52) * Fraction(gwa[g, k])
    # unit weight, K = 1: the slot gradient is the output gradient itself
    slot = np.arange(6, dtype=np.int32).reshape(6, 1)
    go = _bf16_rows(ora, rng, 6, 8)
    gy, _, _, _ = ora.combine_backward(slot, np.ones((6, 1), np.float32), go, go)
    assert np.array_equal(gy, go)


def pin_dispatch_backward(ora):
    rng = np.random.default_rng(22)
    F = lambda b: Fraction(_bits_to_f32(int(b)))
    for K in (1, 3, 16):
        n, H = 5, 8
        slot = _perm_slots(rng, n, K)
        x = _bf16_rows(ora, rng, n, H)
        gb = _bf16_rows(ora, rng, n * K, H)
        gx, ex, ab = ora.dispatch_backward(slot, gb)
        # adjoint: <dispatch(x), grad_buf> == <x, grad_x_exact>
        src = np.empty(n * K, np.int32)
        src[slot.reshape(-1)] = np.arange(n * K, dtype=np.int32)
        buf = ora.dispatch(K, src, x)
        lhs = sum((F(buf[p, h]) * F(gb[p, h]) for p in range(n * K) for h in range(H)), Fraction(0))
        rhs = sum((F(x[g, h]) * Fraction(ex[g, h]) for g in range(n) for h in range(H)), Fraction(0))
        assert lhs == rhs
        for g in range(n):
            for h in range(H):
                v = sum((F(gb[slot[g, k], h]) for k in range(K)), Fraction(0))
                assert Fraction(ex[g, h]) == v
                assert gx[g, h] == bf16_round_by_search(float(v))
    # rows of constant value c_p: grad_x[g] = sum_k c_{slot[g,k]}
    n, K, H = 3, 4, 8
    slot = _perm_slots(rng, n, K)
    gb = np.array([[ora.f64_to_bf16(float(p + 1))] * H for p in range(n * K)], np.uint16)
    gx, ex, _ = ora.dispatch_backward(slot, gb)
    assert np.array_equal(ex, np.repeat((slot + 1).sum(axis=1, keepdims=True).astype(np.float64), H, axis=1))


def pin_prefetch_replicas(ora):
    # brute-force replica list from sorted(); row e of w_home holds e in every byte
    rng = np.random.default_rng(31)
    for (R, S, E, K) in [(2, 3, 4, 2), (4, 16, 16, 2), (8, 5, 16, 4), (5, 4, 20, 7)]:
        idx = _random_idx(rng, R, S, E, K, True, 2.0)
        pl = ora.plan(R, S, E, K, idx)
        ref = brute_plan(R, S, E, K, idx)
        w_home = np.repeat(np.arange(E, dtype=np.uint8)[:, None], 48, axis=1)
        got = ora.prefetch_replicas(pl, w_home)
        want = [ref["seg"][s][0] for s in ref["replica_seg"]]
        assert got.shape[0] == len(want)
        assert all(np.all(got[j] == want[j]) for j in range(len(want)))
    # adversarial closed form: replicas are experts 0 (x3) then 1..7 (x4 each)
    R, S, E, K = 32, 4096, 256, 8
    idx = np.argsort(-np.random.default_rng(0).standard_normal((R * S, K)), axis=1).astype(np.int32)
    pl = ora.plan(R, S, E, K, idx)
    w_home = (np.arange(E, dtype=np.float32)[:, None] + np.arange(4, dtype=np.float32) / 8)
    got = ora.prefetch_replicas(pl, w_home)
    experts = [0] * 3 + [e for e in range(1, 8) for _ in range(4)]
    assert np.array_equal(got, w_home[experts])


# ---------------------------------------------------- home-first schedule

def brute_home_first(R, S, E, K, idx):
    """The home-first plan as a simulation with queues: ranks are bins of
    S*K slots; each bin takes its home experts' pairs (ascending experts,
    (g,k) order) while it has room; what does not fit joins one overflow
    queue; bins are then topped up from the queue in rank order."""
    idx = np.asarray(idx).reshape(R * S, K)
    C, B = S * K, E // R
    lists = [[] for _ in range(E)]
    for g in range(R * S):
        for k in range(K):
            lists[int(idx[g, k])].append(g * K + k)
    bins = [[] for _ in range(R)]
    queue = []
    for r in range(R):
        for e in range(r * B, (r + 1) * B):
            room = C - len(bins[r])
            bins[r] += [(e, q) for q in lists[e][:room]]
            queue += [(e, q) for q in lists[e][room:]]
    qi = 0
    for r in range(R):
        while len(bins[r]) < C:
            bins[r].append(queue[qi])
            qi += 1
    assert qi == len(queue)
    slot = np.zeros((R * S, K), np.int64)
    runs = []                                   # (expert, rank, start, count) in slot order
    for r in range(R):
        for i, (e, q) in enumerate(bins[r]):
            slot[q // K, q % K] = r * C + i
            if runs and runs[-1][0] == e and runs[-1][1] == r:
                runs[-1][3] += 1
            else:
                runs.append([e, r, i, 1])
    table = sorted(range(len(runs)), key=lambda j: (runs[j][0], runs[j][1]))
    where = {j: a for a, j in enumerate(table)}
    seg = [tuple(runs[j]) for j in table]
    return dict(slot=slot, seg=seg, rank_seg_idx=[where[j] for j in range(len(runs))],
                replica_seg=[a for a, sg in enumerate(seg) if sg[1] != sg[0] // B],
                expert_seg_ptr=[next((a for a, sg in enumerate(seg) if sg[0] >= e), len(seg))
                                for e in range(E + 1)],
                rank_seg_ptr=[next((j for j in range(len(runs)) if runs[j][1] >= r), len(runs))
                              for r in range(R + 1)])


def _check_hf_equal(pl, ref, what=""):
    ns = pl["num_seg"]
    assert np.array_equal(pl["slot"], ref["slot"]), what
    assert [tuple(x) for x in pl["seg"][:ns].tolist()] == ref["seg"], what
    assert list(pl["rank_seg_idx"][:ns]) == ref["rank_seg_idx"], what
    assert list(pl["rank_seg_ptr"]) == ref["rank_seg_ptr"], what
    assert list(pl["expert_seg_ptr"]) == ref["expert_seg_ptr"], what
    assert pl["num_replicas"] == len(ref["replica_seg"]), what
    assert list(pl["replica_seg"][:pl["num_replicas"]]) == ref["replica_seg"], what


def check_home_first_invariants(pl, R, S, E, K, idx):
    idx = np.asarray(idx).reshape(-1)
    NK, C, B = R * S * K, S * K, E // R
    slot = np.asarray(pl["slot"]).reshape(-1).astype(np.int64)
    src = np.asarray(pl["src_pair"]).astype(np.int64)
    assert np.array_equal(np.sort(slot), np.arange(NK))           # each pair placed once
    assert np.array_equal(src[slot], np.arange(NK))
    ns = pl["num_seg"]
    seg = np.asarray(pl["seg"])[:ns]
    assert np.array_equal(np.bincount(seg[:, 1], weights=seg[:, 3], minlength=R), np.full(R, C))
    e_of_p = idx[src]
    for e, r, st, cnt in seg:                                       # runs hold one expert
        assert np.all(e_of_p[r * C + st: r * C + st + cnt] == e)
    counts = np.bincount(idx, minlength=E)
    home_load = np.array([counts[r * B:(r + 1) * B].sum() for r in range(R)])
    over_e = np.zeros(E, np.int64)
    for e, r, st, cnt in seg:
        if r != e // B:
            over_e[e] += cnt
    for e in range(E):                 # an expert leaves home only if its home rank is full
        if over_e[e]:
            assert home_load[e // B] >= C
    assert ns <= E + R - 1                                          # the static bound
    deficit_ranks = int((home_load < C).sum())
    overflowing = int((over_e > 0).sum())
    if overflowing:
        assert pl["num_replicas"] <= overflowing + deficit_ranks - 1
    else:
        assert pl["num_replicas"] == 0


def pin_home_first(ora):
    gd = load_golden("example_c_home_first.json")
    pl = ora.plan_home_first(gd["R"], gd["S"], gd["E"], gd["K"], np.array(gd["idx"], np.int32))
    assert list(pl["counts"]) == gd["counts"] and pl["maxvio"] == gd["maxvio"]
    assert pl["slot"].tolist() == gd["slot"] and list(pl["src_pair"]) == gd["src_pair"]
    assert pl["seg"][:pl["num_seg"]].tolist() == gd["segments"]
    assert list(pl["replica_seg"][:pl["num_replicas"]]) == gd["replica_seg"]
    assert list(pl["rank_seg_ptr"]) == gd["rank_seg_ptr"]
    assert list(pl["rank_seg_idx"]) == gd["rank_seg_idx"]
    assert list(pl["expert_seg_ptr"]) == gd["expert_seg_ptr"]
    rng = np.random.default_rng(41)
    for (R, S, E, K) in SMALL_SHAPES:
        for distinct, skew in ((True, 0.0), (True, 2.5), (False, 0.0)):
            idx = _random_idx(rng, R, S, E, K, distinct, skew)
            pl = ora.plan_home_first(R, S, E, K, idx)
            _check_hf_equal(pl, brute_home_first(R, S, E, K, idx), str((R, S, E, K)))
            check_home_first_invariants(pl, R, S, E, K, idx)
    import workloads
    for name, S in (("kimi_r64_e896_k16", 23), ("skew_r32_zipf1.5", 61), ("r8_e64_h2048", 97)):
        wl = workloads.reduced(workloads.WORKLOADS[name], S=S)
        idx, _ = workloads.routing(wl)
        pl = ora.plan_home_first(wl.R, wl.S, wl.E, wl.K, idx)
        check_home_first_invariants(pl, wl.R, wl.S, wl.E, wl.K, idx)
        assert pl["num_replicas"] <= ora.plan(wl.R, wl.S, wl.E, wl.K, idx)["num_replicas"]


def pin_home_first_closed_forms(ora):
    """Where every rank's home experts exactly fill it (round-robin routing)
    or the overflow order coincides with expert order (adversarial routing),
    the home-first plan equals the contiguous cut."""
    import workloads
    for (R, S, E, K) in [(4, 64, 16, 2), (8, 512, 64, 6), (2, 3, 6, 4)]:
        idx, _ = workloads.roundrobin_routing(R, S, E, K)
        a, b = ora.plan_home_first(R, S, E, K, idx), ora.plan(R, S, E, K, idx)
        assert np.array_equal(a["slot"], b["slot"]) and a["num_replicas"] == 0
    R, S, E, K = 32, 4096, 256, 8
    idx = np.argsort(-np.random.default_rng(0).standard_normal((R * S, K)), axis=1).astype(np.int32)
    a, b = ora.plan_home_first(R, S, E, K, idx), ora.plan(R, S, E, K, idx)
    assert np.array_equal(a["slot"], b["slot"])
    assert a["num_seg"] == 32 and a["num_replicas"] == 31


# ---------------------------------------------------- capped schedule

def brute_capped(R, S, E, K, B, idx):
    """The capped plan as a simulation with pair queues: every expert's pairs
    queue up in (g, k) order; each rank, taking its home experts smallest
    count first, keeps the head of each queue while it has room; the
    overflowing experts line up by overflow (largest first), the ranks with
    room by room (largest first); the short queues (shorter than the largest
    room) are offered whole to the rooms in turn, at most B - 2 per room; the
    queues left over are poured into the rooms' remaining space in line
    order.  Ranks list home runs by expert, then arrivals in arrival order."""
    idx = np.asarray(idx).reshape(R * S, K)
    C, Bh = S * K, E // R
    queue = [[] for _ in range(E)]
    for g in range(R * S):
        for k in range(K):
            queue[int(idx[g, k])].append(g * K + k)
    kept = [0] * E
    for r in range(R):
        room = C
        for e in sorted(range(r * Bh, (r + 1) * Bh), key=lambda e: (len(queue[e]), e)):
            kept[e] = min(len(queue[e]), room)
            room -= kept[e]
    home = [[(e, q) for e in range(r * Bh, (r + 1) * Bh) for q in queue[e][:kept[e]]]
            for r in range(R)]
    rest = {e: queue[e][kept[e]:] for e in range(E) if len(queue[e]) > kept[e]}
    line = sorted(rest, key=lambda e: (-len(rest[e]), e))
    space = {r: C - len(home[r]) for r in range(R) if len(home[r]) < C}
    rooms = sorted(space, key=lambda r: (-space[r], r))
    arrivals = {r: [] for r in range(R)}       # (expert, [pairs]) in arrival order
    poured = []
    if rooms:
        dmax = space[rooms[0]]
        short = [e for e in line if len(rest[e]) < dmax]
        for f, e in enumerate(short):
            r = rooms[f % len(rooms)]
            if f // len(rooms) < B - 2 and space[r] >= len(rest[e]):
                arrivals[r].append((e, rest[e]))
                space[r] -= len(rest[e])
            else:
                poured.append(e)
        unplaced = len(poured)
        poured = [e for e in line if e not in short or e in poured]
        stream = [(e, q) for e in poured for q in rest[e]]
        at = 0
        for r in rooms:
            take = stream[at:at + space[r]]
            at += space[r]
            # group the poured pairs of this room into runs of one expert
            runs = []
            for e, q in take:
                if runs and runs[-1][0] == e:
                    runs[-1][1].append(q)
                else:
                    runs.append((e, [q]))
            arrivals[r] += runs
        assert at == len(stream)
    else:
        unplaced = 0
    slot = np.zeros((R * S, K), np.int64)
    runs = []                                   # [expert, rank, start, count] in slot order
    for r in range(R):
        order = [(e, [q]) for e, q in home[r]] + [(e, qs) for e, qs in arrivals[r]]
        i = 0
        for e, qs in order:
            for q in qs:
                slot[q // K, q % K] = r * C + i
                if runs and runs[-1][0] == e and runs[-1][1] == r:
                    runs[-1][3] += 1
                else:
                    runs.append([e, r, i, 1])
                i += 1
        assert i == C
    table = sorted(range(len(runs)), key=lambda j: (runs[j][0], runs[j][1]))
    where = {j: a for a, j in enumerate(table)}
    seg = [tuple(runs[j]) for j in table]
    per_rank = [sum(1 for sg in seg if sg[1] == r and sg[1] != sg[0] // Bh) for r in range(R)]
    return dict(slot=slot, seg=seg, rank_seg_idx=[where[j] for j in range(len(runs))],
                replica_seg=[a for a, sg in enumerate(seg) if sg[1] != sg[0] // Bh],
                expert_seg_ptr=[next((a for a, sg in enumerate(seg) if sg[0] >= e), len(seg))
                                for e in range(E + 1)],
                rank_seg_ptr=[next((j for j in range(len(runs)) if runs[j][1] >= r), len(runs))
                              for r in range(R + 1)],
                max_rank_replicas=max(per_rank), unplaced=unplaced)


def check_capped_invariants(pl, R, S, E, K, B, idx):
    """Exact S*K per rank, each pair once, one expert per run, the static
    segment bound, replicas never on the home rank, the small-first home
    fill, and the cap: no rank above B replicas when every filler found a
    room and B >= 3."""
    check_home_first_invariants_basic(pl, R, S, E, K, idx)
    idx = np.asarray(idx).reshape(-1)
    C, Bh = S * K, E // R
    counts = np.bincount(idx, minlength=E)
    ns = pl["num_seg"]
    seg = np.asarray(pl["seg"])[:ns]
    kept = np.zeros(E, np.int64)
    per_rank = np.zeros(R, np.int64)
    for e, r, st, cnt in seg:
        if r == e // Bh:
            kept[e] += cnt
        else:
            per_rank[r] += 1
    assert int(per_rank.max()) == pl["max_rank_replicas"]
    for r in range(R):                  # smallest home experts are kept whole first
        order = sorted(range(r * Bh, (r + 1) * Bh), key=lambda e: (counts[e], e))
        room = C
        for e in order:
            assert kept[e] == min(counts[e], room), (r, e)
            room -= kept[e]
    if B >= 3 and pl["unplaced"] == 0:
        assert pl["max_rank_replicas"] <= B
    overflowing = int((kept < counts).sum())
    rooms = int(sum(1 for r in range(R) if kept[r * Bh:(r + 1) * Bh].sum() < C))
    assert pl["num_replicas"] <= max(0, overflowing + rooms - 1)


def check_home_first_invariants_basic(pl, R, S, E, K, idx):
    idx = np.asarray(idx).reshape(-1)
    NK, C, Bh = R * S * K, S * K, E // R
    slot = np.asarray(pl["slot"]).reshape(-1).astype(np.int64)
    src = np.asarray(pl["src_pair"]).astype(np.int64)
    assert np.array_equal(np.sort(slot), np.arange(NK))
    assert np.array_equal(src[slot], np.arange(NK))
    ns = pl["num_seg"]
    seg = np.asarray(pl["seg"])[:ns]
    assert ns <= E + R - 1
    assert np.array_equal(np.bincount(seg[:, 1], weights=seg[:, 3], minlength=R), np.full(R, C))
    e_of_p = idx[src]
    for e, r, st, cnt in seg:
        assert np.all(e_of_p[r * C + st: r * C + st + cnt] == e)
    assert len({(int(e), int(r)) for e, r, _, _ in seg}) == ns      # one run per (expert, rank)


def _check_capped_equal(pl, ref, what=""):
    _check_hf_equal(pl, ref, what)
    assert pl["max_rank_replicas"] == ref["max_rank_replicas"], what
    assert pl["unplaced"] == ref["unplaced"], what


def pin_capped(ora):
    gd = load_golden("example_d_capped.json")
    idx = np.array(gd["idx"], np.int32)
    for c in gd["cases"]:
        pl = ora.plan_capped(gd["R"], gd["S"], gd["E"], gd["K"], c["B"], idx)
        assert list(pl["counts"]) == gd["counts"]
        assert pl["maxvio"] == gd["maxvio_num"] / gd["maxvio_den"] - 1.0
        assert pl["slot"].tolist() == c["slot"], c["B"]
        assert pl["seg"][:pl["num_seg"]].tolist() == c["segments"], c["B"]
        assert list(pl["replica_seg"][:pl["num_replicas"]]) == c["replica_seg"]
        assert list(pl["rank_seg_ptr"]) == c["rank_seg_ptr"]
        assert list(pl["rank_seg_idx"]) == c["rank_seg_idx"]
        assert list(pl["expert_seg_ptr"]) == c["expert_seg_ptr"]
        assert pl["max_rank_replicas"] == c["max_rank_replicas"]
        assert pl["unplaced"] == c["unplaced"]
    rng = np.random.default_rng(43)
    for (R, S, E, K) in SMALL_SHAPES:
        for distinct, skew in ((True, 0.0), (True, 2.5), (False, 0.0), (False, 4.0)):
            idx = _random_idx(rng, R, S, E, K, distinct, skew)
            for B in (1, 2, 3, 4, E // R):
                pl = ora.plan_capped(R, S, E, K, B, idx)
                _check_capped_equal(pl, brute_capped(R, S, E, K, B, idx), str((R, S, E, K, B)))
                check_capped_invariants(pl, R, S, E, K, B, idx)
    import workloads
    for name, S in (("kimi_r64_e896_k16", 23), ("skew_r32_zipf1.5", 61), ("r8_e64_h2048", 97),
                    ("skew_r32_uniform", 40)):
        wl = workloads.reduced(workloads.WORKLOADS[name], S=S)
        idx, _ = workloads.routing(wl)
        for B in (3, 4, wl.E // wl.R):
            pl = ora.plan_capped(wl.R, wl.S, wl.E, wl.K, B, idx)
            check_capped_invariants(pl, wl.R, wl.S, wl.E, wl.K, B, idx)
            _check_capped_equal(pl, brute_capped(wl.R, wl.S, wl.E, wl.K, B, idx), name)


def pin_capped_closed_forms(ora):
    """Round-robin routing fills every rank from home: no replica at all.
    Adversarial routing (every token on experts 0..7, R = 32, E = 256, S*K =
    32768): rank 0 keeps 32768 pairs of expert 0 (ties go to the lower id),
    experts 1..7 overflow whole (131072 each) and expert 0 by 98304; the 31
    empty ranks are rooms of 32768; no overflow is below the largest room, so
    the stream gives experts 1..7 four ranks each (1-4, ..., 25-28) and expert
    0 ranks 29-31: 31 replicas, one per rank."""
    import workloads
    for (R, S, E, K) in [(4, 64, 16, 2), (8, 512, 64, 6), (2, 3, 6, 4)]:
        idx, _ = workloads.roundrobin_routing(R, S, E, K)
        for B in (1, 4):
            pl = ora.plan_capped(R, S, E, K, B, idx)
            assert pl["num_replicas"] == 0 and pl["max_rank_replicas"] == 0
            assert np.array_equal(pl["slot"], ora.plan(R, S, E, K, idx)["slot"])
    R, S, E, K = 32, 4096, 256, 8
    idx = np.argsort(-np.random.default_rng(0).standard_normal((R * S, K)), axis=1).astype(np.int32)
    pl = ora.plan_capped(R, S, E, K, 4, idx)
    assert pl["num_seg"] == 32 and pl["num_replicas"] == 31 and pl["max_rank_replicas"] == 1
    want = [(0, 0, 0, 32768)] + [(0, r, 0, 32768) for r in (29, 30, 31)]
    for e in range(1, 8):
        want += [(e, 4 * (e - 1) + 1 + j, 0, 32768) for j in range(4)]
    want.sort()
    assert [tuple(x) for x in pl["seg"][:32].tolist()] == want


ALL_PINS = [pin_bf16_widen, pin_bf16_rounding, pin_plan_golden, pin_plan_bruteforce,
            pin_plan_invariants, pin_closed_forms, pin_errors, pin_dispatch,
            pin_combine, pin_reduce, pin_combine_backward, pin_dispatch_backward,
            pin_prefetch_replicas, pin_home_first, pin_home_first_closed_forms,
            pin_capped, pin_capped_closed_forms]
