"""Combine and replica-gradient reduce are exact where a float32 running sum is not.

The oracle adds the terms of every output in binary64, in the method's fixed
order (k ascending for the weighted combine of the top-K expert outputs back
to token order; segment index ascending for the sum of an expert's duplicate
gradients into its home copy -- MoonEP release page, "Why expert parallelism
is needed" and "How MoonEP works"), and rounds once.  These tests feed both
sides inputs chosen to break a float32 accumulator:

* heavy cancellation: pairs of large terms that cancel up to a small
  remainder, plus small terms -- a float32 chain of fused multiply-adds is
  off by many bf16 units here (checked on the host, so the case has teeth);
* special values: signed zeros, bf16 and float32 subnormals, the largest
  finite values, infinities and NaNs, in expert outputs, weights and
  gradients.

The bar is bit-exact equality with the oracle (NaN matching NaN).
"""
import numpy as np
import pytest
import torch

import oracle
import parity
import token_dispatch_mep_b200 as mep

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


@pytest.fixture(scope="module")
def ora():
    return oracle.get()


def _u16(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def _bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bit patterns, round to nearest even (finite inputs)."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def _bits_tensor(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits.astype(np.uint16).view(np.int16)).view(torch.bfloat16)


def _plan(R, S, E, K, seed=0):
    """A plan whose tokens each pick K distinct experts."""
    rng = np.random.default_rng(seed)
    idx = np.argsort(rng.random((R * S, E)), axis=1)[:, :K].astype(np.int32)
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    return s, idx, plan


def _combine_both(ora, s, plan, idx, y_pairs_bits, w):
    """GPU combine and oracle combine of per-(token, k) rows y_pairs_bits
    [N, K, H] placed at their slots."""
    N, K, H = y_pairs_bits.shape
    pl = ora.plan(s.R, s.S, s.E, s.K, idx)
    y_rows = np.empty((s.NK, H), dtype=np.uint16)
    y_rows[pl["slot"].reshape(-1)] = y_pairs_bits.reshape(N * K, H)
    out = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_combine(s, H, plan, _bits_tensor(y_rows).to(DEV), torch.from_numpy(w).to(DEV), out)
    assert mep.mep_read_status(plan) == 0
    ob, exact, _ = ora.combine(pl["slot"], w, y_rows)
    return _u16(out), ob, exact, pl, y_rows


def _f32_fma_chain_bf16(w, y_pairs_bits, ora):
    """What a float32 accumulator (one fused multiply-add per term, k order)
    would give, rounded to bf16: host emulation, test side only."""
    N, K, H = y_pairs_bits.shape
    y = (y_pairs_bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    acc = np.zeros((N, H), dtype=np.float32)
    for k in range(K):
        acc = (w[:, k:k + 1].astype(np.float64) * y[:, k, :] + acc.astype(np.float64)).astype(np.float32)
    return np.vectorize(ora.f64_to_bf16, otypes=[np.uint16])(acc.astype(np.float64))


@pytest.mark.parametrize("H", [256, 1032])
def test_combine_under_cancellation_is_bit_exact(ora, H):
    R, S, E, K = 2, 32, 8, 8
    s, idx, plan = _plan(R, S, E, K)
    N = s.N
    rng = np.random.default_rng(1)
    big = rng.uniform(1e4, 2e4, size=(N, H)).astype(np.float32)
    small = rng.standard_normal((N, K, H)).astype(np.float32) * 1e-2
    y = small.copy()
    y[:, 0, :] = big
    y[:, 1, :] = -big                        # cancels term 0 up to the weights' difference
    w = rng.uniform(0.05, 0.2, size=(N, K)).astype(np.float32)
    w[:, 1] = np.nextafter(w[:, 0], np.float32(1.0))   # w1 = w0 + 1 ulp: a tiny remainder
    ybits = _bf16_bits(y)
    got, ob, exact, _, _ = _combine_both(ora, s, plan, idx, ybits, w)
    parity.check_combine(got, ob, exact, what=f"cancellation H={H}")
    # the case is meaningful: a float32 chain misses the oracle on many elements
    f32 = _f32_fma_chain_bf16(w, ybits, ora)
    d = np.abs(parity.bf16_ordered(f32) - parity.bf16_ordered(ob))
    assert (d > 1).mean() > 0.05, (d > 1).mean()


SPECIAL_BF16 = np.array([0x0000, 0x8000, 0x0001, 0x8001, 0x007F, 0x0080, 0x7F7F, 0xFF7F,
                         0x7F80, 0xFF80, 0x7FC0, 0xFFC0, 0x3F80, 0xBF80, 0x0040], dtype=np.uint16)
SPECIAL_F32 = np.array([0.0, -0.0, 1e-45, -1e-45, 1.17549435e-38, 3.4028235e38, -3.4028235e38,
                        np.inf, -np.inf, np.nan, 1.0, 0.5, 2.0 ** -100], dtype=np.float32)


def _specials(rng, shape, table, frac):
    pick = rng.random(shape) < frac
    return pick, table[rng.integers(0, len(table), size=shape)]


@pytest.mark.parametrize("frac", [0.002, 0.2])
def test_combine_special_values_are_bit_exact(ora, frac):
    R, S, E, K, H = 2, 48, 16, 6, 520
    s, idx, plan = _plan(R, S, E, K, seed=2)
    N = s.N
    rng = np.random.default_rng(3)
    ybits = _bf16_bits(rng.standard_normal((N, K, H)).astype(np.float32))
    pick, sp = _specials(rng, ybits.shape, SPECIAL_BF16, frac)
    ybits = np.where(pick, sp, ybits).astype(np.uint16)
    w = rng.random((N, K)).astype(np.float32)
    wpick, wsp = _specials(rng, w.shape, SPECIAL_F32, frac)
    w = np.where(wpick, wsp, w).astype(np.float32)
    got, ob, exact, _, _ = _combine_both(ora, s, plan, idx, ybits, w)
    parity.check_combine(got, ob, exact, what=f"special values {frac}")


def test_dispatch_backward_special_values_and_cancellation(ora):
    R, S, E, K, H = 2, 40, 8, 8, 264
    s, idx, plan = _plan(R, S, E, K, seed=4)
    N = s.N
    rng = np.random.default_rng(5)
    g = rng.standard_normal((N, K, H)).astype(np.float32) * 1e-2
    g[:, 0, :] = 300.0
    g[:, 3, :] = -300.0
    gbits = _bf16_bits(g)
    pick, sp = _specials(rng, gbits.shape, SPECIAL_BF16, 0.01)
    gbits = np.where(pick, sp, gbits).astype(np.uint16)
    pl = ora.plan(R, S, E, K, idx)
    rows = np.empty((s.NK, H), dtype=np.uint16)
    rows[pl["slot"].reshape(-1)] = gbits.reshape(N * K, H)
    gx = torch.empty((N, H), dtype=torch.bfloat16, device=DEV)
    mep.mep_dispatch_backward(s, H, plan, _bits_tensor(rows).to(DEV), gx)
    assert mep.mep_read_status(plan) == 0
    want, exact, _ = ora.dispatch_backward(pl["slot"], rows)
    parity.check_combine(_u16(gx), want, exact, what="dispatch backward")


@pytest.mark.parametrize("P", [1000, 1024])
def test_reduce_under_cancellation_and_special_values(ora, P):
    # every token on expert 0: it spans all four ranks (four segments)
    R, S, E, K = 4, 16, 4, 1
    s = mep.Shape(R, S, E, K)
    idx = np.zeros((R * S, K), dtype=np.int32)
    idx[::7, 0] = 2
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    pl = ora.plan(R, S, E, K, idx)
    rng = np.random.default_rng(6)
    G = rng.standard_normal((s.seg_rows, P)).astype(np.float32)
    # expert 0's four segments are rows 0..3: a large row, a small one, the
    # large row negated, a smaller one -- a float32 running sum loses the
    # small row's low bits to the large one, the binary64 sum keeps them
    G[0] = (1e8 * (1.0 + rng.random(P))).astype(np.float32)
    G[2] = -G[0]
    G[3] *= 1e-3
    pick, sp = _specials(rng, G.shape, SPECIAL_F32, 0.01)
    G = np.where(pick, sp, G).astype(np.float32)
    home = torch.empty((E, P), dtype=torch.float32, device=DEV)
    mep.mep_reduce_replica_grads(s, plan, P, torch.from_numpy(G).to(DEV), home)
    assert mep.mep_read_status(plan) == 0
    exact, absum = ora.reduce(pl["expert_seg_ptr"], G)
    parity.check_reduce(home.cpu().numpy(), exact, absum, what=f"reduce P={P}")
    # a float32 running sum misses the oracle rounded to float32 somewhere
    e0 = pl["expert_seg_ptr"]
    f32 = np.zeros(P, dtype=np.float32)
    for r in range(e0[0], e0[1]):
        f32 = (f32 + G[r]).astype(np.float32)
    fin = np.isfinite(exact[0])
    assert (f32[fin] != exact[0][fin].astype(np.float32)).any()
