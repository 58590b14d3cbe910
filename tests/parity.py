"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (derived from the arithmetic, stated here once):
  * plan, counts, slots, segments, dispatch: bit-exact.
  * maxvio: bit-exact (both sides evaluate one binary64 quotient of the same
    two integers, minus 1).
  * combine: the oracle sums the K products in binary64 (exact to ~2^-53) and
    rounds once to bf16.  The kernel accumulates K float32 FMAs (one rounding
    each, error <= K * 2^-24 * sum|w*y|) and rounds to bf16.  Every element
    must be within 1 bf16 ulp of the oracle, except where cancellation makes
    the float32 bound itself exceed half a bf16 ulp; there the element must lie
    within half an ulp plus that bound of the exact sum.
  * replica-gradient reduce: the oracle sums in binary64; the kernel sums n
    float32 rows in ascending order (error <= n * 2^-24 * sum|G|).  Required:
    |gpu - exact| <= max(1e-6, n * 2^-24) * sum|G|.
"""
from __future__ import annotations

import numpy as np

U32 = 2.0 ** -24


def bf16_ordered(bits: np.ndarray) -> np.ndarray:
    """Map bf16 bit patterns to integers that are monotonic in value."""
    b = bits.astype(np.int64) & 0xFFFF
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    return ((bits.astype(np.uint32) & 0xFFFF) << 16).view(np.float32).astype(np.float64)


def bf16_ulp(v: np.ndarray) -> np.ndarray:
    """Spacing of the bf16 grid at |v| (normal range: 2^(floor(log2|v|) - 7))."""
    a = np.abs(v)
    e = np.floor(np.log2(np.where(a > 0, a, 1.0)))
    e = np.maximum(e, -126)
    return np.where(a > 0, 2.0 ** (e - 7), 2.0 ** -133)


def check_combine(gpu_bits, ora_bits, exact, absum, K, what=""):
    gpu_bits = np.asarray(gpu_bits).astype(np.uint16)
    ora_bits = np.asarray(ora_bits).astype(np.uint16)
    d = np.abs(bf16_ordered(gpu_bits) - bf16_ordered(ora_bits))
    bound = K * U32 * absum * (1 + 1e-9)
    gv = bf16_value(gpu_bits)
    ulp = np.maximum(bf16_ulp(gv), bf16_ulp(exact))
    cancel = bound > 0.5 * ulp
    ok = (d <= 1) | (cancel & (np.abs(gv - exact) <= 0.5 * ulp + bound))
    if not ok.all():
        bad = np.argwhere(~ok)[:5]
        raise AssertionError(f"combine {what}: {int((~ok).sum())} elements out of tolerance, "
                             f"first at {bad.tolist()}: gpu {gv[tuple(bad[0])]} "
                             f"oracle {bf16_value(ora_bits)[tuple(bad[0])]} exact {exact[tuple(bad[0])]}")
    return dict(bitexact=float((d == 0).mean()), max_ulp=int(d.max()) if d.size else 0)


def check_reduce(gpu, exact, absum, nseg_per_expert, what=""):
    gpu = np.asarray(gpu, dtype=np.float64)
    n = np.asarray(nseg_per_expert, dtype=np.float64).reshape(-1, 1)
    tol = np.maximum(1e-6, n * U32) * absum
    err = np.abs(gpu - exact)
    ok = err <= tol
    if not ok.all():
        bad = np.argwhere(~ok)[:5]
        raise AssertionError(f"reduce {what}: {int((~ok).sum())} out of tolerance at {bad.tolist()}")
    return dict(bitexact=float((gpu == exact.astype(np.float32)).mean()))


def check_plan(gpu: dict, ora: dict, what=""):
    """Bit-exact comparison of every plan field (segments up to num_seg)."""
    for k in ("counts", "expert_offset", "rank_seg_ptr", "expert_seg_ptr"):
        assert np.array_equal(np.asarray(gpu[k]), np.asarray(ora[k])), f"{what}: {k}"
    assert np.array_equal(np.asarray(gpu["slot"]).reshape(-1), np.asarray(ora["slot"]).reshape(-1)), \
        f"{what}: slot"
    assert np.array_equal(gpu["src_pair"], ora["src_pair"]), f"{what}: src_pair"
    for k in ("num_seg", "num_replicas", "max_count"):
        assert int(gpu[k]) == int(ora[k]), f"{what}: {k} {gpu[k]} vs {ora[k]}"
    ns, nr = ora["num_seg"], ora["num_replicas"]
    assert np.array_equal(np.asarray(gpu["seg"])[:ns], np.asarray(ora["seg"])[:ns]), f"{what}: seg"
    assert np.array_equal(np.asarray(gpu["replica_seg"])[:nr], np.asarray(ora["replica_seg"])[:nr]), \
        f"{what}: replica_seg"
    assert np.array_equal(np.asarray(gpu["rank_seg_idx"])[:ns], np.asarray(ora["rank_seg_idx"])[:ns]), \
        f"{what}: rank_seg_idx"
    assert gpu["maxvio"] == ora["maxvio"], f"{what}: maxvio {gpu['maxvio']!r} vs {ora['maxvio']!r}"
    assert gpu["status"] == 0, f"{what}: status {gpu['status']}"
