"""Comparison helpers for the GPU-vs-oracle parity tests.

Tolerances (derived from the arithmetic, stated here once):
  * plan, counts, slots, segments, dispatch: bit-exact.
  * maxvio: bit-exact (both sides evaluate one binary64 quotient of the same
    two integers, minus 1).
  * combine (and the backward of dispatch, the same sum with unit weights):
    bit-exact.  The oracle adds the K products w*y in binary64, k ascending,
    and rounds the sum once to bf16 (nearest-even).  Every product of a
    float32 weight and a bf16 value is exact in binary64, so the kernel's
    k-ordered chain of binary64 fused multiply-adds performs the same
    roundings, and its one rounding to bf16 gives the same bits.  This meets
    the contract's "within 1 bf16 ulp" everywhere, cancellation included.
    NaN outputs must be NaN on both sides (payloads may differ).
  * replica-gradient reduce: bit-exact against the oracle's ascending binary64
    sum rounded once to float32 (the kernel sums in binary64 in the same
    order), hence within 2^-24 relative of the binary64 sum -- inside the
    contract's 1e-6 relative, cancellation included.
"""
from __future__ import annotations

import numpy as np


def bf16_ordered(bits: np.ndarray) -> np.ndarray:
    """Map bf16 bit patterns to integers that are monotonic in value."""
    b = bits.astype(np.int64) & 0xFFFF
    mag = b & 0x7FFF
    return np.where(b & 0x8000, -mag, mag)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    return ((bits.astype(np.uint32) & 0xFFFF) << 16).view(np.float32).astype(np.float64)


def _bf16_nan(bits: np.ndarray) -> np.ndarray:
    b = bits.astype(np.uint32) & 0x7FFF
    return b > 0x7F80


def check_combine(gpu_bits, ora_bits, exact=None, absum=None, K=None, what=""):
    """Bit-exact comparison of bf16 outputs with the oracle's (NaN matches any
    NaN).  `exact`, `absum` and `K` are accepted for the report only."""
    gpu_bits = np.asarray(gpu_bits).astype(np.uint16)
    ora_bits = np.asarray(ora_bits).astype(np.uint16)
    assert gpu_bits.shape == ora_bits.shape, (what, gpu_bits.shape, ora_bits.shape)
    gn, on = _bf16_nan(gpu_bits), _bf16_nan(ora_bits)
    same = (gpu_bits == ora_bits) | (gn & on)
    if not same.all():
        bad = np.argwhere(~same)
        d = np.abs(bf16_ordered(gpu_bits) - bf16_ordered(ora_bits))[~same]
        first = tuple(bad[0])
        msg = (f"combine {what}: {len(bad)} of {same.size} elements differ from the oracle "
               f"(largest distance {int(d.max())} bf16 ulp), first at {list(first)}: "
               f"gpu {bf16_value(gpu_bits)[first]} oracle {bf16_value(ora_bits)[first]}")
        if exact is not None:
            msg += f" exact {np.asarray(exact)[first]}"
        raise AssertionError(msg)
    return dict(bitexact=1.0, max_ulp=0, n=int(same.size))


def check_reduce(gpu, exact, absum=None, nseg_per_expert=None, what=""):
    """Bit-exact comparison of float32 home gradients with the oracle's binary64
    sums rounded once to float32 (NaN matches any NaN); reports the largest
    relative distance from the binary64 sums."""
    gpu = np.ascontiguousarray(np.asarray(gpu, dtype=np.float32))
    exact = np.asarray(exact, dtype=np.float64)
    want = exact.astype(np.float32)                 # IEEE nearest-even
    assert gpu.shape == want.shape, (what, gpu.shape, want.shape)
    gb, wb = gpu.view(np.uint32), np.ascontiguousarray(want).view(np.uint32)
    same = (gb == wb) | (np.isnan(gpu) & np.isnan(want))
    if not same.all():
        bad = np.argwhere(~same)
        first = tuple(bad[0])
        raise AssertionError(f"reduce {what}: {len(bad)} of {same.size} elements differ from "
                             f"the oracle rounded to float32, first at {list(first)}: "
                             f"gpu {gpu[first]!r} oracle {want[first]!r} exact {exact[first]!r}")
    # relative bound of one rounding, in float32's normal range
    fin = np.isfinite(exact) & (np.abs(exact) >= 2.0 ** -126) & np.isfinite(gpu)
    rel = float(np.max(np.abs(gpu[fin] - exact[fin]) / np.abs(exact[fin]))) if fin.any() else 0.0
    assert rel <= 2.0 ** -24, (what, rel)
    return dict(bitexact=1.0, max_rel=rel, n=int(same.size))


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
