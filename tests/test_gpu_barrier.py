"""The device barrier between ranks (mep_rank_barrier) on one GPU, without two
kernels that wait on each other: "rank 0" is the barrier kernel; "rank 1"
arrives through a copy the host issues on an independent stream (after a
delay, or never).  All flag words are device memory.

* The host arrives after 50 ms: the kernel waits for it, then returns with a
  clean status, having stored its own arrival into every rank's array.
* Nobody arrives: the kernel gives up after the wait limit with
  MEP_ERR_TIMEOUT, and the context stays usable (a plan runs clean after).
* Epochs compare modulo 2^32; a NULL peer pointer is reported, not used.
"""
import time

import numpy as np
import pytest
import torch

import oracle
import parity
import token_dispatch_mep_b200 as mep

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _setup(R=2):
    flags = [torch.zeros(R, dtype=torch.int32, device=DEV) for _ in range(R)]
    table = torch.tensor([f.data_ptr() for f in flags], dtype=torch.int64, device=DEV)
    status = torch.zeros(1, dtype=torch.int32, device=DEV)
    return flags, table, status


def _timed_barrier(table, my_flags, rank, epoch, status, stream):
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(stream):
        e0.record(stream)
        mep.mep_rank_barrier(table, my_flags, rank, epoch, status)
        e1.record(stream)
    return e0, e1


def test_barrier_waits_for_the_peer_then_passes():
    old = mep.mep_get_wait_limit_ns()
    try:
        mep.mep_set_wait_limit_ns(5_000_000_000)
        flags, table, status = _setup()
        torch.cuda.synchronize()
        a, b = torch.cuda.Stream(DEV), torch.cuda.Stream(DEV)
        one = torch.ones(1, dtype=torch.int32).pin_memory()
        e0, e1 = _timed_barrier(table, flags[0], 0, 1, status, a)
        time.sleep(0.05)
        with torch.cuda.stream(b):                       # rank 1 arrives at rank 0's array
            flags[0][1:2].copy_(one, non_blocking=True)
        torch.cuda.synchronize()
        assert int(status.item()) == 0
        assert flags[0].tolist() == [1, 1]               # own arrival + the peer's
        assert flags[1].tolist() == [1, 0]               # rank 0 arrived at rank 1's array
        assert e0.elapsed_time(e1) >= 40.0               # it did wait for the peer
    finally:
        mep.mep_set_wait_limit_ns(old)


def test_barrier_times_out_and_the_context_stays_usable():
    old = mep.mep_get_wait_limit_ns()
    try:
        mep.mep_set_wait_limit_ns(20_000_000)            # 20 ms
        flags, table, status = _setup()
        torch.cuda.synchronize()
        a = torch.cuda.Stream(DEV)
        e0, e1 = _timed_barrier(table, flags[0], 0, 7, status, a)
        torch.cuda.synchronize()
        assert int(status.item()) == 6                   # MEP_ERR_TIMEOUT
        assert 15.0 <= e0.elapsed_time(e1) < 1000.0
    finally:
        mep.mep_set_wait_limit_ns(old)
    # the context is fine: a plan runs clean and right
    s = mep.Shape(4, 64, 16, 2)
    idx = np.random.default_rng(0).integers(0, 16, size=(256, 2)).astype(np.int32)
    plan = mep.Plan(s, DEV)
    mep.mep_plan(s, torch.from_numpy(idx).to(DEV), plan)
    assert mep.mep_read_status(plan) == 0
    parity.check_plan(plan.host(), oracle.get().plan(4, 64, 16, 2, idx), "after a timeout")


def test_epochs_compare_modulo_2_32_and_bad_pointers_are_reported():
    flags, table, status = _setup(R=3)
    for f in flags:
        f.fill_(-1)                                      # 2^32 - 1: epoch 0xFFFFFFFF reached
    mep.mep_rank_barrier(table, flags[1], 1, 0xFFFFFFFF, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    for f in flags:
        f.fill_(2)                                       # 2 is "after" 0xFFFFFFFF
    mep.mep_rank_barrier(table, flags[2], 2, 0xFFFFFFFF, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0 and flags[0].tolist()[2] == -1
    bad = table.clone()
    bad[0] = 0                                           # NULL peer array
    flags[1].fill_(9)
    mep.mep_rank_barrier(bad, flags[1], 1, 9, status)
    torch.cuda.synchronize()
    assert int(status.item()) == 5                       # reported, never stored through
