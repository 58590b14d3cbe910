"""Multi-rank pieces on CPU with world-size-2 gloo process groups.

* bench.py under torchrun runs one independent replica per GPU and reports
  the whole-job rate from the slowest rank's time: max_over_ranks must give
  every rank the same maximum, and whole_job_rate must count every rank's
  tokens once.
* The plan shards with a single exchange: if each rank holds only its own
  tokens' top-K ids, one all-gather of the R x E per-rank histograms is enough
  for every rank to place its own pairs exactly where the single-device plan
  places them (checked against the oracle).  This is the exchange the
  multi-GPU form of the path needs before its dispatch.
* The reference arm prints only on rank 0.
"""
import io
import os
import socket
import sys
from contextlib import redirect_stdout
from datetime import timedelta

import numpy as np
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, case, q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        q.put((rank, CASES[case](rank, world)))
    except Exception as e:  # report instead of hanging the parent
        q.put((rank, f"error: {e!r}"))
    finally:
        dist.destroy_process_group()


def _case_max(rank, world):
    import torch

    import bench
    ms = [1.25, 3.5][rank]
    m = bench.max_over_ranks(ms, world, torch.device("cpu"))
    return m, bench.whole_job_rate(1000, world, m)


def _case_sharded_plan(rank, world):
    import torch
    import torch.distributed as dist

    import oracle
    R, S, E, K = world, 300, 16, 4
    rng = np.random.default_rng(42)
    logits = rng.standard_normal((R * S, E)) - 1.2 * np.log(np.arange(1, E + 1))
    idx = np.argsort(-logits, axis=1, kind="stable")[:, :K].astype(np.int32)
    mine = idx[rank * S:(rank + 1) * S].reshape(-1)            # this rank's pairs only
    hist = torch.from_numpy(np.bincount(mine, minlength=E).astype(np.int64))
    hists = [torch.zeros(E, dtype=torch.int64) for _ in range(world)]
    dist.all_gather(hists, hist)                                 # the one exchange
    H = torch.stack(hists).numpy()
    T = H.sum(axis=0)
    off = np.concatenate([[0], np.cumsum(T)[:-1]])
    base = off + H[:rank].sum(axis=0)
    # stable rank of each own pair among own pairs with the same expert
    order = np.argsort(mine, kind="stable")
    first = np.searchsorted(mine[order], np.arange(E))
    local = np.empty_like(mine)
    local[order] = np.arange(mine.size) - first[mine[order]]
    slots = base[mine] + local
    want = oracle.get().plan(R, S, E, K, idx)["slot"][rank * S:(rank + 1) * S].reshape(-1)
    return bool(np.array_equal(slots, want)), int(T.sum())


def _case_gather_ids(rank, world):
    """ep.gather_router_ids over gloo: every rank ends with all ranks' ids in
    global token order, and the oracle plan of them gives each rank a
    segment list (ep.local_segments) that covers its S*K slots in order."""
    import torch

    import oracle
    from token_dispatch_mep_b200 import ep
    R, S, E, K = world, 257, 16, 3
    rng = np.random.default_rng(7)
    logits = rng.standard_normal((R * S, E)) - 1.1 * np.log(np.arange(1, E + 1))
    idx = np.argsort(-logits, axis=1, kind="stable")[:, :K].astype(np.int32)
    got = ep.gather_router_ids(torch.from_numpy(idx[rank * S:(rank + 1) * S].copy()))
    same = bool(np.array_equal(got.numpy(), idx))
    covered = []
    for plan in (oracle.get().plan(R, S, E, K, idx), oracle.get().plan_home_first(R, S, E, K, idx)):
        segs = ep.local_segments(plan, rank)
        starts = [st for _, _, st, _ in segs]
        experts = [e for _, e, _, _ in segs]
        covered.append((sum(c for _, _, _, c in segs) == S * K,
                        starts == sorted(starts) and (not starts or starts[0] == 0),
                        len(segs) <= ep.max_local_segments(type("Sh", (), dict(E=E, SK=S * K))()),
                        len(set(experts)) == len(experts)))
    errors = []
    for shape, sched in (((3, 4, 6, 2), "contiguous"), ((2, 4, 6, 2), "fastest")):
        try:
            ep.ExchangeGroup(shape, 8, 0, device="cpu", schedule=sched)
            errors.append(None)
        except ValueError as e:           # rejected before any buffer is made
            errors.append(type(e).__name__)
    return same, covered, errors


CASES = {"max": _case_max, "sharded_plan": _case_sharded_plan, "gather_ids": _case_gather_ids}


def _run(case, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, case, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return out


def test_max_over_ranks_and_whole_job_rate():
    out = _run("max")
    assert out[0] == out[1], out
    m, rate = out[0]
    assert m == 3.5
    assert abs(rate - 2 * 1000 / 3.5e-3) < 1e-6


def test_sharded_plan_needs_one_histogram_allgather():
    out = _run("sharded_plan")
    for rank in (0, 1):
        ok, total = out[rank]
        assert ok is True, out
        assert total == 2 * 300 * 4


def test_reference_arm_prints_on_rank_zero_only(monkeypatch):
    sys.path.insert(0, ROOT)
    import bench
    monkeypatch.setenv("RANK", "1")
    args = type("A", (), dict(workload="tiny_r4_e16", steps=1, warmup=0, gpus=2))()
    buf = io.StringIO()
    with redirect_stdout(buf):
        bench.run_reference(args)
    assert buf.getvalue() == ""


def test_router_id_gather_and_local_segment_lists():
    out = _run("gather_ids")
    for rank in (0, 1):
        same, covered, errors = out[rank]
        assert same is True, out
        for flags in covered:                   # contiguous, home-first
            assert all(flags), (rank, flags)
        assert errors == ["ValueError", "ValueError"], errors  # R != world size; unknown schedule
