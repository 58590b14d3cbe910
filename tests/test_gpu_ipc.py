"""The exchange across processes: two EP ranks as two processes (a gloo
process group for the host-side exchange), their buffers shared by CUDA IPC
handles, each rank dispatching, combining and reducing its own share through
the peer mappings (``token_dispatch_mep_b200.ep``).

The test needs only one GPU: both processes use cuda:0 -- which CUDA IPC
supports -- and the ranks are ordered by host barriers only: no kernel of
one rank waits on a kernel of the other.  Every rank checks its own
receive buffer, combine output and home-expert gradients against the oracle
(bit-exact dispatch; combine within 1 bf16 ulp; reduce within the fp32
bound)."""
import dataclasses
import os
import queue
import socket
import sys
from datetime import timedelta

import pytest
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, schedule, q):
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import numpy as np
    import torch
    import torch.distributed as dist

    import oracle
    import parity
    import token_dispatch_mep_b200 as mep
    import workloads
    from token_dispatch_mep_b200 import ep

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    try:
        dev = torch.device("cuda", 0)
        torch.cuda.set_device(dev)
        u16 = lambda t: t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
        wl = dataclasses.replace(workloads.WORKLOADS["tiny_r4_e16"], name="two_ranks", R=world,
                                 S=300, H=256, grad=(96,))
        R, S, E, K, H, P, N, NK, SK = wl.R, wl.S, wl.E, wl.K, wl.H, wl.P, wl.N, wl.NK, wl.SK
        idx, w = workloads.routing(wl)              # same seed on every rank
        x = workloads.hidden(N, H, seed=1)
        y = workloads.expert_outputs(NK, H, seed=2)
        G = workloads.seg_grads(wl.seg_rows, P, seed=3)
        mine = slice(rank * S, (rank + 1) * S)

        grp = ep.ExchangeGroup(mep.Shape(R, S, E, K), H, P, device=dev, schedule=schedule,
                               B=4 if schedule == "capped" else 0)
        plan = grp.make_plan(torch.from_numpy(idx[mine].copy()))
        recv = grp.dispatch(x[mine].to(dev))
        grp.y.copy_(y[rank * SK:(rank + 1) * SK].to(dev))        # this rank's expert outputs
        out = torch.empty((S, H), dtype=torch.bfloat16, device=dev)
        grp.combine(torch.from_numpy(w[mine].copy()).to(dev), out)
        ph = plan.host()
        for j, (sidx, _, _, _) in enumerate(ep.local_segments(ph, rank)):
            grp.grads[j].copy_(G[sidx].to(dev))
        home = grp.reduce()
        grp.check()

        ora = oracle.get()
        if schedule == "contiguous":
            pl = ora.plan(R, S, E, K, idx)
        elif schedule == "home_first":
            pl = ora.plan_home_first(R, S, E, K, idx)
        else:
            pl = ora.plan_capped(R, S, E, K, 4, idx)
        res = {}
        # this rank's own pairs' slots and every table (the plan came from the
        # gathered histograms: the other ranks' slot rows are not this rank's)
        res["plan"] = bool(np.array_equal(ph["slot"][mine], pl["slot"][mine]) and
                           grp.gathered_bytes == R * E * 4)
        parity.check_plan(dict(ph, slot=pl["slot"], src_pair=pl["src_pair"]), pl, f"rank {rank}")
        want = ora.dispatch(K, pl["src_pair"], u16(x))[rank * SK:(rank + 1) * SK]
        res["dispatch"] = bool(np.array_equal(u16(recv), want))
        ob, ex, ab = ora.combine(pl["slot"], w, u16(y))
        try:
            parity.check_combine(u16(out), ob[mine], ex[mine], ab[mine], K, f"rank {rank}")
            res["combine"] = True
        except AssertionError as e:
            res["combine"] = str(e)
        hexact, habs = ora.reduce(pl["expert_seg_ptr"], G.numpy())
        B = E // R
        hs = slice(rank * B, (rank + 1) * B)
        try:
            parity.check_reduce(home[:, :P].cpu().numpy(), hexact[hs], habs[hs],
                                np.diff(pl["expert_seg_ptr"])[hs], f"rank {rank}")
            res["reduce"] = True
        except AssertionError as e:
            res["reduce"] = str(e)
        res["replicas"] = int(ph["num_replicas"])
        grp.close()
        q.put((rank, res))
    except Exception as e:  # report instead of leaving the parent waiting
        q.put((rank, f"error: {e!r}"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("schedule", ["contiguous", "home_first", "capped"])
def test_two_process_exchange_over_ipc(schedule):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, schedule, q)) for r in range(world)]
    for p in procs:
        p.start()
    results = {}
    try:
        for _ in range(world):
            r, res = q.get(timeout=240)
            results[r] = res
    except queue.Empty:
        pass
    finally:
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
                p.join()
    assert set(results) == set(range(world)), results
    for r, res in results.items():
        assert isinstance(res, dict), f"rank {r}: {res}"
        for k in ("plan", "dispatch", "combine", "reduce"):
            assert res[k] is True, f"rank {r} {k}: {res[k]}"
    assert results[0]["replicas"] == results[1]["replicas"]
