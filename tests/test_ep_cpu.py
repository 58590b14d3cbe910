"""The host orchestration of the exchange (token_dispatch_mep_b200.ep) on two
gloo ranks on the CPU, with the library's IPC and kernel calls replaced by
recording fakes: which buffers each rank exports, which peer handles it
opens and where their addresses go in the pointer arrays, the token range
and tables each step passes to the kernels, the plan's one exchange (the
R x E per-rank histograms, gathered rank by rank; the ids stay local), and
that every mapping is closed again."""
import os
import socket
import sys
from datetime import timedelta

import numpy as np
import pytest
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank(rank, world, port, sync, q):
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import token_dispatch_mep_b200 as mep
    from token_dispatch_mep_b200 import ep

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=timedelta(seconds=60))
    log = []
    try:
        def fake_export(t):
            h = mep.IpcHandle()
            h.handle[0], h.handle[1] = rank, len([x for x in log if x[0] == "export"])
            h.offset, h.bytes = 256, t.numel() * t.element_size()
            log.append(("export", t.data_ptr()))
            return h

        def fake_open(h, device):
            log.append(("open", h.handle[0], h.handle[1]))
            return 0x10000000 * (h.handle[0] + 1) + 0x1000 * h.handle[1] + h.offset

        ep.mep_ipc_export = fake_export
        ep.mep_ipc_open = fake_open
        ep.mep_ipc_close = lambda h, p, d: log.append(("close", h.handle[0], h.handle[1], p))
        ep.mep_rank_histogram = lambda s, idx, plan: torch.bincount(
            idx.reshape(-1).long(), minlength=s.E).to(torch.int32)
        ep.mep_plan_rank = lambda s, sched, r, idx, counts, plan, B: log.append(
            ("plan", sched, r, idx.clone(), counts.clone()))
        ep.mep_dispatch_ranked_tokens = lambda s, H, plan, b, x, tab, token_count: log.append(
            ("dispatch", b, token_count, tab.tolist(), x.shape[0]))
        ep.mep_combine_ranked_tokens = lambda s, H, plan, b, tab, w, out, token_count: log.append(
            ("combine", b, token_count, tab.tolist()))
        ep.mep_reduce_replica_grads_ranked = lambda s, plan, P, hr, tab, rows, home: log.append(
            ("reduce", hr, rows, tab.tolist()))
        ep.mep_rank_barrier = lambda tab, flags, r, epoch, status: log.append(
            ("device_barrier", r, epoch, tab.tolist(), flags.data_ptr()))
        real_barrier = ep.dist.barrier

        def counting_barrier(*a, **k):
            log.append(("host_barrier",))
            return real_barrier(*a, **k)
        ep.dist.barrier = counting_barrier

        R, S, E, K, H, P = world, 5, 4, 2, 16, 12
        g = ep.ExchangeGroup(mep.Shape(R, S, E, K), H, P, device="cpu", sync=sync)
        idx_local = torch.full((S, K), rank, dtype=torch.int32)
        g.make_plan(idx_local)
        gathered = g.gathered_bytes
        g.dispatch(torch.zeros((S, H), dtype=torch.bfloat16))
        g.combine(torch.zeros((S, K)), torch.zeros((S, H), dtype=torch.bfloat16))
        g.reduce()
        tables = (g.recv_table.tolist(), g.y_table.tolist(), g.grad_table.tolist())
        own = (g.recv.data_ptr(), g.y.data_ptr(), g.grads.data_ptr())
        if sync == "device":
            tables += (g.flag_table.tolist(),)
            own += (g.flags.data_ptr(),)
        rows = g.grads.shape[0]
        g.close()
        q.put((rank, dict(log=[(e[0],) + tuple(x for x in e[1:] if not isinstance(x, torch.Tensor))
                               for e in log],
                          plan_in=[(e[1], e[2], e[3].numpy(), e[4].numpy())
                                   for e in log if e[0] == "plan"],
                          gathered=gathered, tables=tables, own=own, rows=rows, S=S, E=E,
                          K=K)))
    except Exception as e:
        q.put((rank, f"error: {e!r}"))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("sync", ["host", "device"])
def test_exchange_orchestration_on_gloo_ranks(sync):
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, sync, q)) for r in range(world)]
    for p in procs:
        p.start()
    out = dict(q.get(timeout=120) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, res in out.items():
        assert isinstance(res, dict), res
        peer = 1 - rank
        kinds = [e[0] for e in res["log"]]
        nbuf = 3 if sync == "host" else 4            # + the flag array
        assert kinds.count("export") == nbuf and kinds.count("open") == nbuf
        assert kinds.count("close") == nbuf
        # every peer handle opened is the peer's, once per buffer kind
        assert sorted((e[1], e[2]) for e in res["log"] if e[0] == "open") == \
            [(peer, b) for b in range(nbuf)]
        # pointer arrays: own buffer at the own index, the mapped peer buffer at the peer's
        for kind, (tab, own) in enumerate(zip(res["tables"], res["own"])):
            assert tab[rank] == own
            assert tab[peer] == 0x10000000 * (peer + 1) + 0x1000 * kind + 256
        # the plan's one exchange: every rank's histogram, row r from rank r
        # (rank r routes all its S*K pairs to expert r); the ids stay local
        (sched, prank, pidx, counts) = res["plan_in"][0]
        S, E, K = res["S"], res["E"], res["K"]
        assert sched == "contiguous" and prank == rank
        assert np.array_equal(pidx, np.full((S, K), rank))
        want = np.zeros((world, E), np.int32)
        want[0, 0] = want[1, 1] = S * K
        assert np.array_equal(counts, want)
        assert res["gathered"] == world * E * 4
        # each step gets this rank's token range and the right table
        (d,) = [e for e in res["log"] if e[0] == "dispatch"]
        assert d[1:3] == (rank * res["S"], res["S"]) and list(d[3]) == res["tables"][0]
        (c,) = [e for e in res["log"] if e[0] == "combine"]
        assert c[1:3] == (rank * res["S"], res["S"]) and list(c[3]) == res["tables"][1]
        (r,) = [e for e in res["log"] if e[0] == "reduce"]
        assert r[1] == rank and r[2] == res["rows"] and list(r[3]) == res["tables"][2]
        # mappings are closed last, after every step
        assert kinds.index("close") > kinds.index("reduce")
        # ordering between the phases: a host barrier before and after each
        # exchange kernel, or the device barrier with epochs 1..6 and no host
        # barrier until close
        steps = [k for k in kinds if k in ("dispatch", "combine", "reduce", "host_barrier",
                                           "device_barrier")]
        steps = steps[:steps.index("reduce") + 2]
        bar = "host_barrier" if sync == "host" else "device_barrier"
        assert steps == [bar, "dispatch", bar, bar, "combine", bar, bar, "reduce", bar]
        if sync == "device":
            dev = [e for e in res["log"] if e[0] == "device_barrier"]
            assert [e[2] for e in dev] == [1, 2, 3, 4, 5, 6]
            assert all(e[1] == rank and list(e[3]) == res["tables"][3] and e[4] == res["own"][3]
                       for e in dev)
            assert "host_barrier" not in kinds[kinds.index("dispatch") - 1:kinds.index("reduce") + 2]
