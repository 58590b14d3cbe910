"""The whole step -- plan, dispatch, combine, replica-gradient reduce, replica
weight prefetch -- is captured once in a CUDA graph and replayed on new
routing and new data written into the same static buffers, without any host
synchronisation or re-sizing ("Why this matters to engineers": fixed buffer
shapes, no host round trip per layer).  Each replay is checked against the
oracle."""
import numpy as np
import pytest
import torch

import oracle
import parity
import token_dispatch_mep_b200 as mep
import workloads

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _u16(t):
    return t.contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def test_step_replays_from_a_cuda_graph():
    ora = oracle.get()
    wl = workloads.reduced(workloads.WORKLOADS["kimi_r64_e896_k16"], S=37, H=520, P=1028)
    R, S, E, K, H, P, N, NK = wl.R, wl.S, wl.E, wl.K, wl.H, wl.P, wl.N, wl.NK
    s = mep.Shape(R, S, E, K)
    dev = torch.device(DEV)
    idx = torch.empty((N, K), dtype=torch.int32, device=dev)
    w = torch.empty((N, K), dtype=torch.float32, device=dev)
    x = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
    y = torch.empty((NK, H), dtype=torch.bfloat16, device=dev)
    G = torch.empty((wl.seg_rows, P), dtype=torch.float32, device=dev)
    Wh = torch.empty((E, P), dtype=torch.float32, device=dev)
    plan = mep.Plan(s, dev)
    buf = torch.empty((NK, H), dtype=torch.bfloat16, device=dev)
    out = torch.empty((N, H), dtype=torch.bfloat16, device=dev)
    home = torch.empty((E, P), dtype=torch.float32, device=dev)
    wrep = torch.empty((wl.seg_rows, P), dtype=torch.float32, device=dev)

    def load(seed):
        i, ww = workloads.routing(wl, seed=seed)
        idx.copy_(torch.from_numpy(i))
        w.copy_(torch.from_numpy(ww))
        x.copy_(workloads.hidden(N, H, seed=seed + 1))
        y.copy_(workloads.expert_outputs(NK, H, seed=seed + 2))
        G.copy_(workloads.seg_grads(wl.seg_rows, P, seed=seed + 3))
        Wh.copy_(workloads.seg_grads(E, P, seed=seed + 4))
        return i, ww

    def step():
        mep.mep_plan(s, idx, plan)
        mep.mep_dispatch(s, H, plan, x, buf)
        mep.mep_combine(s, H, plan, y, w, out)
        mep.mep_reduce_replica_grads(s, plan, P, G, home)
        mep.mep_prefetch_replica_weights(s, plan, Wh, wrep)

    load(100)
    side = torch.cuda.Stream(dev)
    side.wait_stream(torch.cuda.current_stream(dev))
    with torch.cuda.stream(side):
        step()                                   # warm-up outside capture
    torch.cuda.current_stream(dev).wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        step()

    for seed in (0, 5):
        i_h, w_h = load(seed)
        graph.replay()
        torch.cuda.synchronize()
        assert mep.mep_read_status(plan) == 0
        pl = ora.plan(R, S, E, K, i_h)
        parity.check_plan(plan.host(), pl, f"graph replay {seed}")
        assert np.array_equal(_u16(buf), ora.dispatch(K, pl["src_pair"], _u16(x)))
        ob, ex, ab = ora.combine(pl["slot"], w_h, _u16(y))
        parity.check_combine(_u16(out), ob, ex, ab, K, f"graph replay {seed}")
        hx, ha = ora.reduce(pl["expert_seg_ptr"], G.cpu().numpy())
        parity.check_reduce(home.cpu().numpy(), hx, ha, np.diff(pl["expert_seg_ptr"]))
        nr = pl["num_replicas"]
        assert np.array_equal(wrep[:nr].cpu().numpy(), ora.prefetch_replicas(pl, Wh.cpu().numpy()))
