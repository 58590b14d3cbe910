"""The plan at the ABI's size limit: R*S*K just under 2^31 pairs, E = R = 1024,
K = 16 (64-bit row addressing, int32 slots at their limit, warps whose ranges
overflow their shared-memory id buffers).

The oracle would need tens of GB of host memory here, so the test checks, on
the device and in chunks, properties that together determine the
contiguous-cut plan uniquely: T_e are the histogram of the ids; slot is a
bijection onto [0, R*S*K) with src_pair its inverse; slots are ordered by
expert and, inside an expert, by pair index (the stable sort); the segment
table cuts the sorted slots at every rank boundary and expert change, with
exactly S*K slots per rank."""
import numpy as np
import pytest
import torch

import token_dispatch_mep_b200 as mep

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def test_plan_at_int32_limit():
    R, S, E, K = 1024, 131071, 1024, 16
    NK, SK = R * S * K, S * K
    assert NK < 2 ** 31
    dev = torch.device(DEV)
    g = torch.Generator(device=dev)
    g.manual_seed(5)
    # skewed ids: squares of uniforms put more mass on low experts
    u = torch.rand(NK, generator=g, device=dev)
    idx = (u * u * E).to(torch.int32).clamp_(0, E - 1)
    del u
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, dev)
    mep.mep_plan(s, idx, plan)
    assert mep.mep_read_status(plan) == 0
    counts = torch.bincount(idx.long(), minlength=E)
    assert torch.equal(plan.counts.long(), counts)
    off = torch.cumsum(counts, 0) - counts
    assert torch.equal(plan.expert_offset[:E].long(), off)
    slot = plan.slot.view(-1)
    src = plan.src_pair
    step = 1 << 27
    prev_e, prev_q = -1, -1
    for c0 in range(0, NK, step):
        c1 = min(NK, c0 + step)
        # src_pair is the inverse of slot
        sp = src[c0:c1].long()
        assert bool(((sp >= 0) & (sp < NK)).all())
        assert torch.equal(slot.index_select(0, sp).long(),
                           torch.arange(c0, c1, device=dev, dtype=torch.long))
        # expert order, stable inside an expert
        ex = idx.index_select(0, sp).long()
        assert int(ex[0]) >= prev_e and bool((ex[1:] >= ex[:-1]).all())
        same = ex[1:] == ex[:-1]
        assert bool((sp[1:][same] > sp[:-1][same]).all())
        if int(ex[0]) == prev_e:
            assert int(sp[0]) > prev_q
        prev_e, prev_q = int(ex[-1]), int(sp[-1])
        del sp, ex, same
    # every slot is the image of exactly one pair: slot values are a permutation
    seen = torch.zeros(NK, dtype=torch.bool, device=dev)
    for c0 in range(0, NK, step):
        seen[slot[c0:min(NK, c0 + step)].long()] = True
    assert bool(seen.all())
    del seen
    # segments: rank cuts and expert changes, S*K slots per rank
    h = plan.host()
    ns = h["num_seg"]
    seg = h["seg"][:ns].astype(np.int64)
    assert ns <= E + R - 1
    assert np.array_equal(np.bincount(seg[:, 1], weights=seg[:, 3], minlength=R), np.full(R, SK))
    p0 = seg[:, 1] * SK + seg[:, 2]
    assert p0[0] == 0 and np.array_equal(p0[1:], p0[:-1] + seg[:-1, 3])
    cnt = counts.cpu().numpy()
    per_e = np.bincount(seg[:, 0], weights=seg[:, 3], minlength=E)
    assert np.array_equal(per_e, cnt)
    starts = np.cumsum(cnt) - cnt
    assert np.all(p0 >= starts[seg[:, 0]]) and np.all(p0 + seg[:, 3] <= starts[seg[:, 0]] + cnt[seg[:, 0]])
    # maxvio from the counts, in binary64
    assert h["maxvio"] == float(cnt.max()) * E / NK - 1.0
    assert h["num_replicas"] == int(np.sum(seg[:, 1] != seg[:, 0] // (E // R)))


def test_home_first_plan_at_int32_limit():
    R, S, E, K = 1024, 131071, 1024, 16
    NK, SK = R * S * K, S * K
    dev = torch.device(DEV)
    g = torch.Generator(device=dev)
    g.manual_seed(6)
    u = torch.rand(NK, generator=g, device=dev)
    idx = (u * u * E).to(torch.int32).clamp_(0, E - 1)
    del u
    s = mep.Shape(R, S, E, K)
    plan = mep.Plan(s, dev)
    mep.mep_plan_home_first(s, idx, plan)
    assert mep.mep_read_status(plan) == 0
    slot, src = plan.slot.view(-1), plan.src_pair
    step = 1 << 27
    for c0 in range(0, NK, step):
        c1 = min(NK, c0 + step)
        sp = src[c0:c1].long()
        assert torch.equal(slot.index_select(0, sp).long(),
                           torch.arange(c0, c1, device=dev, dtype=torch.long))
        del sp
    h = plan.host()
    ns = h["num_seg"]
    seg = h["seg"][:ns].astype(np.int64)
    assert ns <= E + R - 1
    assert np.array_equal(np.bincount(seg[:, 1], weights=seg[:, 3], minlength=R), np.full(R, SK))
    # each segment holds one expert: check its first and last slot on the device
    first = torch.from_numpy(seg[:, 1] * SK + seg[:, 2]).to(dev)
    last = first + torch.from_numpy(seg[:, 3] - 1).to(dev)
    ex = torch.from_numpy(seg[:, 0]).to(dev)
    for q in (first, last):
        assert torch.equal(idx.index_select(0, src.index_select(0, q).long()).long(), ex)
    # per expert, the segments hold exactly its pairs; replicas only where the home rank is full
    cnt = torch.bincount(idx.long(), minlength=E).cpu().numpy()
    assert np.array_equal(np.bincount(seg[:, 0], weights=seg[:, 3], minlength=E), cnt)
    B = E // R
    load = cnt.reshape(R, B).sum(axis=1)
    rep = seg[:, 1] != seg[:, 0] // B
    assert np.all(load[seg[rep, 0] // B] >= SK)
    assert h["num_replicas"] == int(rep.sum())
