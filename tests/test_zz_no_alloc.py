"""mep_plan_noalloc: the plan for callers that cannot allocate device memory.

Some callers cannot hand the library a workspace: their runtime has no device
allocator, or a host framework owns the device memory pool and forbids
allocation once it has started.  mep_plan_noalloc serves them from a scratch
array compiled into the library.  These tests call it through the C ABI and
check that its plan equals the one mep_plan (with a caller workspace)
produces, bit for bit, on two calls in a row.  The file is collected last so
that a run stopping at the first failure has already run every other test;
it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import token_dispatch_mep_b200 as mep
import workloads


def test_rejects_shapes_beyond_the_limits():
    """Shapes outside the library's rules are refused before anything runs."""
    L = mep.load_library()
    p = mep._PlanStruct()
    idx = ctypes.c_void_p(0x100000)
    for bad in (mep.Shape(2, 4, 2048, 2),     # E above MEP_MAX_EXPERTS: beyond the scratch
                mep.Shape(2, 4, 3, 2),        # E % R != 0
                mep.Shape(2, 4, 64, 17)):     # K above MEP_MAX_TOPK
        assert L.mep_plan_noalloc(bad, idx, ctypes.byref(p), None) == 1
    assert L.mep_plan_noalloc(mep.Shape(2, 4, 8, 2), None, ctypes.byref(p), None) == 1
    assert L.mep_plan_noalloc(mep.Shape(2, 4, 8, 2), idx, None, None) == 1


def test_checks_every_plan_field_before_queueing_anything():
    """A NULL or misaligned plan field is reported by the host-side checks,
    before the scratch memset is queued: these calls reach no CUDA API at all
    (they run here without a GPU)."""
    L = mep.load_library()
    fields = [f for f, _ in mep._PlanStruct._fields_]
    aligned = {f: 0x100000 + 0x1000 * i for i, f in enumerate(fields)}
    s = mep.Shape(2, 4, 8, 2)
    idx = ctypes.c_void_p(0x900000)
    for f in fields:
        p = mep._PlanStruct(**aligned)
        setattr(p, f, aligned[f] + 2)           # off every alignment the plan needs
        assert L.mep_plan_noalloc(s, idx, ctypes.byref(p), None) == 2, f
        p = mep._PlanStruct(**aligned)
        setattr(p, f, None)
        assert L.mep_plan_noalloc(s, idx, ctypes.byref(p), None) == 1, f
    p = mep._PlanStruct(**aligned)
    assert L.mep_plan_noalloc(s, ctypes.c_void_p(0x900002), ctypes.byref(p), None) == 2


def _host_fields(plan):
    h = plan.host()
    ns, nr = h["num_seg"], h["num_replicas"]
    return dict(counts=h["counts"], expert_offset=h["expert_offset"], slot=h["slot"],
                src_pair=h["src_pair"], seg=h["seg"][:ns], rank_seg_ptr=h["rank_seg_ptr"],
                expert_seg_ptr=h["expert_seg_ptr"], replica_seg=h["replica_seg"][:nr],
                scalars=(ns, nr, h["max_count"], h["status"]), maxvio=h["maxvio"])


@pytest.mark.gpu
@pytest.mark.parametrize("name", ["kimi_r64_e896_k16", "r8_e64_h2048"])
def test_noalloc_plan_equals_workspace_plan_twice(name):
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    wl = workloads.WORKLOADS[name]
    s = mep.Shape(*wl.shape())
    L = mep.load_library()
    stream = ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)
    ref = mep.Plan(s, dev)
    got = mep.Plan(s, dev)
    for call, seed in enumerate((0, 1)):        # two calls in a row, different routing
        idx_h, _ = workloads.routing(wl, seed=seed)
        idx = torch.from_numpy(idx_h).to(dev)
        mep.mep_plan(s, idx, ref)                  # existing entry point, caller workspace
        rc = L.mep_plan_noalloc(s, ctypes.c_void_p(idx.data_ptr()), ctypes.byref(got.struct),
                                stream)
        assert rc == 0, mep.mep_status_string(rc)
        assert mep.mep_read_status(got) == 0
        a, b = _host_fields(ref), _host_fields(got)
        for key in a:
            if isinstance(a[key], np.ndarray):
                assert np.array_equal(a[key], b[key]), (name, call, key)
            else:
                assert a[key] == b[key], (name, call, key)
