"""The C-ABI library builds, loads and exports every symbol include/mep.h
declares; host-side argument checks reject bad calls before any CUDA call.
CPU only: no kernel is launched here."""
import ctypes
import os
import re

import pytest

import token_dispatch_mep_b200 as mep
from token_dispatch_mep_b200 import build as mep_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    mep_build.build()
    return mep.load_library()


def header_symbols():
    names = set()
    for f in os.listdir(os.path.join(ROOT, "include")):
        if f.endswith(".h"):
            text = open(os.path.join(ROOT, "include", f)).read()
            names |= set(re.findall(r"MEP_API\s+[^;(]*?\b(mep_\w+)\s*\(", text))
    return names


def test_header_declares_the_calls():
    names = header_symbols()
    for n in ("mep_maxvio", "mep_plan", "mep_dispatch", "mep_combine",
              "mep_reduce_replica_grads", "mep_plan_workspace_bytes", "mep_read_status"):
        assert n in names
    assert names == set(mep.ABI_SYMBOLS)


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(mep.library_path())
    for n in header_symbols():
        assert hasattr(raw, n), n


def test_version_and_strings(lib):
    assert mep.mep_version() == 4
    for code, name in mep.STATUS.items():
        assert mep.mep_status_string(code)
    assert mep.mep_status_string(99) == "unknown status"


def test_wait_limit_roundtrip(lib):
    old = mep.mep_get_wait_limit_ns()
    try:
        mep.mep_set_wait_limit_ns(5_000_000)
        assert mep.mep_get_wait_limit_ns() == 5_000_000
        mep.mep_set_wait_limit_ns(3)
        assert mep.mep_get_wait_limit_ns() == 1000
    finally:
        mep.mep_set_wait_limit_ns(old)


def test_workspace_bytes(lib):
    S = mep.Shape
    assert mep.mep_plan_workspace_bytes(S(8, 4096, 64, 6)) >= 64 * 4
    assert mep.mep_plan_workspace_bytes(S(2, 2, 3, 2)) == 0          # E % R != 0
    assert mep.mep_plan_workspace_bytes(S(1, 1, 2048, 1)) == 0       # E > 1024
    assert mep.mep_plan_workspace_bytes(S(1, 4, 32, 17)) == 0        # K > 16
    assert mep.mep_plan_workspace_bytes(S(1 << 10, 1 << 20, 1024, 16)) == 0  # R*S*K >= 2^31
    a = mep.mep_plan_workspace_bytes(S(64, 2048, 896, 16))
    b = mep.mep_plan_workspace_bytes(S(64, 8, 896, 16))
    assert a == b  # sized from E alone: static across token counts


def _plan_struct(base=0x10000):
    p = mep._PlanStruct()
    for i, (name, _) in enumerate(mep._PlanStruct._fields_):
        setattr(p, name, base + 256 * i)
    return p


def test_host_side_rejections_launch_nothing(lib):
    L = lib
    s = mep.Shape(2, 4, 4, 2)
    vp = ctypes.c_void_p
    good = vp(0x100000)
    p = _plan_struct()
    # bad shapes
    for bad in [mep.Shape(0, 4, 4, 2), mep.Shape(2, 4, 3, 2), mep.Shape(2, 4, 4, 5),
                mep.Shape(2, -1, 4, 2), mep.Shape(2, 4, 4, 0)]:
        assert L.mep_plan(bad, good, ctypes.byref(p), good, 1 << 30, None) == 1
        assert L.mep_dispatch(bad, 8, ctypes.byref(p), good, good, None) == 1
    # NULL pointers
    assert L.mep_plan(s, None, ctypes.byref(p), good, 1 << 30, None) == 1
    assert L.mep_plan(s, good, None, good, 1 << 30, None) == 1
    assert L.mep_dispatch(s, 8, ctypes.byref(p), None, good, None) == 1
    assert L.mep_combine(s, 8, ctypes.byref(p), good, None, good, None) == 1
    assert L.mep_reduce_replica_grads(s, ctypes.byref(p), 16, None, good, None) == 1
    assert L.mep_reduce_replica_grads(s, ctypes.byref(p), -1, good, good, None) == 1
    assert L.mep_reduce_replica_grads(s, ctypes.byref(p), 0, None, None, None) == 0  # no-op
    # misalignment and hidden-size rules
    assert L.mep_dispatch(s, 8, ctypes.byref(p), vp(0x100002), good, None) == 2
    assert L.mep_dispatch(s, 12, ctypes.byref(p), good, good, None) == 2
    assert L.mep_dispatch(s, 4, ctypes.byref(p), good, good, None) == 1
    assert L.mep_dispatch(s, 65536, ctypes.byref(p), good, good, None) == 1
    assert L.mep_combine(s, 8, ctypes.byref(p), good, vp(0x100002), good, None) == 2
    assert L.mep_reduce_replica_grads(s, ctypes.byref(p), 16, vp(0x100004), good, None) == 2
    q = _plan_struct()
    q.seg = 0x100008
    assert L.mep_plan(s, good, ctypes.byref(q), good, 1 << 30, None) == 2
    # workspace rules
    assert L.mep_plan(s, good, ctypes.byref(p), None, 1 << 30, None) == 3
    assert L.mep_plan(s, good, ctypes.byref(p), vp(0x100080), 1 << 30, None) == 3
    assert L.mep_plan(s, good, ctypes.byref(p), good, 16, None) == 3
    i4 = vp(0x100000)
    assert L.mep_maxvio(s, i4, i4, i4, vp(0x100004), i4, good, 1 << 30, None) == 2
    assert L.mep_maxvio(s, i4, i4, i4, good, i4, good, 8, None) == 3
    # the capped plan: B >= 1, a cap output, then the plan rules
    assert L.mep_plan_capped(s, 0, good, ctypes.byref(p), i4, good, 1 << 30, None) == 1
    assert L.mep_plan_capped(s, 4, good, ctypes.byref(p), None, good, 1 << 30, None) == 1
    assert L.mep_plan_capped(s, 4, good, ctypes.byref(p), vp(0x100002), good, 1 << 30, None) == 2
    assert L.mep_plan_capped(s, 4, good, ctypes.byref(q), i4, good, 1 << 30, None) == 2
    assert L.mep_plan_capped(s, 4, good, ctypes.byref(p), i4, good, 16, None) == 3
    assert L.mep_plan_capped(mep.Shape(2, 4, 3, 2), 4, good, ctypes.byref(p), i4, good,
                             1 << 30, None) == 1


def test_package_has_no_cpu_fallback(tmp_path, monkeypatch):
    monkeypatch.setattr(mep, "_lib", None)
    monkeypatch.setattr(mep, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        mep.load_library()


def test_host_side_rejections_of_the_exchange_calls(lib):
    """Token ranges, home ranks, NULL and misaligned pointers of the per-rank
    exchange calls are rejected on the host; an empty range is a no-op."""
    L = lib
    s = mep.Shape(2, 4, 4, 2)           # N = 8 tokens
    vp = ctypes.c_void_p
    good = vp(0x100000)
    p = _plan_struct()
    pp = ctypes.byref(p)
    # token ranges
    for b, n in [(-1, 1), (0, -1), (0, 9), (8, 1), (9, 0), (4, 5)]:
        assert L.mep_dispatch_ranked_tokens(s, 8, pp, b, n, good, good, None) == 1, (b, n)
        assert L.mep_combine_ranked_tokens(s, 8, pp, b, n, good, good, good, None) == 1, (b, n)
    for b in (0, 3, 8):
        assert L.mep_dispatch_ranked_tokens(s, 8, pp, b, 0, None, None, None) == 0
        assert L.mep_combine_ranked_tokens(s, 8, pp, b, 0, None, None, None, None) == 0
    # NULL, misaligned, hidden size
    assert L.mep_dispatch_ranked_tokens(s, 8, pp, 0, 4, None, good, None) == 1
    assert L.mep_dispatch_ranked_tokens(s, 8, pp, 0, 4, good, None, None) == 1
    assert L.mep_dispatch_ranked_tokens(s, 8, pp, 0, 4, vp(0x100008), good, None) == 2
    assert L.mep_dispatch_ranked_tokens(s, 8, pp, 0, 4, good, vp(0x100004), None) == 2
    assert L.mep_dispatch_ranked_tokens(s, 12, pp, 0, 4, good, good, None) == 2
    assert L.mep_combine_ranked_tokens(s, 8, pp, 0, 4, good, None, good, None) == 1
    assert L.mep_combine_ranked_tokens(s, 8, pp, 0, 4, good, good, vp(0x100008), None) == 2
    # ranked reduce: home rank, P, pointers
    for hr in (-1, 2):
        assert L.mep_reduce_replica_grads_ranked(s, pp, 16, hr, good, 4, good, None) == 1
    assert L.mep_reduce_replica_grads_ranked(s, pp, -1, 0, good, 4, good, None) == 1
    assert L.mep_reduce_replica_grads_ranked(s, pp, 0, 0, None, 4, None, None) == 0
    assert L.mep_reduce_replica_grads_ranked(s, pp, 16, 0, None, 4, good, None) == 1
    assert L.mep_reduce_replica_grads_ranked(s, pp, 16, 0, good, 0, good, None) == 1
    assert L.mep_reduce_replica_grads_ranked(s, pp, 16, 0, good, 4, None, None) == 1
    assert L.mep_reduce_replica_grads_ranked(s, pp, 16, 0, vp(0x100004), 4, good, None) == 2
    assert L.mep_reduce_replica_grads_ranked(s, pp, 16, 0, good, 4, vp(0x100004), None) == 2
    q = _plan_struct()
    q.rank_seg_idx = None
    assert L.mep_reduce_replica_grads_ranked(s, ctypes.byref(q), 16, 0, good, 4, good, None) == 1
    # IPC: NULL arguments never reach CUDA
    h = mep.IpcHandle()
    assert L.mep_ipc_export(None, 16, ctypes.byref(h)) == 1
    assert L.mep_ipc_export(good, 0, ctypes.byref(h)) == 1
    assert L.mep_ipc_export(good, 16, None) == 1
    out = vp()
    assert L.mep_ipc_open(None, ctypes.byref(out)) == 1
    assert L.mep_ipc_open(ctypes.byref(h), None) == 1
    assert L.mep_ipc_close(None, good) == 1
    assert L.mep_ipc_close(ctypes.byref(h), None) == 1


def test_python_modules_import_without_a_gpu():
    """The autograd wrappers and the exchange module load on a CPU-only host;
    their work happens only when called on CUDA tensors."""
    from token_dispatch_mep_b200 import autograd, ep
    assert callable(autograd.dispatch) and callable(autograd.combine)
    assert callable(ep.gather_router_ids) and ep.max_local_segments(mep.Shape(8, 4096, 64, 6)) == 64


def test_rank_pointer_table_keeps_its_buffers_alive():
    """A table made from temporary rank buffers must not outlive them: the
    table holds references, so the addresses it carries stay allocated."""
    import gc
    import weakref

    import torch
    s = mep.Shape(2, 3, 4, 2)
    H = 8
    table = mep.rank_pointer_table([torch.zeros((s.SK, H), dtype=torch.bfloat16) for _ in range(2)],
                                   s, H, "cpu")
    refs = [weakref.ref(b) for b in table.keepalive]
    gc.collect()
    assert all(r() is not None for r in refs)
    assert table.tolist() == [b.data_ptr() for b in table.keepalive]
    del table
    gc.collect()
    assert all(r() is None for r in refs)


def test_the_header_is_plain_c_and_the_library_links_from_c(lib, tmp_path):
    """A C99 program that includes only include/mep.h (no CUDA or C++ header)
    compiles with -Wall -Werror, links against the library and gets the
    documented answers from the host-side calls."""
    import subprocess
    exe = tmp_path / "abi_from_c"
    src = os.path.join(ROOT, "tests", "c", "abi_from_c.c")
    libdir = os.path.dirname(mep.library_path())
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Wextra", "-Werror", "-pedantic",
                    "-I", os.path.join(ROOT, "include"), src, "-o", str(exe),
                    f"-L{libdir}", "-l:libmep.so", f"-Wl,-rpath,{libdir}"], check=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert out.returncode == 0, out.stderr
    assert out.stdout.strip() == "c abi ok"
