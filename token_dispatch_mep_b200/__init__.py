"""Python binding of libmep, MoonEP's balanced expert-parallel token plan and
its data movement as CUDA kernels for B200 (sm_100a).

Argument marshalling only: every step runs in the CUDA kernels behind the C
ABI declared in ``include/mep.h``; PyTorch supplies device memory and
streams.  The functions carry the C names (``mep_plan``, ``mep_dispatch``,
...) and take torch tensors; they check dtypes, devices and sizes (the C ABI
cannot see sizes), pass raw pointers and the current stream, and raise
``MepError`` on a non-zero status.  There is no CPU fallback: without the
built library every call raises.
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = [
    "MepError", "Shape", "Plan", "load_library", "library_path",
    "mep_plan_workspace_bytes", "mep_maxvio", "mep_plan", "mep_plan_home_first", "mep_plan_noalloc",
    "mep_plan_capped", "mep_rank_histogram", "mep_plan_rank", "SCHEDULES", "mep_rank_barrier",
    "mep_dispatch_bulk",
    "mep_dispatch",
    "mep_combine", "mep_combine_backward", "mep_dispatch_backward", "mep_prefetch_replica_weights",
    "mep_dispatch_ranked", "mep_combine_ranked", "rank_pointer_table", "pointer_table",
    "mep_dispatch_ranked_tokens", "mep_combine_ranked_tokens", "mep_reduce_replica_grads_ranked",
    "IpcHandle", "mep_ipc_export", "mep_ipc_open", "mep_ipc_close",
    "mep_reduce_replica_grads", "mep_read_status", "mep_status_string",
    "mep_set_wait_limit_ns", "mep_get_wait_limit_ns", "mep_version", "STATUS",
]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libmep.so")

STATUS = {0: "MEP_OK", 1: "MEP_ERR_INVALID_ARG", 2: "MEP_ERR_MISALIGNED", 3: "MEP_ERR_WORKSPACE",
          4: "MEP_ERR_CUDA", 5: "MEP_ERR_DEVICE_DATA", 6: "MEP_ERR_TIMEOUT"}

# Symbols the header declares; the CPU test suite checks they are exported.
ABI_SYMBOLS = ("mep_plan_workspace_bytes", "mep_maxvio", "mep_plan", "mep_dispatch", "mep_combine",
               "mep_reduce_replica_grads", "mep_read_status", "mep_status_string",
               "mep_set_wait_limit_ns", "mep_get_wait_limit_ns", "mep_version",
               "mep_plan_noalloc", "mep_combine_backward", "mep_dispatch_backward",
               "mep_prefetch_replica_weights", "mep_plan_home_first", "mep_dispatch_ranked",
               "mep_combine_ranked", "mep_dispatch_ranked_tokens", "mep_combine_ranked_tokens",
               "mep_reduce_replica_grads_ranked", "mep_ipc_export", "mep_ipc_open",
               "mep_ipc_close", "mep_plan_capped", "mep_rank_histogram", "mep_plan_rank",
               "mep_rank_barrier", "mep_dispatch_bulk")


class MepError(RuntimeError):
    def __init__(self, code: int, where: str = ""):
        self.code = int(code)
        super().__init__(f"{where}: {STATUS.get(self.code, self.code)}")


class Shape(ctypes.Structure):
    """``mep_shape_t``: R ranks, S tokens per rank, E experts, K experts per token."""
    _fields_ = [("R", ctypes.c_int32), ("S", ctypes.c_int32), ("E", ctypes.c_int32),
                ("K", ctypes.c_int32)]

    @property
    def N(self) -> int:
        return self.R * self.S

    @property
    def NK(self) -> int:
        return self.R * self.S * self.K

    @property
    def SK(self) -> int:
        return self.S * self.K

    @property
    def seg_rows(self) -> int:
        return self.E + self.R - 1

    def __repr__(self):
        return f"Shape(R={self.R}, S={self.S}, E={self.E}, K={self.K})"


class IpcHandle(ctypes.Structure):
    """``mep_ipc_handle_t``: a CUDA IPC handle of an allocation, the exported
    range's offset in it and its length.  ``bytes(h)`` / ``IpcHandle.from_buffer_copy``
    move it between processes."""
    _fields_ = [("handle", ctypes.c_ubyte * 64), ("offset", ctypes.c_uint64),
                ("bytes", ctypes.c_uint64)]


class _PlanStruct(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "counts", "expert_offset", "slot", "src_pair", "seg", "rank_seg_ptr", "expert_seg_ptr",
        "replica_seg", "num_seg", "num_replicas", "max_count", "status", "maxvio", "rank_seg_idx")]


_lib = None


def library_path() -> str:
    return _LIB_PATH


def load_library():
    """Load ``libmep.so`` (built in-tree by ``token_dispatch_mep_b200.build``)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(_LIB_PATH):
        raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                           "`python -m token_dispatch_mep_b200.build` (nvcc, sm_100a)")
    L = ctypes.CDLL(_LIB_PATH)
    vp, i32, i64, u64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64
    sz = ctypes.c_size_t
    P = ctypes.POINTER(_PlanStruct)
    sig = {
        "mep_plan_workspace_bytes": ([Shape], sz),
        "mep_maxvio": ([Shape, vp, vp, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "mep_plan": ([Shape, vp, P, vp, sz, vp], ctypes.c_int),
        "mep_dispatch": ([Shape, i32, P, vp, vp, vp], ctypes.c_int),
        "mep_dispatch_bulk": ([Shape, i32, P, vp, vp, vp], ctypes.c_int),
        "mep_combine": ([Shape, i32, P, vp, vp, vp, vp], ctypes.c_int),
        "mep_reduce_replica_grads": ([Shape, P, i64, vp, vp, vp], ctypes.c_int),
        "mep_read_status": ([P, vp], ctypes.c_int),
        "mep_status_string": ([ctypes.c_int], ctypes.c_char_p),
        "mep_set_wait_limit_ns": ([u64], None),
        "mep_get_wait_limit_ns": ([], u64),
        "mep_version": ([], i32),
        "mep_plan_noalloc": ([Shape, vp, P, vp], ctypes.c_int),
        "mep_combine_backward": ([Shape, i32, P, vp, vp, vp, vp, vp, vp], ctypes.c_int),
        "mep_dispatch_backward": ([Shape, i32, P, vp, vp, vp], ctypes.c_int),
        "mep_prefetch_replica_weights": ([Shape, P, i64, vp, vp, vp], ctypes.c_int),
        "mep_plan_home_first": ([Shape, vp, P, vp, sz, vp], ctypes.c_int),
        "mep_plan_capped": ([Shape, i32, vp, P, vp, vp, sz, vp], ctypes.c_int),
        "mep_rank_histogram": ([Shape, vp, vp, vp, vp, sz, vp], ctypes.c_int),
        "mep_plan_rank": ([Shape, i32, i32, i32, vp, vp, P, vp, vp, sz, vp], ctypes.c_int),
        "mep_rank_barrier": ([vp, vp, i32, i32, ctypes.c_uint32, vp, vp], ctypes.c_int),
        "mep_dispatch_ranked": ([Shape, i32, P, vp, vp, vp], ctypes.c_int),
        "mep_combine_ranked": ([Shape, i32, P, vp, vp, vp, vp], ctypes.c_int),
        "mep_dispatch_ranked_tokens": ([Shape, i32, P, i64, i64, vp, vp, vp], ctypes.c_int),
        "mep_combine_ranked_tokens": ([Shape, i32, P, i64, i64, vp, vp, vp, vp], ctypes.c_int),
        "mep_reduce_replica_grads_ranked": ([Shape, P, i64, i32, vp, i64, vp, vp], ctypes.c_int),
        "mep_ipc_export": ([vp, u64, ctypes.POINTER(IpcHandle)], ctypes.c_int),
        "mep_ipc_open": ([ctypes.POINTER(IpcHandle), ctypes.POINTER(vp)], ctypes.c_int),
        "mep_ipc_close": ([ctypes.POINTER(IpcHandle), vp], ctypes.c_int),
    }
    for name, (args, res) in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = res
    _lib = L
    return L


def _shape(shape) -> Shape:
    if isinstance(shape, Shape):
        return shape
    return Shape(*[int(v) for v in shape])


def _stream(dev: torch.device):
    return ctypes.c_void_p(torch.cuda.current_stream(dev).cuda_stream)


def _need(t: torch.Tensor, name: str, dtype, numel: int, device: torch.device):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name}: dtype {t.dtype}, expected {dtype}")
    if t.device != device:
        raise ValueError(f"{name}: on {t.device}, expected {device}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if t.numel() < numel:
        raise ValueError(f"{name}: {t.numel()} elements, need {numel}")
    return ctypes.c_void_p(t.data_ptr())


def _ok(code: int, where: str):
    if code != 0:
        raise MepError(code, where)


class Plan:
    """Device buffers of one plan (``mep_plan_t``), sized from the shape alone,
    plus a zero-filled workspace for ``mep_plan`` / ``mep_maxvio``."""

    def __init__(self, shape, device=None):
        self.shape = _shape(shape)
        s = self.shape
        if device is None:
            device = torch.device("cuda", torch.cuda.current_device())
        self.device = torch.device(device)
        i32 = dict(dtype=torch.int32, device=self.device)
        self.counts = torch.zeros(s.E, **i32)
        self.expert_offset = torch.zeros(s.E + 1, **i32)
        self.slot = torch.zeros((s.N, s.K), **i32)
        self.src_pair = torch.zeros(s.NK, **i32)
        self.seg = torch.zeros((s.seg_rows, 4), **i32)
        self.rank_seg_ptr = torch.zeros(s.R + 1, **i32)
        self.expert_seg_ptr = torch.zeros(s.E + 1, **i32)
        self.replica_seg = torch.zeros(s.seg_rows, **i32)
        self.rank_seg_idx = torch.zeros(s.seg_rows, **i32)
        self.scalars = torch.zeros(4, **i32)  # num_seg, num_replicas, max_count, status
        self.maxvio_t = torch.zeros(1, dtype=torch.float64, device=self.device)
        nbytes = mep_plan_workspace_bytes(s)
        if nbytes == 0:
            raise MepError(1, "Plan")
        self.workspace = torch.zeros(nbytes, dtype=torch.uint8, device=self.device)
        a = lambda t: t.data_ptr()
        sc = self.scalars.data_ptr()
        self.struct = _PlanStruct(
            a(self.counts), a(self.expert_offset), a(self.slot), a(self.src_pair), a(self.seg),
            a(self.rank_seg_ptr), a(self.expert_seg_ptr), a(self.replica_seg),
            sc, sc + 4, sc + 8, sc + 12, a(self.maxvio_t), a(self.rank_seg_idx))

    @property
    def status_tensor(self) -> torch.Tensor:
        return self.scalars[3:4]

    def reset_workspace(self):
        """Zero the workspace again (needed after MEP_ERR_TIMEOUT / MEP_ERR_CUDA)."""
        self.workspace.zero_()

    def host(self) -> dict:
        """Copy every field to host numpy arrays (synchronises)."""
        sc = self.scalars.cpu().tolist()
        return dict(
            counts=self.counts.cpu().numpy(), expert_offset=self.expert_offset.cpu().numpy(),
            slot=self.slot.cpu().numpy(), src_pair=self.src_pair.cpu().numpy(),
            seg=self.seg.cpu().numpy(), rank_seg_ptr=self.rank_seg_ptr.cpu().numpy(),
            expert_seg_ptr=self.expert_seg_ptr.cpu().numpy(),
            replica_seg=self.replica_seg.cpu().numpy(), rank_seg_idx=self.rank_seg_idx.cpu().numpy(),
            num_seg=sc[0], num_replicas=sc[1],
            max_count=sc[2], status=sc[3], maxvio=float(self.maxvio_t.item()))


# ---------------------------------------------------------------- the calls

def mep_plan_workspace_bytes(shape) -> int:
    return int(load_library().mep_plan_workspace_bytes(_shape(shape)))


def mep_maxvio(shape, topk_idx, counts, max_count, maxvio, status, workspace):
    """T_e, max T_e and maxvio (device outputs)."""
    L, s = load_library(), _shape(shape)
    dev = topk_idx.device
    args = [_need(topk_idx, "topk_idx", torch.int32, s.NK, dev),
            _need(counts, "counts", torch.int32, s.E, dev),
            _need(max_count, "max_count", torch.int32, 1, dev),
            _need(maxvio, "maxvio", torch.float64, 1, dev),
            _need(status, "status", torch.int32, 1, dev)]
    ws = _need(workspace, "workspace", torch.uint8, mep_plan_workspace_bytes(s), dev)
    _ok(L.mep_maxvio(s, *args, ws, workspace.numel(), _stream(dev)), "mep_maxvio")


def mep_plan(shape, topk_idx, plan: Plan, workspace=None):
    """The balanced plan of ``topk_idx`` (int32 [N, K]) into ``plan``."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    idx = _need(topk_idx, "topk_idx", torch.int32, s.NK, dev)
    ws_t = plan.workspace if workspace is None else workspace
    ws = _need(ws_t, "workspace", torch.uint8, mep_plan_workspace_bytes(s), dev)
    _ok(L.mep_plan(s, idx, ctypes.byref(plan.struct), ws, ws_t.numel(), _stream(dev)), "mep_plan")


def mep_plan_home_first(shape, topk_idx, plan: Plan, workspace=None):
    """The home-first (low-replica) plan of ``topk_idx`` into ``plan``: every
    expert stays home while its home rank has room; only overflow becomes
    replicas.  Same buffers and workspace as ``mep_plan``."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    idx = _need(topk_idx, "topk_idx", torch.int32, s.NK, dev)
    ws_t = plan.workspace if workspace is None else workspace
    ws = _need(ws_t, "workspace", torch.uint8, mep_plan_workspace_bytes(s), dev)
    _ok(L.mep_plan_home_first(s, idx, ctypes.byref(plan.struct), ws, ws_t.numel(), _stream(dev)),
        "mep_plan_home_first")


def mep_plan_capped(shape, B: int, topk_idx, plan: Plan, max_rank_replicas=None, workspace=None):
    """The capped plan of ``topk_idx`` into ``plan``: at most ``B`` replica
    experts per rank when every filler finds a room (always when ``B >= 3``
    and the overflow is large next to the rooms; see ``include/mep.h``).
    ``max_rank_replicas`` (int32 [1] on the device; default: a new tensor)
    receives the most replica segments on one rank and is returned."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    idx = _need(topk_idx, "topk_idx", torch.int32, s.NK, dev)
    if max_rank_replicas is None:
        max_rank_replicas = torch.zeros(1, dtype=torch.int32, device=dev)
    mr = _need(max_rank_replicas, "max_rank_replicas", torch.int32, 1, dev)
    ws_t = plan.workspace if workspace is None else workspace
    ws = _need(ws_t, "workspace", torch.uint8, mep_plan_workspace_bytes(s), dev)
    _ok(L.mep_plan_capped(s, int(B), idx, ctypes.byref(plan.struct), mr, ws, ws_t.numel(),
                          _stream(dev)), "mep_plan_capped")
    return max_rank_replicas


# mep_schedule_t
SCHEDULES = {"contiguous": 0, "home_first": 1, "capped": 2}


def mep_rank_histogram(shape, local_idx, counts=None, plan: Plan = None, workspace=None):
    """One rank's histogram: ``counts[e]`` = pairs of ``local_idx`` (int32
    [S, K]) routed to expert e.  ``workspace``/``plan`` supply the workspace
    and status word (default: ``plan``'s).  Returns ``counts`` (int32 [E])."""
    L, s = load_library(), _shape(shape)
    dev = local_idx.device
    if counts is None:
        counts = torch.zeros(s.E, dtype=torch.int32, device=dev)
    if plan is None:
        raise ValueError("mep_rank_histogram needs a Plan (workspace and status word)")
    li = _need(local_idx, "local_idx", torch.int32, s.SK, dev)
    cp = _need(counts, "counts", torch.int32, s.E, dev)
    ws_t = plan.workspace if workspace is None else workspace
    ws = _need(ws_t, "workspace", torch.uint8, mep_plan_workspace_bytes(s), dev)
    st = ctypes.c_void_p(plan.status_tensor.data_ptr())
    _ok(L.mep_rank_histogram(s, li, cp, st, ws, ws_t.numel(), _stream(dev)), "mep_rank_histogram")
    return counts


def mep_plan_rank(shape, schedule: str, rank: int, local_idx, rank_counts, plan: Plan, B: int = 0,
                  max_rank_replicas=None, workspace=None):
    """Rank ``rank``'s share of the plan from the gathered histograms
    ``rank_counts`` (int32 [R, E]): every table of the whole-range plan of
    ``schedule`` ("contiguous", "home_first" or "capped"), and the slots of
    the rank's own pairs (``local_idx``, int32 [S, K]).  Returns
    ``max_rank_replicas`` for the capped schedule (else None)."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    if schedule not in SCHEDULES:
        raise ValueError(f"unknown schedule {schedule!r}")
    li = _need(local_idx, "local_idx", torch.int32, s.SK, dev)
    rc = _need(rank_counts, "rank_counts", torch.int32, s.R * s.E, dev)
    mr = None
    if schedule == "capped":
        if max_rank_replicas is None:
            max_rank_replicas = torch.zeros(1, dtype=torch.int32, device=dev)
        mr = _need(max_rank_replicas, "max_rank_replicas", torch.int32, 1, dev)
    ws_t = plan.workspace if workspace is None else workspace
    ws = _need(ws_t, "workspace", torch.uint8, mep_plan_workspace_bytes(s), dev)
    _ok(L.mep_plan_rank(s, SCHEDULES[schedule], int(B), int(rank), li, rc, ctypes.byref(plan.struct),
                        mr, ws, ws_t.numel(), _stream(dev)), "mep_plan_rank")
    return max_rank_replicas if schedule == "capped" else None


def mep_rank_barrier(peer_flags, my_flags, rank: int, epoch: int, status):
    """The device barrier between R ranks (``include/mep.h``): ``peer_flags``
    int64 [R] device array of the ranks' flag-array addresses, ``my_flags``
    uint32-sized words of this rank (an int32 [R] tensor), ``status`` int32
    [1] on the device.  Runs on the current stream of ``my_flags``' device
    (or of ``status``' device when the flags live in host memory)."""
    L = load_library()
    dev = status.device
    R = int(my_flags.numel())
    tp = _need(peer_flags, "peer_flags", torch.int64, R, peer_flags.device)
    if my_flags.dtype != torch.int32 or not my_flags.is_contiguous():
        raise TypeError("my_flags must be a contiguous int32 tensor")
    sp = _need(status, "status", torch.int32, 1, dev)
    _ok(L.mep_rank_barrier(tp, ctypes.c_void_p(my_flags.data_ptr()), R, int(rank),
                           int(epoch) & 0xFFFFFFFF, sp, _stream(dev)), "mep_rank_barrier")


def mep_plan_noalloc(shape, topk_idx, plan: Plan):
    """``mep_plan`` without a workspace argument: for callers that cannot
    allocate device memory.  The library's own static device scratch is used
    instead (shared by every call on the device; calls that overlap on the
    GPU race)."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    idx = _need(topk_idx, "topk_idx", torch.int32, s.NK, dev)
    _ok(L.mep_plan_noalloc(s, idx, ctypes.byref(plan.struct), _stream(dev)), "mep_plan_noalloc")


def mep_dispatch(shape, H: int, plan: Plan, x, buf):
    """``buf[slot[g,k]] = x[g]``; x bf16 [N, H], buf bf16 [R, S*K, H]."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    xp = _need(x, "x", torch.bfloat16, s.N * H, dev)
    bp = _need(buf, "buf", torch.bfloat16, s.NK * H, dev)
    _ok(L.mep_dispatch(s, int(H), ctypes.byref(plan.struct), xp, bp, _stream(dev)), "mep_dispatch")


def mep_dispatch_bulk(shape, H: int, plan: Plan, x, buf):
    """``mep_dispatch`` through the bulk-copy engine (rows staged in shared
    memory); the same result, kept for comparison (slower on B200)."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    xp = _need(x, "x", torch.bfloat16, s.N * H, dev)
    bp = _need(buf, "buf", torch.bfloat16, s.NK * H, dev)
    _ok(L.mep_dispatch_bulk(s, int(H), ctypes.byref(plan.struct), xp, bp, _stream(dev)),
        "mep_dispatch_bulk")


def mep_combine(shape, H: int, plan: Plan, y, topk_w, out):
    """``out[g] = bf16(sum_k w[g,k] y[slot[g,k]])``; y bf16 [R, S*K, H], w fp32 [N, K]."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    yp = _need(y, "y", torch.bfloat16, s.NK * H, dev)
    wp = _need(topk_w, "topk_w", torch.float32, s.NK, dev)
    op = _need(out, "out", torch.bfloat16, s.N * H, dev)
    _ok(L.mep_combine(s, int(H), ctypes.byref(plan.struct), yp, wp, op, _stream(dev)), "mep_combine")


def mep_combine_backward(shape, H: int, plan: Plan, grad_out, topk_w, y, grad_y, grad_w):
    """Adjoint of mep_combine: ``grad_y[slot[g,k]] = bf16(w[g,k] * grad_out[g])``,
    ``grad_w[g,k] = <grad_out[g], y[slot[g,k]]>``."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    args = [_need(grad_out, "grad_out", torch.bfloat16, s.N * H, dev),
            _need(topk_w, "topk_w", torch.float32, s.NK, dev),
            _need(y, "y", torch.bfloat16, s.NK * H, dev),
            _need(grad_y, "grad_y", torch.bfloat16, s.NK * H, dev),
            _need(grad_w, "grad_w", torch.float32, s.NK, dev)]
    _ok(L.mep_combine_backward(s, int(H), ctypes.byref(plan.struct), *args, _stream(dev)),
        "mep_combine_backward")


def mep_dispatch_backward(shape, H: int, plan: Plan, grad_buf, grad_x):
    """Adjoint of mep_dispatch: ``grad_x[g] = bf16(sum_k grad_buf[slot[g,k]])``."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    gb = _need(grad_buf, "grad_buf", torch.bfloat16, s.NK * H, dev)
    gx = _need(grad_x, "grad_x", torch.bfloat16, s.N * H, dev)
    _ok(L.mep_dispatch_backward(s, int(H), ctypes.byref(plan.struct), gb, gx, _stream(dev)),
        "mep_dispatch_backward")


def mep_prefetch_replica_weights(shape, plan: Plan, w_home, w_rep):
    """``w_rep[j] = w_home[expert of replica j]`` for j < num_replicas (device
    count); ``w_home`` ``[E, ...]`` and ``w_rep`` ``[E+R-1, ...]`` of one dtype,
    rows a multiple of 16 bytes."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    if w_home.dtype != w_rep.dtype:
        raise TypeError("w_home and w_rep must have the same dtype")
    row_bytes = w_home.numel() * w_home.element_size() // max(1, s.E)
    hp = _need(w_home, "w_home", w_home.dtype, s.E * (row_bytes // w_home.element_size()), dev)
    rp = _need(w_rep, "w_rep", w_rep.dtype, s.seg_rows * (row_bytes // w_rep.element_size()), dev)
    _ok(L.mep_prefetch_replica_weights(s, ctypes.byref(plan.struct), int(row_bytes), hp, rp,
                                       _stream(dev)), "mep_prefetch_replica_weights")


def rank_pointer_table(bufs, shape, H: int, device) -> torch.Tensor:
    """Device array of the R rank buffers' addresses (each [S*K, H] bf16).
    The returned table holds references to the buffers, so they stay
    allocated for as long as the table is alive."""
    s = _shape(shape)
    bufs = list(bufs)
    if len(bufs) != s.R:
        raise ValueError(f"{len(bufs)} rank buffers, need {s.R}")
    for r, b in enumerate(bufs):
        _need(b, f"rank buffer {r}", torch.bfloat16, s.SK * H, torch.device(device))
    table = torch.tensor([b.data_ptr() for b in bufs], dtype=torch.int64, device=device)
    table.keepalive = bufs
    return table


def mep_dispatch_ranked(shape, H: int, plan: Plan, x, rank_table):
    """Dispatch into R separate rank buffers; ``rank_table`` from
    ``rank_pointer_table`` (keep the buffers alive while it is used)."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    xp = _need(x, "x", torch.bfloat16, s.N * H, dev)
    tp = _need(rank_table, "rank_table", torch.int64, s.R, dev)
    _ok(L.mep_dispatch_ranked(s, int(H), ctypes.byref(plan.struct), xp, tp, _stream(dev)),
        "mep_dispatch_ranked")


def mep_combine_ranked(shape, H: int, plan: Plan, rank_table, topk_w, out):
    """Combine reading expert outputs from R separate rank buffers."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    tp = _need(rank_table, "rank_table", torch.int64, s.R, dev)
    wp = _need(topk_w, "topk_w", torch.float32, s.NK, dev)
    op = _need(out, "out", torch.bfloat16, s.N * H, dev)
    _ok(L.mep_combine_ranked(s, int(H), ctypes.byref(plan.struct), tp, wp, op, _stream(dev)),
        "mep_combine_ranked")


def pointer_table(ptrs, device) -> torch.Tensor:
    """Device array of raw device addresses (e.g. peers' buffers mapped by
    ``mep_ipc_open``), for the rank-addressed calls.  The caller keeps the
    memory behind every address alive while the table is used."""
    return torch.tensor([int(p) for p in ptrs], dtype=torch.int64, device=device)


def _token_range(s: Shape, token_begin: int, token_count: int):
    if token_begin < 0 or token_count < 0 or token_begin + token_count > s.N:
        raise ValueError(f"token range [{token_begin}, {token_begin + token_count}) outside [0, {s.N})")


def mep_dispatch_ranked_tokens(shape, H: int, plan: Plan, token_begin: int, x, rank_table,
                               token_count: int | None = None):
    """Dispatch of the tokens [token_begin, token_begin + token_count) (default:
    all rows of ``x``) into R rank buffers; ``x`` holds those tokens' rows."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    n = x.shape[0] if token_count is None else int(token_count)
    _token_range(s, int(token_begin), n)
    xp = _need(x, "x", torch.bfloat16, n * H, dev)
    tp = _need(rank_table, "rank_table", torch.int64, s.R, dev)
    _ok(L.mep_dispatch_ranked_tokens(s, int(H), ctypes.byref(plan.struct), int(token_begin), n,
                                     xp, tp, _stream(dev)), "mep_dispatch_ranked_tokens")


def mep_combine_ranked_tokens(shape, H: int, plan: Plan, token_begin: int, rank_table, topk_w,
                              out, token_count: int | None = None):
    """Combine of the tokens [token_begin, token_begin + token_count) (default:
    all rows of ``out``) from R rank buffers; ``topk_w`` and ``out`` hold those
    tokens' rows."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    n = out.shape[0] if token_count is None else int(token_count)
    _token_range(s, int(token_begin), n)
    tp = _need(rank_table, "rank_table", torch.int64, s.R, dev)
    wp = _need(topk_w, "topk_w", torch.float32, n * s.K, dev)
    op = _need(out, "out", torch.bfloat16, n * H, dev)
    _ok(L.mep_combine_ranked_tokens(s, int(H), ctypes.byref(plan.struct), int(token_begin), n,
                                    tp, wp, op, _stream(dev)), "mep_combine_ranked_tokens")


def mep_reduce_replica_grads_ranked(shape, plan: Plan, P: int, home_rank: int, rank_table,
                                    rank_rows: int, home_grads):
    """Home rank ``home_rank``'s share of the replica-gradient reduction: rank
    r's segment gradients are the ``rank_rows`` rows of the buffer at
    ``rank_table[r]``, in r's slot order; ``home_grads`` fp32 [E/R, P]."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    tp = _need(rank_table, "rank_table", torch.int64, s.R, dev)
    hp = _need(home_grads, "home_grads", torch.float32, (s.E // s.R) * P, dev)
    _ok(L.mep_reduce_replica_grads_ranked(s, ctypes.byref(plan.struct), int(P), int(home_rank),
                                          tp, int(rank_rows), hp, _stream(dev)),
        "mep_reduce_replica_grads_ranked")


def mep_ipc_export(t: torch.Tensor) -> IpcHandle:
    """IPC description of the CUDA tensor ``t``'s memory (contiguous)."""
    if not t.is_cuda or not t.is_contiguous():
        raise ValueError("mep_ipc_export needs a contiguous CUDA tensor")
    h = IpcHandle()
    with torch.cuda.device(t.device):
        _ok(load_library().mep_ipc_export(ctypes.c_void_p(t.data_ptr()),
                                          t.numel() * t.element_size(), ctypes.byref(h)),
            "mep_ipc_export")
    return h


def mep_ipc_open(h: IpcHandle, device) -> int:
    """Map another process's exported range on ``device``; returns its address."""
    p = ctypes.c_void_p()
    with torch.cuda.device(torch.device(device)):
        _ok(load_library().mep_ipc_open(ctypes.byref(h), ctypes.byref(p)), "mep_ipc_open")
    return int(p.value)


def mep_ipc_close(h: IpcHandle, ptr: int, device):
    """Unmap what ``mep_ipc_open`` returned for ``h``."""
    with torch.cuda.device(torch.device(device)):
        _ok(load_library().mep_ipc_close(ctypes.byref(h), ctypes.c_void_p(int(ptr))),
            "mep_ipc_close")


def mep_reduce_replica_grads(shape, plan: Plan, P: int, seg_grads, home_grads):
    """``home[e] = sum of seg_grads rows of e's segments``; seg_grads fp32
    [E+R-1, P], home_grads fp32 [E, P]."""
    L, s = load_library(), _shape(shape)
    dev = plan.device
    gp = _need(seg_grads, "seg_grads", torch.float32, s.seg_rows * P, dev)
    hp = _need(home_grads, "home_grads", torch.float32, s.E * P, dev)
    _ok(L.mep_reduce_replica_grads(s, ctypes.byref(plan.struct), int(P), gp, hp, _stream(dev)),
        "mep_reduce_replica_grads")


def mep_read_status(plan: Plan) -> int:
    """Synchronise the current stream and return the plan's device status."""
    return int(load_library().mep_read_status(ctypes.byref(plan.struct), _stream(plan.device)))


def mep_status_string(code: int) -> str:
    return load_library().mep_status_string(int(code)).decode()


def mep_set_wait_limit_ns(ns: int):
    load_library().mep_set_wait_limit_ns(int(ns))


def mep_get_wait_limit_ns() -> int:
    return int(load_library().mep_get_wait_limit_ns())


def mep_version() -> int:
    return int(load_library().mep_version())
