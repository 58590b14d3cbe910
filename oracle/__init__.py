"""ctypes front end of the CPU oracle (``mep_oracle.c``).

TEST INFRASTRUCTURE ONLY.  The product path (``token_dispatch_mep_b200``)
never imports this package; only ``tests/``, ``__graft_entry__.smoke()`` and
the CPU-baseline leg of ``bench.py`` do.  The oracle shares no code with the
CUDA library: it is plain single-threaded C, compiled with gcc.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "mep_oracle.c")
LIB = os.path.join(HERE, "libmep_oracle.so")
CFLAGS = ["-std=c99", "-O2", "-ffp-contract=off", "-fno-fast-math", "-Wall",
          "-Wextra", "-shared", "-fPIC"]

OK, ERR_ARG, ERR_DATA = 0, 1, 2


def build(src: str = SRC, out: str = LIB, defines=()) -> str:
    """Compile the oracle with gcc into a shared library; returns its path."""
    cmd = ["gcc", *CFLAGS, *[f"-D{d}" for d in defines], "-o", out, src, "-lm"]
    subprocess.run(cmd, check=True)
    return out


def _needs_build(lib: str, src: str) -> bool:
    return not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src)


_i32p = ctypes.POINTER(ctypes.c_int32)
_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_u16p = ctypes.POINTER(ctypes.c_uint16)


def _p(a: np.ndarray | None, t):
    if a is None:
        return ctypes.cast(None, t)
    assert a.flags.c_contiguous
    return a.ctypes.data_as(t)


class OracleError(RuntimeError):
    def __init__(self, code: int):
        super().__init__({ERR_ARG: "invalid shape", ERR_DATA: "expert id out of range"}.get(code, str(code)))
        self.code = code


class Oracle:
    """Typed wrappers over the oracle's C entry points (numpy in, numpy out)."""

    def __init__(self, lib_path: str | None = None):
        if lib_path is None:
            lib_path = LIB
            if _needs_build(LIB, SRC):
                build()
        self.path = lib_path
        L = ctypes.CDLL(lib_path)
        L.ora_bf16_to_f32.argtypes = [ctypes.c_uint16]
        L.ora_bf16_to_f32.restype = ctypes.c_float
        L.ora_f64_to_bf16.argtypes = [ctypes.c_double]
        L.ora_f64_to_bf16.restype = ctypes.c_uint16
        L.ora_counts.argtypes = [ctypes.c_int] * 4 + [_i32p, _i32p]
        L.ora_counts.restype = ctypes.c_int
        L.ora_maxvio_from_counts.argtypes = [ctypes.c_int] * 4 + [_i32p, _i32p]
        L.ora_maxvio_from_counts.restype = ctypes.c_double
        L.ora_plan.argtypes = [ctypes.c_int] * 4 + [_i32p] * 11 + [_i32p, _f64p]
        L.ora_plan.restype = ctypes.c_int
        L.ora_dispatch.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int64, _i32p, _u16p, _u16p]
        L.ora_dispatch.restype = None
        L.ora_combine.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int64, _i32p, _f32p,
                                  _u16p, _u16p, _f64p, _f64p]
        L.ora_combine.restype = None
        L.ora_reduce.argtypes = [ctypes.c_int, _i32p, ctypes.c_int64, _f32p, _f64p, _f64p]
        L.ora_reduce.restype = None
        L.ora_combine_backward.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int64, _i32p, _f32p,
                                           _u16p, _u16p, _u16p, _f64p, _f64p, _f64p]
        L.ora_combine_backward.restype = None
        L.ora_dispatch_backward.argtypes = [ctypes.c_int64, ctypes.c_int, ctypes.c_int64, _i32p, _u16p,
                                            _u16p, _f64p, _f64p]
        L.ora_dispatch_backward.restype = None
        L.ora_prefetch_replicas.argtypes = [ctypes.c_int32, _i32p, _i32p, ctypes.c_int64,
                                            ctypes.c_void_p, ctypes.c_void_p]
        L.ora_prefetch_replicas.restype = None
        L.ora_plan_home_first.argtypes = [ctypes.c_int] * 4 + [_i32p] * 12 + [_i32p, _f64p, _i32p]
        L.ora_plan_home_first.restype = ctypes.c_int
        L.ora_plan_capped.argtypes = [ctypes.c_int] * 5 + [_i32p] * 12 + [_i32p, _f64p, _i32p,
                                                                          _i32p, _i32p]
        L.ora_plan_capped.restype = ctypes.c_int
        self.lib = L

    # -- scalars -----------------------------------------------------------
    def bf16_to_f32(self, b: int) -> float:
        return float(self.lib.ora_bf16_to_f32(int(b)))

    def f64_to_bf16(self, d: float) -> int:
        return int(self.lib.ora_f64_to_bf16(float(d)))

    # -- T_e and maxvio ------------------------------------------------------
    def counts(self, R, S, E, K, idx) -> np.ndarray:
        idx = np.ascontiguousarray(idx, dtype=np.int32)
        c = np.zeros(E, dtype=np.int32)
        st = self.lib.ora_counts(R, S, E, K, _p(idx, _i32p), _p(c, _i32p))
        if st:
            raise OracleError(st)
        return c

    def maxvio(self, R, S, E, K, idx):
        c = self.counts(R, S, E, K, idx)
        m = np.zeros(1, dtype=np.int32)
        v = self.lib.ora_maxvio_from_counts(R, S, E, K, _p(c, _i32p), _p(m, _i32p))
        return c, int(m[0]), float(v)

    # -- plan --------------------------------------------------------------
    def plan(self, R, S, E, K, idx) -> dict:
        idx = np.ascontiguousarray(idx, dtype=np.int32).reshape(-1)
        NK = R * S * K
        nseg_max = E + R - 1
        out = dict(
            counts=np.zeros(E, np.int32), expert_offset=np.zeros(E + 1, np.int32),
            slot=np.zeros(NK, np.int32), src_pair=np.zeros(NK, np.int32),
            seg=np.zeros((nseg_max, 4), np.int32), num_seg=np.zeros(1, np.int32),
            num_replicas=np.zeros(1, np.int32), rank_seg_ptr=np.zeros(R + 1, np.int32),
            expert_seg_ptr=np.zeros(E + 1, np.int32), replica_seg=np.zeros(nseg_max, np.int32),
            max_count=np.zeros(1, np.int32), maxvio=np.zeros(1, np.float64))
        names = ["counts", "expert_offset", "slot", "src_pair", "seg", "num_seg",
                 "num_replicas", "rank_seg_ptr", "expert_seg_ptr", "replica_seg", "max_count"]
        st = self.lib.ora_plan(R, S, E, K, _p(idx, _i32p), *[_p(out[n], _i32p) for n in names],
                               _p(out["maxvio"], _f64p))
        if st:
            raise OracleError(st)
        for n in ("num_seg", "num_replicas", "max_count"):
            out[n] = int(out[n][0])
        out["maxvio"] = float(out["maxvio"][0])
        out["slot"] = out["slot"].reshape(R * S, K)
        # the contiguous plan lists segments in slot order: each rank's own
        # segments are the entries rank_seg_ptr[r] .. rank_seg_ptr[r+1]
        out["rank_seg_idx"] = np.arange(out["num_seg"], dtype=np.int32)
        return out

    def plan_home_first(self, R, S, E, K, idx) -> dict:
        """The home-first (low-replica) plan; same fields as ``plan`` plus
        ``rank_seg_idx``; segments listed by (expert, rank), at most E + R - 1."""
        idx = np.ascontiguousarray(idx, dtype=np.int32).reshape(-1)
        NK = R * S * K
        nseg_max = 2 * E + R
        out = dict(
            counts=np.zeros(E, np.int32), expert_offset=np.zeros(E + 1, np.int32),
            slot=np.zeros(NK, np.int32), src_pair=np.zeros(NK, np.int32),
            seg=np.zeros((nseg_max, 4), np.int32), num_seg=np.zeros(1, np.int32),
            num_replicas=np.zeros(1, np.int32), rank_seg_ptr=np.zeros(R + 1, np.int32),
            rank_seg_idx=np.zeros(nseg_max, np.int32),
            expert_seg_ptr=np.zeros(E + 1, np.int32), replica_seg=np.zeros(nseg_max, np.int32),
            max_count=np.zeros(1, np.int32), maxvio=np.zeros(1, np.float64))
        scratch = np.zeros(6 * E + 3 * R + 2, np.int32)
        names = ["counts", "expert_offset", "slot", "src_pair", "seg", "num_seg",
                 "num_replicas", "rank_seg_ptr", "rank_seg_idx", "expert_seg_ptr", "replica_seg",
                 "max_count"]
        st = self.lib.ora_plan_home_first(R, S, E, K, _p(idx, _i32p), *[_p(out[n], _i32p) for n in names],
                                          _p(out["maxvio"], _f64p), _p(scratch, _i32p))
        if st:
            raise OracleError(st)
        for n in ("num_seg", "num_replicas", "max_count"):
            out[n] = int(out[n][0])
        out["maxvio"] = float(out["maxvio"][0])
        out["slot"] = out["slot"].reshape(R * S, K)
        out["rank_seg_idx"] = out["rank_seg_idx"][:out["num_seg"]].copy()
        return out

    def plan_capped(self, R, S, E, K, B, idx) -> dict:
        """The capped plan (at most B replica experts per rank when every
        filler is placed and B >= 3); same fields as ``plan_home_first`` plus
        ``max_rank_replicas`` (most replica segments on one rank) and
        ``unplaced`` (fillers left to the stream)."""
        idx = np.ascontiguousarray(idx, dtype=np.int32).reshape(-1)
        NK = R * S * K
        nseg_max = 2 * E + R
        out = dict(
            counts=np.zeros(E, np.int32), expert_offset=np.zeros(E + 1, np.int32),
            slot=np.zeros(NK, np.int32), src_pair=np.zeros(NK, np.int32),
            seg=np.zeros((nseg_max, 4), np.int32), num_seg=np.zeros(1, np.int32),
            num_replicas=np.zeros(1, np.int32), rank_seg_ptr=np.zeros(R + 1, np.int32),
            rank_seg_idx=np.zeros(nseg_max, np.int32),
            expert_seg_ptr=np.zeros(E + 1, np.int32), replica_seg=np.zeros(nseg_max, np.int32),
            max_count=np.zeros(1, np.int32), maxvio=np.zeros(1, np.float64),
            max_rank_replicas=np.zeros(1, np.int32), unplaced=np.zeros(1, np.int32))
        scratch = np.zeros(12 * E + 10 * R + 1, np.int32)
        names = ["counts", "expert_offset", "slot", "src_pair", "seg", "num_seg",
                 "num_replicas", "rank_seg_ptr", "rank_seg_idx", "expert_seg_ptr", "replica_seg",
                 "max_count"]
        st = self.lib.ora_plan_capped(R, S, E, K, int(B), _p(idx, _i32p),
                                      *[_p(out[n], _i32p) for n in names],
                                      _p(out["maxvio"], _f64p), _p(out["max_rank_replicas"], _i32p),
                                      _p(out["unplaced"], _i32p), _p(scratch, _i32p))
        if st:
            raise OracleError(st)
        for n in ("num_seg", "num_replicas", "max_count", "max_rank_replicas", "unplaced"):
            out[n] = int(out[n][0])
        out["maxvio"] = float(out["maxvio"][0])
        out["slot"] = out["slot"].reshape(R * S, K)
        out["rank_seg_idx"] = out["rank_seg_idx"][:out["num_seg"]].copy()
        return out

    # -- data movement ---------------------------------------------------------
    def dispatch(self, K, src_pair, x) -> np.ndarray:
        """Rows ``buf[p] = x[src_pair[p] // K]`` for every entry of src_pair.
        ``x`` is bf16 as uint16 ``[N, H]``."""
        src_pair = np.ascontiguousarray(src_pair, dtype=np.int32).reshape(-1)
        x = np.ascontiguousarray(x, dtype=np.uint16)
        H = x.shape[1]
        buf = np.empty((src_pair.size, H), dtype=np.uint16)
        self.lib.ora_dispatch(src_pair.size, K, H, _p(src_pair, _i32p), _p(x, _u16p), _p(buf, _u16p))
        return buf

    def combine(self, slot, w, y):
        """``slot`` int32 ``[n, K]``, ``w`` float32 ``[n, K]``, ``y`` bf16-as-uint16
        ``[rows, H]``; returns (bf16 out ``[n, H]`` as uint16, binary64 sum,
        sum of |terms|)."""
        slot = np.ascontiguousarray(slot, dtype=np.int32)
        w = np.ascontiguousarray(w, dtype=np.float32)
        y = np.ascontiguousarray(y, dtype=np.uint16)
        n, K = slot.shape
        H = y.shape[1]
        out = np.empty((n, H), np.uint16)
        exact = np.empty((n, H), np.float64)
        absum = np.empty((n, H), np.float64)
        self.lib.ora_combine(n, K, H, _p(slot, _i32p), _p(w, _f32p), _p(y, _u16p),
                             _p(out, _u16p), _p(exact, _f64p), _p(absum, _f64p))
        return out, exact, absum

    def reduce(self, expert_seg_ptr, G):
        """``G`` float32 ``[rows, P]`` (one row per segment); returns (binary64
        home sums ``[E, P]``, sums of |G|)."""
        ptr = np.ascontiguousarray(expert_seg_ptr, dtype=np.int32)
        G = np.ascontiguousarray(G, dtype=np.float32)
        E = ptr.size - 1
        P = G.shape[1]
        home = np.empty((E, P), np.float64)
        absum = np.empty((E, P), np.float64)
        self.lib.ora_reduce(E, _p(ptr, _i32p), P, _p(G, _f32p), _p(home, _f64p), _p(absum, _f64p))
        return home, absum

    # -- backward of combine and dispatch --------------------------------------
    def combine_backward(self, slot, w, grad_out, y):
        """``slot`` int32 ``[n, K]`` (rows of ``y``), ``w`` float32 ``[n, K]``,
        ``grad_out`` bf16-as-uint16 ``[n, H]``, ``y`` ``[rows, H]``.  Returns
        (grad_y bf16 ``[rows, H]`` -- rows not named by ``slot`` stay zero --,
        its unrounded binary64 values, grad_w binary64 ``[n, K]``, sum of
        |terms| of each dot product)."""
        slot = np.ascontiguousarray(slot, dtype=np.int32)
        w = np.ascontiguousarray(w, dtype=np.float32)
        go = np.ascontiguousarray(grad_out, dtype=np.uint16)
        y = np.ascontiguousarray(y, dtype=np.uint16)
        n, K = slot.shape
        H = go.shape[1]
        gy = np.zeros((y.shape[0], H), np.uint16)
        gye = np.zeros((y.shape[0], H), np.float64)
        gw = np.empty((n, K), np.float64)
        gwa = np.empty((n, K), np.float64)
        self.lib.ora_combine_backward(n, K, H, _p(slot, _i32p), _p(w, _f32p), _p(go, _u16p),
                                      _p(y, _u16p), _p(gy, _u16p), _p(gye, _f64p), _p(gw, _f64p),
                                      _p(gwa, _f64p))
        return gy, gye, gw, gwa

    def dispatch_backward(self, slot, grad_buf):
        """``slot`` int32 ``[n, K]`` (rows of ``grad_buf``), ``grad_buf``
        bf16-as-uint16 ``[rows, H]``; returns (grad_x bf16 ``[n, H]``, binary64
        sum, sum of |terms|)."""
        slot = np.ascontiguousarray(slot, dtype=np.int32)
        gb = np.ascontiguousarray(grad_buf, dtype=np.uint16)
        n, K = slot.shape
        H = gb.shape[1]
        gx = np.empty((n, H), np.uint16)
        ex = np.empty((n, H), np.float64)
        ab = np.empty((n, H), np.float64)
        self.lib.ora_dispatch_backward(n, K, H, _p(slot, _i32p), _p(gb, _u16p), _p(gx, _u16p),
                                       _p(ex, _f64p), _p(ab, _f64p))
        return gx, ex, ab

    # -- replica weight prefetch -------------------------------------------
    def prefetch_replicas(self, plan: dict, w_home: np.ndarray) -> np.ndarray:
        """Rows ``w_rep[j] = w_home[expert of replica j]`` for the plan's
        replicas (``w_home`` any dtype, ``[E, ...]``)."""
        w_home = np.ascontiguousarray(w_home)
        nr = int(plan["num_replicas"])
        rep = np.ascontiguousarray(plan["replica_seg"], dtype=np.int32)
        seg = np.ascontiguousarray(plan["seg"], dtype=np.int32)
        row = w_home[0].nbytes if w_home.shape[0] else 0
        out = np.zeros((max(nr, 0),) + w_home.shape[1:], dtype=w_home.dtype)
        self.lib.ora_prefetch_replicas(nr, _p(rep, _i32p), _p(seg, _i32p), row,
                                       w_home.ctypes.data_as(ctypes.c_void_p),
                                       out.ctypes.data_as(ctypes.c_void_p))
        return out


_default: Oracle | None = None


def get() -> Oracle:
    """The oracle built from ``mep_oracle.c`` next to this file (built on
    first use if missing or stale)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default
