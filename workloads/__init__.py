"""Seeded synthetic workloads for the balanced expert-parallel token plan.

This module only *generates inputs*: router top-K ids and weights, hidden rows,
expert outputs and per-segment weight gradients.  It holds none of the plan's,
dispatch's, combine's or reduction's arithmetic, so both the CPU oracle and the
CUDA path can be fed from it without sharing any of the method's code.

The router side is a stand-in for the model above the library ("the router
sends each token to several top-K experts", MoonEP news page, section "Why
expert parallelism is needed").  Recipes, all seeded:

* logits ``N(0,1)`` float32 ``[N, E]``, drawn row-chunk by row-chunk from
  ``numpy.random.default_rng(seed)``;
* plus an expert bias: Zipf ``bias_e = -s * ln(e + 1)`` (expert ``e`` has Zipf
  rank ``e + 1``, no permutation), optionally ``+hot_bias`` on ``hot`` experts
  drawn first with ``rng.choice(E, hot, replace=False)``;
* top-K by descending logit, ties to the lower expert id; ``k`` is the rank in
  that order;
* weights: softmax over the K chosen logits, or ``sigmoid(l_k) / sum_j
  sigmoid(l_j)``, evaluated in float64 and stored as float32;
* ``adversarial``: every token's K experts are ``0..K-1`` ordered by their own
  N(0,1) logits; ``uniform``: no bias; ``roundrobin``: ``idx[g,k] = (g*K+k) mod
  E`` with weights ``1/K`` (a closed-form balanced case).

Tokens are numbered rank-major, ``g = r*S + s``.
"""
from __future__ import annotations

import dataclasses
import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "BENCH_WORKLOAD", "routing", "roundrobin_routing",
    "hidden", "expert_outputs", "seg_grads", "reduced",
]


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic configuration of the plan/dispatch/combine/reduce path."""

    name: str
    R: int                      # simulated EP ranks
    S: int                      # tokens per rank
    E: int                      # experts (E % R == 0; home(e) = e // (E // R))
    K: int                      # experts per token
    H: int                      # hidden size (bf16 elements per row)
    routing: str = "zipf"       # zipf | uniform | adversarial | roundrobin
    zipf_s: float = 0.0
    hot: int = 0
    hot_bias: float = 0.0
    weights: str = "softmax"    # softmax | sigmoid
    grad: tuple = ()            # per-expert fp32 gradient shape, () for none

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
    def P(self) -> int:
        return int(np.prod(self.grad)) if self.grad else 0

    @property
    def seg_rows(self) -> int:
        """Static bound on the number of (rank, expert) segments: E + R - 1."""
        return self.E + self.R - 1

    def shape(self) -> tuple:
        return (self.R, self.S, self.E, self.K)


_SKEW = dict(R=32, S=4096, E=256, K=8, H=4096, grad=(3, 4096, 1024))

WORKLOADS = {
    w.name: w for w in [
        Workload("tiny_r4_e16", R=4, S=64, E=16, K=2, H=128, zipf_s=1.2),
        Workload("r8_e64_h2048", R=8, S=4096, E=64, K=6, H=2048, zipf_s=1.0,
                 grad=(3, 2048, 1024)),
        Workload("r16_e256_h7168", R=16, S=8192, E=256, K=8, H=7168, zipf_s=0.8,
                 hot=8, hot_bias=2.0, weights="sigmoid"),
        Workload("kimi_r64_e896_k16", R=64, S=2048, E=896, K=16, H=1024,
                 zipf_s=1.1, grad=(3, 1024, 512)),
        Workload("skew_r32_uniform", routing="uniform", **_SKEW),
        Workload("skew_r32_zipf1.5", zipf_s=1.5, **_SKEW),
        Workload("skew_r32_adversarial", routing="adversarial", **_SKEW),
    ]
}

# The configuration the headline throughput is quoted on: the largest one
# that fits one GPU (16 x 65536 x 7168 bf16 dispatch buffer, 15 GB).
BENCH_WORKLOAD = "r16_e256_h7168"

_ROW_CHUNK = 8192


def reduced(wl: Workload, S: int, H: int | None = None, P: int | None = None) -> Workload:
    """Same routing recipe, ranks, experts and K, with fewer tokens per rank
    (and optionally a smaller hidden size / gradient row) so the oracle runs
    in seconds."""
    grad = wl.grad if P is None else ((P,) if P else ())
    return dataclasses.replace(wl, name=f"{wl.name}@S{S}", S=S,
                               H=wl.H if H is None else H, grad=grad)


def _topk_rows(logits: np.ndarray, K: int) -> np.ndarray:
    """Indices of the K largest entries per row, ordered by descending value,
    ties resolved toward the lower column index."""
    n, E = logits.shape
    if K == E:
        return np.argsort(-logits, axis=1, kind="stable").astype(np.int32)
    part = np.argpartition(-logits, K - 1, axis=1)[:, K - 1]
    kth = logits[np.arange(n), part][:, None]
    gt = logits > kth
    eq = logits == kth
    need = K - gt.sum(axis=1, keepdims=True)
    chosen = gt | (eq & (np.cumsum(eq, axis=1) <= need))
    cols = np.nonzero(chosen)[1].reshape(n, K)          # ascending expert id
    vals = np.take_along_axis(logits, cols, axis=1)
    order = np.argsort(-vals, axis=1, kind="stable")     # stable: lower id first on ties
    return np.take_along_axis(cols, order, axis=1).astype(np.int32)


def _weights(chosen_logits: np.ndarray, kind: str) -> np.ndarray:
    l64 = chosen_logits.astype(np.float64)
    if kind == "softmax":
        z = np.exp(l64 - l64.max(axis=1, keepdims=True))
    elif kind == "sigmoid":
        z = 1.0 / (1.0 + np.exp(-l64))
    else:
        raise ValueError(kind)
    return (z / z.sum(axis=1, keepdims=True)).astype(np.float32)


def roundrobin_routing(R: int, S: int, E: int, K: int):
    """idx[g,k] = (g*K + k) mod E, w = 1/K: every expert gets R*S*K/E pairs
    whenever E divides R*S*K."""
    N = R * S
    idx = (np.arange(N * K, dtype=np.int64) % E).astype(np.int32).reshape(N, K)
    w = np.full((N, K), 1.0 / K, dtype=np.float32)
    return idx, w


def routing(wl: Workload, seed: int = 0):
    """Router top-K ids ``int32 [N, K]`` and weights ``float32 [N, K]``."""
    N, E, K = wl.N, wl.E, wl.K
    if wl.routing == "roundrobin":
        return roundrobin_routing(wl.R, wl.S, E, K)
    rng = np.random.default_rng(seed)
    bias = np.zeros(E, dtype=np.float32)
    if wl.hot:
        hot = rng.choice(E, wl.hot, replace=False)
    if wl.routing == "zipf":
        bias -= (wl.zipf_s * np.log(np.arange(1, E + 1, dtype=np.float64))).astype(np.float32)
    if wl.hot:
        bias[hot] += np.float32(wl.hot_bias)
    idx = np.empty((N, K), dtype=np.int32)
    w = np.empty((N, K), dtype=np.float32)
    for r0 in range(0, N, _ROW_CHUNK):
        n = min(_ROW_CHUNK, N - r0)
        if wl.routing == "adversarial":
            lg = rng.standard_normal((n, K), dtype=np.float32)
            top = _topk_rows(lg, K)
        else:
            lg = rng.standard_normal((n, E), dtype=np.float32)
            if wl.routing == "zipf":
                lg += bias
            top = _topk_rows(lg, K)
        idx[r0:r0 + n] = top
        w[r0:r0 + n] = _weights(np.take_along_axis(lg, top, axis=1), wl.weights)
    return idx, w


def _torch_gen(seed: int, device):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def hidden(N: int, H: int, seed: int = 1, device="cpu"):
    """Hidden rows ``x``: N(0,1) rounded to bf16, ``[N, H]``.  CPU and CUDA
    generators give different streams; a caller that needs both copies makes
    one and moves it."""
    import torch
    g = _torch_gen(seed, device)
    out = torch.empty((N, H), dtype=torch.bfloat16, device=device)
    step = max(1, (64 << 20) // max(1, H))
    for r0 in range(0, N, step):
        r1 = min(N, r0 + step)
        out[r0:r1] = torch.randn((r1 - r0, H), generator=g, device=device,
                                 dtype=torch.float32).to(torch.bfloat16)
    return out


def expert_outputs(rows: int, H: int, seed: int = 2, device="cpu"):
    """Synthetic expert outputs ``y`` (the combine input): N(0,1) bf16 ``[rows, H]``."""
    return hidden(rows, H, seed=seed, device=device)


def seg_grads(rows: int, P: int, seed: int = 3, device="cpu"):
    """Per-segment expert weight gradients: N(0,1) float32 ``[rows, P]``."""
    import torch
    g = _torch_gen(seed, device)
    out = torch.empty((rows, P), dtype=torch.float32, device=device)
    step = max(1, (64 << 20) // max(1, P))
    for r0 in range(0, rows, step):
        r1 = min(rows, r0 + step)
        out[r0:r1] = torch.randn((r1 - r0, P), generator=g, device=device,
                                 dtype=torch.float32)
    return out
