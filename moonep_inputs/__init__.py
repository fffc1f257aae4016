"""Seeded synthetic inputs for the MoonEP balanced expert-parallel hot path.

This module is shared by the CPU oracle tests, the GPU parity tests and the
benchmark.  It draws random numbers and shapes them into the workloads the
MoonEP pages describe (router top-k output swept over imbalance, softmax gates,
bf16 hidden rows); it holds none of the planning, dispatch, combine or
reduce_grad arithmetic.

Workload recipe (the pages' own routing generator, ``tests/generate_topk_routing.py``
named in "MoonshotAI/MoonEP 딥다이브" §8 exercise B, is not published, so this
stands in for it):

* expert popularity ``p_i ∝ 1/(i+1)**alpha`` (Zipf), expert ``i`` holding Zipf
  rank ``i`` so that hot experts cluster on the lowest home ranks;
* each token draws K *distinct* experts weighted by ``p`` through Gumbel-top-k
  (equivalent to Efraimidis–Spirakis weighted sampling without replacement),
  the K picks ordered by descending key;
* ``alpha`` is bisected on the realised imbalance of that very draw (common
  random numbers) until ``maxvio = max/mean expert load - 1`` is within 1% of
  the target — maxvio is the x-axis of the pages' DeepEP comparison
  ("Moonshot AI Open-Sources MoonEP", benchmark paragraph);
* gates are a softmax over the K picks of N(0,1) draws, stored as fp32;
* hidden rows are N(0,1) rounded to bf16 (round-to-nearest-even), carried as
  raw ``uint16`` bit patterns.

Every draw comes from ``numpy`` PCG64 streams keyed by ``(seed, stream id)``.
"""
from __future__ import annotations

import dataclasses
from typing import Dict, List, Optional, Tuple

import numpy as np

# independent random streams per input kind
_STREAM_ROUTING = 0
_STREAM_GATES = 1
_STREAM_X = 2
_STREAM_DOUT = 3
_STREAM_GRAD = 4
_STREAM_Y = 5

MODE_TRAIN = 0
MODE_INFER = 1


@dataclasses.dataclass(frozen=True)
class Workload:
    """One benchmark / parity workload (shapes of the pages' EP=8 and decode settings)."""

    name: str
    R: int          # simulated EP ranks
    E: int          # experts
    K: int          # top-k
    S: int          # tokens per rank
    H: int          # hidden size (bf16 elements per row)
    budget: int     # replica weight slots per rank
    mode: int       # MODE_TRAIN or MODE_INFER
    maxvio: Tuple[float, ...]
    seeds: Tuple[int, ...] = (0,)
    P: int = 0      # elements of one expert's gradient (reduce_grad), 0 if unused
    align: int = 1

    @property
    def T(self) -> int:
        return self.R * self.S


# The five workloads.  Names state what they are.
WORKLOADS: Dict[str, Workload] = {
    w.name: w
    for w in [
        # small parity case (fits in L2)
        Workload("ep8_e32_k4_s256_h512", 8, 32, 4, 256, 512, 4, MODE_TRAIN, (0.2,)),
        # headline forward: dispatch + identity expert + combine at maxvio 0.2
        Workload("ep8_e256_k8_s4096_h7168", 8, 256, 8, 4096, 7168, 32, MODE_TRAIN, (0.2,),
                 P=2048 * 7168),
        # imbalance sweep of the headline shape
        Workload("ep8_e256_k8_s4096_h7168_sweep", 8, 256, 8, 4096, 7168, 32, MODE_TRAIN,
                 (0.2, 1.0, 2.0, 5.0, 10.0, 20.0), seeds=(0, 1, 2, 3, 4)),
        # training backward: combine-backward + reduce_grad of [2048 x 7168] expert grads
        Workload("ep8_e384_k8_s8192_h7168_bwd", 8, 384, 8, 8192, 7168, 48, MODE_TRAIN, (20.0,),
                 P=2048 * 7168),
        # inference decode: 64 ranks, 4 replica slots, remote-read overflow
        Workload("ep64_e256_k8_s128_h7168_decode", 64, 256, 8, 128, 7168, 4, MODE_INFER,
                 (1.0, 20.0)),
    ]
}


def _rng(seed: int, stream: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([int(seed), int(stream)]))


# ---------------------------------------------------------------- routing ---
def zipf_log_popularity(E: int, alpha: float) -> np.ndarray:
    """log p_i for p_i ∝ 1/(i+1)**alpha (unnormalised; top-k is shift invariant)."""
    return -float(alpha) * np.log(np.arange(1, E + 1, dtype=np.float64))


def gumbel_noise(T: int, E: int, seed: int) -> np.ndarray:
    """Standard Gumbel draws [T, E] for the routing stream of ``seed``."""
    return _rng(seed, _STREAM_ROUTING).gumbel(size=(T, E))


def topk_from_keys(gumbel: np.ndarray, alpha: float, K: int) -> np.ndarray:
    """K distinct experts per token: the K largest ``log p + gumbel`` keys, descending."""
    import torch  # CPU, multithreaded top-k; a library selection primitive

    keys = torch.from_numpy(gumbel) + torch.from_numpy(zipf_log_popularity(gumbel.shape[1], alpha))
    idx = torch.topk(keys, K, dim=1, largest=True, sorted=True).indices
    return idx.to(torch.int32).numpy()


def realized_maxvio(topk_idx: np.ndarray, E: int) -> float:
    """max/mean expert load - 1 over all (token, k) picks."""
    cnt = np.bincount(np.asarray(topk_idx).ravel(), minlength=E).astype(np.float64)
    return float(cnt.max() / cnt.mean() - 1.0)


def make_routing(R: int, E: int, K: int, S: int, maxvio: float, seed: int,
                 steps: int = 30) -> Tuple[np.ndarray, float, float]:
    """Router top-k output int32 [R, S, K] tuned to ``maxvio``.

    Returns (topk_idx, alpha, realised maxvio).  The Gumbel noise is drawn once
    and reused for every bisection step, so the realised imbalance is a
    monotone-in-practice function of alpha.
    """
    T = R * S
    if T == 0:
        return np.zeros((R, S, K), np.int32), 0.0, 0.0
    g = gumbel_noise(T, E, seed)
    lo, hi = 0.0, 6.0
    best = None
    for _ in range(steps):
        a = 0.5 * (lo + hi)
        idx = topk_from_keys(g, a, K)
        m = realized_maxvio(idx, E)
        if best is None or abs(m - maxvio) < abs(best[2] - maxvio):
            best = (idx, a, m)
        if abs(m - maxvio) <= 0.01 * maxvio:
            break
        if m < maxvio:
            lo = a
        else:
            hi = a
    idx, a, m = best
    return idx.reshape(R, S, K), float(a), float(m)


def uniform_routing(R: int, E: int, K: int, S: int, seed: int,
                    distinct: bool = True) -> np.ndarray:
    """Router output without popularity skew (alpha = 0); optional repeats within a token."""
    T = R * S
    if distinct:
        return topk_from_keys(gumbel_noise(T, E, seed), 0.0, K).reshape(R, S, K)
    return _rng(seed, _STREAM_ROUTING).integers(0, E, size=(R, S, K), dtype=np.int32)


# ------------------------------------------------------------------ gates ---
def make_gates(R: int, S: int, K: int, seed: int) -> np.ndarray:
    """fp32 [R, S, K]: softmax over the K picks of N(0,1) logits."""
    z = _rng(seed, _STREAM_GATES).standard_normal(size=(R, S, K))
    z = z - z.max(axis=-1, keepdims=True) if K > 0 and R * S > 0 else z
    e = np.exp(z)
    return (e / e.sum(axis=-1, keepdims=True)).astype(np.float32) if K > 0 else e.astype(np.float32)


# -------------------------------------------------------------- bf16 rows ---
def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (nearest, ties to even) and return the uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)
    r = ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16))
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16(shape, seed: int, stream: int = _STREAM_X, scale: float = 1.0) -> np.ndarray:
    """N(0, scale^2) rounded to bf16, as uint16 bits."""
    z = _rng(seed, stream).standard_normal(size=shape, dtype=np.float32)
    if scale != 1.0:
        z *= np.float32(scale)
    return f32_to_bf16_bits(z)


def integer_bf16(shape, seed: int, stream: int = _STREAM_GRAD, bound: int = 64) -> np.ndarray:
    """Integers in [-bound, bound] stored as bf16 (exact for |v| <= 256)."""
    v = _rng(seed, stream).integers(-bound, bound + 1, size=shape).astype(np.float32)
    return f32_to_bf16_bits(v)


def make_x(R: int, S: int, H: int, seed: int) -> np.ndarray:
    return normal_bf16((R, S, H), seed, _STREAM_X)


def make_dout(R: int, S: int, H: int, seed: int) -> np.ndarray:
    return normal_bf16((R, S, H), seed, _STREAM_DOUT)


def row_pool(n_rows: int, H: int, seed: int, stream: int = _STREAM_Y) -> np.ndarray:
    """A pool of ``n_rows`` N(0,1) bf16 rows used to build large buffers cheaply."""
    return normal_bf16((n_rows, H), seed, stream)


def pool_index(n: int, pool_rows: int, seed: int) -> np.ndarray:
    """Deterministic pseudo-random map row -> pool row (int64 [n])."""
    if n == 0:
        return np.zeros(0, np.int64)
    return _rng(seed, _STREAM_Y + 100).integers(0, pool_rows, size=n, dtype=np.int64)


def workload_inputs(w: Workload, maxvio: float, seed: int, with_x: bool = True) -> dict:
    """topk_idx, gates (and x) for one (workload, maxvio, seed)."""
    idx, alpha, realized = make_routing(w.R, w.E, w.K, w.S, maxvio, seed)
    out = dict(topk_idx=idx, gates=make_gates(w.R, w.S, w.K, seed), alpha=alpha,
               maxvio=realized)
    if with_x:
        out["x"] = make_x(w.R, w.S, w.H, seed)
    return out


__all__ = [
    "Workload", "WORKLOADS", "MODE_TRAIN", "MODE_INFER", "make_routing", "uniform_routing",
    "realized_maxvio", "make_gates", "f32_to_bf16_bits", "bf16_bits_to_f32", "normal_bf16",
    "integer_bf16", "make_x", "make_dout", "row_pool", "pool_index", "workload_inputs",
    "zipf_log_popularity", "gumbel_noise", "topk_from_keys",
]
