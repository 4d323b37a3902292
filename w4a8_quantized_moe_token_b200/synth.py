"""Seeded synthetic inputs for the W4A8 MoE expert FFN.

This module only draws random numbers and rounds them to bf16; it holds none of
the layer's arithmetic (no quantisation, no routing selection, no GEMM).  Both
the CUDA path's callers (tests, bench) and the CPU oracle receive the arrays it
returns, so the two sides always see bit-identical inputs.

Every array is drawn from ``numpy.random.default_rng([seed, tag, index...])``
so that any single tensor (one expert's weights, the activations, the routing)
can be regenerated on its own without drawing the others first.

Workload shapes follow the five layers the method is exercised on: one dense
GEMM and four MoE layers (toy, decode, large decode with Zipf-skewed routing,
prefill).  Weights are N(0, 0.02), activations N(0, 1), both rounded to bf16.
"""

from __future__ import annotations

import concurrent.futures as _cf
import os
from dataclasses import dataclass, field

import numpy as np

# tags that separate the random streams of the different tensors
_TAG_X, _TAG_W_UP, _TAG_W_DOWN, _TAG_LOGITS, _TAG_IDS, _TAG_WTS, _TAG_OUTL, _TAG_RANK, _TAG_DENSE_W, _TAG_KV = range(10)

WEIGHT_STD = 0.02


@dataclass(frozen=True)
class Workload:
    """One synthetic layer: a dense GEMM or a MoE expert FFN."""

    name: str
    kind: str  # "gemm" | "moe" | "kv"
    # dense GEMM
    M: int = 0
    K: int = 0
    N: int = 0
    # MoE
    E: int = 0
    topk: int = 0
    T: int = 0
    H: int = 0
    F: int = 0
    routing: str = ""  # "uniform" | "softmax" | "zipf"
    zipf_s: float = 0.0
    outlier_frac: float = 0.0
    outlier_mult: float = 1.0
    extra: dict = field(default_factory=dict)


WORKLOADS = {
    "dense_gemm": Workload("dense_gemm", "gemm", M=16, K=512, N=256),
    "toy_moe": Workload("toy_moe", "moe", E=8, topk=1, T=4096, H=2048, F=1024, routing="uniform"),
    "decode": Workload("decode", "moe", E=64, topk=6, T=64, H=4096, F=1408, routing="softmax",
                       outlier_frac=0.001, outlier_mult=20.0),
    "large_decode": Workload("large_decode", "moe", E=384, topk=8, T=256, H=7168, F=2048,
                             routing="zipf", zipf_s=1.1),
    "prefill": Workload("prefill", "moe", E=384, topk=8, T=16384, H=7168, F=2048, routing="uniform"),
    # reduced layers of the same per-expert shapes, small enough for a full ncu capture:
    # 16 experts with ~341 rows each (the prefill layer's mean), and 48 experts under
    # the large decode layer's Zipf routing (~5 rows each)
    "prefill_slice": Workload("prefill_slice", "moe", E=16, topk=8, T=682, H=7168, F=2048, routing="uniform"),
    "large_decode_slice": Workload("large_decode_slice", "moe", E=48, topk=8, T=32, H=7168, F=2048,
                                   routing="zipf", zipf_s=1.1),
    # INT8 KV cache of one attention layer: 32768 tokens x 8 KV heads x 128 channels,
    # static per-head scales calibrated on the first 1024 tokens
    "kv_int8": Workload("kv_int8", "kv", T=32768, extra={"heads": 8, "head_dim": 128, "calib_tokens": 1024}),
}


def _rng(seed: int, *tags: int) -> np.random.Generator:
    return np.random.default_rng([int(seed)] + [int(t) for t in tags])


def bf16_round(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    r = ((u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000).astype(np.uint32)
    return r.view(np.float32)


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) of float32 values that are already bf16-exact."""
    a = np.ascontiguousarray(a, dtype=np.float32)
    return (a.view(np.uint32) >> 16).astype(np.uint16)


def bf16_from_bits(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def normal_bf16(rng: np.random.Generator, shape, std: float = 1.0) -> np.ndarray:
    x = rng.standard_normal(size=shape, dtype=np.float32)
    if std != 1.0:
        x *= np.float32(std)
    return bf16_round(x)


def outlier_channels(seed: int, H: int, frac: float) -> np.ndarray:
    """Indices of the activation channels that carry outliers (0.1% of H, at least one)."""
    n = max(1, int(round(frac * H))) if frac > 0 else 0
    return np.sort(_rng(seed, _TAG_OUTL).permutation(H)[:n])


def activations(seed: int, T: int, H: int, outlier_frac: float = 0.0, outlier_mult: float = 1.0) -> np.ndarray:
    """Token activations x [T][H], N(0,1) in bf16; optional fixed outlier channels scaled by outlier_mult."""
    x = _rng(seed, _TAG_X).standard_normal(size=(T, H), dtype=np.float32)
    if outlier_frac > 0:
        x[:, outlier_channels(seed, H, outlier_frac)] *= np.float32(outlier_mult)
    return bf16_round(x)


def expert_weight(seed: int, e: int, which: str, rows: int, cols: int) -> np.ndarray:
    """Weights of one expert in nn.Linear orientation [out][in], N(0, 0.02) in bf16.

    which == "up": rows = 2F (gate rows [0,F), up rows [F,2F)), cols = H.
    which == "down": rows = H, cols = F.
    """
    tag = _TAG_W_UP if which == "up" else _TAG_W_DOWN
    return normal_bf16(_rng(seed, tag, e), (rows, cols), WEIGHT_STD)


def expert_weights_parallel(seed: int, E: int, which: str, rows: int, cols: int, threads: int | None = None):
    """Yield (e, weight) for every expert, drawing several experts at once on a thread pool."""
    threads = threads or min(16, os.cpu_count() or 1)
    with _cf.ThreadPoolExecutor(max_workers=threads) as pool:
        window = []
        nxt = 0
        while nxt < E or window:
            while nxt < E and len(window) < threads:
                window.append((nxt, pool.submit(expert_weight, seed, nxt, which, rows, cols)))
                nxt += 1
            e, fut = window.pop(0)
            yield e, fut.result()


def dense_gemm_inputs(seed: int, M: int, K: int, N: int):
    """x [M][K] N(0,1) and W [N][K] N(0,0.02), both bf16-exact float32."""
    x = normal_bf16(_rng(seed, _TAG_X), (M, K))
    w = normal_bf16(_rng(seed, _TAG_DENSE_W), (N, K), WEIGHT_STD)
    return x, w


def kv_cache(seed: int, T: int, H: int, D: int) -> np.ndarray:
    """Keys or values of one attention layer [T][H][D]: N(0,1) times a seeded
    per-head magnitude in [0.5, 4), in bf16 (heads differ in range, as the per-head
    scales assume)."""
    mag = _rng(seed, _TAG_KV, 0).uniform(0.5, 4.0, size=(1, H, 1)).astype(np.float32)
    return bf16_round(normal_bf16(_rng(seed, _TAG_KV, 1), (T, H, D)) * mag)


def router_logits(seed: int, T: int, E: int) -> np.ndarray:
    """Router logits [T][E], N(0,1) in bf16."""
    return normal_bf16(_rng(seed, _TAG_LOGITS), (T, E))


def _gate_weights(seed: int, T: int, k: int) -> np.ndarray:
    if k == 1:
        return np.ones((T, 1), dtype=np.float32)
    g = _rng(seed, _TAG_WTS).standard_normal(size=(T, k)).astype(np.float64)
    g = np.exp(g - g.max(axis=1, keepdims=True))
    return (g / g.sum(axis=1, keepdims=True)).astype(np.float32)


def synthetic_routing(seed: int, T: int, E: int, k: int, kind: str, zipf_s: float = 0.0):
    """Expert ids [T][k] (distinct per token) and gate weights [T][k] for synthetic routing.

    kind == "uniform": every expert equally likely.
    kind == "zipf": expert e is drawn with probability proportional to (1 + rank(e))**(-zipf_s)
    for a seeded random ranking of the experts.
    k distinct experts per token are drawn without replacement (Gumbel top-k).
    Gate weights: 1 for k == 1, else a softmax of k seeded N(0,1) values.
    """
    rng = _rng(seed, _TAG_IDS)
    if kind == "uniform":
        logp = np.zeros(E)
    elif kind == "zipf":
        rank = _rng(seed, _TAG_RANK).permutation(E)
        logp = -zipf_s * np.log1p(rank.astype(np.float64))
    else:
        raise ValueError(kind)
    if k == 1:
        p = np.exp(logp - logp.max())
        p /= p.sum()
        ids = rng.choice(E, size=(T, 1), p=p)
    else:
        gumbel = -np.log(-np.log(rng.random(size=(T, E))))
        keys = logp[None, :] + gumbel
        ids = np.argsort(-keys, axis=1, kind="stable")[:, :k]
    return ids.astype(np.int32), _gate_weights(seed, T, k)


def moe_inputs(w: Workload, seed: int = 0):
    """x and routing inputs of a MoE workload (weights are drawn per expert by expert_weight).

    Returns dict with x [T][H]; for routing == "softmax" the router logits [T][E];
    otherwise ids [T][k] and gate weights [T][k].
    """
    out = {"x": activations(seed, w.T, w.H, w.outlier_frac, w.outlier_mult)}
    if w.routing == "softmax":
        out["logits"] = router_logits(seed, w.T, w.E)
    else:
        out["ids"], out["wts"] = synthetic_routing(seed, w.T, w.E, w.topk, w.routing, w.zipf_s)
    return out
