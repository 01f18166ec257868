"""Seeded synthetic inputs for MoE token dispatch / combine.

This module only draws inputs.  It holds none of the dispatch/combine
arithmetic, imports neither the CUDA binding nor the CPU oracle, and is the one
piece both sides share.

Every workload is a dict with

* ``x``            -- ``numpy.uint16 [T, H]``: bf16 bit patterns of the token rows,
* ``topk_idx``     -- ``numpy.int64 [T, k]``: chosen experts, ``-1`` = no route,
* ``topk_weights`` -- ``numpy.float32 [T, k]``: gate weights (0 on ``-1`` routes),
* ``T, H, E, R, k`` and a ``name``.

Shapes follow the workloads the pages discuss:

* the DeepEP decode/prefill shape (hidden 7168, 256 experts, top-8) from the
  amazon-contributing DeepEP PR "feat(jit): forward sub-part geometry env vars
  to the JIT", section "Measured effect of the knob it exposes";
* the low-batch combine shape (hidden 3584, 896 experts over 32 ranks, top-16,
  one real row with experts ``i * 28`` and weights ``1/16``) from DeepEP issue
  #760 "[Performance] DeepEP V2 combine epilogue low batch performance",
  section "Reproduction";
* the DP batch ``[120, 1, 1, 1, 1, 1, 1, 1]`` laid out compact (sum) and padded
  to ``8 * 120`` rows (max) from SGLang PR #6092's discussion of sum vs max
  token padding.

Recipe (fixed draw order per seed, ``numpy.random.default_rng(seed)``):
x ~ N(0,1) in fp32, rounded to bf16 (round-to-nearest-even, done by torch's CPU
cast); then the expert choice; then N(0,1) fp32 logits whose softmax over the
k chosen experts gives the weights.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "CONFIGS",
    "make",
    "make_uniform",
    "make_zipf",
    "make_lowbatch",
    "make_dp",
    "to_bf16_bits",
    "bf16_bits_to_f32",
]

# name -> keyword arguments of ``make``
CONFIGS = {
    "tiny": dict(kind="uniform", T=128, H=256, E=16, R=4, k=4),
    "decode": dict(kind="uniform", T=128, H=7168, E=256, R=16, k=8),
    "prefill": dict(kind="zipf", T=4096, H=7168, E=256, R=16, k=8, s=1.2),
    "lowbatch1": dict(kind="lowbatch", T=1, H=3584, E=896, R=32, k=16),
    "lowbatch2": dict(kind="lowbatch", T=2, H=3584, E=896, R=32, k=16),
    "lowbatch4": dict(kind="lowbatch", T=4, H=3584, E=896, R=32, k=16),
    "lowbatch8": dict(kind="lowbatch", T=8, H=3584, E=896, R=32, k=16),
    "dp_compact": dict(kind="dp", padded=False, H=7168, E=256, R=16, k=8),
    "dp_padded": dict(kind="dp", padded=True, H=7168, E=256, R=16, k=8),
}

DP_GROUPS = (120, 1, 1, 1, 1, 1, 1, 1)


def to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 array -> bf16 bit patterns (uint16), round-to-nearest-even via torch."""
    import torch

    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> exact fp32 values."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _softmax_f32(logits: np.ndarray) -> np.ndarray:
    z = logits.astype(np.float64)
    z = z - z.max(axis=1, keepdims=True)
    p = np.exp(z)
    return (p / p.sum(axis=1, keepdims=True)).astype(np.float32)


def _pack(name, x, idx, w, E, R):
    T, H = x.shape
    return dict(name=name, x=np.ascontiguousarray(x, dtype=np.uint16),
                topk_idx=np.ascontiguousarray(idx, dtype=np.int64),
                topk_weights=np.ascontiguousarray(w, dtype=np.float32),
                T=int(T), H=int(H), E=int(E), R=int(R), k=int(idx.shape[1]))


def make_uniform(T, H, E, R, k, seed=0, name="uniform"):
    """k distinct experts per token, uniform over E."""
    rng = np.random.default_rng(seed)
    x = to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    # k smallest of E iid uniforms per row = a uniform k-subset in random order
    keys = rng.random((T, E))
    idx = np.argsort(keys, axis=1, kind="stable")[:, :k]
    logits = rng.standard_normal((T, k), dtype=np.float32)
    return _pack(name, x, idx, _softmax_f32(logits), E, R)


def make_zipf(T, H, E, R, k, s=1.2, seed=0, name="zipf"):
    """k distinct experts per token drawn without replacement from a Zipf(s)
    popularity over a seeded permutation of the experts; column order is the
    order of the draws (successive sampling, via the Gumbel-top-k identity)."""
    rng = np.random.default_rng(seed)
    x = to_bf16_bits(rng.standard_normal((T, H), dtype=np.float32))
    perm = rng.permutation(E)
    p = np.empty(E)
    p[perm] = (np.arange(E) + 1.0) ** (-s)   # expert perm[i] has rank i+1
    p /= p.sum()
    g = rng.gumbel(size=(T, E))
    keys = np.log(p)[None, :] + g
    idx = np.argsort(-keys, axis=1, kind="stable")[:, :k]
    logits = rng.standard_normal((T, k), dtype=np.float32)
    return _pack(name, x, idx, _softmax_f32(logits), E, R)


def make_lowbatch(T, H=3584, E=896, R=32, k=16, value=1.0, name="lowbatch"):
    """One real row (row 0) routed to experts i * (E/R) for i < k with weight
    1/k and x filled with ``value``; rows 1..T-1 carry only -1 routes, zero
    weights and zero x.  Deterministic (no seed)."""
    epr = E // R
    x = np.zeros((T, H), dtype=np.float32)
    idx = np.full((T, k), -1, dtype=np.int64)
    w = np.zeros((T, k), dtype=np.float32)
    x[0, :] = value
    idx[0, :] = np.arange(k) * epr
    w[0, :] = np.float32(1.0) / np.float32(k)
    return _pack(name, to_bf16_bits(x), idx, w, E, R)


def make_dp(H, E, R, k, padded, groups=DP_GROUPS, seed=0, name="dp"):
    """DP groups' real tokens (uniform top-k), laid out compact (sum of group
    sizes rows) or padded (each group at a stride of max(group) rows, the gap
    rows zero with -1 routes).  Both layouts hold the same real tokens in the
    same order."""
    n_real = int(sum(groups))
    real = make_uniform(n_real, H, E, R, k, seed=seed)
    if not padded:
        real["name"] = name
        return real
    stride = max(groups)
    T = stride * len(groups)
    x = np.zeros((T, H), dtype=np.uint16)
    idx = np.full((T, k), -1, dtype=np.int64)
    w = np.zeros((T, k), dtype=np.float32)
    src = 0
    for g, b in enumerate(groups):
        dst = g * stride
        x[dst:dst + b] = real["x"][src:src + b]
        idx[dst:dst + b] = real["topk_idx"][src:src + b]
        w[dst:dst + b] = real["topk_weights"][src:src + b]
        src += b
    return _pack(name, x, idx, w, E, R)


def make(name: str, seed: int = 0) -> dict:
    """Build a named workload from ``CONFIGS``."""
    cfg = dict(CONFIGS[name])
    kind = cfg.pop("kind")
    if kind == "uniform":
        return make_uniform(seed=seed, name=name, **cfg)
    if kind == "zipf":
        return make_zipf(seed=seed, name=name, **cfg)
    if kind == "lowbatch":
        return make_lowbatch(name=name, **cfg)
    if kind == "dp":
        return make_dp(seed=seed, name=name, **cfg)
    raise KeyError(name)
