"""Seeded synthetic rank buffers -- shared by the tests, the bench and smoke().

This module draws random numbers and lays them out per rank.  It holds none of
the collectives' arithmetic: no reduction, no rounding rule, no ordering.  Both
the CPU oracle and the CUDA library consume what it returns.

Each generator returns a list of ``p`` contiguous host numpy arrays, one per
simulated rank, drawn in rank order 0..p-1 from ONE ``torch.Generator`` seeded
with ``seed``.  Storage types: float32 ("f32"), uint16 bf16 bit patterns
("bf16", the fp32 draw narrowed by torch's round-to-nearest-even ``.to``),
int32 ("i32").

Workloads (sizes and value distributions as the collectives' pages and their
reproduction recipe state them):
  * worked example: x_r = [0,1,2,3] + r, p = 4;
  * uniform[lo, hi), normal N(0, sigma) (sigma is a standard deviation),
    integers uniform[lo, hi);
  * the transformer-layer parameter count 4*4096*4096 + 3*4096*11008 of a
    Llama-2-7B decoder layer (Q, K, V, O projections and gate, up, down);
  * optimizer state for the sharded AdamW step: fp32 master weights
    uniform[-1, 1), first moments N(0, 1e-3), second moments the squares of
    an N(0, 1e-3) draw, each split into p shards; the step's hyperparameters
    (ZERO1_ADAMW) are a synthetic recipe, since the pages give none.
"""
from __future__ import annotations

from typing import List

import numpy as np
import torch

# Llama-2-7B decoder layer: W_Q, W_K, W_V, W_O are 4096x4096; W_gate, W_up are
# 4096x11008 and W_down is 11008x4096.
LLAMA2_7B_LAYER_ELEMS = 4 * 4096 * 4096 + 3 * 4096 * 11008  # 202,375,168

NP = {"f32": np.float32, "bf16": np.uint16, "i32": np.int32}

# AdamW hyperparameters of the sharded-optimizer workload (synthetic recipe).
ZERO1_ADAMW = dict(lr=3e-4, beta1=0.9, beta2=0.95, eps=1e-8, weight_decay=0.1, step=10)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    return g


def _store(t: torch.Tensor, dt: str) -> np.ndarray:
    if dt == "f32":
        return t.to(torch.float32).contiguous().numpy()
    if dt == "bf16":
        return t.to(torch.float32).to(torch.bfloat16).view(torch.int16).contiguous().numpy().view(np.uint16)
    if dt == "i32":
        return t.to(torch.int32).contiguous().numpy()
    raise ValueError(dt)


def worked_example(p: int = 4, n: int = 4, dt: str = "f32") -> List[np.ndarray]:
    """x_r[i] = i + r (the pages' four-rank example for n = 4)."""
    return [_store(torch.arange(n, dtype=torch.float64) + r, dt) if dt != "i32"
            else (np.arange(n, dtype=np.int64) + r).astype(np.int32) for r in range(p)]


def uniform(p: int, n: int, seed: int, dt: str = "f32", lo: float = -1.0, hi: float = 1.0) -> List[np.ndarray]:
    g = _gen(seed)
    out = []
    for _ in range(p):
        t = torch.rand(n, generator=g, dtype=torch.float32) * (hi - lo) + lo
        out.append(_store(t, dt))
    return out


def normal(p: int, n: int, seed: int, sigma: float = 1.0, dt: str = "f32") -> List[np.ndarray]:
    g = _gen(seed)
    out = []
    for _ in range(p):
        t = torch.randn(n, generator=g, dtype=torch.float32) * sigma
        out.append(_store(t, dt))
    return out


def int_uniform(p: int, n: int, seed: int, lo: int = -(1 << 20), hi: int = 1 << 20) -> List[np.ndarray]:
    g = _gen(seed)
    return [torch.randint(lo, hi, (n,), generator=g, dtype=torch.int32).numpy() for _ in range(p)]


def sweep_data(p: int, n: int, seed: int, dt: str) -> List[np.ndarray]:
    """The sweep's value distributions: floats uniform[-1,1), ints uniform[-2^20, 2^20)."""
    if dt == "i32":
        return int_uniform(p, n, seed)
    return uniform(p, n, seed, dt)


def sweep_data_device(p: int, n: int, seed: int, dt: str, device: str = "cuda") -> List[torch.Tensor]:
    """The sweep's value distributions drawn on the device (torch's seeded
    Philox generator for that device), for the per-rank sizes too large to
    draw on the host in a test: floats uniform[-1, 1) (bf16: the fp32 draw
    narrowed by torch, round-to-nearest-even), ints uniform[-2^20, 2^20).
    Returns p device tensors (float32, bfloat16 or int32)."""
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = []
    for _ in range(p):
        if dt == "i32":
            out.append(torch.randint(-(1 << 20), 1 << 20, (n,), generator=g, device=device,
                                     dtype=torch.int32))
            continue
        t = torch.rand(n, generator=g, device=device, dtype=torch.float32) * 2.0 - 1.0
        out.append(t if dt == "f32" else t.to(torch.bfloat16))
    return out


def special_values(p: int, n: int, seed: int, dt: str = "f32") -> List[np.ndarray]:
    """Values that stress ordering and rounding: signed zeros, large/small
    magnitudes that cancel, exact powers of two, bf16 rounding ties."""
    rng = np.random.default_rng(seed)
    if dt == "i32":
        pool = np.array([0, 1, -1, 2**31 - 1, -2**31, 2**30, -2**30, 12345, -7], dtype=np.int64)
        return [pool[rng.integers(0, pool.size, n)].astype(np.int32) for _ in range(p)]
    pool = np.array([0.0, -0.0, 1.0, -1.0, 2.0**24, -2.0**24, 2.0**-24, 3.0, 1e-3, -1e-3,
                     1.0 + 2.0**-8, 1.0 + 3 * 2.0**-9, 65504.0, -0.5, 2.0**-126, 7.25e9],
                    dtype=np.float32)
    out = []
    for _ in range(p):
        v = pool[rng.integers(0, pool.size, n)]
        if dt == "f32":
            out.append(v.astype(np.float32))
        else:
            out.append(_store(torch.from_numpy(v.astype(np.float32)), "bf16"))
    return out


def config(name: str):
    """The named workloads: a dict with everything needed to draw them."""
    cfgs = {
        "worked_example": dict(p=4, n=4, dt="f32", gen="worked"),
        "uniform_p4_64k": dict(p=4, n=65536, dt="f32", gen="uniform", seed=0),
        "ring_p8_2m_f32": dict(p=8, n=2097152, dt="f32", gen="normal", seed=1, sigma=1e-2),
        "hier_2x4_4m_bf16": dict(p=8, n=4194304, dt="bf16", gen="normal", seed=2, sigma=1.0, group=4),
        "llama_layer_param_shards_bf16": dict(p=8, n=LLAMA2_7B_LAYER_ELEMS // 8, dt="bf16", gen="uniform", seed=3),
        "llama_layer_grads_f32": dict(p=8, n=LLAMA2_7B_LAYER_ELEMS, dt="f32", gen="normal", seed=4, sigma=1e-3),
        "zero1_state": dict(p=8, n=LLAMA2_7B_LAYER_ELEMS, gen="adam_state", seed=5),
    }
    return cfgs[name]


def draw(cfg: dict) -> List[np.ndarray]:
    g = cfg["gen"]
    if g == "worked":
        return worked_example(cfg["p"], cfg["n"], cfg["dt"])
    if g == "uniform":
        return uniform(cfg["p"], cfg["n"], cfg["seed"], cfg["dt"])
    if g == "normal":
        return normal(cfg["p"], cfg["n"], cfg["seed"], cfg.get("sigma", 1.0), cfg["dt"])
    if g == "adam_state":
        return adam_state(cfg["p"], cfg["n"], cfg["seed"])
    raise ValueError(g)


def adam_state(p: int, n: int, seed: int):
    """(master, exp_avg, exp_avg_sq): three lists of p fp32 shards of n // p
    elements -- master uniform[-1, 1), exp_avg N(0, 1e-3), exp_avg_sq the
    squares of an N(0, 1e-3) draw -- from one generator, in that order."""
    g = _gen(seed)
    m = n // p
    master = [(torch.rand(m, generator=g, dtype=torch.float32) * 2 - 1).numpy() for _ in range(p)]
    ea = [(torch.randn(m, generator=g, dtype=torch.float32) * 1e-3).numpy() for _ in range(p)]
    es = [(torch.randn(m, generator=g, dtype=torch.float32) * 1e-3).square().numpy() for _ in range(p)]
    return master, ea, es
