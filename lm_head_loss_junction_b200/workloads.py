"""Seeded synthetic inputs for the junction and the multi-exit LM-head loss.

This module only draws random numbers and rounds them to the storage dtype.
It holds none of the method's arithmetic, so both the CUDA path and the CPU
oracle can consume the same bytes without sharing any computation.

Shapes follow the Matryoshka suite of "Matryoshka Language Model Suites"
(agihunt.info summary, architecture paragraph: widths 1024/2304/4352,
sequence length 2048) and the block/embedding definitions of "Editing the
methods of sub-models are made of blocks" (Modeling paragraph, after version:
block m has width D_m, residual table e_m is V x (D_m - D_{m-1}), head W^m is
V x D_m).  The vocabulary V = 49152 is the size consistent with the pages'
head-size remarks ("Visualizing Core ideas", caveats: the two small heads add
about 0.16B parameters; "Is nesting the cheapest way...", section 2: one head is
about 0.23 GB).

Every generator is numpy ``Generator(PCG64(seed))``; bf16 rounding is
round-to-nearest-even through torch's CPU conversion.
"""
from __future__ import annotations

import dataclasses
from typing import List, Optional

import numpy as np

try:  # torch is only needed for the bf16 rounding of inputs
    import torch
except Exception:  # pragma: no cover - torch is part of the image
    torch = None


@dataclasses.dataclass(frozen=True)
class SuiteConfig:
    name: str
    D: tuple            # widths D_1 < ... < D_M
    V: int
    batch: int
    seq: int
    dtype: str          # "f32" or "bf16" (storage and MMA input type)
    o_std: float = 4.0
    e_std: float = 0.02
    ids: str = "uniform"  # "uniform" or "zipf"
    zipf_s: float = 1.1
    aligned: bool = False  # shared-base block outputs and shared-prefix heads
    teacher_scale: float = 1.0
    alpha_d: float = 0.3
    seed: int = 0

    @property
    def M(self) -> int:
        return len(self.D)

    @property
    def T(self) -> int:
        return self.batch * self.seq

    @property
    def deltas(self) -> tuple:
        prev = (0,) + tuple(self.D[:-1])
        return tuple(d - p for d, p in zip(self.D, prev))

    def describe(self) -> dict:
        return {"workload": self.name, "M": self.M, "D": list(self.D),
                "delta": list(self.deltas), "V": self.V, "T": self.T,
                "batch": self.batch, "seq_len": self.seq, "dtype": self.dtype,
                "ids": self.ids, "alpha_d": self.alpha_d, "seed": self.seed}


# The five synthetic workloads.  Sizes and distributions are the ones the
# method's problem statement fixes for this path; the names say what each is.
CONFIGS = {
    "tiny3": SuiteConfig("tiny3_D64-128-192_V512_T256_f32", (64, 128, 192), 512, 1, 256,
                         "f32", o_std=4.0),
    "proxy2": SuiteConfig("proxy2_D512-1024_V32768_T16384_bf16", (512, 1024), 32768, 8, 2048,
                          "bf16", o_std=3.0),
    "main3": SuiteConfig("main3_D1024-2304-4352_V49152_T8192_bf16", (1024, 2304, 4352), 49152,
                         4, 2048, "bf16", o_std=4.0, ids="zipf"),
    "main3_aligned": SuiteConfig("main3aligned_D1024-2304-4352_V49152_T32768_bf16",
                                 (1024, 2304, 4352), 49152, 16, 2048, "bf16", ids="zipf",
                                 aligned=True, teacher_scale=3.0),
    "suite4": SuiteConfig("suite4_D640-1024-1536-2048_V49152_T32768_bf16",
                          (640, 1024, 1536, 2048), 49152, 16, 2048, "bf16", o_std=4.0),
}
CONFIG_ORDER = ["tiny3", "proxy2", "main3", "main3_aligned", "suite4"]


def small_variant(cfg: SuiteConfig, batch: int, seq: int, V: Optional[int] = None,
                  name_suffix: str = "small") -> SuiteConfig:
    """Same widths and distributions, fewer tokens (and optionally a smaller V)."""
    return dataclasses.replace(cfg, name=f"{cfg.name}_{name_suffix}", batch=batch, seq=seq,
                               V=cfg.V if V is None else V)


def to_storage(a: np.ndarray, dtype: str):
    """Round an fp32/fp64 array to the storage dtype.

    Returns a torch CPU tensor (bf16 or f32).  The oracle reads these exact
    values upcast to fp64; the GPU reads the same bytes.
    """
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32))
    if dtype == "bf16":
        return t.to(torch.bfloat16)
    if dtype == "f32":
        return t
    raise ValueError(dtype)


def as_f64(t) -> np.ndarray:
    """Exact fp64 copy of a stored input tensor."""
    return t.to(torch.float64).numpy()


def _ids(rng: np.random.Generator, cfg: SuiteConfig, n: int) -> np.ndarray:
    if cfg.ids == "uniform":
        return rng.integers(0, cfg.V, size=n, dtype=np.int64)
    if cfg.ids == "zipf":
        # rank k (1-based) has probability proportional to k^-s; rank k -> id k-1
        k = np.arange(1, cfg.V + 1, dtype=np.float64)
        p = k ** (-cfg.zipf_s)
        cdf = np.cumsum(p)
        cdf /= cdf[-1]
        u = rng.random(n)
        return np.minimum(np.searchsorted(cdf, u, side="right"), cfg.V - 1).astype(np.int64)
    raise ValueError(cfg.ids)


def _normal(rng, shape, std):
    return rng.standard_normal(size=shape, dtype=np.float32) * np.float32(std)


@dataclasses.dataclass
class SuiteInputs:
    cfg: SuiteConfig
    x: np.ndarray            # int32 [T] input ids
    y: np.ndarray            # int32 [T] next-token targets
    o: List                  # M tensors [T, D_m] (block outputs = head inputs)
    E: List                  # M tensors [V, delta_m] residual embedding tables
    W: List                  # M tensors [V, D_m] heads


def make_inputs(cfg: SuiteConfig, with_heads: bool = True, with_tables: bool = True) -> SuiteInputs:
    """Draw the workload's inputs.  Deterministic in ``cfg.seed``.

    Draw order (fixed, so sub-selections stay reproducible): ids, final-position
    targets, block outputs o_1..o_M, tables e_1..e_M, heads W^1..W^M.
    """
    rng = np.random.Generator(np.random.PCG64(cfg.seed))
    T, V, M = cfg.T, cfg.V, cfg.M
    x = _ids(rng, cfg, T).reshape(cfg.batch, cfg.seq)
    last = _ids(rng, cfg, cfg.batch)
    y = np.empty_like(x)
    y[:, :-1] = x[:, 1:]          # next-token targets within each sequence
    y[:, -1] = last               # final position drawn from the id distribution
    x = x.reshape(T).astype(np.int32)
    y = y.reshape(T).astype(np.int32)

    o = []
    if cfg.aligned:
        base = _normal(rng, (T, cfg.D[-1]), 1.0)
        for m in range(M):
            o.append(to_storage(base[:, :cfg.D[m]] + _normal(rng, (T, cfg.D[m]), 0.5), cfg.dtype))
        del base
    else:
        for m in range(M):
            o.append(to_storage(_normal(rng, (T, cfg.D[m]), cfg.o_std), cfg.dtype))

    E = []
    if with_tables:
        for m in range(M):
            E.append(to_storage(_normal(rng, (V, cfg.deltas[m]), cfg.e_std), cfg.dtype))

    W = []
    if with_heads:
        if cfg.aligned:
            G = _normal(rng, (V, cfg.D[-1]), 1.0)
            for m in range(M):
                w = G[:, :cfg.D[m]] / np.float32(np.sqrt(cfg.D[m]))
                if m == M - 1:
                    w = w * np.float32(cfg.teacher_scale)
                W.append(to_storage(w, cfg.dtype))
            del G
        else:
            for m in range(M):
                W.append(to_storage(_normal(rng, (V, cfg.D[m]), 1.0 / np.sqrt(cfg.D[m])), cfg.dtype))
    return SuiteInputs(cfg, x, y, o, E, W)


def make_grad(cfg: SuiteConfig, m: int, std: float = 1e-3, seed_offset: int = 1000):
    """Seeded incoming gradient dy for junction m -> m+1, shape [T, D_{m+1}]."""
    rng = np.random.Generator(np.random.PCG64(cfg.seed + seed_offset + m))
    return to_storage(_normal(rng, (cfg.T, cfg.D[m + 1]), std), cfg.dtype)
