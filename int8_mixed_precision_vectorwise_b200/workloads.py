"""Seeded synthetic inputs shaped like the OPT / Llama linears the pages discuss.

This module draws random numbers and nothing else: it holds none of the
method's arithmetic (no scaling rule, no quantisation), so both the CUDA path
and the CPU oracle can be fed from it.  Everything is numpy on the host; callers
move arrays to the device themselves.

Recipe (all float32 draws rounded once to fp16):
  * activations X ~ N(0, 1); ``n_out`` columns chosen by a seeded permutation
    are overwritten, every row, with a random sign times U(lo, hi);
  * weights W ~ N(0, 0.02); biases ~ N(0, 0.01) where the modelled layer has
    one (OPT), none for the Llama shapes.
"""

from __future__ import annotations

from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np

BASE_SEED = 1234


def rng(seed: int) -> np.random.Generator:
    return np.random.default_rng(seed)


def activation(seed: int, M: int, K: int, n_out: int = 0,
               mag: Tuple[float, float] = (20.0, 60.0)):
    """X fp16 [M, K] ~ N(0,1) with ``n_out`` seeded columns of magnitude U(mag)."""
    g = rng(seed)
    X = g.standard_normal((M, K), dtype=np.float32)
    cols = np.sort(g.permutation(K)[:n_out]) if n_out > 0 else np.zeros(0, np.int64)
    if n_out > 0:
        lo, hi = mag
        m = g.uniform(lo, hi, size=(M, n_out)).astype(np.float32)
        s = np.where(g.random((M, n_out)) < 0.5, -1.0, 1.0).astype(np.float32)
        X[:, cols] = s * m
    return X.astype(np.float16), cols


def weight(seed: int, N: int, K: int, std: float = 0.02) -> np.ndarray:
    g = rng(seed)
    W = g.standard_normal((N, K), dtype=np.float32)
    W *= np.float32(std)
    return W.astype(np.float16)


def bias(seed: int, N: int, std: float = 0.01) -> np.ndarray:
    g = rng(seed)
    return (g.standard_normal(N, dtype=np.float32) * np.float32(std)).astype(np.float16)


def grad_output(seed: int, M: int, N: int) -> np.ndarray:
    """dY fp16 [M, N] ~ N(0, 1): the gradient arriving at a layer's output."""
    g = rng(seed)
    return g.standard_normal((M, N), dtype=np.float32).astype(np.float16)


@dataclass
class Linear:
    """One Linear8bitLt call: X [M, K] -> out [M, N]."""
    name: str
    M: int
    K: int
    N: int
    has_bias: bool
    n_out: int                     # planted outlier columns in X
    mag: Tuple[float, float]
    threshold: float
    x_from: Optional[str] = None   # feed from a previous layer's output (after ReLU)

    @property
    def ops(self) -> int:
        return 2 * self.M * self.N * self.K


@dataclass
class Workload:
    key: str
    title: str
    layers: List[Linear] = field(default_factory=list)

    @property
    def ops(self) -> int:
        return sum(l.ops for l in self.layers)


def _llama7b_prefill(tokens: int = 4096) -> Workload:
    f = 0.001
    mag = (20.0, 60.0)
    ls = []
    for nm in ("q_proj", "k_proj", "v_proj", "o_proj"):
        ls.append(Linear(nm, tokens, 4096, 4096, False, round(f * 4096), mag, 6.0))
    for nm in ("gate_proj", "up_proj"):
        ls.append(Linear(nm, tokens, 4096, 11008, False, round(f * 4096), mag, 6.0))
    ls.append(Linear("down_proj", tokens, 11008, 4096, False, round(f * 11008), mag, 6.0))
    return Workload("llama7b_prefill", "Llama-7B-shaped prefill linears, 4096 tokens", ls)


def workloads() -> dict:
    """The five workload families, keyed C1..C5 (plus sweep points)."""
    w = {}
    w["C1"] = Workload("single_linear", "single Linear8bitLt 16x1024 -> 1024", [
        Linear("linear", 16, 1024, 1024, True, 2, (19.5, 20.5), 6.0)])
    w["C2"] = Workload("opt350m_mlp", "OPT-350m-shaped MLP pair 512x1024 -> 4096 -> 1024", [
        Linear("fc1", 512, 1024, 4096, True, round(0.002 * 1024), (8.0, 40.0), 6.0),
        Linear("fc2", 512, 4096, 1024, True, 0, (0.0, 0.0), 6.0, x_from="fc1")])
    w["C3"] = _llama7b_prefill(4096)
    for t in (1, 4, 16):
        for n_o in (0, 1, 8):
            w[f"C4_t{t}_o{n_o}"] = Workload(
                f"llama70b_decode_t{t}_o{n_o}",
                f"Llama-70B FFN decode, {t} tokens, {n_o} outlier columns", [
                    Linear("up_28672x8192", t, 8192, 28672, False, n_o, (30.0, 30.0), 6.0),
                    Linear("down_8192x28672", t, 28672, 8192, False, n_o, (30.0, 30.0), 6.0)])
    for frac in (0.0, 0.001, 0.01, 0.05):
        for thr in (0.0, 6.0):
            n_o = round(frac * 5120)
            w[f"C5_f{frac}_t{thr:g}"] = Workload(
                f"llama13b_mlp_f{frac}_t{thr:g}",
                f"Llama-13B MLP 2048x5120 -> 13824, outlier fraction {frac}, threshold {thr:g}", [
                    Linear("mlp", 2048, 5120, 13824, False, n_o, (6.0, 80.0), thr)])
    return w


def layer_inputs(wl_seed: int, layer_idx: int, L: Linear):
    """Seeded (X, outlier cols, W, bias) for one layer of a workload."""
    s = BASE_SEED + 97 * wl_seed + 7 * layer_idx
    X, cols = activation(s, L.M, L.K, L.n_out, L.mag) if L.x_from is None else (None, None)
    W = weight(s + 1, L.N, L.K)
    b = bias(s + 2, L.N) if L.has_bias else None
    return X, cols, W, b


def seed_of(key: str) -> int:
    """Stable small integer per workload key."""
    return sum((i + 1) * ord(c) for i, c in enumerate(key)) % 10007
