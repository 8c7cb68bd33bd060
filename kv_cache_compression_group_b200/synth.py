"""Seeded synthetic prefill caches shaped like the workloads the JoLT pages measure on.

The pages evaluate on real Mistral-7B-v0.3, LLaMA-2-13B and LLaMA-3.1-8B caches
("A JoLT for the KV Cache ... Joint Tucker and JL-Residual Allocation for LLMs",
introduction; "A JoLT for the KV cache: Near-Lossless KV Cache Compression via
Joint Rank-bit Allocation", abstract).  No weights or caches exist here, so these
generators stand in for them with the same shapes: every (layer, head) slice of
K or V is a decaying sum of random rank-one terms plus Gaussian noise, and the
key slices get per-channel lognormal outlier scales.

This module holds none of the compressor's arithmetic.  It is the one piece of
code that both the CUDA path's tests and the float64 checker consume, so that
the two see bit-identical inputs.
"""
from __future__ import annotations

import os
from concurrent.futures import ThreadPoolExecutor
from dataclasses import dataclass, asdict

import numpy as np
import torch


@dataclass(frozen=True)
class Workload:
    """Shape of one K (or V) cache tensor [n_layers, n_heads, T, D] plus the generator recipe."""

    name: str
    n_layers: int
    n_heads: int
    T: int
    D: int
    layers_per_group: int
    n_components: int      # rank-one terms per slice
    decay: float           # s_i = exp(-i / decay)
    noise: float           # additive N(0, noise^2)
    key_sigma: float       # key channel scales ~ lognormal(0, key_sigma)
    dtype: str             # "bf16" or "f32"

    def as_dict(self):
        return asdict(self)

    @property
    def n_groups(self) -> int:
        return self.n_layers // self.layers_per_group

    @property
    def elems(self) -> int:
        return self.n_layers * self.n_heads * self.T * self.D

    def bf16_bytes(self) -> int:
        """Bytes of K plus V if they were held in bf16 (the reference size for "x-fold")."""
        return 2 * 2 * self.elems

    def input_bytes(self) -> int:
        """Bytes of K plus V in their own dtype."""
        return 2 * self.elems * (2 if self.dtype == "bf16" else 4)


WORKLOADS = {
    # one layer group, fp32, the size the float64 checker runs in a blink
    "tiny": Workload("tiny", 2, 2, 64, 16, 2, 8, 2.0, 0.01, 0.5, "f32"),
    # Mistral-7B-v0.3: 32 layers, 8 KV heads (GQA), head_dim 128, 1024 tokens
    "mistral7b": Workload("mistral7b", 32, 8, 1024, 128, 4, 32, 8.0, 0.05, 1.0, "bf16"),
    # LLaMA-2-13B: 40 layers, 40 heads (MHA), 4096 tokens
    "llama2_13b": Workload("llama2_13b", 40, 40, 4096, 128, 4, 64, 16.0, 0.05, 1.0, "bf16"),
    # LLaMA-3.1-8B at 64K context (GQA)
    "llama31_8b_64k": Workload("llama31_8b_64k", 32, 8, 65536, 128, 4, 128, 32.0, 0.05, 1.0, "bf16"),
}


def sweep_workload(T: int) -> Workload:
    """Mistral-shaped generator at another context length (the compression-time sweep)."""
    w = WORKLOADS["mistral7b"]
    return Workload(f"mistral7b_T{T}", w.n_layers, w.n_heads, T, w.D, w.layers_per_group,
                    w.n_components, w.decay, w.noise, w.key_sigma, w.dtype)


def small_workload(base: str, n_layers: int | None = None, n_heads: int | None = None,
                   T: int | None = None, name: str | None = None) -> Workload:
    """A cut-down copy of a named workload (same recipe, fewer layers/heads/tokens)."""
    w = WORKLOADS[base]
    nl = w.n_layers if n_layers is None else n_layers
    nh = w.n_heads if n_heads is None else n_heads
    t = w.T if T is None else T
    return Workload(name or f"{base}_{nl}x{nh}x{t}", nl, nh, t, w.D, min(w.layers_per_group, nl),
                    w.n_components, w.decay, w.noise, w.key_sigma, w.dtype)


def slice_f64(w: Workload, seed: int, kv: int, layer: int, head: int) -> np.ndarray:
    """One (layer, head) slice, T x D, float64, before the cast to the storage dtype.

    Draw order inside the slice's own stream (seeded by [seed, kv, layer, head]):
    A (T x k), B (D x k), E (T x D), then, for keys only, the D channel scales.
    """
    rng = np.random.default_rng([seed, kv, layer, head])
    k = w.n_components
    a = rng.standard_normal((w.T, k))
    b = rng.standard_normal((w.D, k))
    e = rng.standard_normal((w.T, w.D))
    s = np.exp(-np.arange(k) / w.decay)
    x = (a * s) @ b.T + w.noise * e
    if kv == 0:
        x = x * rng.lognormal(0.0, w.key_sigma, w.D)[None, :]
    return x


def make_cache(w: Workload, seed: int = 0, kv: int | None = None, layers: range | None = None,
               workers: int | None = None):
    """K and V as CPU torch tensors [n_layers, H, T, D] in the workload's dtype.

    With ``kv`` given, returns only that tensor; with ``layers`` given, only those layers
    (the slices are drawn independently, so any sub-range is bit-identical to the same
    layers of the full tensor).  Slices are generated on ``workers`` threads (default: the
    CPUs this process may use); every slice has its own stream, so the result does not
    depend on the thread count.
    """
    tdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    lay = range(w.n_layers) if layers is None else layers
    if workers is None:
        workers = max(1, len(os.sched_getaffinity(0)))
    out = []
    for which in ((0, 1) if kv is None else (kv,)):
        t = torch.empty((len(lay), w.n_heads, w.T, w.D), dtype=tdt)

        def fill(job, which=which, t=t):
            li, layer, h = job
            x = slice_f64(w, seed, which, layer, h)
            t[li, h] = torch.from_numpy(x.astype(np.float32)).to(tdt)

        jobs = [(li, layer, h) for li, layer in enumerate(lay) for h in range(w.n_heads)]
        if workers > 1 and len(jobs) > 1:
            with ThreadPoolExecutor(workers) as ex:
                list(ex.map(fill, jobs))
        else:
            for j in jobs:
                fill(j)
        out.append(t)
    return tuple(out) if kv is None else out[0]


def to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact float64 copy of a bf16 / fp32 tensor (both embed exactly in float64)."""
    return t.to(torch.float64).numpy()
