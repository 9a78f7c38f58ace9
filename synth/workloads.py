"""Seeded synthetic workloads for causal IVF top-k selection.

This module only draws random inputs: keys, queries, head weights and
encoder weights.  It holds none of the selection arithmetic, so both the
CPU oracle and the CUDA path may use it without sharing any method code.

Key/query model (the evaluation sets and model weights of the AttentionIndex
paper are not available; these inputs stand in for them):

* M mixture centres mu_j ~ N(0, I_d).
* Key at position p: a centre j drawn uniformly from the active set
  A(p) = {(floor(p*M/L) + i) mod M : i < M/4}, plus 0.3 * N(0, I_d).  The
  active set drifts slowly with position, so keys that are close in position
  tend to be close in content but not always.
* Query head q_{t,h} = sum_{r<3} alpha_r mu_{j_r} + 0.3 * N(0, I_d) with
  alpha ~ Dirichlet(1,1,1) and j_r uniform over all M centres, so that old
  keys stay relevant at long range.
* Head weights w_{t,h} ~ N(0, 1) * w_scale.

Every chunk of keys and queries is drawn from its own sub-seed, so position
p has the same key no matter how the prefix is split into chunks.
"""
from __future__ import annotations

import dataclasses
import math

import numpy as np

GEN_CHUNK = 8192  # positions per generator sub-seed


@dataclasses.dataclass(frozen=True)
class Workload:
    """One synthetic causal-prefill workload (all sizes in tokens)."""

    name: str
    L: int            # prefix length (keys)
    T: int            # queries per prefill chunk
    d: int            # key / query head dimension
    H: int            # indexer heads
    M: int            # mixture components
    w_scale: float    # head-weight std
    k: int            # top-k
    n_sinks: int      # S
    window: int       # W
    clusters_per_window: int  # m
    refit_period: int  # R (0 = never)
    budget: int       # C
    key_dtype: str    # "fp32" | "bf16" | "fp8"
    q_dtype: str      # "fp32" | "bf16"
    seed: int = 0
    refit_new_seeds: int = 0      # 0 -> R*m/W
    refit_seed_window: int = 0    # 0 -> R
    seal_iters: int = 10
    encoder: str = "none"         # "none" | "random" | "zero_out"
    block_routing: bool = False   # contiguous-block baseline instead of the IVF index

    @property
    def n_chunks(self) -> int:
        return self.L // self.T


# Workloads by what they are (sizes in the name).
WORKLOADS = {
    "tiny_fp32_L4k": Workload(
        name="tiny_fp32_L4k", L=4096, T=512, d=32, H=4, M=64, w_scale=0.5,
        k=64, n_sinks=4, window=256, clusters_per_window=8, refit_period=2048,
        budget=1024, key_dtype="fp32", q_dtype="fp32"),
    "glm_bf16_L128k": Workload(
        name="glm_bf16_L128k", L=131072, T=8192, d=128, H=32, M=4096,
        w_scale=1.0 / math.sqrt(32), k=2048, n_sinks=4, window=1024,
        clusters_per_window=8, refit_period=16384, budget=8192,
        key_dtype="bf16", q_dtype="bf16"),
    "v4flash_fp8_L256k": Workload(
        name="v4flash_fp8_L256k", L=262144, T=8192, d=128, H=64, M=4096,
        w_scale=1.0 / math.sqrt(64), k=2048, n_sinks=4, window=1024,
        clusters_per_window=8, refit_period=16384, budget=8192,
        key_dtype="fp8", q_dtype="bf16"),
    # indexed by the regular seal/refit schedule (~128 keys per cluster); the
    # extra timed refit over the whole prefix takes 64 seeds from the last
    # 16384 keys (bench.py --refit-overlap)
    "glm_bf16_L1m": Workload(
        name="glm_bf16_L1m", L=1048576, T=8192, d=128, H=32, M=4096,
        w_scale=1.0 / math.sqrt(32), k=2048, n_sinks=4, window=1024,
        clusters_per_window=8, refit_period=16384, budget=8192,
        key_dtype="bf16", q_dtype="bf16"),
    "glm_bf16_L128k_encoder": Workload(
        name="glm_bf16_L128k_encoder", L=131072, T=8192, d=128, H=32, M=4096,
        w_scale=1.0 / math.sqrt(32), k=2048, n_sinks=4, window=1024,
        clusters_per_window=8, refit_period=16384, budget=8192,
        key_dtype="bf16", q_dtype="bf16", encoder="random"),
}


def scaled(wl: Workload, **kw) -> Workload:
    """A copy of a workload with some fields replaced (smaller test cases)."""
    return dataclasses.replace(wl, **kw)


def _rng(seed: int, tag: int, idx: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64([seed, tag, idx]))


def centres(wl: Workload) -> np.ndarray:
    return _rng(wl.seed, 1, 0).standard_normal((wl.M, wl.d))


def _keys_block(wl: Workload, mu: np.ndarray, b: int) -> np.ndarray:
    p0 = b * GEN_CHUNK
    n = min(GEN_CHUNK, wl.L - p0)
    g = _rng(wl.seed, 2, b)
    pos = np.arange(p0, p0 + n, dtype=np.int64)
    base = (pos * wl.M) // wl.L
    off = g.integers(0, max(1, wl.M // 4), size=n)
    comp = (base + off) % wl.M
    return mu[comp] + 0.3 * g.standard_normal((n, wl.d))


def keys_f64(wl: Workload, p0: int = 0, p1: int | None = None) -> np.ndarray:
    """Keys at positions [p0, p1) in float64 (before any dtype cast)."""
    p1 = wl.L if p1 is None else p1
    mu = centres(wl)
    out = np.empty((p1 - p0, wl.d))
    for b in range(p0 // GEN_CHUNK, (p1 + GEN_CHUNK - 1) // GEN_CHUNK):
        blk = _keys_block(wl, mu, b)
        lo = max(p0, b * GEN_CHUNK)
        hi = min(p1, b * GEN_CHUNK + blk.shape[0])
        out[lo - p0:hi - p0] = blk[lo - b * GEN_CHUNK:hi - b * GEN_CHUNK]
    return out


def _queries_block(wl: Workload, mu: np.ndarray, b: int):
    p0 = b * GEN_CHUNK
    n = min(GEN_CHUNK, wl.L - p0)
    g = _rng(wl.seed, 3, b)
    comp = g.integers(0, wl.M, size=(n, wl.H, 3))
    alpha = g.dirichlet(np.ones(3), size=(n, wl.H))
    q = np.einsum("thr,thrd->thd", alpha, mu[comp])
    q += 0.3 * g.standard_normal((n, wl.H, wl.d))
    w = g.standard_normal((n, wl.H)) * wl.w_scale
    return q, w


def queries_f64(wl: Workload, p0: int, p1: int):
    """Queries [p1-p0, H, d] and head weights [p1-p0, H] in float64."""
    mu = centres(wl)
    q = np.empty((p1 - p0, wl.H, wl.d))
    w = np.empty((p1 - p0, wl.H))
    for b in range(p0 // GEN_CHUNK, (p1 + GEN_CHUNK - 1) // GEN_CHUNK):
        qb, wb = _queries_block(wl, mu, b)
        lo = max(p0, b * GEN_CHUNK)
        hi = min(p1, b * GEN_CHUNK + qb.shape[0])
        q[lo - p0:hi - p0] = qb[lo - b * GEN_CHUNK:hi - b * GEN_CHUNK]
        w[lo - p0:hi - p0] = wb[lo - b * GEN_CHUNK:hi - b * GEN_CHUNK]
    return q, w


def encoder_weights(wl: Workload, zero_out: bool = False) -> dict:
    """Seeded random weights of the representative-correction encoder.

    PyTorch-default-style uniform(+-1/sqrt(fan_in)) init.  Shapes:
    A [d,d], a [d] (phi layer), B1 [d, 3d+1], b1 [d], B2 [d,d], b2 [d].
    With zero_out the output layer (B2, b2) is zero.
    """
    d = wl.d
    g = _rng(wl.seed, 4, 0)

    def u(shape, fan_in):
        bound = 1.0 / math.sqrt(fan_in)
        return g.uniform(-bound, bound, size=shape)

    wts = {
        "A": u((d, d), d), "a": u((d,), d),
        "B1": u((d, 3 * d + 1), 3 * d + 1), "b1": u((d,), 3 * d + 1),
        "B2": u((d, d), d), "b2": u((d,), d),
    }
    if zero_out:
        wts["B2"] = np.zeros((d, d))
        wts["b2"] = np.zeros((d,))
    # stored as float32: that is what the library is given
    return {k: v.astype(np.float32) for k, v in wts.items()}


# ---- dtype casts (storage formats only; no method arithmetic) -------------

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """float -> bfloat16 bit patterns (uint16), round to nearest even.

    Goes through float32 first (the generator's draws are float64; the
    caller's tensors are produced in float32 and then cast, as a model
    would)."""
    f = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (f >> 16) & 1
    r = (f + np.uint32(0x7FFF) + lsb) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    return (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
