"""Seeded synthetic workloads for block-draft verification.

This module only draws inputs; it holds no step of the verification method.
It is the one piece shared by the CUDA path's tests/benchmark and the CPU
oracle's tests, so both always see bit-identical inputs.

The five workloads stand in for Qwen3-4B/8B verify steps at concurrency
8-64 (Qwen3 vocabulary of 151,936 entries, draft block of 16): logits are
Gaussian with a few peaked tokens, drafts are the target plus Gaussian
noise, survival scores are Beta(6, 2) sorted descending per request. No
dataset or trained weight is reproduced.

Recipe. numpy SeedSequence([seed, config id]) is split into eight child
streams, one per component, so each component can be drawn request by
request without holding fp64 copies of a whole tensor:
  0 target normals, 1 peak indices, 2 draft noise, 3 mixture weights,
  4 survival scores, 5 uniforms u, 6 Gumbel noise g, 7 draft-token noise.
Normals are drawn in float32; bf16 logits are the round-to-nearest-even
bf16 of the float32 value and are stored as their uint16 bit patterns.
Draft logits are built from the stored (already rounded) target values.
Gumbel noise is g = -log(-log U), U uniform in (0, 1), computed in float64
and stored as float32. Drafted tokens are sampled from the proposal the
verifier sees by Gumbel-max over the stored draft logits / T (for a latent
mixture: first z by Gumbel-max over log q(z|y), then every position from
branch z), with stream 7.
"""
from dataclasses import dataclass, field
from functools import lru_cache
from typing import Optional

import numpy as np

V_QWEN3 = 151936


@dataclass(frozen=True)
class Workload:
    cid: int
    name: str
    B: int
    L: int
    V: int
    K: int
    T: float
    dtype: str                 # "bf16" or "f32"
    target_sigma: float
    n_peaks: int
    peak: float
    draft_sigma: float
    budget: Optional[int] = None   # DVL budget (None: dense verify of all L positions)


WORKLOADS = {
    1: Workload(1, "tiny B2 L4 V64 K1 f32", 2, 4, 64, 1, 1.0, "f32", 2.0, 0, 0.0, 0.5),
    2: Workload(2, "block B8 L16 V151936 K1 bf16", 8, 16, V_QWEN3, 1, 1.0, "bf16", 1.0, 32, 8.0, 1.0),
    3: Workload(3, "mixture B32 L16 V151936 K4 bf16 T1.5", 32, 16, V_QWEN3, 4, 1.5, "bf16", 0.7, 8, 4.0, 1.5),
    4: Workload(4, "dvl B32 L16 V151936 K1 bf16 budget272", 32, 16, V_QWEN3, 1, 1.0, "bf16", 1.0, 32, 8.0, 1.0,
                budget=272),
    5: Workload(5, "stress B64 L16 V151936 K4 bf16 budget544", 64, 16, V_QWEN3, 4, 1.0, "bf16", 1.0, 32, 8.0, 2.0,
                budget=544),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return uint16 bit patterns."""
    b = np.ascontiguousarray(x, np.float32).view(np.uint32)
    b = b + (((b >> 16) & np.uint32(1)) + np.uint32(0x7FFF))
    return (b >> 16).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.ascontiguousarray(h, np.uint16).astype(np.uint32) << 16).view(np.float32)


def gumbel(rng: np.random.Generator, shape) -> np.ndarray:
    """Standard Gumbel noise in float64: -log(-log U) with U in (0, 1)."""
    u = rng.random(shape) + 2.0 ** -54
    return -np.log(-np.log(u))


@dataclass
class Inputs:
    w: Workload
    target: np.ndarray                 # [B, L+1, V] (uint16 bf16 bits or float32)
    draft: np.ndarray                  # [B, L, V] if K == 1 else [B, K, L, V]
    tokens: np.ndarray                 # [B, L] int32
    u: np.ndarray                      # [B, L] float32 in [0, 1)
    g: np.ndarray                      # [B, L+1, V] float32
    mix_w: Optional[np.ndarray] = None     # [B, K] float32
    scores: Optional[np.ndarray] = None    # [B, L] float32
    extra: dict = field(default_factory=dict)


def _streams(seed: int, cid: int):
    ss = np.random.SeedSequence([int(seed), int(cid)])
    return [np.random.default_rng(c) for c in ss.spawn(8)]


def make_inputs(w: Workload, seed: int = 0) -> Inputs:
    """Draw every input of workload `w` from `seed` (see the module recipe)."""
    rt, rp, rd, rw, rs, ru, rg, rx = _streams(seed, w.cid)
    B, L, V, K = w.B, w.L, w.V, w.K
    bf16 = w.dtype == "bf16"
    st = np.uint16 if bf16 else np.float32
    target = np.empty((B, L + 1, V), st)
    draft = np.empty((B, L, V) if K == 1 else (B, K, L, V), st)
    tokens = np.empty((B, L), np.int32)
    g = np.empty((B, L + 1, V), np.float32)

    mix_w = None
    if K > 1:
        a = rw.standard_normal((B, K))
        e = np.exp(a - a.max(axis=1, keepdims=True))
        mix_w = (e / e.sum(axis=1, keepdims=True)).astype(np.float32)
    scores = None
    if w.budget is not None:
        scores = -np.sort(-rs.beta(6.0, 2.0, size=(B, L)), axis=1).astype(np.float32)
    u = ru.random((B, L), dtype=np.float32)

    for b in range(B):
        t = rt.standard_normal((L + 1, V), dtype=np.float32) * np.float32(w.target_sigma)
        for i in range(L + 1):
            if w.n_peaks:
                t[i, rp.choice(V, size=w.n_peaks, replace=False)] += np.float32(w.peak)
        if bf16:
            target[b] = f32_to_bf16_bits(t)
            tv = bf16_bits_to_f32(target[b])
        else:
            target[b] = t
            tv = t
        branches = np.empty((K, L, V), np.float32)
        for z in range(K):
            d = tv[:L] + rd.standard_normal((L, V), dtype=np.float32) * np.float32(w.draft_sigma)
            if bf16:
                hb = f32_to_bf16_bits(d)
                branches[z] = bf16_bits_to_f32(hb)
                if K == 1:
                    draft[b] = hb
                else:
                    draft[b, z] = hb
            else:
                branches[z] = d
                if K == 1:
                    draft[b] = d
                else:
                    draft[b, z] = d
        g[b] = gumbel(rg, (L + 1, V)).astype(np.float32)
        # drafter's sample of the block from the proposal the verifier sees
        zb = 0
        if K > 1:
            zb = int(np.argmax(np.log(mix_w[b].astype(np.float64)) + gumbel(rx, K)))
        for i in range(L):
            tokens[b, i] = int(np.argmax(branches[zb, i].astype(np.float64) / w.T + gumbel(rx, V)))
    return Inputs(w, target, draft, tokens, u, g, mix_w, scores)


@lru_cache(maxsize=2)
def workload_inputs(cid: int, seed: int = 0) -> Inputs:
    """Cached make_inputs for one of the five named workloads."""
    return make_inputs(WORKLOADS[cid], seed)


def custom(B, L, V, K=1, T=1.0, dtype="bf16", target_sigma=1.0, n_peaks=0, peak=0.0, draft_sigma=1.0,
           budget=None, seed=0, cid=100) -> Inputs:
    """Inputs for an arbitrary shape with the same recipe (tests and edge cases)."""
    return make_inputs(Workload(cid, "custom", B, L, V, K, T, dtype, target_sigma, n_peaks, peak,
                                draft_sigma, budget), seed)
