"""Seeded synthetic inputs for XAttention block-sparse prefill attention.

This module is shared by the CPU oracle (tests) and the CUDA path (tests, bench,
smoke). It holds only the input recipes: random draws, the structure each workload
plants into Q/K/V, and the fp32 -> bf16 rounding. It holds none of the method's
arithmetic (no scoring, no selection, no attention).

Workloads follow the shapes the XAttention pages name:
- Llama-3.1-8B: 32 query heads, head dim 128, grouped into 8 KV heads, prefill up
  to 128K/256K tokens (XAttention summary page, "Key results"; DuSA rebuttal,
  Response to Q1 and its Table R4-1 caption).
- A video DiT: non-causal attention over a frame x spatial-position token grid
  (XAttention summary page, "Key results" and "Limitations", HunyuanVideo).

Recipes (plain readings of the workload descriptions):
- Q, K, V ~ N(0, 1) in fp32, rounded once to bf16 (round to nearest even).
- "Shared unit direction" u = g/|g|, g ~ N(0, I_C), one per KV head; every query
  head of the group uses its KV head's u. q_i += 1.0*u for every token i;
  k_j += 3.0*u only at the heavy positions (token 0 plus n_heavy-1 positions
  drawn uniformly without replacement from 1..M-1).
- Slash term: 64 vectors r_0..r_63 ~ N(0, I_C), one set shared by all heads;
  q_i += 0.5*r_(i mod 64), k_j += 0.5*r_(j mod 64).
- Video grid: token index = t*frame_tokens + s; per head, per-frame vectors
  f_t ~ 0.7*N(0, I_C) and per-position vectors p_s ~ 0.7*N(0, I_C), added to both
  q and k of that token.
- Per-head thresholds: tau_h ~ U[lo, hi], one per query head, from its own stream.

Every array is drawn from its own counter-keyed numpy Generator
(SeedSequence([seed, stream, index])), so any single head can be regenerated
without drawing the others, and the bits never depend on which side asks.
"""
from __future__ import annotations

import concurrent.futures
import dataclasses
import os
from typing import Optional

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "workload", "bf16_round", "bf16_bits_to_f32",
    "head_inputs", "layer_inputs", "tau_vector", "DEFAULT_SEED",
]

DEFAULT_SEED = 1234

# stream identifiers for SeedSequence keys
_S_Q, _S_K, _S_V, _S_U, _S_HEAVY, _S_SLASH, _S_VIDEO, _S_TAU = range(1, 9)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    M: int
    C: int
    causal: bool
    stride: int
    block: int = 128
    tau: float = 0.9                  # used when tau_range is None
    tau_range: Optional[tuple] = None  # per-head U[lo, hi]
    n_heavy: int = 0                  # heavy key tokens per KV head (0: none)
    q_shift: float = 1.0              # q_i += q_shift*u
    k_shift: float = 3.0              # k_heavy += k_shift*u
    slash: bool = False               # add the period-64 slash term
    slash_scale: float = 0.5
    slash_period: int = 64
    video: bool = False               # frame x position structure
    frame_tokens: int = 4096
    video_scale: float = 0.7

    @property
    def nb(self) -> int:
        return self.M // self.block

    @property
    def group(self) -> int:
        return self.Hq // self.Hkv

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS = {
    # 1 head, M=2048, C=64, 16 heavy tokens, causal, S=8, tau=0.9
    "tiny_1h_2k": Workload("tiny_1h_2k", B=1, Hq=1, Hkv=1, M=2048, C=64,
                           causal=True, stride=8, tau=0.9, n_heavy=16),
    # Llama-3.1-8B-shaped GQA prefill at 32K
    "llama8b_gqa_32k": Workload("llama8b_gqa_32k", B=1, Hq=32, Hkv=8, M=32768, C=128,
                                causal=True, stride=8, tau=0.9, n_heavy=64, slash=True),
    # the same at 128K; the stride sweep uses stride in {4, 8, 16}
    "llama8b_gqa_128k": Workload("llama8b_gqa_128k", B=1, Hq=32, Hkv=8, M=131072, C=128,
                                 causal=True, stride=8, tau=0.9, n_heavy=64, slash=True),
    # the same at 256K with per-head tau ~ U[0.80, 0.95]
    "llama8b_gqa_256k": Workload("llama8b_gqa_256k", B=1, Hq=32, Hkv=8, M=262144, C=128,
                                 causal=True, stride=8, tau_range=(0.80, 0.95),
                                 n_heavy=64, slash=True),
    # video DiT: 24 heads, 29 frames x 4096 positions = 118784 tokens, non-causal
    "video_dit_118k": Workload("video_dit_118k", B=1, Hq=24, Hkv=24, M=118784, C=128,
                               causal=False, stride=8, tau=0.95, video=True),
}


def workload(name: str, **overrides) -> Workload:
    w = WORKLOADS[name]
    return w.with_(**overrides) if overrides else w


def _rng(seed: int, stream: int, index: int = 0, sub: int = 0) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, stream, index, sub])))


def bf16_round(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest, ties to even."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    bias = ((u >> 16) & 1) + np.uint32(0x7FFF)
    return ((u + bias) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def _unit(rng: np.random.Generator, C: int) -> np.ndarray:
    g = rng.standard_normal(C)
    return (g / np.linalg.norm(g)).astype(np.float32)


def _heavy_positions(w: Workload, seed: int, kv: int, b: int) -> np.ndarray:
    rng = _rng(seed, _S_HEAVY, kv, b)
    rest = rng.choice(np.arange(1, w.M), size=w.n_heavy - 1, replace=False)
    return np.concatenate([[0], np.sort(rest)]).astype(np.int64)


def _slash(w: Workload, seed: int) -> np.ndarray:
    return _rng(seed, _S_SLASH).standard_normal((w.slash_period, w.C), dtype=np.float32)


def _video_terms(w: Workload, seed: int, h: int, b: int):
    rng = _rng(seed, _S_VIDEO, h, b)
    frames = -(-w.M // w.frame_tokens)
    f = rng.standard_normal((frames, w.C), dtype=np.float32) * np.float32(w.video_scale)
    p = rng.standard_normal((w.frame_tokens, w.C), dtype=np.float32) * np.float32(w.video_scale)
    return f, p


def _add_video(x: np.ndarray, f: np.ndarray, p: np.ndarray, frame_tokens: int) -> None:
    M = x.shape[0]
    for t in range(f.shape[0]):
        lo, hi = t * frame_tokens, min(M, (t + 1) * frame_tokens)
        x[lo:hi] += f[t]
        x[lo:hi] += p[: hi - lo]


def _add_slash(x: np.ndarray, r: np.ndarray, scale: float) -> None:
    M, P = x.shape[0], r.shape[0]
    rs = (np.float32(scale) * r).astype(np.float32)
    full = M // P
    x[: full * P] += np.tile(rs, (full, 1))
    if M % P:
        x[full * P:] += rs[: M % P]


def kv_head_inputs(w: Workload, kv: int, b: int = 0, seed: int = DEFAULT_SEED):
    """(K, V) for one KV head as bf16 bits, each [M, C] uint16."""
    k = _rng(seed, _S_K, kv, b).standard_normal((w.M, w.C), dtype=np.float32)
    v = _rng(seed, _S_V, kv, b).standard_normal((w.M, w.C), dtype=np.float32)
    if w.n_heavy:
        u = _unit(_rng(seed, _S_U, kv, b), w.C)
        k[_heavy_positions(w, seed, kv, b)] += np.float32(w.k_shift) * u
    if w.slash:
        _add_slash(k, _slash(w, seed), w.slash_scale)
    if w.video:
        f, p = _video_terms(w, seed, kv, b)
        _add_video(k, f, p, w.frame_tokens)
    return bf16_round(k), bf16_round(v)


def q_head_inputs(w: Workload, h: int, b: int = 0, seed: int = DEFAULT_SEED):
    """Q for one query head as bf16 bits, [M, C] uint16."""
    q = _rng(seed, _S_Q, h, b).standard_normal((w.M, w.C), dtype=np.float32)
    kv = h // w.group
    if w.n_heavy:
        u = _unit(_rng(seed, _S_U, kv, b), w.C)
        q += np.float32(w.q_shift) * u
    if w.slash:
        _add_slash(q, _slash(w, seed), w.slash_scale)
    if w.video:
        f, p = _video_terms(w, seed, kv, b)
        _add_video(q, f, p, w.frame_tokens)
    return bf16_round(q)


def head_inputs(w: Workload, h: int, b: int = 0, seed: int = DEFAULT_SEED):
    """(q, k, v) bf16 bits for query head h of batch b; k/v are its KV head's."""
    k, v = kv_head_inputs(w, h // w.group, b, seed)
    return q_head_inputs(w, h, b, seed), k, v


def layer_inputs(w: Workload, seed: int = DEFAULT_SEED, out=None, heads=None, threads=None):
    """Full (Q, K, V) bf16 bits: Q [B,Hq,M,C], K/V [B,Hkv,M,C] (uint16).

    `out` may hold three preallocated uint16 arrays (e.g. pinned host memory
    viewed through numpy) to fill in place. `heads` = (kv_lo, kv_hi) generates only
    the KV heads kv_lo..kv_hi-1 and their query heads (the arrays then hold those
    heads only, in order); every head is drawn from its own keyed stream, so a
    slice has the same bits as the same heads of the whole layer. Heads are drawn
    on `threads` host threads (default: the cores this process may use); the bits
    do not depend on it.
    """
    kv_lo, kv_hi = (0, w.Hkv) if heads is None else heads
    g = w.group
    nkv, nq = kv_hi - kv_lo, (kv_hi - kv_lo) * g
    if out is None:
        Q = np.empty((w.B, nq, w.M, w.C), np.uint16)
        K = np.empty((w.B, nkv, w.M, w.C), np.uint16)
        V = np.empty((w.B, nkv, w.M, w.C), np.uint16)
    else:
        Q, K, V = out

    def kv_job(b, kv):
        K[b, kv - kv_lo], V[b, kv - kv_lo] = kv_head_inputs(w, kv, b, seed)

    def q_job(b, h):
        Q[b, h - kv_lo * g] = q_head_inputs(w, h, b, seed)

    jobs = [(kv_job, b, kv) for b in range(w.B) for kv in range(kv_lo, kv_hi)] + \
        [(q_job, b, h) for b in range(w.B) for h in range(kv_lo * g, kv_hi * g)]
    n = threads or max(1, min(16, len(os.sched_getaffinity(0))))
    if n == 1:
        for f, b, i in jobs:
            f(b, i)
    else:
        with concurrent.futures.ThreadPoolExecutor(n) as ex:
            for fut in [ex.submit(f, b, i) for f, b, i in jobs]:
                fut.result()
    return Q, K, V


def tau_vector(w: Workload, seed: int = DEFAULT_SEED) -> np.ndarray:
    """Per-query-head thresholds, fp32 [Hq]."""
    if w.tau_range is None:
        return np.full(w.Hq, w.tau, np.float32)
    lo, hi = w.tau_range
    return np.array([_rng(seed, _S_TAU, h).uniform(lo, hi) for h in range(w.Hq)], np.float32)
