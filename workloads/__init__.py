"""Seeded synthetic decode workloads for COBS block-sparse attention.

This module only draws numbers: keys, values and queries with the shapes,
value distributions and structure of the long-context decode settings the
COBS explainer (gist.science paper 2607.09052, §4.1: 32k retrieval with
planted "needles") talks about.  It holds none of the method's arithmetic and
is the one module that both the oracle tests and the CUDA tests/bench read.

Stand-in note: the pages measure retrieval quality on the 32k RULER suite.
That suite is not used or reproduced here; the "needle" recipe below only
mimics its shape (a few keys aligned with the query hidden in wide blocks).

All arrays of bf16 values are returned as their raw uint16 bit patterns
(round-to-nearest-even from fp32), the exact bytes uploaded to the GPU; the
oracle widens the same bits to fp64 with :func:`bits_to_f64`.
"""

from __future__ import annotations

import dataclasses
import math
from dataclasses import dataclass

import numpy as np

__all__ = [
    "Workload", "WORKLOADS", "workload", "to_bf16_bits", "bits_to_f64",
    "make_queries", "make_kv_slice", "make_kv", "needle_blocks",
]

_TAG_K, _TAG_V, _TAG_Q, _TAG_BLOCKS = 1, 2, 3, 4


@dataclass(frozen=True)
class Workload:
    """One synthetic decode setting.  Sizes are tokens unless stated."""
    name: str
    batch: int
    q_heads: int
    kv_heads: int
    head_dim: int
    seq_len: int
    block: int = 64
    rank: int = 8
    top_k: int = 16
    sink_blocks: int = 1
    local_tokens: int = 512
    keys: str = "tight_spread"       # offset_scale | tight_spread | lowrank16
    values: str = "normal"           # normal | offset_scale
    needles: int = 0                 # planted query-aligned keys per (b, kv-head)
    capacity: int = 0                # cache capacity; 0 -> seq_len rounded up
    append_chunk: int = 0            # tokens per append (stats built per chunk)
    decode_steps: int = 1            # query sets (step t is seeded by t)
    seed: int = 0

    @property
    def group(self) -> int:
        return self.q_heads // self.kv_heads

    @property
    def cap(self) -> int:
        if self.capacity:
            return self.capacity
        return -(-self.seq_len // self.block) * self.block

    def scaled(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five settings the hot path is measured and checked on.
WORKLOADS = {
    # Tiny decode step (parity in seconds on the CPU).
    "tiny_4k": Workload("tiny_4k", batch=1, q_heads=4, kv_heads=1, head_dim=64,
                        seq_len=4096, rank=4, top_k=8, sink_blocks=1,
                        local_tokens=64, keys="offset_scale",
                        values="offset_scale"),
    # One layer, one sequence, 32k context.
    "single_32k": Workload("single_32k", batch=1, q_heads=16, kv_heads=4,
                           head_dim=128, seq_len=32768, rank=8, top_k=16,
                           local_tokens=512),
    # Batched 32k decode with planted needles (the throughput workload).
    "batched_needles_32k": Workload("batched_needles_32k", batch=32, q_heads=32,
                                    kv_heads=8, head_dim=128, seq_len=32768,
                                    rank=8, top_k=16, local_tokens=512,
                                    needles=4),
    # 128k context, keys from per-block rank-16 Gaussians.
    "long_128k": Workload("long_128k", batch=8, q_heads=32, kv_heads=8,
                          head_dim=128, seq_len=131072, rank=16, top_k=32,
                          local_tokens=1024, keys="lowrank16"),
    # 256k context built by 4096-token appends, then 64 decode steps.
    "build_256k": Workload("build_256k", batch=1, q_heads=64, kv_heads=8,
                           head_dim=128, seq_len=262144, rank=16, top_k=64,
                           local_tokens=1024, append_chunk=4096,
                           decode_steps=64),
}


def workload(name: str) -> Workload:
    return WORKLOADS[name]


# ---------------------------------------------------------------------------
# bf16 bit patterns
# ---------------------------------------------------------------------------

def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bits, round to nearest even (finite inputs only)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    u = u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))
    return (u >> np.uint32(16)).astype(np.uint16)


def bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """bf16 bits -> the exact values as fp64."""
    u = np.ascontiguousarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return u.view(np.float32).astype(np.float64)


def _rng(w: Workload, tag: int, *idx: int) -> np.random.Generator:
    return np.random.default_rng(np.random.SeedSequence([w.seed, tag, *idx]))


# ---------------------------------------------------------------------------
# Queries
# ---------------------------------------------------------------------------

def make_queries(w: Workload, step: int = 0) -> np.ndarray:
    """q ~ N(0, 1), [batch, q_heads, head_dim] bf16 bits; step t seeded by t."""
    g = _rng(w, _TAG_Q, step)
    q = g.standard_normal((w.batch, w.q_heads, w.head_dim), dtype=np.float32)
    return to_bf16_bits(q)


# ---------------------------------------------------------------------------
# Keys and values of one (batch, kv-head) slice
# ---------------------------------------------------------------------------

def needle_blocks(w: Workload, b: int, h: int, spread: np.ndarray) -> np.ndarray:
    """Blocks that receive a needle: distinct spread blocks away from the
    first ``sink_blocks`` blocks and from the last ``local_tokens`` tokens."""
    hi = max(0, w.seq_len - w.local_tokens) // w.block - 1
    pool = [j for j in range(w.sink_blocks, max(w.sink_blocks, hi))
            if spread[j]]
    g = _rng(w, _TAG_BLOCKS, b, h)
    if len(pool) < w.needles:
        raise ValueError("not enough spread blocks for the needles")
    return np.sort(g.choice(np.asarray(pool), size=w.needles, replace=False))


def needle_block_list(w: Workload, b: int, h: int) -> np.ndarray:
    """The blocks that make_kv_slice plants needles in for slice (b, h),
    without drawing the keys: the same generator replays only the draws that
    decide them (the block means, then the spread flags of the tight/spread
    recipe), which must stay in step with _per_block."""
    if not w.needles or w.keys != "tight_spread":
        return np.zeros(0, np.int64)
    n_blocks = -(-w.seq_len // w.block)
    gk = _rng(w, _TAG_K, b, h)
    gk.standard_normal((n_blocks, 1, w.head_dim), dtype=np.float32)   # block means
    spread = gk.random(n_blocks) < 0.5
    return needle_blocks(w, b, h, spread)


def _per_block(g, n_blocks, B, d, recipe):
    """Draw [n_blocks * B, d] fp32 values for one recipe (plus spread flags)."""
    if recipe == "offset_scale":
        off = 0.5 * g.standard_normal((n_blocks, 1, d), dtype=np.float32)
        sc = g.uniform(0.3, 2.0, size=(n_blocks, 1, 1)).astype(np.float32)
        z = g.standard_normal((n_blocks, B, d), dtype=np.float32)
        return (off + sc * z).reshape(n_blocks * B, d), np.zeros(n_blocks, bool)
    if recipe == "tight_spread":
        mean = 0.5 * g.standard_normal((n_blocks, 1, d), dtype=np.float32)
        spread = g.random(n_blocks) < 0.5
        std = np.where(spread, 1.0, 0.5).astype(np.float32)[:, None, None]
        z = g.standard_normal((n_blocks, B, d), dtype=np.float32)
        return (mean + std * z).reshape(n_blocks * B, d), spread
    if recipe == "lowrank16":
        mean = 0.5 * g.standard_normal((n_blocks, 1, d), dtype=np.float32)
        a = 0.5 * g.standard_normal((n_blocks, d, 16), dtype=np.float32)
        z = g.standard_normal((n_blocks, B, 16), dtype=np.float32)
        k = mean + np.einsum("nbr,ndr->nbd", z, a)
        return k.reshape(n_blocks * B, d), np.zeros(n_blocks, bool)
    if recipe == "normal":
        return (g.standard_normal((n_blocks * B, d), dtype=np.float32),
                np.zeros(n_blocks, bool))
    raise ValueError(f"unknown recipe {recipe!r}")


def make_kv_slice(w: Workload, b: int, h: int, q_bits: np.ndarray | None = None,
                  poison: str = "zero"):
    """K and V of one (batch b, kv-head h) slice: two [cap, d] bf16-bit arrays.

    Tokens in [seq_len, cap) hold ``poison`` ("zero", or "nan" to prove that
    nothing past the sequence is ever read into a result).  Needles need the
    group's step-0 queries (``q_bits`` [batch, q_heads, d]).
    """
    B, d, T, cap = w.block, w.head_dim, w.seq_len, w.cap
    n_blocks = -(-T // B)
    gk = _rng(w, _TAG_K, b, h)
    k, spread = _per_block(gk, n_blocks, B, d, w.keys)
    if w.needles:
        if q_bits is None:
            raise ValueError("needles need the queries")
        qg = bits_to_f64(q_bits[b, h * w.group:(h + 1) * w.group]).mean(axis=0)
        qhat = qg / np.linalg.norm(qg)
        for j in needle_blocks(w, b, h, spread):
            e = gk.standard_normal(d)
            e -= (e @ qhat) * qhat
            e /= np.linalg.norm(e)
            needle = math.sqrt(d) * (0.9 * qhat + math.sqrt(0.19) * e)
            t = j * B + int(gk.integers(B))
            delta = needle - k[t]
            rows = np.arange(j * B, (j + 1) * B)
            k[rows[rows != t]] -= (delta / (B - 1)).astype(np.float32)
            k[t] = needle.astype(np.float32)
    gv = _rng(w, _TAG_V, b, h)
    v, _ = _per_block(gv, n_blocks, B, d, w.values)

    kb = np.empty((cap, d), np.uint16)
    vb = np.empty((cap, d), np.uint16)
    kb[:T] = to_bf16_bits(k[:T])
    vb[:T] = to_bf16_bits(v[:T])
    fill = {"zero": 0, "nan": 0x7FC0}[poison]
    kb[T:] = fill
    vb[T:] = fill
    return kb, vb


def _slice_job(args):
    w, b, h, q_bits, poison = args
    return b, h, make_kv_slice(w, b, h, q_bits, poison)


def make_kv(w: Workload, q_bits: np.ndarray | None = None, poison: str = "zero",
            workers: int = 1):
    """Full caches [batch, kv_heads, cap, d] (bf16 bits) for K and V.

    ``workers`` > 1 draws slices in a spawn-started process pool (each slice
    has its own seed, so the bytes do not depend on the worker count).
    """
    K = np.empty((w.batch, w.kv_heads, w.cap, w.head_dim), np.uint16)
    V = np.empty_like(K)
    jobs = [(w, b, h, q_bits, poison) for b in range(w.batch)
            for h in range(w.kv_heads)]
    if workers > 1 and len(jobs) > 1:
        import multiprocessing as mp
        from concurrent.futures import ProcessPoolExecutor
        with ProcessPoolExecutor(max_workers=workers,
                                 mp_context=mp.get_context("spawn")) as ex:
            for b, h, (kb, vb) in ex.map(_slice_job, jobs, chunksize=1):
                K[b, h], V[b, h] = kb, vb
    else:
        for job in jobs:
            b, h, (kb, vb) = _slice_job(job)
            K[b, h], V[b, h] = kb, vb
    return K, V
