"""Seeded synthetic workloads for the chunked H2O attention step.

This module only draws random inputs; it holds none of the method's
arithmetic.  The parity tests feed the same tensors to the CPU oracle and to
the CUDA path, and the benchmark uses the same distributions.

The shapes stand in for the long-context runs of *Learning how to Forget:
Fine-tuning for Long-Context Sparse Attention* (Qwen3-4B, Table 2; chunk sizes
1k/2k in Tables 1 and 5), whose Helmet datasets and weights are not available.
Inputs are i.i.d. N(0, 1) with "heavy-hitter" positions whose keys are shifted
by 3.0 along one fixed unit vector, so that some keys attract more attention.

Every (cache, chunk) pair has its own generator, seeded by mixing
(seed, cache index, chunk index) through ``numpy.random.SeedSequence``; so a
chunk of one cache can be regenerated on its own.  The exception is the
drifting-mean workload, whose random walk carries over chunk boundaries: a
``ChunkSource`` caches the walk state at each chunk start.
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass
from typing import Optional, Tuple

import numpy as np
import torch

HEAVY_SHIFT = 3.0


@dataclass(frozen=True)
class Workload:
    """One synthetic workload.

    ``batch`` counts independent caches (layers x sequences); all of them
    advance together, one chunk of ``chunk`` tokens per step.
    """

    name: str
    batch: int
    n_q_heads: int
    n_kv_heads: int
    head_dim: int
    chunk: int
    capacity: int
    window: int
    seq_len: int
    dtype: str                      # "bf16", "f32" or "q8" (int8 cache, bf16 activations)
    heavy_p: float = 0.02           # probability that a position is heavy
    heavy_p_range: Optional[Tuple[float, float]] = None  # per-chunk U[lo, hi]
    drift_step: float = 0.0         # norm of the per-token mean step of K
    layers: int = 1
    seqs: int = 1
    prefill_chunk: int = 0          # chunk of the filling steps (0: ``chunk``)
    policy: str = "h2o"             # eviction policy: "h2o", "lr" or "slr"
    sinks: int = 0                  # "slr": first positions that always stay

    @property
    def fill_chunk(self) -> int:
        return self.prefill_chunk or self.chunk

    @property
    def max_chunk(self) -> int:
        return max(self.chunk, self.fill_chunk)

    @property
    def steps(self) -> int:
        return self.seq_len // self.chunk

    @property
    def group(self) -> int:
        return self.n_q_heads // self.n_kv_heads

    def torch_dtype(self) -> torch.dtype:
        """Element type of q, k_new, v_new and out."""
        return torch.float32 if self.dtype == "f32" else torch.bfloat16

    def cache_dtype(self) -> torch.dtype:
        """The cache's element type as the binding names it (torch.int8: the
        int8 cache with per-row scales)."""
        return torch.int8 if self.dtype == "q8" else self.torch_dtype()

    def scaled(self, **changes) -> "Workload":
        """A copy with some fields replaced (used for scaled-down tests)."""
        return dataclasses.replace(self, **changes)


# The five workloads: a tiny fp32 case, two Qwen3-4B-shaped single caches,
# the 36-layer x 4-sequence stack, and the 1M-token streaming case.
TINY = Workload("tiny_gqa2_d64_f32_c256_q64", batch=1, n_q_heads=4, n_kv_heads=2,
                head_dim=64, chunk=64, capacity=256, window=0, seq_len=1024,
                dtype="f32", heavy_p=0.02)
QWEN_C8K = Workload("qwen3_4b_attn_c8192_q1024_w256", batch=1, n_q_heads=32,
                    n_kv_heads=8, head_dim=128, chunk=1024, capacity=8192,
                    window=256, seq_len=65536, dtype="bf16", heavy_p=0.02)
QWEN_C16K = Workload("qwen3_4b_attn_c16384_q2048_w512", batch=1, n_q_heads=32,
                     n_kv_heads=8, head_dim=128, chunk=2048, capacity=16384,
                     window=512, seq_len=131072, dtype="bf16",
                     heavy_p_range=(0.005, 0.05))
STACK36 = Workload("qwen3_4b_36layer_x4seq_c8192_q1024", batch=144,
                   n_q_heads=32, n_kv_heads=8, head_dim=128, chunk=1024,
                   capacity=8192, window=0, seq_len=32768, dtype="bf16",
                   heavy_p=0.02, layers=36, seqs=4)
STREAM1M = Workload("qwen3_4b_stream_1m_c32768_q1024_w1024", batch=1,
                    n_q_heads=32, n_kv_heads=8, head_dim=128, chunk=1024,
                    capacity=32768, window=1024, seq_len=1 << 20, dtype="bf16",
                    heavy_p=0.01, drift_step=0.01)

# Generation after a chunked prefill: one new token per cache and step (the
# decode step, n_q = 1), for one cache and for the 36-layer x 4-sequence stack.
# The cache is filled by prefill chunks of 1024 tokens.
DECODE_C8K = Workload("qwen3_4b_decode_c8192_w256", batch=1, n_q_heads=32,
                      n_kv_heads=8, head_dim=128, chunk=1, capacity=8192, window=256,
                      seq_len=8192 + 512, dtype="bf16", heavy_p=0.02, prefill_chunk=1024)
DECODE_STACK36 = Workload("qwen3_4b_decode_36layer_x4seq_c8192_w256", batch=144,
                          n_q_heads=32, n_kv_heads=8, head_dim=128, chunk=1,
                          capacity=8192, window=256, seq_len=8192 + 512, dtype="bf16",
                          heavy_p=0.02, layers=36, seqs=4, prefill_chunk=1024)

# The headline cache under the score-free policies (the summary page's
# lr-vs-h2o step-time comparison, Table 6): no summed weights are needed.
LR_C8K = dataclasses.replace(QWEN_C8K, name="qwen3_4b_lr_c8192_q1024_w256", policy="lr")
SLR_C8K = dataclasses.replace(QWEN_C8K, name="qwen3_4b_slr4_c8192_q1024_w256", policy="slr",
                              sinks=4)

# The headline cache quantised (Q-Hitter: H2O with an int8 cache, summary
# page Table 5's qh2o rows), and its decode step.
QH2O_C8K = dataclasses.replace(QWEN_C8K, name="qwen3_4b_qh2o_c8192_q1024_w256", dtype="q8")
QH2O_DECODE_C8K = dataclasses.replace(DECODE_C8K, name="qwen3_4b_qh2o_decode_c8192_w256",
                                      dtype="q8")

WORKLOADS = {w.name: w for w in (TINY, QWEN_C8K, QWEN_C16K, STACK36, STREAM1M, DECODE_C8K,
                                 DECODE_STACK36, LR_C8K, SLR_C8K, QH2O_C8K, QH2O_DECODE_C8K)}
ORDERED = [TINY, QWEN_C8K, QWEN_C16K, STACK36, STREAM1M, DECODE_C8K, DECODE_STACK36, LR_C8K,
           SLR_C8K, QH2O_C8K, QH2O_DECODE_C8K]


def _seed64(*words: int) -> int:
    ss = np.random.SeedSequence([int(w) & 0xFFFFFFFF for w in words])
    a, b = ss.generate_state(2, dtype=np.uint32)
    return (int(a) << 32 | int(b)) & ((1 << 63) - 1)


def _gen(seed: int, *words: int, device: str = "cpu") -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(_seed64(seed, *words))
    return g


def heavy_direction(wl: Workload, seed: int, b: int) -> torch.Tensor:
    """Fixed unit vector of cache b (shared by its KV heads)."""
    g = _gen(seed, 0x5EED, b)
    u = torch.randn(wl.head_dim, generator=g, dtype=torch.float64)
    return (u / u.norm()).to(torch.float32)


class ChunkSource:
    """Yields the (Q, K_new, V_new) chunks of one workload on the CPU.

    Shapes: Q ``[B, n_q, H_q, d]``, K_new and V_new ``[B, n_q, H_kv, d]``,
    in the workload's dtype.  ``n_q`` defaults to the workload's chunk.
    """

    def __init__(self, wl: Workload, seed: int = 0, batch: Optional[int] = None):
        self.wl = wl
        self.seed = seed
        self.batch = wl.batch if batch is None else batch
        self._u = [heavy_direction(wl, seed, b) for b in range(self.batch)]
        # drift state: mean of K per (b, kv head) at the start of chunk c
        self._mu = {0: torch.zeros(self.batch, wl.n_kv_heads, wl.head_dim)}

    def _drift_increments(self, b: int, c: int, n_q: int) -> torch.Tensor:
        g = _gen(self.seed, 0xD21F7, b, c)
        xi = torch.randn(n_q, self.wl.n_kv_heads, self.wl.head_dim, generator=g)
        return self.wl.drift_step * xi / xi.norm(dim=-1, keepdim=True)

    def _mu_at(self, c: int, n_q: int) -> torch.Tensor:
        last = max(k for k in self._mu if k <= c)
        mu = self._mu[last]
        for cc in range(last, c):
            inc = torch.stack([self._drift_increments(b, cc, n_q).sum(0)
                               for b in range(self.batch)])
            mu = mu + inc
            self._mu[cc + 1] = mu
        return mu

    def chunk(self, c: int, n_q: Optional[int] = None):
        wl = self.wl
        n_q = wl.chunk if n_q is None else n_q
        Q = torch.empty(self.batch, n_q, wl.n_q_heads, wl.head_dim)
        K = torch.empty(self.batch, n_q, wl.n_kv_heads, wl.head_dim)
        V = torch.empty_like(K)
        mu0 = self._mu_at(c, n_q) if wl.drift_step > 0 else None
        for b in range(self.batch):
            g = _gen(self.seed, b, c)
            Q[b] = torch.randn(n_q, wl.n_q_heads, wl.head_dim, generator=g)
            K[b] = torch.randn(n_q, wl.n_kv_heads, wl.head_dim, generator=g)
            V[b] = torch.randn(n_q, wl.n_kv_heads, wl.head_dim, generator=g)
            p = wl.heavy_p
            if wl.heavy_p_range is not None:
                lo, hi = wl.heavy_p_range
                p = lo + (hi - lo) * float(torch.rand(1, generator=g))
            heavy = torch.rand(n_q, generator=g) < p
            K[b, heavy] += HEAVY_SHIFT * self._u[b]
            if mu0 is not None:
                inc = self._drift_increments(b, c, n_q)
                K[b] += mu0[b] + torch.cumsum(inc, dim=0)
        dt = wl.torch_dtype()
        return Q.to(dt), K.to(dt), V.to(dt)


class DeviceChunkSource:
    """The distribution of ``ChunkSource`` drawn on ``device`` (for
    throughput runs, where the values only need the right distribution; it
    does not reproduce the CPU draws).

    * Each cache keeps one heavy-hitter direction for the whole run: the same
      unit vector ``ChunkSource`` uses (``heavy_direction``).
    * The heavy density is ``heavy_p``, or drawn per chunk and cache from
      U[lo, hi] when the workload gives a range.
    * A drifting workload's K mean is a per-token random walk per (cache, KV
      head) with steps of norm ``drift_step`` in uniformly random directions,
      carried from one chunk to the next on the device.  Chunks are meant to
      be drawn in order; a call that skips ahead starts the walk from a
      Gaussian draw with the walk's covariance at that token
      (drift_step^2 * tokens / d per coordinate).

    The last chunk's heavy mask, densities and walk are kept in
    ``last_heavy`` ([B, n_q] bool), ``last_p`` ([B]) and ``last_walk``
    ([B, n_q, H_kv, d], or None) for inspection.
    """

    def __init__(self, wl: Workload, seed: int, device, batch: Optional[int] = None):
        self.wl = wl
        self.seed = seed
        self.device = torch.device(device)
        self.batch = wl.batch if batch is None else batch
        self.u = torch.stack([heavy_direction(wl, seed, b) for b in range(self.batch)]).to(
            self.device)
        self.mu = torch.zeros(self.batch, wl.n_kv_heads, wl.head_dim, device=self.device)
        self.next_c = 0
        self.last_heavy = self.last_p = self.last_walk = None

    def chunk(self, c: int, n_q: Optional[int] = None):
        wl = self.wl
        n_q = wl.chunk if n_q is None else n_q
        dev = self.device
        g = _gen(self.seed, 0xC0DA, c, device=str(dev))
        B, d, Hkv = self.batch, wl.head_dim, wl.n_kv_heads
        Q = torch.randn(B, n_q, wl.n_q_heads, d, generator=g, device=dev)
        K = torch.randn(B, n_q, Hkv, d, generator=g, device=dev)
        V = torch.randn(B, n_q, Hkv, d, generator=g, device=dev)
        if wl.heavy_p_range is not None:
            lo, hi = wl.heavy_p_range
            p = lo + (hi - lo) * torch.rand(B, generator=g, device=dev)
        else:
            p = torch.full((B,), wl.heavy_p, device=dev)
        heavy = torch.rand(B, n_q, generator=g, device=dev) < p[:, None]
        K += HEAVY_SHIFT * heavy[:, :, None, None].float() * self.u[:, None, None, :]
        self.last_heavy, self.last_p, self.last_walk = heavy, p, None
        if wl.drift_step > 0:
            if c != self.next_c:   # skipped ahead: the walk's distribution at token c * n_q
                std = wl.drift_step * (c * n_q / d) ** 0.5
                self.mu = std * torch.randn(B, Hkv, d, generator=g, device=dev)
            xi = torch.randn(B, n_q, Hkv, d, generator=g, device=dev)
            inc = wl.drift_step * xi / xi.norm(dim=-1, keepdim=True)
            walk = self.mu[:, None] + torch.cumsum(inc, dim=1)
            K += walk
            self.mu = walk[:, -1].clone()
            self.last_walk = walk
        self.next_c = c + 1
        dt = wl.torch_dtype()
        return Q.to(dt), K.to(dt), V.to(dt)
