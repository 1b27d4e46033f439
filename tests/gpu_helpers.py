"""Shared pieces of the GPU parity tests: moving state between the CUDA
cache (through the C ABI) and the CPU oracle, and the comparison rules.

Tolerances (bf16 inputs, fp32 accumulation):
  * attention output: max |O_gpu - O_ref| <= 2e-2;
  * summed weights: |d| / max(|ref|, 1e-6 * n_q * G) <= 1e-3 elementwise;
  * cache contents, scores, positions: bit-exact whenever the gap between the
    last kept and first dropped unprotected score exceeds 1e-4 (relative),
    and always when the eviction is fed the same summed weights.
"""
from __future__ import annotations

import numpy as np
import torch

from kv_cache_sparse_b200 import binding
from kv_cache_sparse_b200.build import build
from oracle import h2o_oracle as orc

O_TOL = 2e-2
COLSUM_RTOL = 1e-3
GAP_RTOL = 1e-4


def ensure_built():
    build()


def np64(t: torch.Tensor) -> np.ndarray:
    return t.detach().to(torch.float64).cpu().numpy()


def shape_of(B, Hq, Hkv, d, C, max_chunk, W, dtype=torch.bfloat16, scale=0.0):
    return binding.CacheShape(B, Hq, Hkv, d, C, max_chunk, W, dtype, scale)


def oracle_for(shape: binding.CacheShape) -> orc.OracleCache:
    scale = shape.softmax_scale if shape.softmax_scale > 0 else None
    return orc.OracleCache(shape.batch, shape.n_q_heads, shape.n_kv_heads, shape.head_dim,
                           shape.capacity, shape.recent_window, scale=scale,
                           kv_format="q8" if shape.q8 else "bf16")


def push_oracle_state(gpu: binding.H2OCache, ref: orc.OracleCache):
    dt = gpu.shape.dtype
    gpu.write(torch.from_numpy(ref.K).to(dt), torch.from_numpy(ref.V).to(dt),
              torch.from_numpy(ref.scores), torch.from_numpy(ref.pos), ref.n, ref.t0)


def pull_state(gpu: binding.H2OCache):
    st = gpu.read()
    return st


def load_oracle_from_gpu(ref: orc.OracleCache, st):
    if ref.kv_format == "q8":
        ref.load_q8(st["k"].cpu().numpy(), st["k_scale"].cpu().numpy(), st["v"].cpu().numpy(),
                    st["v_scale"].cpu().numpy(), st["scores"].cpu().numpy(),
                    st["pos"].cpu().numpy(), st["n"], st["t0"])
        return
    ref.load(np64(st["k"]), np64(st["v"]), st["scores"].cpu().numpy(),
             st["pos"].cpu().numpy(), st["n"], st["t0"])


def random_state_q8(shape, n, t0, rng, score_levels=None):
    """A plausible int8-cache state: codes and row scales of n valid slots
    (the quantised form of N(0,1) rows), scores and distinct positions."""
    K, V, sc, pos = random_state(shape.__class__(**{**shape.__dict__, "dtype": torch.bfloat16}),
                                 n, t0, rng, score_levels)
    B, Hkv, C, d = shape.batch, shape.n_kv_heads, shape.capacity, shape.head_dim
    out = []
    for X in (K, V):
        codes = np.zeros((B, Hkv, C, d), np.int8)
        scales = np.zeros((B, Hkv, C), np.float32)
        x = X.float().numpy()
        for b in range(B):
            for g in range(Hkv):
                for s_ in range(n):
                    codes[b, g, s_], scales[b, g, s_] = orc.quantize_row_q8(x[b, g, s_])
        out += [codes, scales]
    return out[0], out[1], out[2], out[3], sc, pos


def install_state_q8(gpu, ref, Kq, Ks, Vq, Vs, sc, pos, n, t0):
    gpu.write(torch.from_numpy(Kq), torch.from_numpy(Vq), torch.from_numpy(sc),
              torch.from_numpy(pos), n, t0, k_scale=torch.from_numpy(Ks),
              v_scale=torch.from_numpy(Vs))
    ref.load_q8(Kq, Ks, Vq, Vs, sc, pos, n, t0)


def random_state(shape, n, t0, rng, score_levels=None):
    """A plausible cache state: n valid slots with distinct positions < t0."""
    B, Hkv, C, d = shape.batch, shape.n_kv_heads, shape.capacity, shape.head_dim
    g = torch.Generator().manual_seed(int(rng.integers(1 << 31)))
    K = torch.zeros(B, Hkv, C, d)
    V = torch.zeros(B, Hkv, C, d)
    K[:, :, :n] = torch.randn(B, Hkv, n, d, generator=g)
    V[:, :, :n] = torch.randn(B, Hkv, n, d, generator=g)
    if score_levels:
        sc = rng.integers(0, score_levels, (B, Hkv, C)).astype(np.float32) / score_levels
    else:
        sc = (rng.random((B, Hkv, C)) * 4).astype(np.float32)
    sc[:, :, n:] = 0
    pos = np.full((B, Hkv, C), -1, np.int32)
    for b in range(B):
        for h in range(Hkv):
            pos[b, h, :n] = rng.permutation(t0)[:n]
    dt = shape.dtype
    return K.to(dt), V.to(dt), sc, pos


def install_state(gpu, ref, K, V, sc, pos, n, t0):
    gpu.write(K, V, torch.from_numpy(sc), torch.from_numpy(pos), n, t0)
    ref.load(np64(K), np64(V), sc, pos, n, t0)


def colsum_rel_err(got: np.ndarray, ref: np.ndarray, n_q: int, G: int) -> float:
    denom = np.maximum(np.abs(ref), 1e-6 * n_q * G)
    return float(np.max(np.abs(got - ref) / denom))


def assert_attention_close(O_gpu, cs_gpu, O_ref, cs_ref, n_q, G, what=""):
    O_gpu = np64(O_gpu) if isinstance(O_gpu, torch.Tensor) else O_gpu
    cs_gpu = np64(cs_gpu) if isinstance(cs_gpu, torch.Tensor) else cs_gpu
    err_o = float(np.max(np.abs(O_gpu - O_ref))) if O_ref.size else 0.0
    err_c = colsum_rel_err(cs_gpu, cs_ref, n_q, G)
    assert err_o <= O_TOL, f"{what}: attention output max-abs error {err_o:.3e}"
    assert err_c <= COLSUM_RTOL, f"{what}: summed weights rel error {err_c:.3e}"
    return err_o, err_c


def bits(t: torch.Tensor) -> torch.Tensor:
    t = t.detach().cpu().contiguous()
    return t.view({torch.bfloat16: torch.int16, torch.float32: torch.int32,
                   torch.float16: torch.int16}.get(t.dtype, t.dtype))


def assert_state_equal(st, ref: orc.OracleCache, dtype, what=""):
    """GPU state (from read()) equals the oracle's, bit for bit."""
    assert st["n"] == ref.n and st["t0"] == ref.t0, what
    assert np.array_equal(st["pos"].cpu().numpy(), ref.pos), f"{what}: positions differ"
    assert np.array_equal(st["scores"].cpu().numpy().view(np.uint32),
                          ref.scores.astype(np.float32).view(np.uint32)), f"{what}: scores differ"
    if ref.kv_format == "q8":
        assert np.array_equal(st["k"].cpu().numpy(), ref.Kq), f"{what}: K codes differ"
        assert np.array_equal(st["v"].cpu().numpy(), ref.Vq), f"{what}: V codes differ"
        assert np.array_equal(st["k_scale"].cpu().numpy().view(np.uint32),
                              ref.Ks.view(np.uint32)), f"{what}: K scales differ"
        assert np.array_equal(st["v_scale"].cpu().numpy().view(np.uint32),
                              ref.Vs.view(np.uint32)), f"{what}: V scales differ"
        return
    kref = torch.from_numpy(ref.K).to(dtype)
    vref = torch.from_numpy(ref.V).to(dtype)
    assert torch.equal(bits(st["k"]), bits(kref)), f"{what}: cache K differs"
    assert torch.equal(bits(st["v"]), bits(vref)), f"{what}: cache V differs"


def min_gap(ref: orc.OracleCache, colsum32: np.ndarray, n_q: int) -> float:
    gaps = [orc.gap_at_boundary(ref.scores[b, g], ref.pos[b, g], ref.n, ref.t0,
                                colsum32[b, g], n_q, ref.W)
            for b in range(ref.B) for g in range(ref.H_kv)]
    return min(gaps) if gaps else float("inf")
