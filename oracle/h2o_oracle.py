"""Plain, slow CPU oracle of one chunked H2O sparse-attention step (fp64).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and
the ``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import
this module.  The product (the CUDA library and its Python binding) never
calls it and shares no code with it.

What it computes follows *Learning how to Forget: Fine-tuning for
Long-Context Sparse Attention* (arXiv 2608.19920):

* §1 Introduction: key/value information lives in a fixed-size KV cache;
  when the cache is full a policy evicts slots.  H2O is the policy the paper
  optimises, with dedicated SDPA kernel support.
* §1, second contribution: the SDPA kernel also returns the summed attention
  weights, the input of the H2O policy.
* §2 Related work: SnapKV uses H2O-like summed attention weights.
* Summary page, glossary entry "H2O": entries are scored by how often and
  how strongly they were attended, and the less important ones are evicted.

The page that would define H2O precisely (§3.1.1) is not among the sources.
The readings taken here, where the sources are silent:

* GQA grouping: query head h reads KV head h // G (G = H_q / H_kv).
* Visibility: every valid cache slot precedes the chunk, so every query sees
  it; chunk key j is visible to chunk query i iff j <= i.
* Score: a plain running sum of the attention weight a slot received, summed
  over the G query heads of its KV head and over the chunk's queries; fp32
  storage, one fp32 round-to-nearest addition per step.
* Selection: when the n cached entries plus the N_q new tokens exceed C, keep
  every candidate whose position is within the last W positions
  (pos >= t0 + N_q - W), and fill the remaining C - |protected| places with
  the unprotected candidates of highest score; ties go to the lower candidate
  index, where cache slot s has index s and new token i has index C + i.
* Placement: surviving entries keep their slot; the kept new tokens, in
  ascending order, take the freed (and empty) slots in ascending order.
* The score-free policies ``lr`` and ``slr`` (summary page, Tables 1, 2, 5
  and 6, named only): ``lr`` keeps the most recent tokens, ``slr`` keeps the
  first ``sinks`` positions of the sequence as well ("sink" tokens) and the
  most recent ones otherwise.  Reading: the same selection and placement as
  H2O with the candidate's position in place of its score (positions are
  distinct, so there are no ties), the recent window still protecting, and
  no score kept: old slots keep theirs, placed tokens get 0.
* The quantised cache of Q-Hitter (page 1 §2 Related Work: Q-Hitter combines
  H2O with quantisation; summary page Table 5, ``qh2o`` rows), whose format
  the sources do not give.  Reading: each cache row (one slot of one KV head,
  K and V separately) is stored as int8 codes with one fp32 scale,
  symmetric: s = fl32(max|x| / 127), q = clamp(rint(fl32(x / s)), -127, 127)
  (half to even; q = 0 when the row is all zero); the attention reads the
  dequantised value bf16(fl32(q * s)) (round to nearest even).  A token is
  quantised when it is placed into the cache; the chunk's own keys and
  values enter the step that brings them at their input precision.  The
  H2O scores are the same summed attention weights as without quantisation.

Parity status: the quantiser is pinned by hand-worked rows, its defining
properties (the largest element maps to +-127, the round-trip bound) and a
library bf16 rounding.  The attention output, summed weights and the selection are pinned
by brute force, a library routine (torch SDPA in fp64), closed forms and
invariants in ``tests/test_oracle_*.py``.  The multi-step trajectory is pinned
by an independent token-centric re-implementation.  The backward is pinned by
torch fp64 autograd, central finite differences and closed forms; the
score-free policies by the closed form of the positions they keep.  No worked
numeric example exists in the sources.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import List, Optional, Tuple

import numpy as np

F32 = np.float32


# --------------------------------------------------------------------------
# the quantised cache format (Q-Hitter reading, see the module docstring)
# --------------------------------------------------------------------------

def bf16_round(x: np.ndarray) -> np.ndarray:
    """float32 values rounded to the nearest bfloat16 (ties to even), as
    float32: the upper 16 bits of the float32 pattern after adding half an
    ulp of the kept part (0x7FFF plus the lowest kept bit)."""
    b = np.ascontiguousarray(x, dtype=F32).view(np.uint32).astype(np.uint64)
    r = (b + 0x7FFF + ((b >> 16) & 1)) >> 16 << 16
    return (r & 0xFFFFFFFF).astype(np.uint32).view(F32)


def quantize_row_q8(x: np.ndarray) -> Tuple[np.ndarray, np.float32]:
    """One cache row (d values) -> (int8 codes, fp32 scale)."""
    x = np.asarray(x, dtype=F32)
    amax = F32(np.max(np.abs(x))) if x.size else F32(0)
    s = F32(amax / F32(127))
    if s == 0:
        return np.zeros(x.shape, dtype=np.int8), F32(0)
    q = np.rint(np.asarray(x / s, dtype=F32)).clip(-127, 127)
    return q.astype(np.int8), s


def dequantize_q8(q: np.ndarray, s) -> np.ndarray:
    """int8 codes and their scale(s) -> the value the attention reads,
    bf16(fl32(q * s)), as float64.  One scale per row: s has the shape of q
    without its last axis."""
    q = np.asarray(q, dtype=F32)
    s = np.asarray(s, dtype=F32)
    if s.ndim:
        s = s[..., None]
    return bf16_round((q * s).astype(F32)).astype(np.float64)


# --------------------------------------------------------------------------
# attention with summed weights (one cache)
# --------------------------------------------------------------------------

def kv_head_of(h: int, group: int) -> int:
    """KV head read by query head h (contiguous grouping)."""
    return h // group


def visible_mask(n: int, n_q: int) -> np.ndarray:
    """[n_q, n + n_q] boolean: query i sees all n cache slots and chunk keys j <= i."""
    m = np.zeros((n_q, n + n_q), dtype=bool)
    m[:, :n] = True
    m[:, n:] = np.tril(np.ones((n_q, n_q), dtype=bool))
    return m


def attention_one_cache(q: np.ndarray, kc: np.ndarray, vc: np.ndarray, n: int,
                        kn: np.ndarray, vn: np.ndarray, scale: float):
    """Attention plus summed weights for one cache.

    q  [n_q, H_q, d];  kc, vc [H_kv, C, d] (slots 0..n-1 valid);
    kn, vn [n_q, H_kv, d].
    Returns (o [n_q, H_q, d], colsum [H_kv, C + n_q], lse [H_q, n_q]) where
    colsum[g, s] (s < n) is the weight cache slot s received, colsum[g, C + j]
    the weight chunk key j received, colsum[g, n:C] = 0, and lse the natural
    log-sum-exp of each row's logits.
    """
    q = np.asarray(q, dtype=np.float64)
    n_q, H_q, d = q.shape
    H_kv, C, _ = kc.shape
    G = H_q // H_kv
    o = np.zeros((n_q, H_q, d))
    colsum = np.zeros((H_kv, C + n_q))
    lse = np.zeros((H_q, n_q))
    vis = visible_mask(n, n_q)
    for h in range(H_q):
        g = kv_head_of(h, G)
        keys = np.concatenate([kc[g, :n], kn[:, g]], axis=0)       # [n + n_q, d]
        vals = np.concatenate([vc[g, :n], vn[:, g]], axis=0)
        s = scale * (q[:, h, :] @ keys.T)                          # [n_q, n + n_q]
        s = np.where(vis, s, -np.inf)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        l = e.sum(axis=1, keepdims=True)
        p = e / l
        o[:, h, :] = p @ vals
        lse[h] = (m + np.log(l))[:, 0]
        w = p.sum(axis=0)                                          # column sums
        colsum[g, :n] += w[:n]
        colsum[g, C:] += w[n:]
    return o, colsum, lse


def attention_backward_one_cache(q: np.ndarray, kc: np.ndarray, vc: np.ndarray, n: int,
                                 kn: np.ndarray, vn: np.ndarray, do: np.ndarray,
                                 scale: float):
    """Gradients of the attention output O of ``attention_one_cache`` with
    respect to its inputs, for one cache, given dO = dL/dO [n_q, H_q, d].

    The cache contents and the visibility are held fixed: the eviction that
    follows the attention in a step is a discrete decision and is not
    differentiated (the paper trains through the cache with its policy in
    place, summary page, Tables 1 and 6).  For query head h of KV head g, over
    its visible keys:  P = softmax(scale q k^T);  dV_g += P^T dO_h;
    dP = dO_h V^T;  dS = P * (dP - rowsum(P * dP)) (the softmax Jacobian);
    dq_h = scale dS K;  dK_g += scale dS^T q_h.

    Returns (dq [n_q, H_q, d], dkc [H_kv, C, d], dvc [H_kv, C, d],
    dkn [n_q, H_kv, d], dvn [n_q, H_kv, d]); rows of dkc, dvc past the n
    valid slots are 0.
    """
    q = np.asarray(q, dtype=np.float64)
    do = np.asarray(do, dtype=np.float64)
    n_q, H_q, d = q.shape
    H_kv, C, _ = kc.shape
    G = H_q // H_kv
    dq = np.zeros_like(q)
    dkc = np.zeros((H_kv, C, d))
    dvc = np.zeros((H_kv, C, d))
    dkn = np.zeros((n_q, H_kv, d))
    dvn = np.zeros((n_q, H_kv, d))
    vis = visible_mask(n, n_q)
    for h in range(H_q):
        g = kv_head_of(h, G)
        keys = np.concatenate([kc[g, :n], kn[:, g]], axis=0)       # [n + n_q, d]
        vals = np.concatenate([vc[g, :n], vn[:, g]], axis=0)
        s = scale * (q[:, h, :] @ keys.T)
        s = np.where(vis, s, -np.inf)
        e = np.exp(s - s.max(axis=1, keepdims=True))
        p = e / e.sum(axis=1, keepdims=True)                       # [n_q, n + n_q]
        dv = p.T @ do[:, h, :]
        dp = do[:, h, :] @ vals.T
        ds = p * (dp - (p * dp).sum(axis=1, keepdims=True))
        dq[:, h, :] = scale * (ds @ keys)
        dk = scale * (ds.T @ q[:, h, :])
        dkc[g, :n] += dk[:n]
        dvc[g, :n] += dv[:n]
        dkn[:, g] += dk[n:]
        dvn[:, g] += dv[n:]
    return dq, dkc, dvc, dkn, dvn


# --------------------------------------------------------------------------
# score accumulation, selection and placement (one cache, one KV head)
# --------------------------------------------------------------------------

@dataclass
class Placement:
    """Result of the eviction decision for one (cache, KV head)."""
    slots: List[int] = field(default_factory=list)    # destination slot, ascending
    tokens: List[int] = field(default_factory=list)   # new token placed there, ascending
    evicted: List[int] = field(default_factory=list)  # old slots dropped


POLICIES = ("h2o", "lr", "slr")


def evict_one_head(score: np.ndarray, pos: np.ndarray, n: int, t0: int,
                   colsum32: np.ndarray, n_q: int, window: int, policy: str = "h2o",
                   sinks: int = 0):
    """Score update + selection + placement for one (cache, KV head).

    score [C] float32, pos [C] int32 (-1 empty), colsum32 [C + n_q] float32
    (layout of ``attention_one_cache``; not read by the score-free
    policies).  ``policy``: "h2o" ranks the unprotected candidates by score,
    "lr" and "slr" by position; "slr" also protects positions < ``sinks``.
    Returns (new score, new pos, Placement).  Inputs are not modified.
    """
    assert policy in POLICIES
    C = score.shape[0]
    score = score.astype(F32).copy()
    pos = pos.astype(np.int32).copy()
    if policy == "h2o":
        # one fp32 addition per cached slot
        score[:n] = (score[:n] + colsum32[:n].astype(F32)).astype(F32)
        cand_new = colsum32[C:C + n_q].astype(F32)
    else:
        cand_new = np.zeros(n_q, dtype=F32)
    pl = Placement()
    if n + n_q <= C:
        pl.slots = list(range(n, n + n_q))
        pl.tokens = list(range(n_q))
    else:
        limit = t0 + n_q - window
        # candidates: (index, rank value, position, is_new, slot-or-token)
        if policy == "h2o":
            cands = [(s, float(score[s]), int(pos[s]), False, s) for s in range(n)]
            cands += [(C + i, float(cand_new[i]), t0 + i, True, i) for i in range(n_q)]
        else:
            cands = [(s, float(pos[s]), int(pos[s]), False, s) for s in range(n)]
            cands += [(C + i, float(t0 + i), t0 + i, True, i) for i in range(n_q)]

        def is_protected(c):
            return c[2] >= limit or (policy == "slr" and c[2] < sinks)

        protected = [c for c in cands if is_protected(c)]
        unprot = [c for c in cands if not is_protected(c)]
        k_keep = C - len(protected)
        ranked = sorted(unprot, key=lambda c: (-c[1], c[0]))
        kept = {c[0] for c in protected} | {c[0] for c in ranked[:k_keep]}
        pl.evicted = [s for s in range(n) if s not in kept]
        free = sorted(pl.evicted + list(range(n, C)))
        new_kept = sorted(i for i in range(n_q) if (C + i) in kept)
        assert len(free) == len(new_kept), (len(free), len(new_kept))
        pl.slots, pl.tokens = free, new_kept
    for s, i in zip(pl.slots, pl.tokens):
        score[s] = cand_new[i]
        pos[s] = t0 + i
    return score, pos, pl


# --------------------------------------------------------------------------
# the whole step over a batch of caches
# --------------------------------------------------------------------------

class OracleCache:
    """State of ``batch`` independent H2O caches and the step that advances them.

    K, V: [B, H_kv, C, d] float64 holding the input values exactly;
    scores [B, H_kv, C] float32; pos [B, H_kv, C] int32 (-1 empty);
    n (valid slots, shared) and t0 (position of the next chunk's first token).
    With kv_format "q8" the cache rows are stored quantised: Kq, Vq
    [B, H_kv, C, d] int8 and Ks, Vs [B, H_kv, C] float32, and K, V hold their
    dequantised values (what the attention reads).
    """

    def __init__(self, batch: int, n_q_heads: int, n_kv_heads: int, head_dim: int,
                 capacity: int, window: int, scale: Optional[float] = None,
                 policy: str = "h2o", sinks: int = 0, kv_format: str = "bf16"):
        assert n_q_heads % n_kv_heads == 0
        assert kv_format in ("bf16", "q8")
        self.kv_format = kv_format
        assert 0 <= window <= capacity
        assert policy in POLICIES and 0 <= sinks and (policy != "slr" or sinks + window <= capacity)
        self.policy, self.sinks = policy, sinks
        self.B, self.H_q, self.H_kv, self.d = batch, n_q_heads, n_kv_heads, head_dim
        self.C, self.W = capacity, window
        self.scale = 1.0 / math.sqrt(head_dim) if scale is None else float(scale)
        self.K = np.zeros((batch, n_kv_heads, capacity, head_dim))
        self.V = np.zeros_like(self.K)
        self.scores = np.zeros((batch, n_kv_heads, capacity), dtype=F32)
        self.pos = np.full((batch, n_kv_heads, capacity), -1, dtype=np.int32)
        self.n = 0
        self.t0 = 0
        if kv_format == "q8":
            self.Kq = np.zeros((batch, n_kv_heads, capacity, head_dim), dtype=np.int8)
            self.Vq = np.zeros_like(self.Kq)
            self.Ks = np.zeros((batch, n_kv_heads, capacity), dtype=F32)
            self.Vs = np.zeros_like(self.Ks)

    # snapshot / restore --------------------------------------------------
    def state(self):
        return (self.K.copy(), self.V.copy(), self.scores.copy(), self.pos.copy(),
                self.n, self.t0)

    def load(self, K, V, scores, pos, n, t0):
        self.K = np.array(K, dtype=np.float64)
        self.V = np.array(V, dtype=np.float64)
        self.scores = np.array(scores, dtype=F32)
        self.pos = np.array(pos, dtype=np.int32)
        self.n, self.t0 = int(n), int(t0)

    def load_q8(self, Kq, Ks, Vq, Vs, scores, pos, n, t0):
        """Restores a quantised cache from its codes and scales."""
        assert self.kv_format == "q8"
        self.Kq, self.Vq = np.array(Kq, dtype=np.int8), np.array(Vq, dtype=np.int8)
        self.Ks, self.Vs = np.array(Ks, dtype=F32), np.array(Vs, dtype=F32)
        self.load(dequantize_q8(self.Kq, self.Ks), dequantize_q8(self.Vq, self.Vs), scores, pos,
                  n, t0)

    # the two halves of the step -------------------------------------------
    def attention(self, Q, Kn, Vn):
        """Q [B, n_q, H_q, d], Kn/Vn [B, n_q, H_kv, d] -> (O, colsum, lse).

        O [B, n_q, H_q, d] float64, colsum [B, H_kv, C + n_q] float64,
        lse [B, H_q, n_q].  The state is not changed.
        """
        Q, Kn, Vn = (np.asarray(x, dtype=np.float64) for x in (Q, Kn, Vn))
        B, n_q = Q.shape[0], Q.shape[1]
        O = np.zeros((B, n_q, self.H_q, self.d))
        colsum = np.zeros((B, self.H_kv, self.C + n_q))
        lse = np.zeros((B, self.H_q, n_q))
        for b in range(B):
            O[b], colsum[b], lse[b] = attention_one_cache(
                Q[b], self.K[b], self.V[b], self.n, Kn[b], Vn[b], self.scale)
        return O, colsum, lse

    def attention_backward(self, Q, Kn, Vn, dO):
        """Gradients of ``attention``'s O for the current state (before the
        eviction of the same step): (dQ, dK_cache, dV_cache, dK_new, dV_new)
        with the layouts of Q [B, n_q, H_q, d], the cache [B, H_kv, C, d] and
        Kn [B, n_q, H_kv, d]."""
        Q, Kn, Vn, dO = (np.asarray(x, dtype=np.float64) for x in (Q, Kn, Vn, dO))
        B = Q.shape[0]
        outs = [np.zeros_like(Q), np.zeros_like(self.K), np.zeros_like(self.V),
                np.zeros_like(Kn), np.zeros_like(Vn)]
        for b in range(B):
            r = attention_backward_one_cache(Q[b], self.K[b], self.V[b], self.n, Kn[b], Vn[b],
                                             dO[b], self.scale)
            for o, x in zip(outs, r):
                o[b] = x
        return tuple(outs)

    def evict(self, colsum32, Kn, Vn):
        """Apply the score update, selection and placement with the given fp32
        summed weights ([B, H_kv, C + n_q]); advances n and t0.
        Returns the per-(b, g) placements."""
        Kn, Vn = np.asarray(Kn, dtype=np.float64), np.asarray(Vn, dtype=np.float64)
        n_q = Kn.shape[1]
        placements = []
        for b in range(self.B):
            row = []
            for g in range(self.H_kv):
                sc, ps, pl = evict_one_head(self.scores[b, g], self.pos[b, g], self.n,
                                            self.t0, colsum32[b, g], n_q, self.W,
                                            self.policy, self.sinks)
                self.scores[b, g], self.pos[b, g] = sc, ps
                if pl.slots and self.kv_format == "q8":
                    for s_, i_ in zip(pl.slots, pl.tokens):   # quantised on placement
                        self.Kq[b, g, s_], self.Ks[b, g, s_] = quantize_row_q8(Kn[b, i_, g])
                        self.Vq[b, g, s_], self.Vs[b, g, s_] = quantize_row_q8(Vn[b, i_, g])
                        self.K[b, g, s_] = dequantize_q8(self.Kq[b, g, s_], self.Ks[b, g, s_])
                        self.V[b, g, s_] = dequantize_q8(self.Vq[b, g, s_], self.Vs[b, g, s_])
                elif pl.slots:
                    self.K[b, g, pl.slots] = Kn[b, pl.tokens, g]
                    self.V[b, g, pl.slots] = Vn[b, pl.tokens, g]
                row.append(pl)
            placements.append(row)
        self.n = min(self.C, self.n + n_q)
        self.t0 += n_q
        return placements

    def step(self, Q, Kn, Vn):
        """One full step: attention + summed weights, then eviction.
        Returns (O, colsum) with colsum in float64."""
        O, colsum, _ = self.attention(Q, Kn, Vn)
        self.evict(colsum.astype(F32), Kn, Vn)
        return O, colsum


def gap_at_boundary(scores: np.ndarray, pos: np.ndarray, n: int, t0: int,
                    colsum32: np.ndarray, n_q: int, window: int) -> float:
    """Relative gap between the last kept and the first dropped unprotected
    candidate score of one (cache, KV head); +inf when nothing is evicted.
    Used to decide whether a step is a near-tie."""
    C = scores.shape[0]
    if n + n_q <= C:
        return math.inf
    sc = scores.astype(F32).copy()
    sc[:n] = (sc[:n] + colsum32[:n].astype(F32)).astype(F32)
    limit = t0 + n_q - window
    vals = [float(sc[s]) for s in range(n) if pos[s] < limit]
    vals += [float(colsum32[C + i]) for i in range(n_q) if t0 + i < limit]
    n_prot = (n + n_q) - len(vals)
    k_keep = C - n_prot
    vals.sort(reverse=True)
    if k_keep <= 0 or k_keep >= len(vals):
        return math.inf
    a, b = vals[k_keep - 1], vals[k_keep]
    return (a - b) / max(abs(a), 1e-30)
