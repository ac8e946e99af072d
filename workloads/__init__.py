"""Seeded synthetic inputs for the verify workloads.

This module feeds both the CPU oracle and the GPU library with the same
bytes.  It holds none of the verifier's arithmetic: it draws logits from
normal distributions (numpy's Philox bit generator), rounds them to bf16,
and draws draft tokens the way a draft model's sampler would (inverse CDF
over the draft softmax, or "argmax with probability p, else uniform" for the
greedy and lookahead workloads).

Logit arrays are numpy arrays: float32 for "f32", uint16 bf16 bit patterns
for "bf16".  ``as_torch`` turns one into a torch tensor of the right dtype.

The named workloads (sizes, distributions, temperatures and seeds of the
verify step they stand for; the first five, plus the profiling cases below):

  stoch_b1_k4_v32000_f32   stochastic, B=1 k=4 V=32000, target fp32 ~ N(0, 2^2),
                           draft fp32 = target + N(0, 1), T=1.0, seed 0
  greedy_b64_k4_v128256    greedy, B=64 k=4 V=128256, bf16 ~ N(0, 3^2), draft token
                           = argmax w.p. 0.7 else uniform, seed 2
  stoch_b64_k4_v128256     stochastic, B=64 k=4 V=128256, target bf16 ~ N(0, 3^2),
                           draft fp32 = target + N(0, 1.5^2), T=0.7, seed 1
  stoch_b256_k8_v128256    stochastic, B=256 k=8 V=128256, target bf16 ~ N(0, 3^2),
                           draft bf16 = RNE(target + N(0, 1)), T=1.0, seed 3
  multi_b16_g8_k4_v32000   multi-candidate, B=16 G=8 k=4 V=32000, bf16 ~ N(0, 3^2);
                           half the sequences share a random-length (1..3) prefix
                           of candidate 0 across branches; each other token is the
                           row argmax w.p. 0.6 else uniform, seed 4
  threshold_b64_k4_v128256, multi_rows_b16_g8_k4_v32000, tree_b64_n26_v128256 and
  tree_stoch_b64_n26_v128256 (26-node trees of depth <= 3, node rows bf16 ~
  N(0, 10^2), first child = the row argmax w.p. 0.9, T=1.0, seed 7): see
  WORKLOADS.
"""
from __future__ import annotations

import concurrent.futures as _fut
import os

import numpy as np

# ----------------------------------------------------------- named workloads

WORKLOADS = {
    "stoch_b1_k4_v32000_f32": dict(mode="stochastic", B=1, k=4, V=32000, t_dtype="f32",
                                   d_dtype="f32", t_std=2.0, d_noise=1.0, temperature=1.0,
                                   seed=0),
    "greedy_b64_k4_v128256": dict(mode="greedy", B=64, k=4, V=128256, t_dtype="bf16",
                                  t_std=3.0, p_match=0.7, seed=2),
    "stoch_b64_k4_v128256": dict(mode="stochastic", B=64, k=4, V=128256, t_dtype="bf16",
                                 d_dtype="f32", t_std=3.0, d_noise=1.5, temperature=0.7,
                                 seed=1),
    "stoch_b256_k8_v128256": dict(mode="stochastic", B=256, k=8, V=128256, t_dtype="bf16",
                                  d_dtype="bf16", t_std=3.0, d_noise=1.0, temperature=1.0,
                                  seed=3),
    "multi_b16_g8_k4_v32000": dict(mode="multi", B=16, G=8, k=4, V=32000, t_dtype="bf16",
                                   t_std=3.0, p_match=0.6, p_shared=0.5, seed=4),
    # threshold acceptance on the greedy workload's rows and drafts
    "threshold_b64_k4_v128256": dict(mode="threshold", B=64, k=4, V=128256, t_dtype="bf16",
                                     t_std=3.0, p_match=0.7, seed=2, temperature=1.0,
                                     threshold=1e-3),
    # an EAGLE-style draft tree per sequence (Top-K children, distinct tokens)
    "tree_b64_n26_v128256": dict(mode="tree", B=64, N=26, V=128256, t_dtype="bf16",
                                 t_std=3.0, p_match=0.7, seed=6),
    # the same tree shape under stochastic acceptance; sharper rows (sigma 10:
    # the row maximum holds about 2/3 of the mass) stand for a confident target,
    # and the first child carries it with probability 0.9
    "tree_stoch_b64_n26_v128256": dict(mode="tree_stochastic", B=64, N=26, V=128256,
                                       t_dtype="bf16", t_std=10.0, p_match=0.9,
                                       temperature=1.0, seed=7),
    # the same lookahead step with each distinct candidate prefix's row once
    "multi_rows_b16_g8_k4_v32000": dict(mode="multi_rows", B=16, G=8, k=4, V=32000,
                                        t_dtype="bf16", t_std=3.0, p_match=0.6,
                                        p_shared=0.5, seed=4),
}

ELEM_BYTES = {"f32": 4, "bf16": 2}


def _threads(threads: int | None) -> int:
    return max(1, threads if threads else min(32, os.cpu_count() or 1))


def _rng(seed: int, *stream: int) -> np.random.Generator:
    """Independent Philox stream for (seed, *stream)."""
    return np.random.Generator(np.random.Philox(np.random.SeedSequence([seed, *stream])))


def _pmap(fn, n: int, threads: int | None):
    t = _threads(threads)
    if t == 1 or n < 2:
        return [fn(j) for j in range(n)]
    with _fut.ThreadPoolExecutor(t) as ex:
        return list(ex.map(fn, range(n)))


# ------------------------------------------------------------------- bf16

def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 to bf16 (round to nearest, ties to even); uint16 bits."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    bias = ((b >> np.uint32(16)) & np.uint32(1)) + np.uint32(0x7FFF)
    return ((b + bias) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    return (np.asarray(h).astype(np.uint32) << np.uint32(16)).view(np.float32)


def to_f32(arr: np.ndarray, dtype: str) -> np.ndarray:
    return bf16_bits_to_f32(arr) if dtype == "bf16" else np.asarray(arr, np.float32)


def as_torch(arr: np.ndarray, dtype: str):
    """numpy logits (f32 or bf16 bits) -> CPU torch tensor of that dtype."""
    import torch

    if dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)).view(torch.bfloat16)
    return torch.from_numpy(np.ascontiguousarray(arr, dtype=np.float32))


def from_torch(t) -> tuple[np.ndarray, str]:
    """CPU torch tensor (bf16 or f32) -> (numpy array, dtype)."""
    import torch

    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16), "bf16"
    if t.dtype == torch.float32:
        return t.numpy(), "f32"
    raise TypeError(f"unsupported logit dtype {t.dtype}")


# ------------------------------------------------------------- generators

# stream ids inside one seed
_S_TARGET, _S_DRAFT, _S_TOKENS, _S_SHARE = 1, 2, 3, 4


def _target_rows(seed: int, rows: int, V: int, std: float, dtype: str,
                 threads: int | None) -> np.ndarray:
    """[rows, V] target rows ~ N(0, std^2), row r from stream (seed, 1, r),
    stored as `dtype` (bf16 rounded to nearest even)."""
    out = np.empty((rows, V), np.uint16 if dtype == "bf16" else np.float32)

    def fill(r):
        x = _rng(seed, _S_TARGET, r).standard_normal(V, dtype=np.float32)
        x *= np.float32(std)
        out[r] = f32_to_bf16_bits(x) if dtype == "bf16" else x

    _pmap(fill, rows, threads)
    return out


def make_stochastic(B: int, k: int, V: int, t_dtype: str = "bf16", d_dtype: str = "bf16",
                    t_std: float = 3.0, d_noise: float = 1.0, temperature: float = 1.0,
                    seed: int = 0, threads: int | None = None) -> dict:
    """Target [B,k+1,V] ~ N(0, t_std^2); draft [B,k,V] = target + N(0, d_noise^2);
    draft tokens [B,k] drawn from softmax(draft / T)."""
    target = _target_rows(seed, B * (k + 1), V, t_std, t_dtype, threads).reshape(B, k + 1, V)
    draft = np.empty((B, k, V), np.uint16 if d_dtype == "bf16" else np.float32)
    tokens = np.zeros((B, k), np.int32)
    T = float(np.float32(temperature))

    def fill(r):
        b, i = divmod(r, k)
        noise = _rng(seed, _S_DRAFT, r).standard_normal(V, dtype=np.float32)
        noise *= np.float32(d_noise)
        d32 = to_f32(target[b, i], t_dtype) + noise
        if d_dtype == "bf16":
            draft[b, i] = f32_to_bf16_bits(d32)
            d32 = bf16_bits_to_f32(draft[b, i])
        else:
            draft[b, i] = d32
        tokens[b, i] = _inverse_cdf(d32, T, _rng(seed, _S_TOKENS, r).random())

    _pmap(fill, B * k, threads)
    return dict(mode="stochastic", target=target, t_dtype=t_dtype, draft=draft,
                d_dtype=d_dtype, tokens=tokens, temperature=T, seed=seed, B=B, k=k, V=V)


def _inverse_cdf(row_f32: np.ndarray, T: float, u: float) -> int:
    """Token drawn from softmax(row / T) by inverse CDF with uniform u."""
    z = row_f32.astype(np.float64) / T
    c = np.cumsum(np.exp(z - z.max()))
    return min(int(np.searchsorted(c, u * c[-1], side="right")), row_f32.size - 1)


def make_greedy(B: int, k: int, V: int, t_dtype: str = "bf16", t_std: float = 3.0,
                p_match: float = 0.7, seed: int = 0, threads: int | None = None) -> dict:
    """Target [B,k+1,V] ~ N(0, t_std^2); draft token = row argmax w.p. p_match."""
    target = _target_rows(seed, B * (k + 1), V, t_std, t_dtype, threads).reshape(B, k + 1, V)
    rows = target[:, :k, :].reshape(B * k, V)
    tokens = (_argmax_or_uniform(rows, t_dtype, p_match, seed, threads).reshape(B, k)
              if B * k else np.zeros((B, k), np.int32))
    return dict(mode="greedy", target=target, t_dtype=t_dtype, tokens=tokens, seed=seed,
                B=B, k=k, V=V)


def _argmax_or_uniform(rows: np.ndarray, dtype: str, p_match: float, seed: int,
                       threads: int | None) -> np.ndarray:
    n, V = rows.shape
    am = np.empty(n, np.int64)

    def f(r):
        am[r] = int(np.argmax(to_f32(rows[r], dtype)))

    _pmap(f, n, threads)
    g = _rng(seed, _S_TOKENS)
    hit = g.random(n) < p_match
    uni = g.integers(0, V, n)
    return np.where(hit, am, uni).astype(np.int32)


def make_multi(B: int, G: int, k: int, V: int, t_dtype: str = "bf16", t_std: float = 3.0,
               p_match: float = 0.6, p_shared: float = 0.5, seed: int = 0,
               threads: int | None = None) -> dict:
    """Target [B,G,k+1,V] ~ N(0, t_std^2), i.i.d. rows; candidates [B,G,k].

    With probability p_shared a sequence picks s in {1,2,3} and branches
    1..G-1 copy branch 0's first s tokens; every other token is its own row's
    argmax with probability p_match, else uniform.
    """
    target = _target_rows(seed, B * G * (k + 1), V, t_std, t_dtype, threads)
    target = target.reshape(B, G, k + 1, V)
    rows = target[:, :, :k, :].reshape(B * G * k, V)
    cand = (_argmax_or_uniform(rows, t_dtype, p_match, seed, threads).reshape(B, G, k)
            if B * G * k else np.zeros((B, G, k), np.int32))
    g = _rng(seed, _S_SHARE)
    shared = g.random(B) < p_shared
    s = g.integers(1, 4, B)
    for b in range(B):
        if shared[b] and k > 0:
            m = min(int(s[b]), k)
            cand[b, 1:, :m] = cand[b, 0, :m]
    return dict(mode="multi", target=target, t_dtype=t_dtype, tokens=cand, seed=seed,
                B=B, G=G, k=k, V=V)


def prefix_rows(cand: np.ndarray) -> tuple[np.ndarray, int]:
    """Row map of lookahead candidates [B,G,k]: row (b, g, i) conditions on
    the context plus cand[b,g,:i], so (g, i) pairs with equal prefixes share
    one row.  Returns row_of [B,G,k+1] (int32, rows numbered per sequence in
    order of first appearance, i-major) and R, the most rows any sequence
    needs."""
    B, G, k = cand.shape
    row_of = np.zeros((B, G, k + 1), np.int32)
    R = 1
    for b in range(B):
        seen = {}
        for i in range(k + 1):
            for g in range(G):
                key = tuple(int(t) for t in cand[b, g, :i])
                if key not in seen:
                    seen[key] = len(seen)
                row_of[b, g, i] = seen[key]
        R = max(R, len(seen))
    return row_of, R


def make_multi_rows(B: int, G: int, k: int, V: int, t_dtype: str = "bf16", t_std: float = 3.0,
                    p_match: float = 0.6, p_shared: float = 0.5, seed: int = 0,
                    threads: int | None = None) -> dict:
    """The multi-candidate workload in deduplicated form: the candidates of
    make_multi (same seed), rows [B,R,V] holding one row per distinct prefix
    (the row of the first (g, i) with that prefix), and row_of [B,G,k+1].
    Unused row slots of a sequence repeat its last row."""
    w = make_multi(B, G, k, V, t_dtype, t_std, p_match, p_shared, seed, threads)
    row_of, R = prefix_rows(w["tokens"])
    rows = np.empty((B, R, V), w["target"].dtype)
    for b in range(B):
        first = {}
        for i in range(k + 1):
            for g in range(G):
                first.setdefault(int(row_of[b, g, i]), (g, i))
        for r in range(R):
            g, i = first.get(r, first[max(first)])
            rows[b, r] = w["target"][b, g, i]
    return dict(mode="multi_rows", rows=rows, row_of=row_of, t_dtype=t_dtype,
                tokens=w["tokens"], seed=seed, B=B, G=G, k=k, R=R, V=V)


_S_TREE = 40


def tree_parents(N: int, rng, max_children: int = 4) -> np.ndarray:
    """A draft tree of N nodes in topological order: breadth-first, each node
    taking up to `max_children` children, fewer at deeper levels (a Top-K tree
    whose K shrinks with depth).  parent[0] = -1."""
    parent = np.full(N, -1, np.int32)
    frontier, depth, j = [0], 0, 1
    while j < N:
        nxt = []
        for u in frontier:
            kids = max(1, max_children - depth) if depth < 2 else int(rng.integers(1, 3))
            for _ in range(kids):
                if j >= N:
                    break
                parent[j] = u
                nxt.append(j)
                j += 1
        frontier, depth = (nxt or [j - 1]), depth + 1
    return parent


def make_tree(B: int, N: int, V: int, t_dtype: str = "bf16", t_std: float = 3.0,
              p_match: float = 0.7, seed: int = 0, threads: int | None = None) -> dict:
    """Node rows [B,N,V] ~ N(0, t_std^2); per sequence a tree_parents topology;
    children of a node carry distinct tokens, the first one being the node
    row's argmax with probability p_match (so that paths are accepted)."""
    rows = _target_rows(seed, B * N, V, t_std, t_dtype, threads).reshape(B, N, V)
    am = np.argmax(to_f32(rows, t_dtype), -1)
    g = _rng(seed, _S_TREE)
    parent = np.zeros((B, N), np.int32)
    tokens = np.zeros((B, N), np.int32)
    for b in range(B):
        parent[b] = tree_parents(N, g)
        for u in range(N):
            kids = [j for j in range(1, N) if parent[b, j] == u]
            used = set()
            for r, j in enumerate(kids):
                t = int(am[b, u]) if (r == 0 and g.random() < p_match) else int(g.integers(0, V))
                while t in used:
                    t = (t + 1) % V
                used.add(t)
                tokens[b, j] = t
    return dict(mode="tree", node_logits=rows, parent=parent, tokens=tokens, t_dtype=t_dtype,
                seed=seed, B=B, N=N, V=V)


def make(name: str, threads: int | None = None, **overrides) -> dict:
    """Inputs of a named workload (``WORKLOADS``), with optional overrides
    (e.g. ``B=4`` for a bounded sample of the same workload)."""
    cfg = dict(WORKLOADS[name])
    cfg.update(overrides)
    mode = cfg.pop("mode")
    if mode == "stochastic":
        return make_stochastic(threads=threads, **cfg)
    if mode == "greedy":
        return make_greedy(threads=threads, **cfg)
    if mode == "multi":
        return make_multi(threads=threads, **cfg)
    if mode == "multi_rows":
        return make_multi_rows(threads=threads, **cfg)
    if mode == "tree":
        return make_tree(threads=threads, **cfg)
    if mode == "tree_stochastic":
        T = cfg.pop("temperature")
        w = make_tree(threads=threads, **cfg)
        w.update(mode="tree_stochastic", temperature=T)
        return w
    if mode == "threshold":
        T, tau = cfg.pop("temperature"), cfg.pop("threshold")
        w = make_greedy(threads=threads, **cfg)
        w.update(mode="threshold", temperature=T, threshold=tau)
        return w
    raise ValueError(mode)


def logit_bytes(w: dict) -> int:
    """Bytes of logits a verify call over workload ``w`` streams (all rows)."""
    key = "rows" if "rows" in w else ("node_logits" if "node_logits" in w else "target")
    n = w[key].size * ELEM_BYTES[w["t_dtype"]]
    if "draft" in w:
        n += w["draft"].size * ELEM_BYTES[w["d_dtype"]]
    return n
