"""CPU oracle for the speculative-decoding verify-and-accept step.

TEST INFRASTRUCTURE, NOT PRODUCT CODE.  Only ``tests/``, the smoke check in
``__graft_entry__`` and the CPU-baseline leg of ``bench.py`` may import this
package.  The GPU library never imports it and shares no code with it.

The arithmetic lives in ``spec_verify_oracle.c`` (plain C, fp64); this module
compiles it with gcc on first use and marshals numpy arrays into it.  Logit
arrays are passed as ``(array, dtype)`` where dtype is ``"f32"`` (a float32
array) or ``"bf16"`` (a uint16/int16 array holding bf16 bit patterns).
Strides are taken from the numpy array, in elements; the vocabulary axis
must be contiguous.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "spec_verify_oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")

DTYPE_CODES = {"f32": 0, "bf16": 1}

_lib = None
_lock = threading.Lock()


def build(force: bool = False) -> str:
    """Compile the oracle into ``oracle/_build/liboracle.so`` (gcc -O2)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)) or (
        os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        # -ffp-contract=off: no fused multiply-adds, so each fp64 operation
        # rounds exactly as written.
        cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-ffp-contract=off",
               "-fno-fast-math", "-o", tmp, _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            # SV_ORACLE_LIB names another build of this same source with one
            # planted mistake; the planted-mistake tests run the pins against
            # it to show that they catch the mistake.
            lib = ctypes.CDLL(os.environ.get("SV_ORACLE_LIB") or build())
            P = ctypes.c_void_p
            i64, i32, u32, u64, dbl = (ctypes.c_int64, ctypes.c_int, ctypes.c_uint32,
                                       ctypes.c_uint64, ctypes.c_double)
            lib.oracle_philox_batch.argtypes = [P, i64, u64, P]
            lib.oracle_philox_batch.restype = None
            lib.oracle_verify_stochastic.argtypes = [
                P, i32, i64, i64, P, i32, i64, i64, P, i32, i32, i32, dbl, u64, u32,
                i32, i32, P, P, P, P, P, P]
            lib.oracle_verify_stochastic.restype = i32
            lib.oracle_verify_greedy.argtypes = [
                P, i32, i64, i64, P, i32, i32, i32, i32, i32, P, P, P]
            lib.oracle_verify_greedy.restype = i32
            lib.oracle_verify_multi.argtypes = [
                P, i32, i64, i64, i64, P, i32, i32, i32, i32, i32, i32, P, P, P]
            lib.oracle_verify_multi.restype = i32
            lib.oracle_verify_threshold.argtypes = [
                P, i32, i64, i64, P, i32, i32, i32, dbl, dbl, i32, i32, P, P, P]
            lib.oracle_verify_threshold.restype = i32
            lib.oracle_verify_tree_stochastic.argtypes = [
                P, i32, i64, i64, P, P, i32, i32, i32, dbl, u64, u32, i32, i32, P, P, P, P, P, P]
            lib.oracle_verify_tree_stochastic.restype = i32
            _lib = lib
    return _lib


def _ptr(a: np.ndarray | None):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _logits(arr: np.ndarray, dtype: str, ndim: int):
    if dtype not in DTYPE_CODES:
        raise ValueError(f"unknown logit dtype {dtype!r}")
    want = np.float32 if dtype == "f32" else (np.uint16, np.int16)
    if dtype == "f32" and arr.dtype != np.float32:
        raise TypeError("f32 logits must be a float32 array")
    if dtype == "bf16" and arr.dtype not in want:
        raise TypeError("bf16 logits must be a uint16/int16 array of bit patterns")
    if arr.ndim != ndim:
        raise ValueError(f"expected {ndim}-d logits, got shape {arr.shape}")
    if arr.size > 0 and arr.strides[-1] != arr.itemsize:
        raise ValueError("vocabulary axis must be contiguous")
    strides = tuple(s // arr.itemsize for s in arr.strides[:-1])
    return DTYPE_CODES[dtype], strides


def _ranges(B: int, threads: int):
    threads = max(1, min(threads, B))
    edges = np.linspace(0, B, threads + 1).astype(int)
    return [(int(edges[j]), int(edges[j + 1])) for j in range(threads)]


def _run_parallel(fn, B: int, threads: int):
    parts = _ranges(B, threads)
    if len(parts) == 1:
        rc = [fn(*parts[0])]
    else:
        rc = [None] * len(parts)

        def work(j):
            rc[j] = fn(*parts[j])

        ts = [threading.Thread(target=work, args=(j,)) for j in range(len(parts))]
        for t in ts:
            t.start()
        for t in ts:
            t.join()
    if any(r != 0 for r in rc):
        raise ValueError("oracle rejected its arguments")


def philox4x32_10(counters: np.ndarray, seed: int) -> np.ndarray:
    """Philox4x32-10 of each counter row ([n, 4] uint32) under a 64-bit seed."""
    lib = _load()
    c = np.ascontiguousarray(counters, dtype=np.uint32).reshape(-1, 4)
    out = np.empty_like(c)
    lib.oracle_philox_batch(_ptr(c), c.shape[0], int(seed) & (2**64 - 1), _ptr(out))
    return out


def verify_stochastic(target: np.ndarray, t_dtype: str, draft: np.ndarray, d_dtype: str,
                      tokens: np.ndarray, temperature: float, seed: int,
                      seq_offset: int = 0, threads: int = 1) -> dict:
    """Stochastic verify of target [B,k+1,V] against draft [B,k,V].

    ``temperature`` is rounded to float32 first, exactly as the GPU library
    receives it.  Returns accepted_len [B], out_tokens [B,k+1], probs [B,k,2]
    (p_i(x_i), q_i(x_i)), margins [B,k], gaps [B] and flags [B].
    """
    lib = _load()
    tc, (t_sb, t_sp) = _logits(target, t_dtype, 3)
    dc, (d_sb, d_sp) = _logits(draft, d_dtype, 3)
    B, kp1, V = target.shape
    k = kp1 - 1
    if draft.shape[0] != B or draft.shape[1] != k or draft.shape[2] != V:
        raise ValueError("draft must be [B, k, V]")
    tok = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, k)
    T = float(np.float32(temperature))
    out = {
        "accepted_len": np.zeros(B, np.int32),
        "out_tokens": np.zeros((B, k + 1), np.int32),
        "probs": np.zeros((B, k, 2), np.float64),
        "margins": np.zeros((B, k), np.float64),
        "gaps": np.zeros(B, np.float64),
        "flags": np.zeros(B, np.int32),
    }

    def fn(b0, b1):
        return lib.oracle_verify_stochastic(
            _ptr(target), tc, t_sb, t_sp, _ptr(draft), dc, d_sb, d_sp, _ptr(tok), B, k, V, T,
            int(seed) & (2**64 - 1), int(seq_offset) & 0xFFFFFFFF, b0, b1,
            _ptr(out["accepted_len"]), _ptr(out["out_tokens"]), _ptr(out["probs"]),
            _ptr(out["margins"]), _ptr(out["gaps"]), _ptr(out["flags"]))

    _run_parallel(fn, B, threads)
    return out


def verify_greedy(target: np.ndarray, t_dtype: str, tokens: np.ndarray,
                  threads: int = 1) -> dict:
    """Greedy verify of target [B,k+1,V] against draft tokens [B,k]."""
    lib = _load()
    tc, (t_sb, t_sp) = _logits(target, t_dtype, 3)
    B, kp1, V = target.shape
    k = kp1 - 1
    tok = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, k)
    out = {
        "accepted_len": np.zeros(B, np.int32),
        "out_tokens": np.zeros((B, k + 1), np.int32),
        "row_argmax": np.zeros((B, k + 1), np.int32),
    }

    def fn(b0, b1):
        return lib.oracle_verify_greedy(
            _ptr(target), tc, t_sb, t_sp, _ptr(tok), B, k, V, b0, b1,
            _ptr(out["accepted_len"]), _ptr(out["out_tokens"]), _ptr(out["row_argmax"]))

    _run_parallel(fn, B, threads)
    return out


def verify_multi(target: np.ndarray, t_dtype: str, cand: np.ndarray,
                 threads: int = 1) -> dict:
    """Multi-candidate verify of target [B,G,k+1,V] against candidates [B,G,k]."""
    lib = _load()
    tc, (t_sb, t_sg, t_sp) = _logits(target, t_dtype, 4)
    B, G, kp1, V = target.shape
    k = kp1 - 1
    c = np.ascontiguousarray(cand, dtype=np.int32).reshape(B, G, k)
    out = {
        "best_candidate": np.zeros(B, np.int32),
        "accepted_len": np.zeros(B, np.int32),
        "out_tokens": np.zeros((B, k + 1), np.int32),
    }

    def fn(b0, b1):
        return lib.oracle_verify_multi(
            _ptr(target), tc, t_sb, t_sg, t_sp, _ptr(c), B, G, k, V, b0, b1,
            _ptr(out["best_candidate"]), _ptr(out["accepted_len"]), _ptr(out["out_tokens"]))

    _run_parallel(fn, B, threads)
    return out


def verify_multi_rows(rows: np.ndarray, t_dtype: str, row_of: np.ndarray, cand: np.ndarray,
                      threads: int = 1) -> dict:
    """Multi-candidate verify on deduplicated rows [B,R,V] with row_of [B,G,k+1].

    By definition the result of verify_multi on the gathered logits
    E[b,g,i] = rows[b, row_of[b,g,i]].  A map entry outside [0, R) stands for
    a row whose argmax is -1; then the gather is impossible and the same
    decision (per branch the longest prefix equal to the row argmaxes, the
    longest branch, lowest g on a tie) is taken on the row argmaxes directly.
    Also returns "invalid_row": whether such an entry occurred.
    """
    B, R, V = rows.shape
    rmap = np.ascontiguousarray(row_of, dtype=np.int32)
    G, kp1 = rmap.shape[1], rmap.shape[2]
    k = kp1 - 1
    c = np.ascontiguousarray(cand, dtype=np.int32).reshape(B, G, k)
    valid = (rmap >= 0) & (rmap < R)
    if valid.all():
        gathered = np.ascontiguousarray(rows[np.arange(B)[:, None, None], rmap])
        out = verify_multi(gathered, t_dtype, c, threads=threads)
        out["invalid_row"] = False
        return out
    # argmax of every distinct row (first maximum), through the greedy oracle
    flat = np.ascontiguousarray(rows.reshape(B * R, 1, V))
    amax = verify_greedy(flat, t_dtype, np.zeros((B * R, 0), np.int32),
                         threads=threads)["row_argmax"].reshape(B, R)
    out = {"best_candidate": np.zeros(B, np.int32), "accepted_len": np.zeros(B, np.int32),
           "out_tokens": np.full((B, kp1), -1, np.int32), "invalid_row": True}
    for b in range(B):
        a = np.where(valid[b], amax[b][np.clip(rmap[b], 0, R - 1)], -1)  # [G, k+1]
        best_n, best_g = -1, 0
        for g in range(G):
            n = 0
            while n < k and c[b, g, n] == a[g, n]:
                n += 1
            if n > best_n:
                best_n, best_g = n, g
        out["best_candidate"][b] = best_g
        out["accepted_len"][b] = best_n
        out["out_tokens"][b, :best_n] = c[b, best_g, :best_n]
        out["out_tokens"][b, best_n] = a[best_g, best_n]
    return out


def commit(accepted_len: np.ndarray, out_tokens: np.ndarray, seq_len: np.ndarray,
           token_buf: np.ndarray) -> dict:
    """Device-side commit, written out: for each sequence, n = accepted_len
    clamped to [0, k], L = max(seq_len, 0); tokens out_tokens[b, :n+1] go to
    token_buf[b, L:L+n+1] (those at or past the capacity are dropped), the
    length becomes min(L + n + 1, capacity), the next input is out_tokens[b, n].
    Returns copies: seq_len, token_buf, next_input, capacity_hit."""
    out = np.asarray(out_tokens, np.int32)
    B, kp1 = out.shape
    k = kp1 - 1
    buf = np.array(token_buf, np.int32, copy=True)
    cap = buf.shape[1]
    lens = np.array(seq_len, np.int32, copy=True)
    nxt = np.zeros(B, np.int32)
    hit = False
    for b in range(B):
        n = min(max(int(accepted_len[b]), 0), k)
        L = max(int(lens[b]), 0)
        for j in range(n + 1):
            if L + j < cap:
                buf[b, L + j] = out[b, j]
            else:
                hit = True
        lens[b] = min(L + n + 1, cap)
        nxt[b] = out[b, n]
    return {"seq_len": lens, "token_buf": buf, "next_input": nxt, "capacity_hit": hit}


def verify_tree_greedy(node_logits: np.ndarray, t_dtype: str, parent: np.ndarray,
                       tokens: np.ndarray, threads: int = 1) -> dict:
    """Greedy verify of a draft token tree [B,N,V] with parent/tokens [B,N].

    From the root (node 0), step to the lowest-index child whose token equals
    the argmax of the current node's row, until no child matches; commit the
    tokens of the accepted nodes and the argmax of the last one.  A node whose
    parent is outside [0, j) is never entered ("invalid_tree" reports it).
    """
    B, N, V = node_logits.shape
    par = np.ascontiguousarray(parent, dtype=np.int32).reshape(B, N)
    tok = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, N)
    flat = np.ascontiguousarray(node_logits.reshape(B * N, 1, V))
    amax = verify_greedy(flat, t_dtype, np.zeros((B * N, 0), np.int32),
                         threads=threads)["row_argmax"].reshape(B, N)
    out = {"accepted_len": np.zeros(B, np.int32), "path": np.full((B, N), -1, np.int32),
           "out_tokens": np.full((B, N), -1, np.int32), "invalid_tree": False}
    for b in range(B):
        valid = [j >= 1 and 0 <= par[b, j] < j for j in range(N)]
        if any(not valid[j] for j in range(1, N)):
            out["invalid_tree"] = True
        u, n = 0, 0
        out["path"][b, 0] = 0
        while True:
            nxt = [j for j in range(1, N) if valid[j] and par[b, j] == u and tok[b, j] == amax[b, u]]
            if not nxt:
                break
            u = nxt[0]
            out["out_tokens"][b, n] = tok[b, u]
            n += 1
            out["path"][b, n] = u
        out["out_tokens"][b, n] = amax[b, u]
        out["accepted_len"][b] = n
    return out


def verify_tree_stochastic(node_logits: np.ndarray, t_dtype: str, parent: np.ndarray,
                           tokens: np.ndarray, temperature: float, seed: int,
                           seq_offset: int = 0, threads: int = 1) -> dict:
    """Stochastic verify of a draft token tree [B,N,V] with parent/tokens
    [B,N] (node 0 the root; Top-K siblings tried in node order, each accepted
    with probability p(x)/R of the target's distribution left after the
    rejected siblings; the final token drawn from p outside the rejected
    tokens).  ``temperature`` is rounded to float32 first.  Returns
    accepted_len [B], path [B,N], out_tokens [B,N], margins [B,N], gaps [B],
    flags [B] and invalid_tree."""
    lib = _load()
    tc, (sb, sn) = _logits(node_logits, t_dtype, 3)
    B, N, V = node_logits.shape
    par = np.ascontiguousarray(parent, dtype=np.int32).reshape(B, N)
    tok = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, N)
    T = float(np.float32(temperature))
    out = {
        "accepted_len": np.zeros(B, np.int32),
        "path": np.full((B, N), -1, np.int32),
        "out_tokens": np.full((B, N), -1, np.int32),
        "margins": np.full((B, N), np.nan, np.float64),
        "gaps": np.zeros(B, np.float64),
        "flags": np.zeros(B, np.int32),
    }

    def fn(b0, b1):
        return lib.oracle_verify_tree_stochastic(
            _ptr(node_logits), tc, sb, sn, _ptr(par), _ptr(tok), B, N, V, T,
            int(seed) & (2**64 - 1), int(seq_offset) & 0xFFFFFFFF, b0, b1,
            _ptr(out["accepted_len"]), _ptr(out["path"]), _ptr(out["out_tokens"]),
            _ptr(out["margins"]), _ptr(out["gaps"]), _ptr(out["flags"]))

    _run_parallel(fn, B, threads)
    out["invalid_tree"] = bool((out["flags"] & 32).any())
    return out


def verify_threshold(target: np.ndarray, t_dtype: str, tokens: np.ndarray, temperature: float,
                     threshold: float, threads: int = 1) -> dict:
    """Threshold acceptance of target [B,k+1,V] against draft tokens [B,k]:
    n = the longest prefix whose probability under softmax(target/T) is at
    least `threshold`, then the argmax of row n.  temperature and threshold
    are rounded to float32 first, as the GPU library receives them.  Returns
    accepted_len, out_tokens and log_scores [B,k] (ln of the prefix score for
    the examined positions, NaN after)."""
    lib = _load()
    tc, (t_sb, t_sp) = _logits(target, t_dtype, 3)
    B, kp1, V = target.shape
    k = kp1 - 1
    tok = np.ascontiguousarray(tokens, dtype=np.int32).reshape(B, k)
    T = float(np.float32(temperature))
    tau = float(np.float32(threshold))
    out = {"accepted_len": np.zeros(B, np.int32), "out_tokens": np.zeros((B, k + 1), np.int32),
           "log_scores": np.zeros((B, k), np.float64)}

    def fn(b0, b1):
        return lib.oracle_verify_threshold(
            _ptr(target), tc, t_sb, t_sp, _ptr(tok), B, k, V, T, tau, b0, b1,
            _ptr(out["accepted_len"]), _ptr(out["out_tokens"]), _ptr(out["log_scores"]))

    _run_parallel(fn, B, threads)
    return out

