"""Pins of the oracle's near-tie report: acceptance margins and Gumbel gaps.

The GPU parity tests excuse a stochastic mismatch only on a sequence whose
oracle report shows a near tie: an acceptance margin |u_i - p_i(x_i)/q_i(x_i)|
below 1e-5 at an examined position, or a gap below 1e-5 between the best and
the second-best Gumbel-max score of the sampled row.  A mistake in that
report would let real mismatches through, so it is recomputed here from
scratch -- scipy's softmax, numpy arithmetic, and the raw Philox4x32-10
words (pinned to the published known answers in test_oracle_pins.py) --
following the rule as the pages and the method state it:

* "Accelerating Sonar through speculation", section "Draft-Target": the
  full draft and target distributions are compared; the rejection rule of
  speculative sampling accepts x_i while u_i q_i(x_i) < p_i(x_i), and the
  first rejection n takes a draw from normalize(max(0, p_n - q_n)), or from
  p_k when all k drafts are accepted.
* Same page, section "EAGLE": a tree of Top-K candidates; siblings are tried
  in node order with the residual mass R and the rejected set E, and the last
  token is drawn from p outside E.

Draws: u_i = (w >> 8) 2^-24 with w = word 0 of Philox(0, i, b + offset, 0);
Gumbel noise g(x) = -ln(-ln(((w >> 9) + 0.5) 2^-23)) with w = word x & 3 of
Philox(x >> 2, position, b + offset, tag), tag 1 for a correction and 2 for a
bonus.  Scores are ln r(x) + g(x) over r = p_n - q_n > 0 (or l/T + g), and the
gap is the best score minus the best of the other entries.
"""
import numpy as np
import pytest
import scipy.special

import oracle
import workloads

TOL_MARGIN = 1e-12  # both sides are fp64 softmax values; only summation order differs
TOL_GAP = 1e-9      # ln of a residual that may be a difference of close values


# ------------------------------------------------------------ the draws

def philox_row(seed, n_ctr, pos, seq, tag):
    ctr = np.zeros((n_ctr, 4), np.uint32)
    ctr[:, 0] = np.arange(n_ctr, dtype=np.uint32)
    ctr[:, 1] = pos
    ctr[:, 2] = seq
    ctr[:, 3] = tag
    return oracle.philox4x32_10(ctr, seed)


def accept_u(seed, pos, seq):
    w = int(philox_row(seed, 1, pos, seq, 0)[0, 0])
    return (w >> 8) * 2.0 ** -24


def gumbel(seed, V, pos, seq, tag):
    w = philox_row(seed, (V + 3) // 4, pos, seq, tag).reshape(-1)[:V]
    u = ((w >> 9).astype(np.float64) + 0.5) * 2.0 ** -23
    return -np.log(-np.log(u))


def best_and_gap(scores, cand):
    """First maximum over the candidate entries and its lead over the best of
    the others (inf when there is no other candidate)."""
    s = np.where(cand, scores, -np.inf)
    idx = np.nonzero(cand)[0]
    best = int(idx[np.argmax(s[idx])])
    rest = np.delete(s, best)[np.delete(cand, best)]
    second = rest.max() if rest.size else -np.inf
    return best, (np.inf if second == -np.inf else float(s[best] - second))


def logits64(arr, dtype):
    return workloads.to_f32(arr, dtype).astype(np.float64)


# -------------------------------------------------- linear drafts

def report_stochastic(target, t_dtype, draft, d_dtype, tokens, T, seed, seq_offset=0):
    T = float(np.float32(T))
    t, d = logits64(target, t_dtype), logits64(draft, d_dtype)
    B, kp1, V = t.shape
    k = kp1 - 1
    out = {"accepted_len": np.zeros(B, np.int32), "out_tokens": np.full((B, k + 1), -1, np.int32),
           "margins": np.zeros((B, k)), "gaps": np.zeros(B)}
    for b in range(B):
        seq = (b + seq_offset) & 0xFFFFFFFF
        n = k
        for i in range(k):
            x = int(tokens[b, i])
            valid = 0 <= x < V
            p = scipy.special.softmax(t[b, i] / T)[x] if valid else 0.0
            q = scipy.special.softmax(d[b, i] / T)[x] if valid else 0.0
            u = accept_u(seed, i, seq)
            out["margins"][b, i] = abs(u - p / q) if (valid and q > 0) else np.inf
            if n == k and not (valid and u * q < p):
                n = i
        if n < k:
            g = gumbel(seed, V, n, seq, 1)
            r = scipy.special.softmax(t[b, n] / T) - scipy.special.softmax(d[b, n] / T)
            cand = r > 0
            if cand.any():
                with np.errstate(divide="ignore"):
                    scores = np.log(np.where(cand, r, 1.0)) + g
            else:  # no positive residual (rounding only): a draw from p_n
                cand, scores = np.ones(V, bool), t[b, n] / T + g
        else:
            cand, scores = np.ones(V, bool), t[b, k] / T + gumbel(seed, V, k, seq, 2)
        y, out["gaps"][b] = best_and_gap(scores, cand)
        out["accepted_len"][b] = n
        out["out_tokens"][b, :n] = tokens[b, :n]
        out["out_tokens"][b, n] = y
    return out


def check_stochastic(target, t_dtype, draft, d_dtype, tokens, T, seed, seq_offset=0):
    o = oracle.verify_stochastic(target, t_dtype, draft, d_dtype, tokens, T, seed, seq_offset)
    ref = report_stochastic(target, t_dtype, draft, d_dtype, tokens, T, seed, seq_offset)
    np.testing.assert_array_equal(o["accepted_len"], ref["accepted_len"])
    np.testing.assert_array_equal(o["out_tokens"], ref["out_tokens"])
    np.testing.assert_array_equal(np.isinf(o["margins"]), np.isinf(ref["margins"]))
    fin = np.isfinite(ref["margins"])
    np.testing.assert_allclose(o["margins"][fin], ref["margins"][fin], atol=TOL_MARGIN, rtol=0)
    np.testing.assert_array_equal(np.isinf(o["gaps"]), np.isinf(ref["gaps"]))
    fin = np.isfinite(ref["gaps"])
    np.testing.assert_allclose(o["gaps"][fin], ref["gaps"][fin], atol=TOL_GAP, rtol=0)
    return o


@pytest.mark.parametrize("t_dtype,d_dtype,T,seed", [
    ("f32", "f32", 1.0, 0), ("bf16", "f32", 0.7, 1), ("bf16", "bf16", 1.3, 2),
    ("f32", "bf16", 0.4, 3)])
def test_margins_and_gaps_recomputed(t_dtype, d_dtype, T, seed):
    # drafts sampled from q (so long prefixes and both draw kinds occur), plus
    # a few invalid tokens and zero-probability tokens
    w = workloads.make_stochastic(B=40, k=5, V=1031, t_dtype=t_dtype, d_dtype=d_dtype,
                                  t_std=2.0, d_noise=0.6, temperature=T, seed=seed + 10)
    tok = w["tokens"].copy()
    tok[3, 1] = -1
    tok[7, 0] = 1031
    o = check_stochastic(w["target"], t_dtype, w["draft"], d_dtype, tok, T, seed, 7)
    n = o["accepted_len"]
    assert (n < 5).any() and (n == 5).any(), "both the correction and the bonus draw"
    assert np.isinf(o["margins"][3, 1]) and np.isinf(o["margins"][7, 0])


def test_margins_and_gaps_with_ties_and_masked_entries():
    """Rows with -inf entries (q = 0 at the token, p = 0 at the token), and
    rows with a single candidate, whose gap is infinite: a bonus row with one
    finite logit, and a correction row where only one entry has p > q."""
    rng = np.random.default_rng(5)
    B, k, V = 30, 3, 64
    t = (rng.standard_normal((B, k + 1, V)) * 1.5).astype(np.float32)
    d = (t[:, :k] + rng.standard_normal((B, k, V)).astype(np.float32)).astype(np.float32)
    t[rng.random(t.shape) < 0.1] = -np.inf
    d[rng.random(d.shape) < 0.1] = -np.inf
    for b in range(B):
        t[b, :, 0] = 0.0  # every row keeps a finite logit
        d[b, :, 0] = 0.0
    tok = rng.integers(0, V, (B, k)).astype(np.int32)
    # identical target and draft rows accept everything; one finite entry in
    # the bonus row of those sequences
    t[:4, :k] = d[:4]
    tok[:4] = 0  # a finite entry: p = q > 0
    t[:4, k, 1:] = -np.inf
    # a target row with all its mass on entry 3 against a draft token with
    # p = 0: rejected at position 0, and only entry 3 has p - q > 0
    t[4:6, 0, :] = -np.inf
    t[4:6, 0, 3] = 0.0
    tok[4:6, 0] = 0
    o = check_stochastic(t, "f32", d, "f32", tok, 1.0, 9)
    assert (o["accepted_len"][:4] == k).all() and np.isinf(o["gaps"][:6]).all()
    assert (o["out_tokens"][:4, k] == 0).all()
    assert (o["accepted_len"][4:6] == 0).all() and (o["out_tokens"][4:6, 0] == 3).all()
    assert np.isfinite(o["gaps"][6:]).any()


def test_zero_drafts_gap_is_the_bonus_rows():
    rng = np.random.default_rng(6)
    t = (rng.standard_normal((25, 1, 300)) * 2).astype(np.float32)
    check_stochastic(t, "f32", np.zeros((25, 0, 300), np.float32), "f32",
                     np.zeros((25, 0), np.int32), 0.9, 4, 3)


# ------------------------------------------------------------------ trees

def report_tree(logits, dtype, parent, tokens, T, seed, seq_offset=0):
    T = float(np.float32(T))
    lg = logits64(logits, dtype)
    B, N, V = lg.shape
    out = {"accepted_len": np.zeros(B, np.int32), "path": np.full((B, N), -1, np.int32),
           "out_tokens": np.full((B, N), -1, np.int32), "margins": np.full((B, N), np.nan),
           "gaps": np.zeros(B)}
    for b in range(B):
        seq = (b + seq_offset) & 0xFFFFFFFF
        u, n, path = 0, 0, [0]
        while True:
            p = scipy.special.softmax(lg[b, u] / T)
            R, E, nxt, has_child = 1.0, [], -1, False
            for j in range(u + 1, N):
                if parent[b, j] != u:
                    continue
                has_child = True
                x = int(tokens[b, j])
                open_ = 0 <= x < V and x not in E
                pj = p[x] if open_ else 0.0
                uj = accept_u(seed, j - 1, seq)
                out["margins"][b, j] = abs(uj - pj / R) if (open_ and R > 0) else np.inf
                if open_ and uj * R < pj:
                    nxt = j
                    break
                if open_:
                    E.append(x)
                    R -= pj
            if nxt < 0:
                break
            u = nxt
            out["out_tokens"][b, n] = tokens[b, u]
            n += 1
            path.append(u)
        scores = lg[b, u] / T + gumbel(seed, V, u, seq, 1 if has_child else 2)
        cand = np.isfinite(lg[b, u])
        cand[E] = False
        if not cand.any():
            cand = np.ones(V, bool)
        y, out["gaps"][b] = best_and_gap(scores, cand)
        out["out_tokens"][b, n] = y
        out["path"][b, : n + 1] = path
        out["accepted_len"][b] = n
    return out


def random_trees(rng, B, N, V, K=3):
    """Breadth-first trees: node j's parent is an earlier node, at most K
    children each; sibling tokens mostly distinct and mostly likely ones."""
    parent = np.full((B, N), -1, np.int32)
    tokens = np.zeros((B, N), np.int32)
    for b in range(B):
        kids = {0: 0}
        for j in range(1, N):
            choices = [u for u in range(j) if kids.get(u, 0) < K]
            u = choices[rng.integers(min(len(choices), 3))]
            parent[b, j] = u
            first = kids.get(u, 0) == 0
            kids[u] = kids.get(u, 0) + 1
            kids[j] = 0
            # a node's first child mostly takes the likely token 0
            tokens[b, j] = 0 if (first and rng.random() < 0.8) else rng.integers(V)
    return parent, tokens


@pytest.mark.parametrize("dtype,T", [("f32", 1.0), ("bf16", 0.6)])
def test_tree_margins_and_gaps_recomputed(dtype, T):
    rng = np.random.default_rng(71)
    B, N, V = 40, 12, 97
    x = (rng.standard_normal((B, N, V)) * 1.5).astype(np.float32)
    x[:, :, 0] += 5.0  # token 0 likely, so that paths get long
    parent, tokens = random_trees(rng, B, N, V)
    tokens[2, 1] = V + 4  # an invalid token
    tokens[4, parent[4] == 0] = 0  # every root child of tree 4 repeats one token
    arr = workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x
    o = oracle.verify_tree_stochastic(arr, dtype, parent, tokens, T, seed=13, seq_offset=5)
    ref = report_tree(arr, dtype, parent, tokens, T, seed=13, seq_offset=5)
    for key in ("accepted_len", "path", "out_tokens"):
        np.testing.assert_array_equal(o[key], ref[key], err_msg=key)
    np.testing.assert_array_equal(np.isnan(o["margins"]), np.isnan(ref["margins"]))
    np.testing.assert_array_equal(np.isinf(o["margins"]), np.isinf(ref["margins"]))
    fin = np.isfinite(ref["margins"])
    np.testing.assert_allclose(o["margins"][fin], ref["margins"][fin], atol=TOL_MARGIN, rtol=0)
    fin = np.isfinite(ref["gaps"])
    np.testing.assert_array_equal(np.isfinite(o["gaps"]), fin)
    np.testing.assert_allclose(o["gaps"][fin], ref["gaps"][fin], atol=TOL_GAP, rtol=0)
    assert o["accepted_len"].max() >= 2 and (o["accepted_len"] == 0).any()
    kids = np.nonzero(parent[4] == 0)[0]
    if o["path"][4, 1] != kids[0]:  # the first root child was rejected: repeats cannot win
        assert np.isinf(o["margins"][4, kids[1:]]).all()
