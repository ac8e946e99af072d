"""Pins of the CPU oracle against what the method and the mathematics fix.

Nothing here compares the oracle with itself: each check is a published
known answer, a library routine, an exact law of speculative sampling
(chi-square over 10^6 seeded trials), a hand case with a known outcome, or
brute force on a tiny input.
"""
import itertools
import math
import os

import numpy as np
import pytest
import scipy.special
import scipy.stats

import oracle
import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
THREADS = min(8, os.cpu_count() or 1)
P_MIN = 0.01


# ------------------------------------------------------------------ helpers

def chi2_pvalue(observed_counts, expected_probs, min_expected=5.0):
    """Chi-square goodness of fit; bins with small expectation are pooled."""
    obs = np.asarray(observed_counts, np.float64)
    exp = np.asarray(expected_probs, np.float64) * obs.sum()
    order = np.argsort(exp)
    o_b, e_b, acc_o, acc_e = [], [], 0.0, 0.0
    for j in order:
        acc_o += obs[j]
        acc_e += exp[j]
        if acc_e >= min_expected:
            o_b.append(acc_o)
            e_b.append(acc_e)
            acc_o = acc_e = 0.0
    if acc_e > 0 or acc_o > 0:
        if e_b:
            o_b[-1] += acc_o
            e_b[-1] += acc_e
        else:
            o_b.append(acc_o)
            e_b.append(acc_e)
    assert not np.any((np.array(e_b) == 0) & (np.array(o_b) > 0)), "impossible outcome observed"
    if len(o_b) < 2:
        return 1.0
    return scipy.stats.chisquare(o_b, e_b).pvalue


def softmax64(logits_f32, T):
    return scipy.special.softmax(np.asarray(logits_f32, np.float64) / float(np.float32(T)), axis=-1)


def draw_tokens(q, trials, seed):
    """tokens[b, i] ~ q_i, independent over b and i (numpy's own sampler)."""
    g = np.random.default_rng(seed)
    k, V = q.shape
    return np.stack([g.choice(V, size=trials, p=q[i]) for i in range(k)], axis=1).astype(np.int32)


def broadcast_run(tl, dl, T, trials, seed, tokens=None, token_seed=123):
    """One fixed set of rows shared by `trials` sequences (stride 0 batch)."""
    k = dl.shape[0]
    target = np.broadcast_to(tl.astype(np.float32), (trials,) + tl.shape)
    draft = np.broadcast_to(dl.astype(np.float32), (trials,) + dl.shape)
    if tokens is None:
        tokens = draw_tokens(softmax64(dl, T), trials, token_seed)
    r = oracle.verify_stochastic(target, "f32", draft, "f32", tokens, T, seed, threads=THREADS)
    return r, tokens


def exact_law(p, q):
    """Closed forms of speculative sampling when drafts x_i ~ q_i independently."""
    k = q.shape[0]
    alpha = np.minimum(p[:k], q).sum(-1)
    P_n = np.array([np.prod(alpha[:j]) * (1.0 - alpha[j]) for j in range(k)]
                   + [np.prod(alpha)])
    resid = np.maximum(p[:k] - q, 0.0)
    with np.errstate(invalid="ignore", divide="ignore"):
        resid = resid / resid.sum(-1, keepdims=True)
    return alpha, P_n, resid


# ---------------------------------------------------------------- Philox

def read_kat():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            w = [int(t, 16) for t in line.split()]
            rows.append((w[0:4], w[4:6], w[6:10]))
    return rows


def test_philox_known_answers():
    kat = read_kat()
    assert len(kat) == 3
    for ctr, key, out in kat:
        seed = key[0] | (key[1] << 32)
        got = oracle.philox4x32_10(np.array([ctr], np.uint32), seed)[0]
        assert [int(v) for v in got] == out


def test_philox_output_bytes_uniform():
    ctr = np.zeros((1 << 15, 4), np.uint32)
    ctr[:, 0] = np.arange(1 << 15)
    ctr[:, 1] = 7
    ctr[:, 2] = 3
    out = oracle.philox4x32_10(ctr, 0x0123456789ABCDEF)
    counts = np.bincount(out.view(np.uint8).ravel(), minlength=256)
    assert chi2_pvalue(counts, np.full(256, 1 / 256)) > P_MIN


# --------------------------------------------------- softmax probabilities

@pytest.mark.parametrize("t_dtype,d_dtype,T", [
    ("f32", "f32", 1.0), ("bf16", "f32", 0.7), ("bf16", "bf16", 1.3), ("f32", "bf16", 0.25)])
def test_probs_match_library_softmax(t_dtype, d_dtype, T):
    B, k, V = 3, 4, 37
    w = workloads.make_stochastic(B, k, V, t_dtype, d_dtype, t_std=3.0, d_noise=1.0,
                                  temperature=T, seed=11)
    r = oracle.verify_stochastic(w["target"], t_dtype, w["draft"], d_dtype, w["tokens"], T, 5)
    p = softmax64(workloads.to_f32(w["target"], t_dtype), T)
    q = softmax64(workloads.to_f32(w["draft"], d_dtype), T)
    bi = np.arange(B)[:, None]
    ii = np.arange(k)[None, :]
    np.testing.assert_allclose(r["probs"][..., 0], p[bi, ii, w["tokens"]], rtol=1e-12, atol=0)
    np.testing.assert_allclose(r["probs"][..., 1], q[bi, ii, w["tokens"]], rtol=1e-12, atol=0)


# ------------------------------------------------- exact laws (chi-square)

@pytest.fixture(scope="module")
def law_case():
    rng = np.random.default_rng(2024)
    k, V, T = 3, 6, 0.8
    tl = (rng.standard_normal((k + 1, V)) * 1.5).astype(np.float32)
    dl = (tl[:k] + rng.standard_normal((k, V))).astype(np.float32)
    trials = 1_000_000
    r, tokens = broadcast_run(tl, dl, T, trials, seed=77)
    p = softmax64(tl, T)
    q = softmax64(dl, T)
    return dict(k=k, V=V, T=T, p=p, q=q, r=r, tokens=tokens, trials=trials)


def test_first_committed_token_follows_target(law_case):
    c = law_case
    counts = np.bincount(c["r"]["out_tokens"][:, 0], minlength=c["V"])
    assert chi2_pvalue(counts, c["p"][0]) > P_MIN


def test_accepted_length_closed_form(law_case):
    c = law_case
    _, P_n, _ = exact_law(c["p"], c["q"])
    counts = np.bincount(c["r"]["accepted_len"], minlength=c["k"] + 1)
    assert chi2_pvalue(counts, P_n) > P_MIN


def test_token_at_each_position_follows_target(law_case):
    """Given positions < m accepted, the token committed at m is ~ p_m."""
    c = law_case
    for m in range(1, c["k"] + 1):
        sel = c["r"]["accepted_len"] >= m
        counts = np.bincount(c["r"]["out_tokens"][sel, m], minlength=c["V"])
        assert chi2_pvalue(counts, c["p"][m]) > P_MIN, m


def test_correction_follows_residual(law_case):
    c = law_case
    _, _, resid = exact_law(c["p"], c["q"])
    for j in range(c["k"]):
        sel = c["r"]["accepted_len"] == j
        counts = np.bincount(c["r"]["out_tokens"][sel, j], minlength=c["V"])
        assert chi2_pvalue(counts, resid[j]) > P_MIN, j


def test_bonus_follows_last_target_row(law_case):
    c = law_case
    sel = c["r"]["accepted_len"] == c["k"]
    assert sel.sum() > 10_000
    counts = np.bincount(c["r"]["out_tokens"][sel, c["k"]], minlength=c["V"])
    assert chi2_pvalue(counts, c["p"][c["k"]]) > P_MIN


def test_accepted_prefix_is_the_drafts(law_case):
    c = law_case
    n = c["r"]["accepted_len"]
    out = c["r"]["out_tokens"]
    for i in range(c["k"]):
        sel = n > i
        assert np.array_equal(out[sel, i], c["tokens"][sel, i])
        assert np.all(out[n < i, i] == -1)


# --------------------------------------------------------------- hand cases

def test_identical_distributions_accept_everything():
    rng = np.random.default_rng(5)
    k, V, T, trials = 4, 7, 1.0, 200_000
    tl = (rng.standard_normal((k + 1, V)) * 2).astype(np.float32)
    dl = tl[:k].copy()
    r, _ = broadcast_run(tl, dl, T, trials, seed=3)
    assert np.all(r["accepted_len"] == k)
    counts = np.bincount(r["out_tokens"][:, k], minlength=V)
    assert chi2_pvalue(counts, softmax64(tl, T)[k]) > P_MIN
    assert np.all(r["flags"] == 0)


def test_disjoint_supports_reject_first_and_resample_target():
    rng = np.random.default_rng(6)
    k, V, T, trials = 3, 8, 0.9, 200_000
    tl = (rng.standard_normal((k + 1, V))).astype(np.float32)
    dl = (rng.standard_normal((k, V))).astype(np.float32)
    tl[:, : V // 2] = -np.inf  # target lives on the upper half
    dl[:, V // 2:] = -np.inf   # draft lives on the lower half
    r, tokens = broadcast_run(tl, dl, T, trials, seed=4)
    assert np.all(tokens < V // 2)
    assert np.all(r["accepted_len"] == 0)
    np.testing.assert_array_equal(r["probs"][:, :, 0], 0.0)
    counts = np.bincount(r["out_tokens"][:, 0], minlength=V)
    assert chi2_pvalue(counts, softmax64(tl, T)[0]) > P_MIN


def test_one_hot_draft_accepts_with_target_probability():
    rng = np.random.default_rng(7)
    k, V, T, trials, xs = 1, 9, 1.0, 400_000, 4
    tl = (rng.standard_normal((k + 1, V)) * 1.2).astype(np.float32)
    dl = np.full((k, V), -np.inf, np.float32)
    dl[0, xs] = 0.0
    r, tokens = broadcast_run(tl, dl, T, trials, seed=9)
    assert np.all(tokens == xs)
    p = softmax64(tl, T)
    acc = int((r["accepted_len"] == 1).sum())
    assert scipy.stats.binomtest(acc, trials, p[0, xs]).pvalue > P_MIN
    sel = r["accepted_len"] == 0
    law = p[0].copy()
    law[xs] = 0.0
    law /= law.sum()
    counts = np.bincount(r["out_tokens"][sel, 0], minlength=V)
    assert counts[xs] == 0
    assert chi2_pvalue(counts, law) > P_MIN


def test_invalid_token_is_rejected_and_residual_fallback_draws_target():
    rng = np.random.default_rng(8)
    k, V, T, trials = 3, 6, 1.0, 200_000
    tl = (rng.standard_normal((k + 1, V))).astype(np.float32)
    dl = tl[:k].copy()
    tokens = draw_tokens(softmax64(dl, T), trials, 99)
    tokens[:, 1] = np.where(np.arange(trials) % 2 == 0, V, -1)  # out of range
    r, _ = broadcast_run(tl, dl, T, trials, seed=10, tokens=tokens)
    assert np.all(r["accepted_len"] == 1)
    assert np.all(r["flags"] == 3)
    np.testing.assert_array_equal(r["probs"][:, 1, :], 0.0)
    counts = np.bincount(r["out_tokens"][:, 1], minlength=V)
    assert chi2_pvalue(counts, softmax64(tl, T)[1]) > P_MIN
    assert np.all(r["out_tokens"][:, 2:] == -1)


def test_bad_temperature_rejected():
    w = workloads.make_stochastic(1, 2, 5, "f32", "f32", seed=1)
    for T in (0.0, -1.0, float("nan")):
        with pytest.raises(ValueError):
            oracle.verify_stochastic(w["target"], "f32", w["draft"], "f32", w["tokens"], T, 0)


def test_rule_reproduces_target_law_by_enumeration():
    """Brute force over every draft tuple (V=4, k=3): the accept/residual
    rule, weighted by the draft law, gives exactly p_m at every position."""
    rng = np.random.default_rng(3)
    k, V = 3, 4
    p = scipy.special.softmax(rng.standard_normal((k + 1, V)) * 1.3, axis=-1)
    q = scipy.special.softmax(rng.standard_normal((k, V)) * 1.3, axis=-1)
    law = np.zeros((k + 1, V))
    mass_reach = np.zeros(k + 1)
    for xs in itertools.product(range(V), repeat=k):
        w = np.prod([q[i, xs[i]] for i in range(k)])
        reach = 1.0
        for i in range(k):
            a = min(1.0, p[i, xs[i]] / q[i, xs[i]])
            mass_reach[i] += w * reach
            law[i, xs[i]] += w * reach * a
            r = np.maximum(p[i] - q[i], 0.0)
            if r.sum() > 0:
                law[i] += w * reach * (1 - a) * r / r.sum()
            reach *= a
        mass_reach[k] += w * reach
        law[k] += w * reach * p[k]
    for m in range(k + 1):
        np.testing.assert_allclose(law[m] / mass_reach[m], p[m], atol=1e-12)


# ---------------------------------------------------------------- greedy

def plain_greedy(rows_f32, tokens):
    """Argmax decoding by numpy: first maximum per row, longest prefix."""
    B, kp1, V = rows_f32.shape
    k = kp1 - 1
    a = np.argmax(rows_f32, axis=-1)
    n = np.full(B, k)
    out = np.full((B, k + 1), -1)
    for b in range(B):
        for i in range(k):
            if tokens[b, i] != a[b, i]:
                n[b] = i
                break
        out[b, : n[b]] = tokens[b, : n[b]]
        out[b, n[b]] = a[b, n[b]]
    return n, out, a


def tie_heavy_rows(rng, shape):
    x = rng.integers(-3, 4, size=shape).astype(np.float32)  # many exact ties
    x[rng.random(shape) < 0.05] = -np.inf
    zeros = x == 0
    x[zeros & (rng.random(shape) < 0.5)] = -0.0
    return x


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_greedy_equals_argmax_decoding(dtype):
    rng = np.random.default_rng(12)
    B, k, V = 200, 5, 33
    x = tie_heavy_rows(rng, (B, k + 1, V))
    arr = workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x
    a = np.argmax(x, axis=-1)
    tokens = np.where(rng.random((B, k)) < 0.8, a[:, :k], rng.integers(0, V, (B, k)))
    tokens[0, 0] = V + 5  # out of range: never matches
    tokens = tokens.astype(np.int32)
    r = oracle.verify_greedy(arr, dtype, tokens)
    n, out, am = plain_greedy(x, tokens)
    np.testing.assert_array_equal(r["accepted_len"], n)
    np.testing.assert_array_equal(r["out_tokens"], out)
    np.testing.assert_array_equal(r["row_argmax"], am)


def test_greedy_signed_zero_and_all_neg_inf():
    x = np.array([[[-0.0, 0.0, -1.0], [-np.inf, -np.inf, -np.inf]]], np.float32)
    r = oracle.verify_greedy(x, "f32", np.array([[0]], np.int32))
    assert r["row_argmax"].tolist() == [[0, 0]]
    assert r["accepted_len"].tolist() == [1]
    assert r["out_tokens"].tolist() == [[0, 0]]


def test_greedy_zero_drafts_is_argmax():
    rng = np.random.default_rng(1)
    x = rng.standard_normal((4, 1, 50)).astype(np.float32)
    r = oracle.verify_greedy(x, "f32", np.zeros((4, 0), np.int32))
    np.testing.assert_array_equal(r["accepted_len"], 0)
    np.testing.assert_array_equal(r["out_tokens"][:, 0], np.argmax(x[:, 0], -1))


# ---------------------------------------------------------- multi-candidate

def plain_multi(rows_f32, cand):
    B, G, kp1, V = rows_f32.shape
    k = kp1 - 1
    a = np.argmax(rows_f32, axis=-1)
    best_g = np.zeros(B, int)
    n_out = np.zeros(B, int)
    out = np.full((B, k + 1), -1)
    for b in range(B):
        ns = []
        for g in range(G):
            m = 0
            while m < k and cand[b, g, m] == a[b, g, m]:
                m += 1
            ns.append(m)
        g = int(np.argmax(ns))  # first of the longest
        best_g[b], n_out[b] = g, ns[g]
        out[b, : ns[g]] = cand[b, g, : ns[g]]
        out[b, ns[g]] = a[b, g, ns[g]]
    return best_g, n_out, out


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_multi_bruteforce(dtype):
    rng = np.random.default_rng(21)
    B, G, k, V = 60, 5, 4, 17
    x = tie_heavy_rows(rng, (B, G, k + 1, V))
    arr = workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x
    a = np.argmax(x, axis=-1)
    cand = np.where(rng.random((B, G, k)) < 0.7, a[:, :, :k], rng.integers(0, V, (B, G, k)))
    cand = cand.astype(np.int32)
    r = oracle.verify_multi(arr, dtype, cand)
    bg, n, out = plain_multi(x, cand)
    np.testing.assert_array_equal(r["best_candidate"], bg)
    np.testing.assert_array_equal(r["accepted_len"], n)
    np.testing.assert_array_equal(r["out_tokens"], out)


def test_multi_single_branch_equals_greedy():
    w = workloads.make_multi(B=12, G=1, k=4, V=300, p_match=0.7, seed=9)
    r = oracle.verify_multi(w["target"], "bf16", w["tokens"])
    g = oracle.verify_greedy(w["target"][:, 0], "bf16", w["tokens"][:, 0])
    np.testing.assert_array_equal(r["best_candidate"], 0)
    np.testing.assert_array_equal(r["accepted_len"], g["accepted_len"])
    np.testing.assert_array_equal(r["out_tokens"], g["out_tokens"])


def test_multi_all_branches_empty_picks_branch_zero():
    x = np.zeros((1, 3, 2, 4), np.float32)
    x[..., 2] = 1.0  # argmax 2 everywhere
    cand = np.zeros((1, 3, 1), np.int32)  # never 2
    r = oracle.verify_multi(x, "f32", cand)
    assert r["best_candidate"].tolist() == [0]
    assert r["accepted_len"].tolist() == [0]
    assert r["out_tokens"].tolist() == [[2, -1]]


# ------------------------------------------------ multi-candidate, rows form

def test_prefix_rows_hand_case():
    # branch 0: 5 6 ; branch 1: 5 7 ; branch 2: 9 6
    cand = np.array([[[5, 6], [5, 7], [9, 6]]], np.int32)
    row_of, R = workloads.prefix_rows(cand)
    # i = 0: all share the empty prefix -> row 0
    # i = 1: prefixes (5,) (5,) (9,) -> rows 1, 1, 2
    # i = 2: prefixes (5,6) (5,7) (9,6) -> rows 3, 4, 5
    assert R == 6
    assert row_of.tolist() == [[[0, 1, 3], [0, 1, 4], [0, 2, 5]]]


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_multi_rows_bruteforce(dtype):
    """Rows form against a plain argmax decision on the gathered rows."""
    rng = np.random.default_rng(31)
    B, G, k, R, V = 40, 5, 3, 9, 13
    x = tie_heavy_rows(rng, (B, R, V))
    arr = workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x
    row_of = rng.integers(0, R, (B, G, k + 1)).astype(np.int32)
    a = np.argmax(x, axis=-1)
    gathered = x[np.arange(B)[:, None, None], row_of]
    ga = np.argmax(gathered, -1)
    cand = np.where(rng.random((B, G, k)) < 0.7, ga[:, :, :k], rng.integers(0, V, (B, G, k)))
    cand = cand.astype(np.int32)
    r = oracle.verify_multi_rows(arr, dtype, row_of, cand)
    bg, n, out = plain_multi(gathered, cand)
    assert not r["invalid_row"]
    np.testing.assert_array_equal(r["best_candidate"], bg)
    np.testing.assert_array_equal(r["accepted_len"], n)
    np.testing.assert_array_equal(r["out_tokens"], out)
    assert a.shape == (B, R)


def test_multi_rows_invalid_entry_hand_case():
    # rows: argmax of row 0 is 1, of row 1 is 2
    rows = np.array([[[0.0, 5.0, 1.0], [0.0, 1.0, 5.0]]], np.float32)
    cand = np.array([[[1, 2], [1, 2]]], np.int32)
    # branch 0: rows 0, 1, 1 -> accepts 1 (=argmax row 0), 2 (=argmax row 1), next = 2
    # branch 1: rows 0, 7 (invalid), 1 -> accepts 1, stops at the invalid row
    row_of = np.array([[[0, 1, 1], [0, 7, 1]]], np.int32)
    r = oracle.verify_multi_rows(rows, "f32", row_of, cand)
    assert r["invalid_row"]
    assert r["best_candidate"].tolist() == [0]
    assert r["accepted_len"].tolist() == [2]
    assert r["out_tokens"].tolist() == [[1, 2, 2]]
    # only the invalid branch left: it commits -1 where it stops
    r = oracle.verify_multi_rows(rows, "f32", row_of[:, 1:], cand[:, 1:])
    assert r["accepted_len"].tolist() == [1]
    assert r["out_tokens"].tolist() == [[1, -1, -1]]


# ------------------------------------------------------ threshold acceptance

def test_threshold_uniform_rows_closed_form():
    # uniform rows over V: every drafted token has p = 1/V, score(j) = V^-j
    B, k, V = 3, 6, 4
    x = np.zeros((B, k + 1, V), np.float32)
    tokens = np.tile(np.arange(k, dtype=np.int32) % V, (B, 1))
    for tau, n in ((0.9, 0), (0.2, 1), (0.05, 2), (0.01, 3), (0.003, 4), (1e-30, k)):
        r = oracle.verify_threshold(x, "f32", tokens, 1.0, tau)
        assert r["accepted_len"].tolist() == [n] * B, tau
        assert r["out_tokens"][:, n].tolist() == [0] * B  # argmax of a flat row: first entry
        assert (r["out_tokens"][:, :n] == tokens[:, :n]).all()


def test_threshold_low_temperature_is_greedy():
    """As T -> 0, p_i(x_i) -> 1 for the row argmax and -> 0 otherwise, so a
    threshold of 1/2 reproduces greedy verify (rows without tied maxima)."""
    w = workloads.make_greedy(B=40, k=5, V=200, t_dtype="f32", p_match=0.7, seed=17)
    srt = np.sort(w["target"], -1)
    assert (srt[..., -1] - srt[..., -2] > 1e-4).all()  # clear maxima
    r = oracle.verify_threshold(w["target"], "f32", w["tokens"], 1e-6, 0.5)
    g = oracle.verify_greedy(w["target"], "f32", w["tokens"])
    np.testing.assert_array_equal(r["accepted_len"], g["accepted_len"])
    np.testing.assert_array_equal(r["out_tokens"], g["out_tokens"])


def test_threshold_monotone_and_invalid_token():
    w = workloads.make_greedy(B=30, k=6, V=100, p_match=0.6, seed=18)
    ns = [oracle.verify_threshold(w["target"], "bf16", w["tokens"], 1.0, tau)["accepted_len"]
          for tau in (1e-12, 1e-6, 1e-3, 0.1, 0.5, 1.0)]
    for a, b in zip(ns, ns[1:]):
        assert (a >= b).all()  # a higher threshold never accepts more
    tok = w["tokens"].copy()
    tok[:, 2] = -1  # probability 0 at position 2
    r = oracle.verify_threshold(w["target"], "bf16", tok, 1.0, 1e-30)
    assert (r["accepted_len"] <= 2).all()
    assert (r["accepted_len"] == 2).sum() > 0


# ---------------------------------------------------------------- tree verify

def longest_matching_path(parent, tokens, amax):
    """Independent formulation: among all root paths whose every node's token
    equals its parent's argmax, the longest (depth-first over all nodes)."""
    N = len(parent)
    best = [0]
    stack = [[0]]
    while stack:
        path = stack.pop()
        if len(path) > len(best):
            best = path
        u = path[-1]
        for j in range(1, N):
            if parent[j] == u and tokens[j] == amax[u]:
                stack.append(path + [j])
    return best


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_tree_walk_is_the_longest_matching_path(dtype):
    rng = np.random.default_rng(41)
    B, N, V = 60, 20, 9
    x = tie_heavy_rows(rng, (B, N, V))
    arr = workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x
    amax = np.argmax(x, -1)
    parent = np.zeros((B, N), np.int32)
    tokens = np.zeros((B, N), np.int32)
    for b in range(B):
        parent[b] = workloads.tree_parents(N, rng)
        for u in range(N):
            kids = [j for j in range(1, N) if parent[b, j] == u]
            toks = rng.permutation(V)[:len(kids)]  # distinct sibling tokens
            if kids and rng.random() < 0.8:
                toks[0] = amax[b, u] if amax[b, u] not in toks[1:] else toks[0]
            tokens[b, kids] = toks
    r = oracle.verify_tree_greedy(arr, dtype, parent, tokens)
    for b in range(B):
        best = longest_matching_path(parent[b], tokens[b], amax[b])
        n = len(best) - 1
        assert r["accepted_len"][b] == n
        assert r["path"][b, :n + 1].tolist() == best
        assert (r["path"][b, n + 1:] == -1).all()
        assert r["out_tokens"][b, :n].tolist() == [int(tokens[b, j]) for j in best[1:]]
        assert r["out_tokens"][b, n] == amax[b, best[-1]]
        assert (r["out_tokens"][b, n + 1:] == -1).all()


def test_tree_chain_equals_greedy():
    w = workloads.make_greedy(B=10, k=6, V=400, p_match=0.8, seed=12)
    B, kp1 = w["target"].shape[:2]
    parent = np.tile(np.arange(-1, kp1 - 1, dtype=np.int32), (B, 1))
    tokens = np.concatenate([np.zeros((B, 1), np.int32), w["tokens"]], axis=1)
    r = oracle.verify_tree_greedy(w["target"], "bf16", parent, tokens)
    g = oracle.verify_greedy(w["target"], "bf16", w["tokens"])
    np.testing.assert_array_equal(r["accepted_len"], g["accepted_len"])
    np.testing.assert_array_equal(r["out_tokens"], g["out_tokens"])


def test_tree_duplicate_siblings_and_invalid_parent_hand_cases():
    # root argmax 2; nodes 1 and 2 both carry token 2 (duplicates), node 3 under
    # node 2 would extend the path, but the walk takes node 1 (lowest index)
    rows = np.zeros((1, 4, 3), np.float32)
    rows[0, :, 2] = 1.0
    parent = np.array([[-1, 0, 0, 2]], np.int32)
    tokens = np.array([[0, 2, 2, 2]], np.int32)
    r = oracle.verify_tree_greedy(rows, "f32", parent, tokens)
    assert r["accepted_len"].tolist() == [1]
    assert r["path"].tolist() == [[0, 1, -1, -1]]
    assert r["out_tokens"].tolist() == [[2, 2, -1, -1]]
    assert not r["invalid_tree"]
    # node 1's parent points forward: it is never entered
    parent = np.array([[-1, 3, 0, 2]], np.int32)
    r = oracle.verify_tree_greedy(rows, "f32", parent, tokens)
    assert r["invalid_tree"]
    assert r["path"].tolist() == [[0, 2, 3, -1]]
    assert r["out_tokens"].tolist() == [[2, 2, 2, -1]]


# ------------------------------------------------------ stochastic tree verify

def chain_tree(B, k):
    parent = np.tile(np.arange(-1, k, dtype=np.int32), (B, 1))
    return parent


def one_hot_draft(tokens, V):
    B, k = tokens.shape
    d = np.full((B, k, V), -np.inf, np.float32)
    for b in range(B):
        d[b, np.arange(k), tokens[b]] = 0.0
    return d


@pytest.mark.parametrize("dtype,T", [("f32", 1.0), ("bf16", 0.7)])
def test_tree_stochastic_chain_is_stochastic_verify_with_one_hot_drafts(dtype, T):
    """A chain tree is linear drafting with a point-mass draft at every
    position: the rejection rule, draws and committed tokens must coincide."""
    rng = np.random.default_rng(61)
    B, k, V = 300, 5, 50
    x = (rng.standard_normal((B, k + 1, V)) * 2.0).astype(np.float32)
    p = softmax64(x, T)
    drafts = np.zeros((B, k), np.int32)
    for b in range(B):
        for i in range(k):  # mostly likely tokens, so that long prefixes occur
            drafts[b, i] = int(np.argmax(p[b, i])) if rng.random() < 0.6 else int(rng.integers(V))
    arr = workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x
    tokens = np.concatenate([np.zeros((B, 1), np.int32), drafts], axis=1)
    r = oracle.verify_tree_stochastic(arr, dtype, chain_tree(B, k), tokens, T, seed=5)
    lin = oracle.verify_stochastic(arr, dtype, one_hot_draft(drafts, V), "f32", drafts, T, seed=5)
    ok = lin["gaps"] > 1e-9
    assert ok.sum() > B - 3
    np.testing.assert_array_equal(r["accepted_len"][ok], lin["accepted_len"][ok])
    np.testing.assert_array_equal(r["out_tokens"][ok], lin["out_tokens"][ok])
    for b in np.nonzero(ok)[0]:
        n = int(r["accepted_len"][b])
        assert r["path"][b, : n + 1].tolist() == list(range(n + 1))
        seen = ~np.isnan(r["margins"][b, 1:])  # children examined on the walk
        assert seen.sum() == min(n + 1, k)
        np.testing.assert_allclose(r["margins"][b, 1:][seen], lin["margins"][b][seen], atol=1e-12)
    assert 0 < r["accepted_len"].mean() < k


def test_tree_stochastic_root_only_is_the_bonus_draw():
    rng = np.random.default_rng(62)
    B, V, T = 200, 70, 0.9
    x = (rng.standard_normal((B, 1, V)) * 1.5).astype(np.float32)
    r = oracle.verify_tree_stochastic(x, "f32", np.full((B, 1), -1, np.int32),
                                      np.zeros((B, 1), np.int32), T, seed=8)
    lin = oracle.verify_stochastic(x, "f32", np.zeros((B, 0, V), np.float32), "f32",
                                   np.zeros((B, 0), np.int32), T, seed=8)
    assert np.all(r["accepted_len"] == 0)
    np.testing.assert_array_equal(r["out_tokens"][:, 0], lin["out_tokens"][:, 0])
    np.testing.assert_array_equal(r["path"], np.zeros((B, 1), np.int32))


@pytest.fixture(scope="module")
def tree_law_case():
    """One 8-node tree shared by 400k sequences (stride-0 batch): root with
    children 1, 2, 3 (node 3 repeats node 2's token), node 1 with children 4
    and 5, node 2 with child 6, node 4 with child 7."""
    rng = np.random.default_rng(63)
    V, T, trials = 6, 0.8, 400_000
    parent = np.array([-1, 0, 0, 0, 1, 1, 2, 4], np.int32)
    tokens = np.array([0, 1, 4, 4, 2, 0, 5, 3], np.int32)
    rows = (rng.standard_normal((8, V)) * 1.2).astype(np.float32)
    r = oracle.verify_tree_stochastic(np.broadcast_to(rows, (trials, 8, V)), "f32",
                                      np.broadcast_to(parent, (trials, 8)),
                                      np.broadcast_to(tokens, (trials, 8)), T, seed=21,
                                      threads=THREADS)
    return dict(V=V, p=softmax64(rows, T), parent=parent, tokens=tokens, r=r, trials=trials)


def test_tree_stochastic_first_token_follows_the_root_row(tree_law_case):
    c = tree_law_case
    counts = np.bincount(c["r"]["out_tokens"][:, 0], minlength=c["V"])
    assert chi2_pvalue(counts, c["p"][0]) > P_MIN


def test_tree_stochastic_each_child_is_taken_with_its_target_probability(tree_law_case):
    c = tree_law_case
    first = c["r"]["path"][:, 1]
    for j in (1, 2):
        hits = int((first == j).sum())
        assert scipy.stats.binomtest(hits, c["trials"], c["p"][0, c["tokens"][j]]).pvalue > P_MIN
    assert not (first == 3).any()  # a repeated sibling token is never taken


def test_tree_stochastic_after_an_accepted_node_its_row_takes_over(tree_law_case):
    c = tree_law_case
    r = c["r"]
    for u in (1, 2, 4):
        sel = (r["path"] == u).any(axis=1)
        depth = {1: 1, 2: 1, 4: 2}[u]
        counts = np.bincount(r["out_tokens"][sel, depth], minlength=c["V"])
        assert sel.sum() > 1000
        assert chi2_pvalue(counts, c["p"][u]) > P_MIN


def test_tree_stochastic_final_draw_skips_rejected_siblings(tree_law_case):
    c = tree_law_case
    r = c["r"]
    stop0 = r["accepted_len"] == 0  # every root child was rejected
    drawn = r["out_tokens"][stop0, 0]
    assert not np.isin(drawn, [1, 4]).any()
    law = c["p"][0].copy()
    law[[1, 4]] = 0.0
    counts = np.bincount(drawn, minlength=c["V"])
    assert chi2_pvalue(counts, law / law.sum()) > P_MIN
    # node 1 accepted, both its children rejected: the draw avoids 2 and 0
    stop1 = (r["accepted_len"] == 1) & (r["path"][:, 1] == 1)
    assert not np.isin(r["out_tokens"][stop1, 1], [2, 0]).any()
    # leaf reached (node 6 under node 2): the bonus draw is unrestricted
    leaf = r["path"][:, 2] == 6
    counts = np.bincount(r["out_tokens"][leaf, 2], minlength=c["V"])
    assert chi2_pvalue(counts, c["p"][6]) > P_MIN


def test_tree_stochastic_sure_and_impossible_children():
    V = 5
    rows = np.zeros((1, 3, V), np.float32)
    rows[0, 0] = [-np.inf, 0.0, -np.inf, -np.inf, -np.inf]  # root puts all mass on 1
    parent = np.array([[-1, 0, 0]], np.int32)
    r = oracle.verify_tree_stochastic(rows, "f32", parent, np.array([[0, 3, 1]], np.int32),
                                      1.0, seed=1)
    # node 1 (token 3, p = 0) is rejected, node 2 (token 1, p / R = 1) accepted
    assert r["path"].tolist() == [[0, 2, -1]]
    assert r["out_tokens"][0, 0] == 1
    assert np.isfinite(r["margins"][0, 1]) and np.isfinite(r["margins"][0, 2])
    # invalid token and a forward parent
    r = oracle.verify_tree_stochastic(rows, "f32", np.array([[-1, 0, 5]], np.int32),
                                      np.array([[0, V, 1]], np.int32), 1.0, seed=1)
    assert r["flags"].tolist() == [1 | 32]
    assert r["invalid_tree"]
    assert r["accepted_len"].tolist() == [0]
    assert r["out_tokens"][0, 0] == 1  # the root's only token with mass
    assert np.isinf(r["margins"][0, 1]) and np.isnan(r["margins"][0, 2])


@pytest.mark.parametrize("T", [0.5, 1.0, 2.0])
def test_tree_stochastic_outcomes_are_valid_walks(T):
    """Random trees with repeated and invalid sibling tokens and a few bad
    parents: every outcome is a root path of accepted children, their tokens,
    and a drawn token outside the final node's children's tokens; and the
    invariant checker itself rejects corrupted outcomes."""
    from tree_checks import valid_tree_outcome

    rng = np.random.default_rng(65)
    B, N, V = 300, 20, 12
    x = (rng.standard_normal((B, N, V)) * 2.5).astype(np.float32)
    am = np.argmax(x, -1)
    parent = np.zeros((B, N), np.int32)
    tokens = rng.integers(0, V, (B, N)).astype(np.int32)
    for b in range(B):
        parent[b] = workloads.tree_parents(N, rng)
        for j in range(1, N):
            if rng.random() < 0.5:
                tokens[b, j] = am[b, parent[b, j]]
            if rng.random() < 0.03:
                tokens[b, j] = V + 2
        if rng.random() < 0.05:
            parent[b, N - 1] = N + 3
    r = oracle.verify_tree_stochastic(x, "f32", parent, tokens, T, seed=13)
    assert r["accepted_len"].max() >= 2
    for b in range(B):
        if r["flags"][b] & 2:
            continue
        assert valid_tree_outcome(parent[b], tokens[b], V, r["accepted_len"][b], r["path"][b],
                                  r["out_tokens"][b]), b
    b = int(np.argmax(r["accepted_len"]))
    n, path, out = int(r["accepted_len"][b]), r["path"][b].copy(), r["out_tokens"][b].copy()
    bad = out.copy()
    bad[0] = (bad[0] + 1) % V  # a committed token that is not the node's
    assert not valid_tree_outcome(parent[b], tokens[b], V, n, path, bad)
    bad = path.copy()
    bad[n], bad[1] = bad[1], bad[n]  # not a parent chain
    assert not valid_tree_outcome(parent[b], tokens[b], V, n, bad, out)
    u = int(path[n])
    kids = [j for j in range(u + 1, N) if parent[b, j] == u and 0 <= tokens[b, j] < V]
    if kids:
        bad = out.copy()
        bad[n] = tokens[b, kids[0]]  # a rejected child's token drawn
        assert not valid_tree_outcome(parent[b], tokens[b], V, n, path, bad)


def test_tree_stochastic_sequence_offset_selects_the_stream():
    rng = np.random.default_rng(64)
    B, N, V = 12, 9, 30
    x = (rng.standard_normal((1, N, V)) * 2).astype(np.float32)
    par = workloads.tree_parents(N, rng)[None, :]
    tok = rng.integers(0, V, (1, N)).astype(np.int32)
    xb = np.broadcast_to(x, (B, N, V))
    full = oracle.verify_tree_stochastic(xb, "f32", np.broadcast_to(par, (B, N)),
                                         np.broadcast_to(tok, (B, N)), 1.0, seed=3)
    for s in (0, 5, 11):
        one = oracle.verify_tree_stochastic(x, "f32", par, tok, 1.0, seed=3, seq_offset=s)
        np.testing.assert_array_equal(one["out_tokens"][0], full["out_tokens"][s])
        np.testing.assert_array_equal(one["path"][0], full["path"][s])


# ------------------------------------------------------------ device commit

def test_commit_hand_case():
    out = np.array([[7, 8, 9, -1], [1, 2, 3, 4]], np.int32)
    acc = np.array([1, 3], np.int32)
    buf = np.full((2, 6), -5, np.int32)
    r = oracle.commit(acc, out, np.array([2, 5], np.int32), buf)
    # sequence 0: n = 1 -> tokens 7, 8 at 2..3; next input 8
    # sequence 1: n = 3 -> tokens 1..4 at 5..8, only position 5 fits
    assert r["token_buf"].tolist() == [[-5, -5, 7, 8, -5, -5], [-5, -5, -5, -5, -5, 1]]
    assert r["seq_len"].tolist() == [4, 6]
    assert r["next_input"].tolist() == [8, 4]
    assert r["capacity_hit"]


def test_commit_clamps_and_appends_the_commit():
    rng = np.random.default_rng(5)
    B, k, cap = 50, 6, 40
    out = rng.integers(0, 1000, (B, k + 1)).astype(np.int32)
    acc = rng.integers(-2, k + 3, B).astype(np.int32)  # includes values outside [0, k]
    lens = rng.integers(-3, 20, B).astype(np.int32)
    buf = rng.integers(0, 1000, (B, cap)).astype(np.int32)
    r = oracle.commit(acc, out, lens, buf)
    for b in range(B):
        n = min(max(int(acc[b]), 0), k)
        L = max(int(lens[b]), 0)
        assert r["seq_len"][b] == L + n + 1
        assert r["token_buf"][b, L:L + n + 1].tolist() == out[b, :n + 1].tolist()
        assert r["token_buf"][b, :L].tolist() == buf[b, :L].tolist()
        assert r["token_buf"][b, L + n + 1:].tolist() == buf[b, L + n + 1:].tolist()
        assert r["next_input"][b] == out[b, n]
    assert not r["capacity_hit"]


# ------------------------------------------------------------------ strides

def test_strided_views_equal_contiguous():
    w = workloads.make_stochastic(5, 3, 40, "bf16", "f32", seed=2)
    big_t = np.zeros((5, 7, 48), np.uint16)
    big_t[:, 1:5, 4:44] = w["target"]
    big_d = np.zeros((5, 3, 2, 40), np.float32)
    big_d[:, :, 1, :] = w["draft"]
    a = oracle.verify_stochastic(w["target"], "bf16", w["draft"], "f32", w["tokens"], 1.0, 8)
    b = oracle.verify_stochastic(big_t[:, 1:5, 4:44], "bf16", big_d[:, :, 1, :], "f32",
                                 w["tokens"], 1.0, 8)
    for key in a:
        np.testing.assert_array_equal(a[key], b[key])


def test_sequence_offset_selects_the_philox_stream():
    """Sharding a batch with seq_offset reproduces the unsharded result."""
    w = workloads.make_stochastic(6, 3, 50, "f32", "f32", seed=4)
    full = oracle.verify_stochastic(w["target"], "f32", w["draft"], "f32", w["tokens"], 1.0, 21)
    lo = oracle.verify_stochastic(w["target"][:2], "f32", w["draft"][:2], "f32",
                                  w["tokens"][:2], 1.0, 21, seq_offset=0)
    hi = oracle.verify_stochastic(w["target"][2:], "f32", w["draft"][2:], "f32",
                                  w["tokens"][2:], 1.0, 21, seq_offset=2)
    for key in ("accepted_len", "out_tokens", "probs"):
        np.testing.assert_array_equal(np.concatenate([lo[key], hi[key]]), full[key])
