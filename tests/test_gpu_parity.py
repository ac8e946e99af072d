"""GPU parity: the CUDA library (through its C ABI) against the CPU oracle.

Greedy, multi-candidate and Philox results must be bit-exact.  Stochastic
results: accepted lengths and tokens must match exactly, except for
sequences where a decision the oracle took was a near tie (an acceptance
margin |u - p/q| < 1e-5 at a position the oracle examined, or a Gumbel-max
score gap < 1e-5 in the sampled row); those are counted.  p_i(x_i) and
q_i(x_i) must agree within 1e-5 absolute.
"""
import os

import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_88_b200 as sv
import workloads
from tree_checks import valid_tree_outcome

pytestmark = pytest.mark.gpu

TOL_PROB = 1e-5
TOL_MARGIN = 1e-5
TOL_GAP = 1e-5
THREADS = os.cpu_count() or 1


@pytest.fixture
def argmax_path(request, monkeypatch):
    """Plain greedy and multi-candidate calls run either as one grid of
    row-chunk blocks (small calls) or on the persistent pipeline with early
    exit (large calls); the size limit between them is overridden here so
    that both paths meet every case."""
    monkeypatch.setenv("SV_ONESHOT_MAX_BYTES", "0" if request.param == "persistent" else
                       str(1 << 62))
    return request.param


both_argmax_paths = pytest.mark.parametrize("argmax_path", ["oneshot", "persistent"],
                                            indirect=True)


@pytest.fixture(scope="module")
def dev():
    from speculative_decoding_verification_88_b200 import build

    build.build()
    assert torch.cuda.is_available(), "the GPU tests need a CUDA device"
    return torch.device("cuda:0")


def to_dev(arr, dtype, dev):
    return workloads.as_torch(arr, dtype).to(dev)


def near_ties(o, k):
    n = o["accepted_len"]
    near = o["gaps"] < TOL_GAP
    if k > 0:
        for b in range(len(n)):
            upto = min(int(n[b]), k - 1)
            near[b] |= bool((o["margins"][b, : upto + 1] < TOL_MARGIN).any())
    return near


def near_tie_bound(B):
    """Most sequences a test may excuse as near ties: the oracle flags a
    sequence with probability about 1e-4 or less on these inputs (a margin or
    a gap below 1e-5), so more than this means a broken report or an input
    that does not test what it should."""
    return max(2, B // 100)


def check_probs(probs, o, gpu_len, what=""):
    """p_i(x_i), q_i(x_i) within TOL_PROB of the oracle on every row up to the
    first rejection (the earlier of the GPU's and the oracle's, which differ
    only at a near tie); a later row is either as exact or (-1, -1): it lies
    past a rejection and may have been retired without being read."""
    k = probs.shape[1]
    retired = (probs == -1.0).all(axis=-1)
    upto = np.arange(k)[None, :] <= np.minimum(o["accepted_len"], gpu_len)[:, None]
    assert not (retired & upto).any(), f"{what}: a row up to the first rejection was retired"
    close = (np.abs(probs - o["probs"]) <= TOL_PROB).all(axis=-1)
    bad = np.argwhere(~(close | retired))
    assert bad.size == 0, f"{what}: probs differ at (b, i) = {bad[0]}: {probs[tuple(bad[0])]} " \
                          f"vs {o['probs'][tuple(bad[0])]}"


def compare_stochastic(r, o, k, what=""):
    acc = r["accepted_len"].cpu().numpy()
    tok = r["out_tokens"].cpu().numpy()
    if "probs" in r and k > 0:
        check_probs(r["probs"].cpu().numpy(), o, acc, what)
    near = near_ties(o, k)
    assert near.sum() <= near_tie_bound(len(near)), f"{what}: {near.sum()} near ties"
    mism = (acc != o["accepted_len"]) | (tok != o["out_tokens"]).any(axis=1)
    bad = np.nonzero(mism & ~near)[0]
    assert bad.size == 0, (
        f"{what}: {bad.size} mismatches outside near ties, first b={bad[0]}: gpu n={acc[bad[0]]} "
        f"tok={tok[bad[0]]} oracle n={o['accepted_len'][bad[0]]} tok={o['out_tokens'][bad[0]]} "
        f"margins={o['margins'][bad[0]]} gap={o['gaps'][bad[0]]}")
    if "inputs" in o:  # a near tie that went the other way still gives a valid commit
        drafts, V = o["inputs"]
        for b in np.nonzero(mism & near)[0]:
            n = int(acc[b])
            assert 0 <= n <= k and (tok[b, :n] == drafts[b, :n]).all(), (what, b)
            assert 0 <= tok[b, n] < V and (tok[b, n + 1:] == -1).all(), (what, b)
    return int(near.sum()), int((mism & near).sum())


def run_stochastic(w, dev, seed=None, seq_offset=0, **views):
    T = w["temperature"]
    seed = w["seed"] if seed is None else seed
    t = views.get("t", to_dev(w["target"], w["t_dtype"], dev))
    d = views.get("d", to_dev(w["draft"], w["d_dtype"], dev))
    tok = torch.from_numpy(w["tokens"]).to(dev)
    r = sv.stochastic(t, d, tok, T, seed, seq_offset, probs=True)
    o = oracle.verify_stochastic(views.get("t_np", w["target"]), w["t_dtype"],
                                 views.get("d_np", w["draft"]), w["d_dtype"], w["tokens"], T,
                                 seed, seq_offset, threads=THREADS)
    o["inputs"] = (w["tokens"], w["target"].shape[-1])
    torch.cuda.synchronize()
    return r, o


# ------------------------------------------------------------------ Philox

def test_philox_matches_oracle(dev):
    rng = np.random.default_rng(0)
    ctr = rng.integers(0, 2**32, size=(1 << 20, 4), dtype=np.uint64).astype(np.uint32)
    ctr[:4] = [[0, 0, 0, 0], [0xFFFFFFFF] * 4, [1, 2, 3, 4], [0, 7, 9, 2]]
    for seed in (0, 1, 0xFFFFFFFFFFFFFFFF, 0xA4093822299F31D0):
        want = oracle.philox4x32_10(ctr, seed)
        got = sv.philox4x32_10(torch.from_numpy(ctr.view(np.int32)).to(dev), seed)
        assert np.array_equal(got.cpu().numpy().view(np.uint32), want)


# ------------------------------------------------------------------ greedy

def tie_heavy(rng, shape):
    x = rng.integers(-4, 5, size=shape).astype(np.float32)
    x[rng.random(shape) < 0.03] = -np.inf
    z = x == 0
    x[z & (rng.random(shape) < 0.5)] = -0.0
    return x


@both_argmax_paths
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,k,V", [(1, 0, 1), (3, 1, 2), (129, 4, 7), (3, 8, 8), (1, 4, 9),
                                   (3, 32, 31), (129, 2, 33), (3, 4, 4095), (1, 8, 4097),
                                   (5, 3, 32000), (2, 4, 128256)])
def test_greedy_parity_shapes(dev, argmax_path, dtype, B, k, V):
    rng = np.random.default_rng(B * 1000 + k * 10 + V)
    if V <= 64:
        x = tie_heavy(rng, (B, k + 1, V))
    else:
        x = rng.standard_normal((B, k + 1, V)).astype(np.float32) * 3
    arr = workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x
    xv = workloads.to_f32(arr, dtype)
    am = np.argmax(xv, -1)
    tok = np.where(rng.random((B, k)) < 0.75, am[:, :k], rng.integers(-2, V + 2, (B, k)))
    tok = tok.astype(np.int32)
    r = sv.greedy(to_dev(arr, dtype, dev), torch.from_numpy(tok).to(dev))
    o = oracle.verify_greedy(arr, dtype, tok, threads=THREADS)
    np.testing.assert_array_equal(r["accepted_len"].cpu().numpy(), o["accepted_len"])
    np.testing.assert_array_equal(r["out_tokens"].cpu().numpy(), o["out_tokens"])


@both_argmax_paths
def test_greedy_strided_unaligned_and_broadcast(dev, argmax_path):
    rng = np.random.default_rng(3)
    B, k, V = 6, 4, 1001
    big = workloads.f32_to_bf16_bits(rng.standard_normal((B, k + 2, V + 3)).astype(np.float32))
    tok = rng.integers(0, V, (B, k)).astype(np.int32)
    tok_d = torch.from_numpy(tok).to(dev)
    big_d = to_dev(big, "bf16", dev)
    # offset by one element: rows are not 16-byte aligned (plain-load path)
    r = sv.greedy(big_d[:, 1:, 1:1 + V], tok_d)
    o = oracle.verify_greedy(big[:, 1:, 1:1 + V], "bf16", tok)
    np.testing.assert_array_equal(r["out_tokens"].cpu().numpy(), o["out_tokens"])
    np.testing.assert_array_equal(r["accepted_len"].cpu().numpy(), o["accepted_len"])
    # stride-0 broadcast of one sequence over the batch
    one = big[:1, :k + 1, :V]
    bc = big_d[:1, :k + 1, :V].expand(B, k + 1, V)
    r = sv.greedy(bc, tok_d)
    o = oracle.verify_greedy(np.broadcast_to(one, (B, k + 1, V)), "bf16", tok)
    np.testing.assert_array_equal(r["out_tokens"].cpu().numpy(), o["out_tokens"])


@both_argmax_paths
def test_greedy_all_accepted_and_none(dev, argmax_path):
    rng = np.random.default_rng(4)
    B, k, V = 40, 6, 5000
    x = workloads.f32_to_bf16_bits(rng.standard_normal((B, k + 1, V)).astype(np.float32))
    am = np.argmax(workloads.to_f32(x, "bf16"), -1).astype(np.int32)
    t = to_dev(x, "bf16", dev)
    r = sv.greedy(t, torch.from_numpy(am[:, :k].copy()).to(dev))
    assert (r["accepted_len"].cpu().numpy() == k).all()
    np.testing.assert_array_equal(r["out_tokens"].cpu().numpy(), am)
    bad = ((am[:, :k] + 1) % V).astype(np.int32)
    r = sv.greedy(t, torch.from_numpy(bad).to(dev))
    assert (r["accepted_len"].cpu().numpy() == 0).all()
    np.testing.assert_array_equal(r["out_tokens"].cpu().numpy()[:, 0], am[:, 0])


@both_argmax_paths
@pytest.mark.parametrize("B,k,V,p_match", [(512, 8, 32000, 0.5), (300, 32, 4000, 0.9),
                                           (1024, 2, 20000, 0.3)])
def test_greedy_early_exit_is_exact_and_leaves_the_workspace_clean(dev, argmax_path, B, k, V, p_match):
    """Batches large enough that rows past a branch's first mismatch are
    retired unread: results stay bit-exact, the flag word stays clear for
    valid drafts, and the workspace (branch states included) is left zero."""
    w = workloads.make_greedy(B, k, V, p_match=p_match, seed=B + k, threads=THREADS)
    t = to_dev(w["target"], "bf16", dev)
    tok = torch.from_numpy(w["tokens"]).to(dev)
    o = oracle.verify_greedy(w["target"], "bf16", w["tokens"], threads=THREADS)
    ws = sv.Workspace(dev)
    for _ in range(2):
        r = sv.greedy(t, tok, workspace=ws)
        torch.cuda.synchronize()
        np.testing.assert_array_equal(r["accepted_len"].cpu().numpy(), o["accepted_len"])
        np.testing.assert_array_equal(r["out_tokens"].cpu().numpy(), o["out_tokens"])
        assert int(ws.buf[256:].cpu().count_nonzero()) == 0
    assert ws.device_status() == 0
    assert 0 < o["accepted_len"].mean() < k


@both_argmax_paths
@pytest.mark.parametrize("B,G,k,V", [(64, 8, 4, 32000), (40, 64, 6, 3000)])
def test_multi_early_exit_is_exact_and_leaves_the_workspace_clean(dev, argmax_path, B, G, k, V):
    w = workloads.make_multi(B, G, k, V, p_match=0.5, seed=G + k, threads=THREADS)
    t = to_dev(w["target"], "bf16", dev)
    tok = torch.from_numpy(w["tokens"]).to(dev)
    o = oracle.verify_multi(w["target"], "bf16", w["tokens"], threads=THREADS)
    ws = sv.Workspace(dev)
    for _ in range(2):
        r = sv.multi_candidate(t, tok, workspace=ws)
        torch.cuda.synchronize()
        for key in ("best_candidate", "accepted_len", "out_tokens"):
            np.testing.assert_array_equal(r[key].cpu().numpy(), o[key], err_msg=key)
        assert int(ws.buf[256:].cpu().count_nonzero()) == 0
    assert ws.device_status() == 0


@both_argmax_paths
def test_greedy_invalid_drafts_raise_the_flag(dev, argmax_path):
    w = workloads.make_greedy(9, 4, 3000, seed=5)
    w["tokens"][4, 2] = -7
    w["tokens"][8, 0] = 3000
    ws = sv.Workspace(dev)
    r = sv.greedy(to_dev(w["target"], "bf16", dev), torch.from_numpy(w["tokens"]).to(dev),
                  workspace=ws)
    o = oracle.verify_greedy(w["target"], "bf16", w["tokens"])
    np.testing.assert_array_equal(r["out_tokens"].cpu().numpy(), o["out_tokens"])
    assert ws.device_status(clear=True) == sv.SV_FLAG_INVALID_TOKEN
    w = workloads.make_greedy(9, 4, 3000, seed=6)  # valid drafts: nothing raised
    sv.greedy(to_dev(w["target"], "bf16", dev), torch.from_numpy(w["tokens"]).to(dev),
              workspace=ws)
    assert ws.device_status() == 0


# ---------------------------------------------------------- multi-candidate

@both_argmax_paths
@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,G,k,V", [(1, 1, 4, 100), (3, 3, 2, 17), (16, 8, 4, 3001),
                                     (2, 64, 3, 50), (4, 5, 32, 40), (2, 2, 0, 10)])
def test_multi_parity_shapes(dev, argmax_path, dtype, B, G, k, V):
    rng = np.random.default_rng(B + G * 7 + k * 13 + V)
    x = tie_heavy(rng, (B, G, k + 1, V)) if V < 64 else \
        rng.standard_normal((B, G, k + 1, V)).astype(np.float32) * 3
    arr = workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x
    am = np.argmax(workloads.to_f32(arr, dtype), -1)
    cand = np.where(rng.random((B, G, k)) < 0.7, am[..., :k], rng.integers(0, V, (B, G, k)))
    cand = cand.astype(np.int32)
    r = sv.multi_candidate(to_dev(arr, dtype, dev), torch.from_numpy(cand).to(dev))
    o = oracle.verify_multi(arr, dtype, cand, threads=THREADS)
    for key in ("best_candidate", "accepted_len", "out_tokens"):
        np.testing.assert_array_equal(r[key].cpu().numpy(), o[key], err_msg=key)


# ------------------------------------------ multi-candidate, rows form

def random_rows_case(rng, B, G, k, V, dtype, share=0.6):
    """Candidates with shared prefixes, their prefix row map and one row of
    logits per distinct prefix."""
    cand = rng.integers(0, max(V, 1), (B, G, k)).astype(np.int32)
    for b in range(B):
        for g in range(1, G):
            if rng.random() < share and k > 0:
                m = int(rng.integers(1, k + 1))
                src = int(rng.integers(0, g))
                cand[b, g, :m] = cand[b, src, :m]
    row_of, R = workloads.prefix_rows(cand)
    x = tie_heavy(rng, (B, R, V)) if V < 64 else \
        rng.standard_normal((B, R, V)).astype(np.float32) * 3
    arr = workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x
    # steer some candidates onto their row's argmax so that prefixes get accepted
    am = np.argmax(workloads.to_f32(arr, dtype), -1)
    for b in range(B):
        for g in range(G):
            for i in range(k):
                if rng.random() < 0.5:
                    cand[b, g, i] = am[b, row_of[b, g, i]]
    row_of, R2 = workloads.prefix_rows(cand)
    if R2 > R:  # steering created new prefixes: give them rows too
        extra = rng.standard_normal((B, R2 - R, V)).astype(np.float32) * 3
        extra = workloads.f32_to_bf16_bits(extra) if dtype == "bf16" else extra
        arr = np.concatenate([arr, extra], axis=1)
    return arr, row_of, cand


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,G,k,V", [(1, 1, 4, 100), (3, 3, 2, 17), (16, 8, 4, 3001),
                                     (2, 64, 3, 50), (4, 5, 32, 40), (2, 2, 0, 10),
                                     (3, 6, 5, 20480 + 17)])
@both_argmax_paths
def test_multi_rows_parity_shapes(dev, argmax_path, dtype, B, G, k, V):
    rng = np.random.default_rng(B * 3 + G * 5 + k * 11 + V)
    arr, row_of, cand = random_rows_case(rng, B, G, k, V, dtype)
    r = sv.multi_candidate_rows(to_dev(arr, dtype, dev), torch.from_numpy(row_of).to(dev),
                                torch.from_numpy(cand).to(dev))
    o = oracle.verify_multi_rows(arr, dtype, row_of, cand, threads=THREADS)
    for key in ("best_candidate", "accepted_len", "out_tokens"):
        np.testing.assert_array_equal(r[key].cpu().numpy(), o[key], err_msg=key)


@both_argmax_paths
def test_multi_rows_equals_expanded_multi(dev, argmax_path):
    """The rows form and the expanded form give the same results."""
    rng = np.random.default_rng(21)
    arr, row_of, cand = random_rows_case(rng, 9, 7, 6, 2000, "bf16")
    t = to_dev(arr, "bf16", dev)
    rm = torch.from_numpy(row_of).to(dev)
    c = torch.from_numpy(cand).to(dev)
    r = sv.multi_candidate_rows(t, rm, c)
    expanded = t[torch.arange(9, device=dev)[:, None, None], rm.long()]
    e = sv.multi_candidate(expanded.contiguous(), c)
    for key in ("best_candidate", "accepted_len", "out_tokens"):
        assert torch.equal(r[key], e[key]), key


@both_argmax_paths
def test_multi_rows_invalid_entries_and_limits(dev, argmax_path):
    rng = np.random.default_rng(22)
    arr, row_of, cand = random_rows_case(rng, 5, 4, 3, 300, "bf16")
    R = arr.shape[1]
    bad = row_of.copy()
    bad[1, 2, 1] = R + 5
    bad[3, 0, 0] = -1
    ws = sv.Workspace(dev)
    r = sv.multi_candidate_rows(to_dev(arr, "bf16", dev), torch.from_numpy(bad).to(dev),
                                torch.from_numpy(cand).to(dev), workspace=ws)
    o = oracle.verify_multi_rows(arr, "bf16", bad, cand)
    assert o["invalid_row"]
    for key in ("best_candidate", "accepted_len", "out_tokens"):
        np.testing.assert_array_equal(r[key].cpu().numpy(), o[key], err_msg=key)
    assert ws.device_status(clear=True) == sv.SV_FLAG_INVALID_ROW
    torch.cuda.synchronize()
    assert int(ws.buf[256:].cpu().count_nonzero()) == 0
    # more rows than G * (k + 1) is refused
    big = np.zeros((1, 2 * 2 + 1, 64), np.uint16)
    with pytest.raises(sv.SpecVerifyError):
        sv.multi_candidate_rows(to_dev(big, "bf16", dev),
                                torch.zeros((1, 2, 2), dtype=torch.int32, device=dev),
                                torch.zeros((1, 2, 1), dtype=torch.int32, device=dev))


# ------------------------------------------------------ threshold acceptance

TOL_SCORE = 1e-4  # |ln score - ln tau| below which a decision is a near tie


def compare_threshold(r, o, tau):
    """Exact except sequences whose examined prefix score is within TOL_SCORE
    of the threshold (natural-log units); returns how many were near."""
    ls = o["log_scores"]
    lt = np.log(np.float32(tau))
    near = np.zeros(len(o["accepted_len"]), bool)
    k = ls.shape[1]
    for b in range(len(near)):
        upto = min(int(o["accepted_len"][b]) + 1, k)
        v = ls[b, :upto]
        near[b] = bool((np.abs(v[np.isfinite(v)] - lt) < TOL_SCORE).any())
    acc = r["accepted_len"].cpu().numpy()
    out = r["out_tokens"].cpu().numpy()
    ok = ~near
    np.testing.assert_array_equal(acc[ok], o["accepted_len"][ok])
    np.testing.assert_array_equal(out[ok], o["out_tokens"][ok])
    return int(near.sum())


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,k,V,T,tau", [(1, 1, 1, 1.0, 0.5), (5, 4, 33, 0.7, 0.01),
                                         (64, 8, 4097, 1.0, 1e-4), (7, 32, 500, 1.3, 1e-30),
                                         (16, 4, 128256, 0.7, 1e-3), (40, 0, 100, 1.0, 0.5)])
def test_threshold_parity(dev, dtype, B, k, V, T, tau):
    w = workloads.make_greedy(B, k, V, t_dtype=dtype, p_match=0.8, seed=B + k + V)
    r = sv.threshold(to_dev(w["target"], dtype, dev), torch.from_numpy(w["tokens"]).to(dev),
                     T, tau)
    o = oracle.verify_threshold(w["target"], dtype, w["tokens"], T, tau, threads=THREADS)
    near = compare_threshold(r, o, tau)
    assert near <= max(1, B // 20)


def test_threshold_invalid_tokens_and_workspace(dev):
    w = workloads.make_greedy(12, 5, 300, p_match=0.9, seed=50)
    tok = w["tokens"].copy()
    tok[3, 1] = 300
    tok[7, 0] = -4
    ws = sv.Workspace(dev)
    r = sv.threshold(to_dev(w["target"], "bf16", dev), torch.from_numpy(tok).to(dev), 1.0,
                     1e-20, workspace=ws)
    o = oracle.verify_threshold(w["target"], "bf16", tok, 1.0, 1e-20)
    compare_threshold(r, o, 1e-20)
    assert int(r["accepted_len"][3]) <= 1 and int(r["accepted_len"][7]) == 0
    torch.cuda.synchronize()
    assert int(ws.buf[256:].cpu().count_nonzero()) == 0
    assert ws.device_status() == 0


# ---------------------------------------------------------------- tree verify

def random_tree_case(rng, B, N, V, dtype, dup=0.1):
    x = tie_heavy(rng, (B, N, V)) if V < 64 else \
        rng.standard_normal((B, N, V)).astype(np.float32) * 3
    arr = workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x
    am = np.argmax(workloads.to_f32(arr, dtype), -1)
    parent = np.zeros((B, N), np.int32)
    tokens = rng.integers(0, V, (B, N)).astype(np.int32)
    for b in range(B):
        parent[b] = workloads.tree_parents(N, rng)
        for j in range(1, N):
            if rng.random() < 0.6:
                tokens[b, j] = am[b, parent[b, j]]  # duplicates among siblings happen
    return arr, parent, tokens


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,N,V", [(1, 1, 10), (3, 5, 17), (16, 26, 3001), (4, 64, 40),
                                   (2, 33, 20480 + 9), (70, 12, 300)])
def test_tree_parity_shapes(dev, dtype, B, N, V):
    rng = np.random.default_rng(B * 7 + N * 3 + V)
    arr, parent, tokens = random_tree_case(rng, B, N, V, dtype)
    r = sv.tree_greedy(to_dev(arr, dtype, dev), torch.from_numpy(parent).to(dev),
                       torch.from_numpy(tokens).to(dev))
    o = oracle.verify_tree_greedy(arr, dtype, parent, tokens, threads=THREADS)
    for key in ("accepted_len", "path", "out_tokens"):
        np.testing.assert_array_equal(r[key].cpu().numpy(), o[key], err_msg=key)


def test_tree_chain_equals_greedy_on_gpu(dev):
    w = workloads.make_greedy(B=20, k=8, V=5000, p_match=0.8, seed=13)
    B = w["B"]
    t = to_dev(w["target"], "bf16", dev)
    parent = torch.arange(-1, 8, dtype=torch.int32, device=dev).repeat(B, 1)
    tokens = torch.cat([torch.zeros((B, 1), dtype=torch.int32),
                        torch.from_numpy(w["tokens"])], 1).to(dev)
    r = sv.tree_greedy(t, parent.contiguous(), tokens.contiguous())
    g = sv.greedy(t, torch.from_numpy(w["tokens"]).to(dev))
    assert torch.equal(r["accepted_len"], g["accepted_len"])
    assert torch.equal(r["out_tokens"], g["out_tokens"])


def test_tree_invalid_parent_flag(dev):
    rng = np.random.default_rng(44)
    arr, parent, tokens = random_tree_case(rng, 6, 10, 200, "bf16")
    parent[2, 4] = 9   # forward pointer
    parent[5, 7] = -3  # negative
    ws = sv.Workspace(dev)
    r = sv.tree_greedy(to_dev(arr, "bf16", dev), torch.from_numpy(parent).to(dev),
                       torch.from_numpy(tokens).to(dev), workspace=ws)
    o = oracle.verify_tree_greedy(arr, "bf16", parent, tokens)
    assert o["invalid_tree"]
    for key in ("accepted_len", "path", "out_tokens"):
        np.testing.assert_array_equal(r[key].cpu().numpy(), o[key], err_msg=key)
    assert ws.device_status(clear=True) == sv.SV_FLAG_INVALID_TREE
    torch.cuda.synchronize()
    assert int(ws.buf[256:].cpu().count_nonzero()) == 0


# ---------------------------------------------------- stochastic tree verify

def stoch_tree_case(rng, B, N, V, dtype, sigma=4.0):
    """Random node rows; children carry their parent row's argmax with
    probability 0.6 (so paths are accepted and sibling tokens repeat), else a
    uniform token."""
    x = (rng.standard_normal((B, N, V)) * sigma).astype(np.float32)
    arr = workloads.f32_to_bf16_bits(x) if dtype == "bf16" else x
    am = np.argmax(workloads.to_f32(arr, dtype), -1)
    parent = np.zeros((B, N), np.int32)
    tokens = rng.integers(0, V, (B, N)).astype(np.int32)
    for b in range(B):
        parent[b] = workloads.tree_parents(N, rng)
        for j in range(1, N):
            if rng.random() < 0.6:
                tokens[b, j] = am[b, parent[b, j]]
    return arr, parent, tokens


def compare_tree_stochastic(r, o, what=""):
    """Exact except sequences with a near-tie decision in the oracle (an
    examined child with |u - p/R| < TOL_MARGIN, or a final-draw gap below
    TOL_GAP); returns (near ties, near ties that differ)."""
    m = np.where(np.isnan(o["margins"]), np.inf, o["margins"])
    near = (m < TOL_MARGIN).any(axis=1) | (o["gaps"] < TOL_GAP)
    assert near.sum() <= near_tie_bound(len(near)), f"{what}: {near.sum()} near ties"
    acc = r["accepted_len"].cpu().numpy()
    path = r["path"].cpu().numpy()
    tok = r["out_tokens"].cpu().numpy()
    mism = (acc != o["accepted_len"]) | (path != o["path"]).any(1) | \
        (tok != o["out_tokens"]).any(1)
    bad = np.nonzero(mism & ~near)[0]
    assert bad.size == 0, (
        f"{what}: {bad.size} mismatches outside near ties, first b={bad[0]}: gpu n={acc[bad[0]]} "
        f"path={path[bad[0]]} tok={tok[bad[0]]} oracle n={o['accepted_len'][bad[0]]} "
        f"path={o['path'][bad[0]]} tok={o['out_tokens'][bad[0]]}")
    # where a near tie went the other way, the GPU's outcome must still be a
    # possible one
    for b in np.nonzero(mism & near)[0]:
        assert valid_tree_outcome(o["inputs"][0][b], o["inputs"][1][b], o["inputs"][2], acc[b],
                                  path[b], tok[b], not (o["flags"][b] & 2)), (what, b)
    return int(near.sum()), int((mism & near).sum())


def run_tree_stochastic(arr, dtype, parent, tokens, T, seed, dev, seq_offset=0, t=None,
                        workspace=None):
    t = to_dev(arr, dtype, dev) if t is None else t
    r = sv.tree_stochastic(t, torch.from_numpy(parent).to(dev), torch.from_numpy(tokens).to(dev),
                           T, seed, seq_offset, workspace=workspace)
    o = oracle.verify_tree_stochastic(arr, dtype, parent, tokens, T, seed, seq_offset,
                                      threads=THREADS)
    o["inputs"] = (parent, tokens, arr.shape[-1])
    torch.cuda.synchronize()
    return r, o


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
@pytest.mark.parametrize("B,N,V,T", [(1, 1, 10, 1.0), (3, 5, 17, 0.7), (16, 26, 3001, 1.0),
                                     (4, 64, 40, 1.3), (2, 33, 2 * 16384 + 9, 1.0),
                                     (70, 12, 300, 0.8), (5, 8, 3 * 8192, 1.0)])
def test_tree_stochastic_parity_shapes(dev, dtype, B, N, V, T):
    rng = np.random.default_rng(B * 11 + N * 5 + V)
    arr, parent, tokens = stoch_tree_case(rng, B, N, V, dtype)
    r, o = run_tree_stochastic(arr, dtype, parent, tokens, T, 17, dev)
    compare_tree_stochastic(r, o, f"{dtype} B={B} N={N} V={V}")
    if N > 1:
        assert o["accepted_len"].max() >= 1 or B < 4


def test_tree_stochastic_strided_unaligned_and_broadcast(dev):
    rng = np.random.default_rng(71)
    B, N, V = 6, 9, 2500
    arr, parent, tokens = stoch_tree_case(rng, B, N, V, "bf16")
    big = np.zeros((B, N + 1, V + 5), np.uint16)
    big[:, 1:, 3:3 + V] = arr
    t = to_dev(big, "bf16", dev)[:, 1:, 3:3 + V]  # rows 6 bytes off alignment
    r, o = run_tree_stochastic(arr, "bf16", parent, tokens, 1.0, 4, dev, t=t)
    compare_tree_stochastic(r, o, "unaligned")
    # one tree's rows shared by every sequence (stride 0): independent draws
    trials = 4000
    one = arr[:1]
    t = to_dev(one, "bf16", dev).expand(trials, N, V)
    par = np.broadcast_to(parent[:1], (trials, N)).copy()
    tok = np.broadcast_to(tokens[:1], (trials, N)).copy()
    r, o = run_tree_stochastic(np.broadcast_to(one, (trials, N, V)), "bf16", par, tok, 1.0, 4,
                               dev, t=t)
    near, flipped = compare_tree_stochastic(r, o, "broadcast")
    assert flipped <= 2


def test_tree_stochastic_chain_equals_stochastic_on_gpu(dev):
    """A chain tree against stochastic verify with one-hot draft rows."""
    rng = np.random.default_rng(72)
    B, k, V = 40, 6, 5000
    x = (rng.standard_normal((B, k + 1, V)) * 4).astype(np.float32)
    am = np.argmax(x, -1)
    drafts = np.where(rng.random((B, k)) < 0.7, am[:, :k],
                      rng.integers(0, V, (B, k))).astype(np.int32)
    tokens = np.concatenate([np.zeros((B, 1), np.int32), drafts], 1)
    parent = np.tile(np.arange(-1, k, dtype=np.int32), (B, 1))
    r, o = run_tree_stochastic(x, "f32", parent, tokens, 1.0, 9, dev)
    compare_tree_stochastic(r, o, "chain")
    d = np.full((B, k, V), -np.inf, np.float32)
    for b in range(B):
        d[b, np.arange(k), drafts[b]] = 0.0
    s = sv.stochastic(to_dev(x, "f32", dev), to_dev(d, "f32", dev),
                      torch.from_numpy(drafts).to(dev), 1.0, 9)
    m = np.where(np.isnan(o["margins"]), np.inf, o["margins"])
    clear = ~((m < TOL_MARGIN).any(1) | (o["gaps"] < TOL_GAP))
    np.testing.assert_array_equal(s["accepted_len"].cpu().numpy()[clear],
                                  r["accepted_len"].cpu().numpy()[clear])
    np.testing.assert_array_equal(s["out_tokens"].cpu().numpy()[clear],
                                  r["out_tokens"].cpu().numpy()[clear])


def test_tree_stochastic_flags_and_clean_workspace(dev):
    rng = np.random.default_rng(73)
    arr, parent, tokens = stoch_tree_case(rng, 8, 12, 400, "f32")
    parent[2, 5] = 11   # forward pointer
    parent[6, 3] = -2   # negative
    tokens[:, 1] = np.where(np.arange(8) % 2 == 0, 400, -1)  # invalid tokens
    parent[:, 1] = 0    # ... under the root, so the walk examines them
    ws = sv.Workspace(dev)
    r, o = run_tree_stochastic(arr, "f32", parent, tokens, 1.0, 2, dev, workspace=ws)
    compare_tree_stochastic(r, o, "flags")
    assert o["invalid_tree"]
    want = sv.SV_FLAG_INVALID_TREE | sv.SV_FLAG_INVALID_TOKEN
    assert int(np.bitwise_or.reduce(o["flags"])) & want == want
    assert ws.device_status(clear=True) == int(np.bitwise_or.reduce(o["flags"]))
    assert int(ws.buf[256:].cpu().count_nonzero()) == 0
    # the clean workspace serves the other modes next
    w = workloads.make_stochastic(5, 3, 3000, "bf16", "f32", seed=19)
    r2 = sv.stochastic(to_dev(w["target"], "bf16", dev), to_dev(w["draft"], "f32", dev),
                       torch.from_numpy(w["tokens"]).to(dev), w["temperature"], w["seed"],
                       probs=True, workspace=ws)
    o2 = oracle.verify_stochastic(w["target"], "bf16", w["draft"], "f32", w["tokens"],
                                  w["temperature"], w["seed"])
    compare_stochastic(r2, o2, 3, "after tree")
    r3, o3 = run_tree_stochastic(arr, "f32", parent, tokens, 0.9, 5, dev, seq_offset=77,
                                 workspace=ws)
    compare_tree_stochastic(r3, o3, "again")
    torch.cuda.synchronize()
    ws.device_status(clear=True)
    assert int(ws.buf[256:].cpu().count_nonzero()) == 0


# ------------------------------------------------------------ device commit

@pytest.mark.parametrize("B,k,cap", [(1, 0, 4), (7, 1, 9), (300, 8, 40), (33, 32, 100),
                                     (20, 4, 3)])
def test_commit_parity(dev, B, k, cap):
    rng = np.random.default_rng(B + k + cap)
    out = rng.integers(-1, 32000, (B, k + 1)).astype(np.int32)
    acc = rng.integers(-1, k + 2, B).astype(np.int32)
    lens = rng.integers(-2, cap + 1, B).astype(np.int32)
    buf = rng.integers(0, 9, (B, cap + 5)).astype(np.int32)  # row stride cap + 5
    o = oracle.commit(acc, out, lens, buf[:, :cap])
    seq = torch.from_numpy(lens).to(dev)
    tb = torch.from_numpy(buf).to(dev)
    nxt = torch.full((B,), -7, dtype=torch.int32, device=dev)
    ws = sv.Workspace(dev)
    ws.ensure(256)
    sv.commit({"accepted_len": torch.from_numpy(acc).to(dev),
               "out_tokens": torch.from_numpy(out).to(dev)},
              seq, tb[:, :cap], next_input=nxt, workspace=ws)
    np.testing.assert_array_equal(seq.cpu().numpy(), o["seq_len"])
    np.testing.assert_array_equal(tb[:, :cap].cpu().numpy(), o["token_buf"])
    np.testing.assert_array_equal(tb[:, cap:].cpu().numpy(), buf[:, cap:])  # untouched
    np.testing.assert_array_equal(nxt.cpu().numpy(), o["next_input"])
    assert ws.device_status(clear=True) == (sv.SV_FLAG_CAPACITY if o["capacity_hit"] else 0)


def test_verify_then_commit_without_host_sync(dev):
    """Greedy verify and the commit enqueued back to back on one stream, twice;
    the host reads nothing in between."""
    B, k, V, cap = 24, 4, 3000, 64
    w = workloads.make_greedy(B, k, V, seed=31)
    w2 = workloads.make_greedy(B, k, V, seed=32)
    seq = torch.zeros(B, dtype=torch.int32, device=dev)
    tb = torch.full((B, cap), -9, dtype=torch.int32, device=dev)
    nxt = torch.empty(B, dtype=torch.int32, device=dev)
    for ww in (w, w2):
        r = sv.greedy(to_dev(ww["target"], "bf16", dev), torch.from_numpy(ww["tokens"]).to(dev))
        sv.commit(r, seq, tb, next_input=nxt)
    lens = np.zeros(B, np.int32)
    buf = np.full((B, cap), -9, np.int32)
    for ww in (w, w2):
        o = oracle.verify_greedy(ww["target"], "bf16", ww["tokens"])
        c = oracle.commit(o["accepted_len"], o["out_tokens"], lens, buf)
        lens, buf, last = c["seq_len"], c["token_buf"], c["next_input"]
    np.testing.assert_array_equal(seq.cpu().numpy(), lens)
    np.testing.assert_array_equal(tb.cpu().numpy(), buf)
    np.testing.assert_array_equal(nxt.cpu().numpy(), last)


# --------------------------------------------------------------- stochastic

@pytest.mark.parametrize("t_dtype,d_dtype", [("bf16", "bf16"), ("bf16", "f32"), ("f32", "f32"),
                                             ("f32", "bf16")])
@pytest.mark.parametrize("B,k,V,T", [(1, 1, 1, 1.0), (3, 1, 2, 1.0), (129, 4, 7, 0.7),
                                     (3, 8, 9, 1.3), (3, 32, 33, 1.0), (5, 4, 4095, 0.7),
                                     (3, 8, 4097, 1.0), (4, 4, 32000, 0.5),
                                     (2, 3, 128256, 1.0)])
def test_stochastic_parity_shapes(dev, t_dtype, d_dtype, B, k, V, T):
    w = workloads.make_stochastic(B, k, V, t_dtype, d_dtype, t_std=3.0, d_noise=1.0,
                                  temperature=T, seed=B * 100 + k * 10 + V)
    r, o = run_stochastic(w, dev)
    compare_stochastic(r, o, k, f"{t_dtype}/{d_dtype} B={B} k={k} V={V}")


@pytest.mark.parametrize("parking", ["parked", "unparked"])
@pytest.mark.parametrize("B,k,V,d_noise", [(1, 4, 32000, 1.0), (64, 4, 32000, 1.5),
                                           (256, 8, 8000, 1.0), (300, 3, 5000, 0.3)])
def test_stochastic_parked_and_unparked_tickets(dev, monkeypatch, parking, B, k, V, d_noise):
    """The producers park chunks of pairs whose earlier rows are undecided
    (every batch size by default); the size limit is overridden here so that
    both ways meet the same cases: results equal the oracle's, and the
    workspace is left zero."""
    monkeypatch.setenv("SV_PARK_MIN_B", "1" if parking == "parked" else str(1 << 30))
    w = workloads.make_stochastic(B, k, V, "bf16", "bf16", t_std=3.0, d_noise=d_noise,
                                  temperature=1.0, seed=B + k + V, threads=THREADS)
    ws = sv.Workspace(dev)
    t = to_dev(w["target"], "bf16", dev)
    d = to_dev(w["draft"], "bf16", dev)
    tok = torch.from_numpy(w["tokens"]).to(dev)
    o = oracle.verify_stochastic(w["target"], "bf16", w["draft"], "bf16", w["tokens"], 1.0,
                                 w["seed"], threads=THREADS)
    o["inputs"] = (w["tokens"], V)
    for _ in range(2):
        r = sv.stochastic(t, d, tok, 1.0, w["seed"], probs=True, workspace=ws)
        torch.cuda.synchronize()
        compare_stochastic(r, o, k, f"{parking} B={B} k={k} V={V}")
        assert int(ws.buf[256:].cpu().count_nonzero()) == 0
    assert ws.device_status() == 0


def test_stochastic_zero_drafts_samples_bonus(dev):
    w = workloads.make_stochastic(50, 0, 3000, "bf16", "bf16", seed=8)
    r, o = run_stochastic(w, dev)
    assert (r["accepted_len"].cpu().numpy() == 0).all()
    compare_stochastic(r, o, 0, "k=0")


def test_stochastic_sharp_and_flat_temperatures(dev):
    for T in (0.05, 4.0):
        w = workloads.make_stochastic(24, 4, 5000, "bf16", "f32", t_std=3.0, d_noise=0.5,
                                      temperature=T, seed=9)
        r, o = run_stochastic(w, dev)
        compare_stochastic(r, o, 4, f"T={T}")


def test_stochastic_neg_inf_logits(dev):
    w = workloads.make_stochastic(16, 4, 3000, "f32", "f32", seed=10)
    rng = np.random.default_rng(1)
    w["target"][rng.random(w["target"].shape) < 0.2] = -np.inf
    w["draft"][rng.random(w["draft"].shape) < 0.2] = -np.inf
    r, o = run_stochastic(w, dev)
    compare_stochastic(r, o, 4, "-inf")


def test_stochastic_strided_unaligned_views(dev):
    """Rows not 16-byte aligned take the plain-load path; same results."""
    B, k, V = 7, 4, 2500
    w = workloads.make_stochastic(B, k, V, "bf16", "f32", seed=12)
    big_t = np.zeros((B, k + 2, V + 5), np.uint16)
    big_t[:, 1:, 3:3 + V] = w["target"]
    big_d = np.zeros((B, k, V + 1), np.float32)
    big_d[:, :, 1:] = w["draft"]
    t = to_dev(big_t, "bf16", dev)[:, 1:, 3:3 + V]
    d = to_dev(big_d, "f32", dev)[:, :, 1:]
    r, o = run_stochastic(w, dev, t=t, d=d)
    compare_stochastic(r, o, k, "unaligned")
    # aligned but padded rows (strides larger than V): bulk-copy path
    big_t = np.zeros((B, k + 1, V + 12), np.uint16)
    big_t[:, :, :V] = w["target"]
    t = to_dev(big_t, "bf16", dev)[:, :, :V]
    r, o = run_stochastic(w, dev, t=t)
    compare_stochastic(r, o, k, "padded")


def test_stochastic_broadcast_rows_statistics(dev):
    """Stride-0 batch of one tiny p/q set: 200k independent trials; the
    GPU's first committed token follows p_0 and matches the oracle."""
    rng = np.random.default_rng(13)
    k, V, T, trials = 3, 6, 0.8, 200_000
    tl = (rng.standard_normal((k + 1, V)) * 1.5).astype(np.float32)
    dl = (tl[:k] + rng.standard_normal((k, V))).astype(np.float32)
    q = np.exp(dl / np.float32(T))
    q /= q.sum(-1, keepdims=True)
    g = np.random.default_rng(5)
    tok = np.stack([g.choice(V, trials, p=q[i]) for i in range(k)], 1).astype(np.int32)
    t = torch.from_numpy(tl).to(dev).expand(trials, k + 1, V)
    d = torch.from_numpy(dl).to(dev).expand(trials, k, V)
    r = sv.stochastic(t, d, torch.from_numpy(tok).to(dev), T, 31, probs=True)
    o = oracle.verify_stochastic(np.broadcast_to(tl, (trials, k + 1, V)), "f32",
                                 np.broadcast_to(dl, (trials, k, V)), "f32", tok, T, 31,
                                 threads=THREADS)
    near, flipped = compare_stochastic(r, o, k, "broadcast")
    assert flipped <= max(5, trials // 10000)


def test_stochastic_invalid_token_and_residual_fallback(dev):
    B, k, V = 10, 3, 700
    w = workloads.make_stochastic(B, k, V, "f32", "f32", seed=14)
    w["draft"] = w["target"][:, :k].copy()  # p == q: every valid draft is accepted
    w["tokens"][:, 1] = np.where(np.arange(B) % 2 == 0, V, -3)
    ws = sv.Workspace(dev)
    t = to_dev(w["target"], "f32", dev)
    d = to_dev(w["draft"], "f32", dev)
    r = sv.stochastic(t, d, torch.from_numpy(w["tokens"]).to(dev), 1.0, 3, probs=True,
                      workspace=ws)
    o = oracle.verify_stochastic(w["target"], "f32", w["draft"], "f32", w["tokens"], 1.0, 3)
    assert (o["flags"] == 3).all()
    compare_stochastic(r, o, k, "fallback")
    flags = ws.device_status(clear=True)
    assert flags == (sv.SV_FLAG_INVALID_TOKEN | sv.SV_FLAG_RESIDUAL_FALLBACK)
    assert ws.device_status() == 0


def test_stochastic_seq_offset_and_repeat(dev):
    w = workloads.make_stochastic(12, 4, 6000, "bf16", "bf16", seed=15)
    r0, o0 = run_stochastic(w, dev, seq_offset=1000)
    compare_stochastic(r0, o0, 4, "offset")
    t = to_dev(w["target"], "bf16", dev)
    d = to_dev(w["draft"], "bf16", dev)
    tok = torch.from_numpy(w["tokens"]).to(dev)
    for _ in range(3):  # the workspace is left clean: repeated calls agree
        r = sv.stochastic(t, d, tok, w["temperature"], w["seed"], 1000, probs=True)
        assert torch.equal(r["out_tokens"], r0["out_tokens"])
        assert torch.equal(r["accepted_len"], r0["accepted_len"])
        # rows past the first rejection may be retired unread in one call and
        # not in another; every row read in full gives the same bits
        a, b = r["probs"].cpu().numpy(), r0["probs"].cpu().numpy()
        both = ~((a == -1).all(-1) | (b == -1).all(-1))
        np.testing.assert_array_equal(a[both], b[both])


@both_argmax_paths
def test_kernel_launch_counts(dev, argmax_path):
    """The library counts its own launches: one kernel per stochastic, commit
    and Philox call, three per stochastic tree call, and per greedy,
    multi-candidate or multi-candidate rows call two on the one-grid path (the
    streaming grid, then the finalize grid) and one on the persistent
    pipeline."""
    ws = sv.Workspace(dev)
    g = workloads.make_greedy(B=3, k=2, V=3000, seed=21)
    t = to_dev(g["target"], "bf16", dev)
    tok = torch.from_numpy(g["tokens"]).to(dev)
    per_argmax = 2 if argmax_path == "oneshot" else 1
    st = workloads.make_stochastic(B=3, k=2, V=3000, t_dtype="bf16", d_dtype="bf16", t_std=2.0,
                                   d_noise=0.5, temperature=1.0, seed=22)
    tr = workloads.make_tree(B=2, N=5, V=3000, seed=23)
    rows, row_of, cand = random_rows_case(np.random.default_rng(24), 3, 2, 2, 3000, "bf16")
    seq = torch.zeros(3, dtype=torch.int32, device=dev)
    buf = torch.full((3, 8), -1, dtype=torch.int32, device=dev)
    calls = [
        (per_argmax, lambda: sv.greedy(t, tok, workspace=ws)),
        (per_argmax, lambda: sv.multi_candidate(t[:, None], tok[:, None], workspace=ws)),
        (per_argmax, lambda: sv.multi_candidate_rows(to_dev(rows, "bf16", dev),
                                                     torch.from_numpy(row_of).to(dev),
                                                     torch.from_numpy(cand).to(dev), workspace=ws)),
        (1, lambda: sv.stochastic(to_dev(st["target"], "bf16", dev), to_dev(st["draft"], "bf16", dev),
                                  torch.from_numpy(st["tokens"]).to(dev), 1.0, 5, workspace=ws)),
        (3, lambda: sv.tree_stochastic(to_dev(tr["node_logits"], "bf16", dev),
                                       torch.from_numpy(tr["parent"]).to(dev),
                                       torch.from_numpy(tr["tokens"]).to(dev), 1.0, 5)),
        (1, lambda: sv.tree_greedy(to_dev(tr["node_logits"], "bf16", dev),
                                   torch.from_numpy(tr["parent"]).to(dev),
                                   torch.from_numpy(tr["tokens"]).to(dev))),
        (1, lambda: sv.philox4x32_10(torch.zeros(5, 4, dtype=torch.int32, device=dev), 3)),
    ]
    for want, fn in calls:
        n0 = sv.launch_count()
        r = fn()
        assert sv.launch_count() - n0 == want
    n0 = sv.launch_count()
    sv.commit(sv.greedy(t, tok, workspace=ws), seq, buf)
    assert sv.launch_count() - n0 == per_argmax + 1
    torch.cuda.synchronize()


def test_one_workspace_across_modes_and_sizes(dev):
    """Calls of every mode and many sizes share one workspace; each call must
    leave it clean for the next."""
    ws = sv.Workspace(dev)
    rng = np.random.default_rng(16)
    for step in range(18):
        mode = ("stochastic", "greedy", "multi", "rows", "tree", "threshold")[step % 6]
        B = int(rng.integers(1, 40))
        k = int(rng.integers(0, 9))
        V = int(rng.integers(2, 3000))
        if mode == "stochastic":
            w = workloads.make_stochastic(B, k, V, "bf16", "f32", seed=step)
            t = to_dev(w["target"], "bf16", dev)
            d = to_dev(w["draft"], "f32", dev)
            r = sv.stochastic(t, d, torch.from_numpy(w["tokens"]).to(dev), w["temperature"], 7,
                              probs=True, workspace=ws)
            o = oracle.verify_stochastic(w["target"], "bf16", w["draft"], "f32", w["tokens"],
                                         w["temperature"], 7)
            compare_stochastic(r, o, k, f"step {step}")
        elif mode == "greedy":
            w = workloads.make_greedy(B, k, V, seed=step)
            r = sv.greedy(to_dev(w["target"], "bf16", dev), torch.from_numpy(w["tokens"]).to(dev),
                          workspace=ws)
            o = oracle.verify_greedy(w["target"], "bf16", w["tokens"])
            np.testing.assert_array_equal(r["out_tokens"].cpu().numpy(), o["out_tokens"])
        elif mode == "multi":
            w = workloads.make_multi(B, 3, k, V, seed=step)
            r = sv.multi_candidate(to_dev(w["target"], "bf16", dev),
                                   torch.from_numpy(w["tokens"]).to(dev), workspace=ws)
            o = oracle.verify_multi(w["target"], "bf16", w["tokens"])
            np.testing.assert_array_equal(r["out_tokens"].cpu().numpy(), o["out_tokens"])
        elif mode == "threshold":
            w = workloads.make_greedy(B, k, V, seed=step)
            r = sv.threshold(to_dev(w["target"], "bf16", dev),
                             torch.from_numpy(w["tokens"]).to(dev), 1.0, 1e-3, workspace=ws)
            o = oracle.verify_threshold(w["target"], "bf16", w["tokens"], 1.0, 1e-3)
            compare_threshold(r, o, 1e-3)
        elif mode == "tree":
            w = workloads.make_tree(B, k + 1, V, seed=step)
            r = sv.tree_greedy(to_dev(w["node_logits"], "bf16", dev),
                               torch.from_numpy(w["parent"]).to(dev),
                               torch.from_numpy(w["tokens"]).to(dev), workspace=ws)
            o = oracle.verify_tree_greedy(w["node_logits"], "bf16", w["parent"], w["tokens"])
            np.testing.assert_array_equal(r["out_tokens"].cpu().numpy(), o["out_tokens"])
        else:
            w = workloads.make_multi_rows(B, 3, k, V, seed=step)
            r = sv.multi_candidate_rows(to_dev(w["rows"], "bf16", dev),
                                        torch.from_numpy(w["row_of"]).to(dev),
                                        torch.from_numpy(w["tokens"]).to(dev), workspace=ws)
            o = oracle.verify_multi_rows(w["rows"], "bf16", w["row_of"], w["tokens"])
            np.testing.assert_array_equal(r["out_tokens"].cpu().numpy(), o["out_tokens"])
        torch.cuda.synchronize()
        body = ws.buf[256:].cpu()
        assert int(body.count_nonzero()) == 0, f"workspace not clean after step {step} ({mode})"
    assert ws.device_status() == 0


# --------------------------------------------- bounded waits (no GPU fault)

def test_device_wait_runs_out_and_the_workspace_recovers(dev):
    """A sequence whose state word already marks every row decided (and none
    rejected) before the call can never be resolved by a row merge -- no
    merge sees it change from unresolved to resolved -- so its phase-2 chunks
    wait for a ready-list entry that nothing writes; that wait gives up after
    its bounded limit (about 2 s), every other wait sees the abort, the
    kernel returns, the status word reports SV_FLAG_TIMEOUT, and a
    re-initialised workspace works again."""
    w = workloads.make_stochastic(4, 3, 5000, "bf16", "f32", seed=3)
    t, d = to_dev(w["target"], "bf16", dev), to_dev(w["draft"], "f32", dev)
    tok = torch.from_numpy(w["tokens"]).to(dev)
    call = lambda ws: sv.stochastic(t, d, tok, w["temperature"], 5, workspace=ws)
    size = sv.workspace_size(4, 1, 3, 5000)
    ws = sv.Workspace(dev)
    ws.ensure(size)
    # sequence 0's state word (bytes 8..15 of its 64-byte record after the
    # 256 control bytes): rows 0..2 decided, none rejected
    ws.buf[264:272] = torch.tensor([0x07, 0, 0, 0, 0, 0, 0, 0], dtype=torch.uint8, device=dev)
    call(ws)
    flags = ws.device_status(clear=True)
    assert flags & sv.SV_FLAG_TIMEOUT, flags
    ws.reset()
    r = call(ws)
    torch.cuda.synchronize()
    assert ws.device_status() == 0
    o = oracle.verify_stochastic(w["target"], "bf16", w["draft"], "f32", w["tokens"],
                                 w["temperature"], 5)
    compare_stochastic(r, o, w["k"], "after recovery")


# ------------------------------------------------------- named workloads

@pytest.mark.parametrize("name", list(workloads.WORKLOADS))
def test_named_workload_full_size(dev, name):
    """Every sequence of the full-size workload against the oracle, in the
    same launch configuration the benchmark times."""
    w = workloads.make(name, threads=THREADS)
    mode = w["mode"]
    if mode == "stochastic":
        r, o = run_stochastic(w, dev)
        near, flipped = compare_stochastic(r, o, w["k"], name)
        print(f"{name}: near ties {near}, of which differing {flipped}")
    elif mode == "greedy":
        r = sv.greedy(to_dev(w["target"], "bf16", dev), torch.from_numpy(w["tokens"]).to(dev))
        o = oracle.verify_greedy(w["target"], "bf16", w["tokens"], threads=THREADS)
        np.testing.assert_array_equal(r["accepted_len"].cpu().numpy(), o["accepted_len"])
        np.testing.assert_array_equal(r["out_tokens"].cpu().numpy(), o["out_tokens"])
    elif mode == "multi":
        r = sv.multi_candidate(to_dev(w["target"], "bf16", dev),
                               torch.from_numpy(w["tokens"]).to(dev))
        o = oracle.verify_multi(w["target"], "bf16", w["tokens"], threads=THREADS)
        for key in ("best_candidate", "accepted_len", "out_tokens"):
            np.testing.assert_array_equal(r[key].cpu().numpy(), o[key], err_msg=key)
    elif mode == "threshold":
        r = sv.threshold(to_dev(w["target"], "bf16", dev), torch.from_numpy(w["tokens"]).to(dev),
                         w["temperature"], w["threshold"])
        o = oracle.verify_threshold(w["target"], "bf16", w["tokens"], w["temperature"],
                                    w["threshold"], threads=THREADS)
        near = compare_threshold(r, o, w["threshold"])
        print(f"{name}: near ties {near}")
    elif mode == "tree_stochastic":
        r, o = run_tree_stochastic(w["node_logits"], "bf16", w["parent"], w["tokens"],
                                   w["temperature"], w["seed"], dev)
        near, flipped = compare_tree_stochastic(r, o, name)
        print(f"{name}: near ties {near}, of which differing {flipped}; "
              f"mean accepted {o['accepted_len'].mean():.2f}")
    elif mode == "tree":
        r = sv.tree_greedy(to_dev(w["node_logits"], "bf16", dev),
                           torch.from_numpy(w["parent"]).to(dev),
                           torch.from_numpy(w["tokens"]).to(dev))
        o = oracle.verify_tree_greedy(w["node_logits"], "bf16", w["parent"], w["tokens"],
                                      threads=THREADS)
        for key in ("accepted_len", "path", "out_tokens"):
            np.testing.assert_array_equal(r[key].cpu().numpy(), o[key], err_msg=key)
    else:
        r = sv.multi_candidate_rows(to_dev(w["rows"], "bf16", dev),
                                    torch.from_numpy(w["row_of"]).to(dev),
                                    torch.from_numpy(w["tokens"]).to(dev))
        o = oracle.verify_multi_rows(w["rows"], "bf16", w["row_of"], w["tokens"], threads=THREADS)
        for key in ("best_candidate", "accepted_len", "out_tokens"):
            np.testing.assert_array_equal(r[key].cpu().numpy(), o[key], err_msg=key)
