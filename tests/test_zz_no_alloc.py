"""The greedy entry point that allocates nothing.

It exists for callers that cannot allocate device memory on the verify path
(an external allocator or pool owns the device, or the call runs where an
allocation may block or fail): the library runs greedy verify on a fixed
device array it carries in its image instead of a caller's workspace.  This
file is collected last, so a run that stops at its first failure has already
run every other test.
"""
import numpy as np
import pytest
import torch

import oracle
import speculative_decoding_verification_88_b200 as sv
import workloads
from speculative_decoding_verification_88_b200 import build as svbuild


@pytest.fixture(scope="module")
def lib():
    svbuild.build()
    return sv.load_library()


def largest_batch(lib, k, V):
    """The largest B whose workspace fits the 2 MiB array."""
    lo, hi = 0, 1 << 16
    while lo < hi:
        m = (lo + hi + 1) // 2
        if lib.spec_verify_workspace_size(m, 1, k, V) <= (2 << 20):
            lo = m
        else:
            hi = m - 1
    return lo


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    # Fails on the host before any device work: one sequence more than the
    # 2 MiB array holds.
    top = largest_batch(lib, 8, 128256)
    assert top >= 700
    rc = lib.spec_verify_greedy_noalloc(None, 1, 0, 0, None, top + 1, 8, 128256, None, None,
                                        None)
    assert rc == 3  # SV_ERR_WORKSPACE
    rc = lib.spec_verify_greedy_noalloc(None, 1, 0, 0, None, 4, 40, 100, None, None, None)
    assert rc == 1  # SV_ERR_INVALID_ARG (k > 32)
    assert lib.spec_verify_greedy_noalloc(None, 1, 0, 0, None, 0, 4, 100, None, None, None) == 0
    assert lib.spec_verify_greedy_noalloc_read_device_status(None, 0, None) == 1


@pytest.mark.gpu
@pytest.mark.parametrize("B,k,V", [(64, 4, 128256), (7, 3, 4097), (760, 8, 2000)])
def test_noalloc_matches_oracle_and_workspace_entry_point_twice(lib, B, k, V):
    dev = torch.device("cuda:0")
    w = workloads.make_greedy(B, k, V, p_match=0.7, seed=B + k)
    t = workloads.as_torch(w["target"], "bf16").to(dev)
    tok = torch.from_numpy(w["tokens"]).to(dev)
    want = oracle.verify_greedy(w["target"], "bf16", w["tokens"])
    ref = sv.greedy(t, tok)
    for _ in range(2):  # two calls in a row share the static scratch
        got = sv.greedy_noalloc(t, tok)
        torch.cuda.synchronize()
        # greedy verify is exact: the tolerance of the other greedy tests
        for key in ("accepted_len", "out_tokens"):
            np.testing.assert_array_equal(got[key].cpu().numpy(), want[key], err_msg=key)
            np.testing.assert_array_equal(got[key].cpu().numpy(), ref[key].cpu().numpy())
    assert sv.greedy_noalloc_device_status() == 0


@pytest.mark.gpu
def test_noalloc_reports_device_errors_until_read(lib):
    dev = torch.device("cuda:0")
    w = workloads.make_greedy(5, 4, 3000, p_match=0.7, seed=3)
    w["tokens"][2, 0] = 3000  # outside [0, V): rejected and flagged
    t = workloads.as_torch(w["target"], "bf16").to(dev)
    tok = torch.from_numpy(w["tokens"]).to(dev)
    got = sv.greedy_noalloc(t, tok)
    good = torch.from_numpy(workloads.make_greedy(5, 4, 3000, seed=4)["tokens"]).to(dev)
    sv.greedy_noalloc(t, good)  # a later call keeps the flag: it is sticky
    assert sv.greedy_noalloc_device_status(clear=False) == sv.SV_FLAG_INVALID_TOKEN
    want = oracle.verify_greedy(w["target"], "bf16", w["tokens"])
    np.testing.assert_array_equal(got["out_tokens"].cpu().numpy(), want["out_tokens"])
    assert want["accepted_len"][2] == 0
    assert sv.greedy_noalloc_device_status(clear=True) == sv.SV_FLAG_INVALID_TOKEN
    assert sv.greedy_noalloc_device_status() == 0
