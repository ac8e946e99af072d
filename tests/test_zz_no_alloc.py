"""The greedy entry point that allocates nothing.

It exists for callers that cannot allocate device memory on the verify path
(an external allocator or pool owns the device, or the call runs where an
allocation may block or fail).  This file is collected last, so a run that
stops at its first failure has already run every other test.
"""
import ctypes

import numpy as np
import pytest
import torch

import speculative_decoding_verification_88_b200 as sv
import workloads
from speculative_decoding_verification_88_b200 import build as svbuild


@pytest.fixture(scope="module")
def lib():
    svbuild.build()
    return sv.load_library()


def test_noalloc_rejects_problems_beyond_its_scratch(lib):
    # Fails on the host before any device work: too large for the 2 MiB array.
    rc = lib.spec_verify_greedy_noalloc(None, 1, 0, 0, None, 4096, 8, 128256, None, None, None)
    assert rc == 3  # SV_ERR_WORKSPACE
    rc = lib.spec_verify_greedy_noalloc(None, 1, 0, 0, None, 4, 40, 100, None, None, None)
    assert rc == 1  # SV_ERR_INVALID_ARG (k > 32)
    assert lib.spec_verify_greedy_noalloc(None, 1, 0, 0, None, 0, 4, 100, None, None, None) == 0


@pytest.mark.gpu
@pytest.mark.parametrize("B,k,V", [(64, 4, 128256), (7, 3, 4097)])
def test_noalloc_matches_workspace_entry_point_twice(lib, B, k, V):
    dev = torch.device("cuda:0")
    w = workloads.make_greedy(B, k, V, p_match=0.7, seed=B + k)
    t = workloads.as_torch(w["target"], "bf16").to(dev)
    tok = torch.from_numpy(w["tokens"]).to(dev)
    ref = sv.greedy(t, tok)
    for _ in range(2):  # two calls in a row share the static scratch
        got = sv.greedy_noalloc(t, tok)
        torch.cuda.synchronize()
        # greedy verify is exact: the tolerance of the other greedy tests
        np.testing.assert_array_equal(got["accepted_len"].cpu().numpy(),
                                      ref["accepted_len"].cpu().numpy())
        np.testing.assert_array_equal(got["out_tokens"].cpu().numpy(),
                                      ref["out_tokens"].cpu().numpy())
