"""Multi-rank host logic on CPU (gloo, world size 2).

Each rank verifies its shard of one batch with the oracle, passing
seq_offset = the shard's first sequence; gathering the shards must give the
unsharded result, and the job time is the slowest rank's.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from speculative_decoding_verification_88_b200.dist import gather_rows, max_over_ranks, shard


def test_shard_covers_the_batch_once():
    for B in (0, 1, 5, 64, 257):
        for world in (1, 2, 3, 8):
            ranges = [shard(B, r, world) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == B
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [b - a for a, b in ranges]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard(4, 2, 2)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        import workloads

        w = workloads.make_stochastic(7, 3, 300, "bf16", "f32", seed=5, threads=1)
        b0, b1 = shard(w["B"], rank, world)
        r = oracle.verify_stochastic(w["target"][b0:b1], "bf16", w["draft"][b0:b1], "f32",
                                     w["tokens"][b0:b1], w["temperature"], 99, seq_offset=b0)
        acc = gather_rows(torch.from_numpy(r["accepted_len"]), w["B"])
        tok = gather_rows(torch.from_numpy(r["out_tokens"]), w["B"])
        # a tree batch shards the same way
        tr = workloads.make_tree(B=5, N=9, V=400, seed=8, threads=1)
        t0, t1 = shard(tr["B"], rank, world)
        rt = oracle.verify_tree_stochastic(tr["node_logits"][t0:t1], "bf16",
                                           tr["parent"][t0:t1], tr["tokens"][t0:t1], 0.8, 41,
                                           seq_offset=t0)
        tree_tok = gather_rows(torch.from_numpy(rt["out_tokens"]), tr["B"])
        tree_path = gather_rows(torch.from_numpy(rt["path"]), tr["B"])
        slowest = max_over_ranks(10.0 + rank)
        if rank == 0:
            np.save(os.path.join(result_dir, "acc.npy"), acc.numpy())
            np.save(os.path.join(result_dir, "tok.npy"), tok.numpy())
            np.save(os.path.join(result_dir, "tree_tok.npy"), tree_tok.numpy())
            np.save(os.path.join(result_dir, "tree_path.npy"), tree_path.numpy())
            np.save(os.path.join(result_dir, "slowest.npy"), np.array([slowest]))
    finally:
        dist.destroy_process_group()


def test_sharded_batch_reproduces_unsharded_result(tmp_path):
    import oracle
    import workloads

    oracle.build()
    mp.spawn(_worker, args=(2, _free_port(), str(tmp_path)), nprocs=2, join=True)
    w = workloads.make_stochastic(7, 3, 300, "bf16", "f32", seed=5, threads=1)
    full = oracle.verify_stochastic(w["target"], "bf16", w["draft"], "f32", w["tokens"],
                                    w["temperature"], 99)
    np.testing.assert_array_equal(np.load(tmp_path / "acc.npy"), full["accepted_len"])
    np.testing.assert_array_equal(np.load(tmp_path / "tok.npy"), full["out_tokens"])
    tr = workloads.make_tree(B=5, N=9, V=400, seed=8, threads=1)
    ft = oracle.verify_tree_stochastic(tr["node_logits"], "bf16", tr["parent"], tr["tokens"],
                                       0.8, 41)
    np.testing.assert_array_equal(np.load(tmp_path / "tree_tok.npy"), ft["out_tokens"])
    np.testing.assert_array_equal(np.load(tmp_path / "tree_path.npy"), ft["path"])
    assert float(np.load(tmp_path / "slowest.npy")[0]) == 11.0
