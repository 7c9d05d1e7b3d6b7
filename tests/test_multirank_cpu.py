"""The multi-GPU path's host logic, run as world-size-2 gloo process groups on the CPU.

The recurrence shards with no exchange step: each rank processes its own documents (or
sequences / heads), and only timings are reduced (max over ranks).  These tests run two
ranks on gloo.  Each rank takes its share of a packed batch from ``shard_documents``, runs
the computation for its documents, and the shares are gathered; the reassembled result must
equal the unsharded computation.  The fp64 oracle stands in for the CUDA kernels, which need
a GPU.  The timing reduction is checked on rank-dependent values.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from gated_deltanet_linear_eqs_b200.dist import max_over_ranks, shard_documents, shard_range


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_documents_balances_and_covers():
    lengths = [16749, 4122, 7000, 4897]
    shards = shard_documents(lengths, 2)
    assert sorted(sum(shards, [])) == [0, 1, 2, 3]
    loads = [sum(lengths[i] for i in s) for s in shards]
    assert max(loads) == 16749 and min(loads) == 16019
    assert shard_documents([5, 1], 4) == [[0], [1], [], []]
    with pytest.raises(ValueError):
        shard_documents([1], 0)


def test_shard_range_partitions():
    for n in (1, 7, 8, 32):
        for world in (1, 2, 3, 8):
            blocks = [shard_range(n, world, r) for r in range(world)]
            assert blocks[0][0] == 0 and blocks[-1][1] == n
            assert all(a[1] == b[0] for a, b in zip(blocks, blocks[1:]))
            sizes = [b - a for a, b in blocks]
            assert max(sizes) - min(sizes) <= 1


def _worker(rank, world, port, lengths, result_path):
    import oracle
    from gated_deltanet_linear_eqs_b200.inputs import make_varlen_inputs

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        # timing reduction: the max over ranks of rank-dependent values
        assert max_over_ranks(1.5 + rank) == 1.5 + world - 1
        H, d = 2, 8
        inp = make_varlen_inputs(lengths, H, d, d, seed=3)
        cu = inp["cu_seqlens"].numpy()
        mine = shard_documents(lengths, world)[rank]
        ys, ss = {}, {}
        for n in mine:  # this rank's documents, computed independently
            a, b = int(cu[n]), int(cu[n + 1])
            sl = {k: inp[k][:, a:b] for k in ("q", "k", "v", "alpha", "beta")}
            y, s = oracle.forward_varlen(sl["q"], sl["k"], sl["v"], sl["alpha"], sl["beta"],
                                         [0, b - a], inp["s0"][n:n + 1])
            ys[n], ss[n] = y, s
        gathered = [None] * world
        dist.all_gather_object(gathered, (ys, ss))
        if rank == 0:
            y_all = np.zeros((1, int(cu[-1]), H, d))
            s_all = np.zeros((len(lengths), H, d, d))
            seen = []
            for part_y, part_s in gathered:
                for n, y in part_y.items():
                    y_all[:, cu[n]:cu[n + 1]] = y
                    s_all[n] = part_s[n][0]
                    seen.append(n)
            assert sorted(seen) == list(range(len(lengths)))
            y_ref, s_ref = oracle.forward_varlen(inp["q"], inp["k"], inp["v"], inp["alpha"],
                                                 inp["beta"], cu, inp["s0"])
            np.testing.assert_allclose(y_all, y_ref, rtol=1e-13, atol=1e-14)
            np.testing.assert_allclose(s_all, s_ref, rtol=1e-13, atol=1e-14)
            with open(result_path, "w") as f:
                f.write("ok")
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_sharded_forward_reassembles(tmp_path):
    result = tmp_path / "result.txt"
    mp.start_processes(_worker, args=(2, _free_port(), [37, 5, 64, 20, 1], str(result)),
                       nprocs=2, join=True, start_method="spawn")
    assert result.read_text() == "ok"
