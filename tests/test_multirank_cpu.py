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


def _oracle_prefill(q, k, v, alpha, beta, s0, scale, l2norm_qk):
    """Stand-in for the kernel call (CPU): the fp64 oracle, states returned as fp32 tensors
    like the kernels'."""
    import oracle
    y, sf = oracle.forward(q, k, v, alpha, beta, s0, scale=scale, l2norm=l2norm_qk)
    return torch.from_numpy(y), torch.from_numpy(sf).to(torch.float32)


def _cp_worker(rank, world, port, cuts, result_path):
    from gated_deltanet_linear_eqs_b200.dist import context_parallel_prefill
    import oracle

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(5)
        B, T, H, d = 2, cuts[-1], 2, 6
        q = torch.from_numpy(rng.standard_normal((B, T, H, d)))
        k = torch.from_numpy(rng.standard_normal((B, T, H, d)))
        v = torch.from_numpy(rng.standard_normal((B, T, H, d)))
        alpha = torch.from_numpy(rng.uniform(0.3, 0.999, (B, T, H)))
        beta = torch.from_numpy(rng.uniform(0.05, 0.95, (B, T, H)))
        s0 = torch.from_numpy(rng.standard_normal((B, H, d, d)) * 0.3).to(torch.float32)
        a, b = cuts[rank], cuts[rank + 1]
        y, s_end = context_parallel_prefill(q[:, a:b], k[:, a:b], v[:, a:b], alpha[:, a:b],
                                            beta[:, a:b], s0, scale=0.5,
                                            prefill=_oracle_prefill)
        gathered = [None] * world
        dist.all_gather_object(gathered, (a, b, y.numpy(), s_end.numpy()))
        if rank == 0:
            y_ref, s_ref = oracle.forward(q, k, v, alpha, beta, s0, scale=0.5)
            y_all = np.zeros_like(y_ref)
            for a_, b_, y_, _ in gathered:
                y_all[:, a_:b_] = y_
            # fp32 states between the ranks: agreement to fp32 rounding
            np.testing.assert_allclose(y_all, y_ref, rtol=1e-5, atol=1e-5)
            np.testing.assert_allclose(gathered[-1][3], s_ref, rtol=1e-5, atol=1e-5)
            # every rank's end state is the sequence's state after its last token
            for a_, b_, _, s_ in gathered:
                _, s_mid = oracle.forward(q[:, :b_], k[:, :b_], v[:, :b_], alpha[:, :b_],
                                          beta[:, :b_], s0, scale=0.5)
                np.testing.assert_allclose(s_, s_mid, rtol=1e-5, atol=1e-5)
            with open(result_path, "w") as f:
                f.write("ok")
        dist.barrier()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("cuts", [[0, 23, 45], [0, 20, 20, 45]])
def test_context_parallel_prefill_matches_one_sequence(tmp_path, cuts):
    """One sequence split along time across gloo ranks (the second case gives a rank no
    tokens): the maps, the all-gather and the scan reproduce the unsplit token loop."""
    result = tmp_path / "result.txt"
    world = len(cuts) - 1
    mp.start_processes(_cp_worker, args=(world, _free_port(), cuts, str(result)),
                       nprocs=world, join=True, start_method="spawn")
    assert result.read_text() == "ok"


def test_context_parallel_prefill_single_rank_is_plain_prefill():
    from gated_deltanet_linear_eqs_b200.dist import context_parallel_prefill
    import oracle
    rng = np.random.default_rng(6)
    q, k, v = (torch.from_numpy(rng.standard_normal((1, 9, 2, 4))) for _ in range(3))
    alpha = torch.from_numpy(rng.uniform(0.3, 0.99, (1, 9, 2)))
    beta = torch.from_numpy(rng.uniform(0.1, 0.9, (1, 9, 2)))
    y, s = context_parallel_prefill(q, k, v, alpha, beta, prefill=_oracle_prefill)
    y_ref, s_ref = oracle.forward(q, k, v, alpha, beta)
    np.testing.assert_allclose(y.numpy(), y_ref, rtol=1e-12)
    np.testing.assert_allclose(s.numpy(), s_ref, rtol=1e-6)
    with pytest.raises(ValueError):
        context_parallel_prefill(q, k, v[..., :3], alpha, beta, prefill=_oracle_prefill)
