"""Sharding across ranks, on CPU with gloo (world size 2): every image is processed by
exactly one rank, the gathered per-rank results equal a single-process run, and the timing
reduction takes the max over ranks. The per-rank compute here is the CPU oracle."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from bi_level_routing_b200.distributed import gather_images, max_over_ranks, shard_range


@pytest.mark.parametrize("B,world", [(64, 2), (7, 2), (1, 2), (0, 3), (10, 4)])
def test_shard_range_partitions_the_batch(B, world):
    seen = []
    for r in range(world):
        a, b = shard_range(B, r, world)
        assert 0 <= a <= b <= B
        seen.extend(range(a, b))
    assert seen == list(range(B))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, B, result_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle
        from bi_level_routing_b200.distributed import forward_local
        from bi_level_routing_b200.workloads import WORKLOADS, make_inputs
        w = WORKLOADS["stage2"].with_(B=B)
        inp = make_inputs(w)
        q, k, v = (torch.from_numpy(inp[n].astype(np.float64)) for n in "qkv")

        def oracle_forward(q, k, v, n_win, topk, heads):
            out, idx = oracle.forward(q.numpy(), k.numpy(), v.numpy(), n_win, topk, heads)
            return torch.from_numpy(out), torch.from_numpy(idx)

        start, stop, out, idx = forward_local(q, k, v, w.n_win, w.topk, w.heads, forward_fn=oracle_forward)
        full_out = gather_images(out, B)
        full_idx = gather_images(idx, B)
        slowest = max_over_ranks(float(rank + 1) * 0.5)
        if rank == 0:
            torch.save({"out": full_out, "idx": full_idx, "slowest": slowest}, os.path.join(result_dir, "r.pt"))
    finally:
        dist.destroy_process_group()


def test_gloo_two_ranks_match_one_process(tmp_path):
    import oracle
    from bi_level_routing_b200.workloads import WORKLOADS, make_inputs
    B = 5
    mp.start_processes(_worker, args=(2, _free_port(), B, str(tmp_path)), nprocs=2, start_method="spawn")
    got = torch.load(tmp_path / "r.pt")
    w = WORKLOADS["stage2"].with_(B=B)
    inp = make_inputs(w)
    out, idx = oracle.forward(inp["q"], inp["k"], inp["v"], w.n_win, w.topk, w.heads)
    assert np.array_equal(got["idx"].numpy(), idx)
    assert np.array_equal(got["out"].numpy(), out)
    assert got["slowest"] == 1.0
