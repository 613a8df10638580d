"""Multi-rank host logic on CPU: two gloo ranks shard a batch by tokens, run
the block per shard (the oracle stands in for the GPU path here) and
reassemble; the result equals the single-process block, and the timing
reduction returns the slowest rank."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from routed_moe_layer_b200.dist import (data_parallel_forward, max_over_ranks, rank_token_seed,
                                        shard_rows)


def test_shard_rows_cover_exactly_once():
    for T in (0, 1, 7, 240, 19412, 38824):
        for world in (1, 2, 3, 4, 8):
            spans = [shard_rows(T, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == T
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [hi - lo for lo, hi in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        shard_rows(10, 2, 2)
    assert rank_token_seed(2, 0) == 2 and rank_token_seed(2, 3) != rank_token_seed(2, 1)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, result_path):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        import oracle
        from routed_moe_layer_b200 import inputs
        T, H, E, I = 91, 64, 16, 32
        d = inputs.make_block_inputs(T, H, seed=7, E=E, I=I, I_shared=I, unit_scale=True)
        dn = {k: v.float().numpy() for k, v in d.items()}
        cfg = oracle.MoeConfig(E=E, I=I, I_shared=I, top_k=4, n_group=4, topk_group=2)

        def block(xs):
            out, _, _, _ = oracle.moe_forward(xs.numpy(), dn["Wr"], dn["bias"], dn["w13"],
                                              dn["w2"], dn["ws13"], dn["ws2"], cfg)
            return torch.from_numpy(out)

        full = data_parallel_forward(d["x"].float(), block)
        slowest = max_over_ranks(float(rank + 1))
        if rank == 0:
            ref, _, _, _ = oracle.moe_forward(dn["x"], dn["Wr"], dn["bias"], dn["w13"], dn["w2"],
                                              dn["ws13"], dn["ws2"], cfg)
            np.save(result_path, np.stack([np.abs(full.numpy() - ref).max(), slowest]))
    finally:
        dist.barrier()
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_and_reassemble(tmp_path):
    world = 2
    path = str(tmp_path / "res.npy")
    mp.start_processes(_worker, args=(world, _free_port(), path), nprocs=world,
                       start_method="spawn", join=True)
    err, slowest = np.load(path)
    assert err < 1e-12
    assert slowest == 2.0
