"""Multi-process host logic on CPU: two gloo ranks shard tokens, run the oracle on
their own shard (stand-in for the per-rank GPU path, which needs no collective),
and reduce their timing with MAX, exactly as bench.py does on GPUs."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from activation_sparse_ffn_twell_b200.dist import token_shard


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def test_token_shard_partitions():
    for M in (0, 1, 7, 4096, 4097):
        for world in (1, 2, 3, 8):
            spans = [token_shard(M, r, world) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == M
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        token_shard(10, 2, 2)


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import oracle as O
    import twell_synth as S
    from activation_sparse_ffn_twell_b200 import dist as D
    r, _, w = D.init("gloo", timeout_s=60)
    assert (r, w) == (rank, world)
    L = S.small_random(64, 64, 256, 32, 8, 0.1, seed=11)
    lo, hi = token_shard(L.M, r, w)
    _, y = O.ffn_forward(L.x[lo:hi], L.w_up, L.b, L.w_down, L.tile_w, L.ell_w)
    D.barrier()
    t_max = D.max_over_ranks(1.0 + rank)
    out[rank] = (lo, hi, y, t_max)
    D.finish()


def test_two_rank_gloo_sharded_forward():
    world, port = 2, _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, port, out), nprocs=world, start_method="spawn", join=True)
    import oracle as O
    import twell_synth as S
    L = S.small_random(64, 64, 256, 32, 8, 0.1, seed=11)
    _, y_all = O.ffn_forward(L.x, L.w_up, L.b, L.w_down, L.tile_w, L.ell_w)
    parts = sorted(out.values(), key=lambda v: v[0])
    assert parts[0][0] == 0 and parts[-1][1] == L.M
    y = np.concatenate([p[2] for p in parts], axis=0)
    assert np.array_equal(y, y_all)                    # sharding over tokens changes nothing
    assert all(p[3] == float(world) for p in parts)    # MAX over ranks seen by every rank
