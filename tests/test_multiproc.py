"""World-size-2 checks of the multi-GPU host logic on CPU (gloo backend).

Each rank runs the CPU oracle on its own token block; the gathered rows must
equal the single-process result bit for bit (tokens are independent), and the
max-over-ranks reduction used to time a step must return the slowest rank.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from activation_sparse_gemm_b200 import dist as rdist


def test_token_blocks_cover_without_overlap():
    for M in (0, 1, 127, 128, 4096, 32760):
        for world in (1, 2, 3, 8):
            for align in (1, 128):
                blocks = [rdist.token_block(M, world, r, align) for r in range(world)]
                assert blocks[0][0] == 0 and blocks[-1][1] == M
                for (a, b), (c, d) in zip(blocks, blocks[1:]):
                    assert b == c and a <= b
                sizes = [b - a for a, b in blocks]
                assert max(sizes) - min(sizes) <= 2 * align  # the last block may also be cut short by M
                for a, b in blocks:
                    assert b == a or a % align == 0  # non-empty blocks start on an aligned token


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world), RANK=str(rank),
                      LOCAL_RANK=str(rank))
    import torch
    import torch.distributed as dist

    import oracle
    from activation_sparse_gemm_b200.inputs import make_custom

    w, r, _ = rdist.init("gloo", timeout_s=60)
    assert (w, r) == (world, rank)
    X, W, L_A, L_B = make_custom(37, 64, 24, 16, seed=21)
    a, b = rdist.token_block(X.shape[0], w, r)
    Y = oracle.linear(X[a:b], W, L_A, L_B)
    rows = [None] * w
    dist.all_gather_object(rows, (a, b, Y))
    slowest = rdist.max_over_ranks(float(10 + rank))
    if rank == 0:
        full = np.concatenate([y for _, _, y in sorted(rows, key=lambda t: t[0])], axis=0)
        np.save(os.path.join(out_dir, "gathered.npy"), full)
        np.save(os.path.join(out_dir, "slowest.npy"), np.array([slowest]))
    rdist.shutdown()


@pytest.mark.timeout(180)
def test_two_rank_token_split_matches_single_process(tmp_path):
    import oracle
    from activation_sparse_gemm_b200.inputs import make_custom
    oracle.build()
    world = 2
    mp.spawn(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    X, W, L_A, L_B = make_custom(37, 64, 24, 16, seed=21)
    ref = oracle.linear(X, W, L_A, L_B)
    got = np.load(tmp_path / "gathered.npy")
    assert got.shape == ref.shape and (got == ref).all()
    assert np.load(tmp_path / "slowest.npy")[0] == 11.0
