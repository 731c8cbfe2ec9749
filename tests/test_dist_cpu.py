"""World-size-2 gloo runs of the multi-rank host logic (no GPU): row sharding
covers every row exactly once on 32-row boundaries, the sharded cast equals
the unsharded one, and timings reduce to the slowest rank."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from microscaling_block_scaled_mx_b200.dist import shard_rows


def test_shard_rows_partition():
    for rows in (0, 1, 31, 32, 33, 8192, 16384 + 96):
        for ws in (1, 2, 3, 4, 8):
            got = [shard_rows(rows, ws, r, 32) for r in range(ws)]
            assert got[0][0] == 0 and got[-1][1] == rows
            for (a, b), (c, d) in zip(got, got[1:]):
                assert b == c
            for a, b in got:
                assert a % 32 == 0 or a == rows
                assert b % 32 == 0 or b == rows


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, ws, port, out_dir):
    import torch.distributed as dist
    import oracle
    from microscaling_block_scaled_mx_b200 import inputs as I
    from microscaling_block_scaled_mx_b200.dist import barrier, max_over_ranks, shard_rows
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        x = I.cast_sweep_input(256, 128)
        r0, r1 = shard_rows(256, ws, rank, 32)
        # blocks along rows: each rank casts whole 32-row blocks of its shard
        codes, scales = oracle.quantize(np.ascontiguousarray(x[r0:r1]), 0, oracle.E4M3)
        np.save(os.path.join(out_dir, f"codes{rank}.npy"), codes)
        np.save(os.path.join(out_dir, f"scales{rank}.npy"), scales)
        barrier()
        t = max_over_ranks(float(rank + 1))
        np.save(os.path.join(out_dir, f"t{rank}.npy"), np.array([t]))
    finally:
        dist.destroy_process_group()


def test_two_rank_sharded_cast_and_timing(tmp_path, oracle):
    ws = 2
    mp.start_processes(_worker, args=(ws, _free_port(), str(tmp_path)), nprocs=ws, start_method="spawn")
    from microscaling_block_scaled_mx_b200 import inputs as I
    x = I.cast_sweep_input(256, 128)
    want_c, want_s = oracle.quantize(x, 0, oracle.E4M3)
    parts_c = [np.load(tmp_path / f"codes{r}.npy") for r in range(ws)]
    parts_s = [np.load(tmp_path / f"scales{r}.npy") for r in range(ws)]
    # codes are 128 x 256 (block-axis-major): shards are column ranges of it
    np.testing.assert_array_equal(np.concatenate(parts_c, axis=1), want_c)
    got_s = np.concatenate([s.reshape(128, -1) for s in parts_s], axis=1)
    np.testing.assert_array_equal(got_s, want_s.reshape(128, -1))
    for r in range(ws):
        assert np.load(tmp_path / f"t{r}.npy")[0] == 2.0
