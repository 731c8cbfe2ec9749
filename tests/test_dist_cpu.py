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


class OracleOps:
    """The oracle's sharded cast and GEMM (fp64), so that the ranks' host logic
    (token placement, the all-reduce / reduce-scatter of partial dW) runs on
    CPU under gloo exactly as it runs on GPUs under NCCL."""

    @staticmethod
    def cast(t, fmt, seed, sign_mask, shard):
        import oracle
        x = np.ascontiguousarray(t.numpy())
        return oracle.quantize(x, 0, oracle.FORMATS[fmt], rnd=oracle.SR, seed=seed, hadamard=True,
                               sign_mask=sign_mask, scale_layout=oracle.MMA, shard=shard)

    @staticmethod
    def gemm(ac, as_, bc, bs, M, N, K, fmt, alpha):
        import oracle
        import torch
        f = oracle.FORMATS[fmt]
        c, _ = oracle.gemm_decoded(ac, as_, f, bc, bs, f, M, N, K, alpha=alpha)
        return torch.from_numpy(c)


WG_T, WG_DO, WG_DI = 1024, 96, 160


def _wgrad_operands():
    from microscaling_block_scaled_mx_b200 import inputs as I
    return I.wgrad_operands(WG_T, WG_DO, WG_DI)


def _wgrad_worker(rank, ws, port, out_dir):
    import torch
    import torch.distributed as dist
    from microscaling_block_scaled_mx_b200 import dist as D
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=ws)
    try:
        dy, xx = _wgrad_operands()
        t0, t1 = D.token_shards(WG_T, ws)[rank]
        dy_l = torch.from_numpy(dy[t0:t1].copy())
        x_l = torch.from_numpy(xx[t0:t1].copy())
        codes = OracleOps.cast(dy_l, "e2m1", 42, 0x6A09E667, (t0, 0, WG_T, WG_DO))[0]
        np.save(os.path.join(out_dir, f"dy_codes{rank}.npy"), codes)
        full = D.wgrad(dy_l, x_l, t0, WG_T, reduce="all_reduce", ops=OracleOps)
        np.save(os.path.join(out_dir, f"dw_full{rank}.npy"), full.numpy())
        part = D.wgrad(dy_l, x_l, t0, WG_T, reduce="reduce_scatter", ops=OracleOps)
        np.save(os.path.join(out_dir, f"dw_rows{rank}.npy"), part.numpy())
    finally:
        dist.destroy_process_group()


def test_two_rank_token_sharded_wgrad(tmp_path, oracle):
    """Data-parallel weight gradient on two gloo ranks: each rank casts its
    token shard of dY and X (Hadamard + SR, placed in the whole tensor) and
    computes a partial dW; the all-reduce gives every rank the unsharded dW
    and the reduce-scatter gives each rank its row block of it."""
    ws = 2
    mp.start_processes(_wgrad_worker, args=(ws, _free_port(), str(tmp_path)), nprocs=ws, start_method="spawn")
    dy, xx = _wgrad_operands()
    mask = 0x6A09E667
    wc, ws_ = oracle.quantize(dy, 0, oracle.E2M1, rnd=oracle.SR, seed=42, hadamard=True, sign_mask=mask,
                              scale_layout=oracle.MMA)
    xc, xs = oracle.quantize(xx, 0, oracle.E2M1, rnd=oracle.SR, seed=43, hadamard=True, sign_mask=mask,
                             scale_layout=oracle.MMA)
    ref, bound = oracle.gemm_decoded(wc, ws_, oracle.E2M1, xc, xs, oracle.E2M1, WG_DO, WG_DI, WG_T, alpha=1.0 / 32)
    from microscaling_block_scaled_mx_b200.dist import token_shards
    for r, (t0, t1) in enumerate(token_shards(WG_T, ws)):
        np.testing.assert_array_equal(np.load(tmp_path / f"dy_codes{r}.npy"), wc[:, t0 // 2:t1 // 2])
        full = np.load(tmp_path / f"dw_full{r}.npy")
        assert np.all(np.abs(full - ref) <= 1e-12 * bound + 1e-300)
        rows = np.load(tmp_path / f"dw_rows{r}.npy")
        h = WG_DO // ws
        assert np.all(np.abs(rows - ref[r * h:(r + 1) * h]) <= 1e-12 * bound[r * h:(r + 1) * h] + 1e-300)


def test_token_shards_boundaries():
    from microscaling_block_scaled_mx_b200.dist import token_shards
    assert token_shards(16384, 2) == [(0, 8192), (8192, 16384)]
    for ws in (1, 3, 4, 8):
        s = token_shards(16384, ws)
        assert s[0][0] == 0 and s[-1][1] == 16384
        assert all(a % 256 == 0 and b % 256 == 0 for a, b in s)
    with pytest.raises(ValueError):
        token_shards(1000, 2)
