"""The N > 1 host path on CPU: two gloo ranks shard tokens, process their own rows, and agree on
the max-over-ranks time; the union of the shards is exactly the single-process result. Two gloo
ranks also calibrate on halves of one calibration set and merge their keys with the library's
all-reduce(MAX): every rank must find the whole set's outlier channel and sign vector."""
import os
import socket
import tempfile

import numpy as np
import pytest
import torch.multiprocessing as mp

from rotation_activation_quantization_b200 import sharding


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_shard_range_partitions():
    for total in (0, 1, 7, 8192, 8193):
        for world in (1, 2, 3, 8):
            spans = [sharding.shard_range(r, world, total) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            assert all(a[1] == b[0] for a, b in zip(spans, spans[1:]))
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    assert sharding.weak_shard(3, 8192) == (3 * 8192, 4 * 8192)
    with pytest.raises(ValueError):
        sharding.shard_range(2, 2, 10)
    assert sharding.aggregate_rate(4 * 8192, 0.5) == 4 * 8192 / 0.5


def _worker(rank, world, port, outdir):
    import torch.distributed as dist

    from oracle import signrot_oracle as o
    from rotation_activation_quantization_b200 import synthetic as syn

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = syn.workload(1)
        t0, t1 = sharding.weak_shard(rank, 16)
        x = o.to_f64(syn.draw_tokens(w, t0, t1), w.dtype)
        d = syn.draw_d(w)
        k, xk = o.calibrate(o.to_f64(syn.draw_calibration(w), w.dtype))
        q, scale, zero = o.rotate_quant(x, d, o.build_sign(w.n, k, xk, d))
        np.savez(os.path.join(outdir, f"r{rank}.npz"), q=q, scale=scale, zero=zero, t0=t0, t1=t1)
        elapsed = 1.0 + rank  # each rank's own step time; the job's is the slowest
        assert sharding.max_over_ranks(elapsed) == float(world)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_shard_tokens():
    world = 2
    with tempfile.TemporaryDirectory() as outdir:
        mp.start_processes(_worker, args=(world, _free_port(), outdir), nprocs=world, join=True,
                           start_method="spawn")
        parts = [np.load(os.path.join(outdir, f"r{r}.npz")) for r in range(world)]
        assert [int(p["t0"]) for p in parts] == [0, 16] and [int(p["t1"]) for p in parts] == [16, 32]

        from oracle import signrot_oracle as o
        from rotation_activation_quantization_b200 import synthetic as syn

        w = syn.workload(1)
        d = syn.draw_d(w)
        k, xk = o.calibrate(o.to_f64(syn.draw_calibration(w), w.dtype))
        q, scale, zero = o.rotate_quant(o.to_f64(syn.draw_tokens(w, 0, 32), w.dtype), d,
                                        o.build_sign(w.n, k, xk, d))
        assert (np.concatenate([p["q"] for p in parts]) == q).all()
        assert (np.concatenate([p["scale"] for p in parts]) == scale).all()
        assert (np.concatenate([p["zero"] for p in parts]) == zero).all()


def _calib_worker(rank, world, port, outdir):
    import torch
    import torch.distributed as dist

    from calib_keys import decode, fold_keys
    from oracle import signrot_oracle as o

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x, d = _calibration_set()
        t0, t1 = sharding.shard_range(rank, world, x.shape[0])
        keys = torch.from_numpy(fold_keys(x[t0:t1], t_offset=t0).astype(np.int64))
        sharding.merge_calibration(keys)
        k, xk = decode(keys.numpy().astype(np.uint64))
        s = o.build_sign(x.shape[1], k, xk, d)
        np.savez(os.path.join(outdir, f"c{rank}.npz"), k=k, xk=xk, s=s)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _calibration_set():
    """256 rows, n = 448, with magnitude ties planted across the two halves: the largest |x| (the
    bf16 value 1232) sits in channel 300 at tokens 100 and 200 (signs + then -) and in channel 301
    at token 50 (sign -), so the lowest channel (300) and its first token (100, rank 0) must win."""
    from rotation_activation_quantization_b200 import synthetic as syn

    x, d, _ = syn.random_rows(448, 256, "f32", seed=77, outlier=0.0)
    x[100, 300], x[200, 300], x[50, 301] = 1232.0, -1232.0, -1232.0
    x[180, 5] = -1000.0  # a smaller magnitude in the second half
    return x.astype(np.float64), d


def test_two_gloo_ranks_merge_calibration():
    world = 2
    with tempfile.TemporaryDirectory() as outdir:
        mp.start_processes(_calib_worker, args=(world, _free_port(), outdir), nprocs=world, join=True,
                           start_method="spawn")
        parts = [np.load(os.path.join(outdir, f"c{r}.npz")) for r in range(world)]

        from oracle import signrot_oracle as o

        x, d = _calibration_set()
        k_ref, xk_ref = o.calibrate(x)
        assert (k_ref, xk_ref) == (300, 1232.0)
        s_ref = o.build_sign(x.shape[1], k_ref, xk_ref, d)
        for p in parts:
            assert (int(p["k"]), float(p["xk"])) == (k_ref, xk_ref)
            assert (p["s"] == s_ref).all()
        # without the merge each rank would see only its own half: rank 1 alone finds token 200
        from calib_keys import decode, fold_keys

        assert decode(fold_keys(x[128:], t_offset=128)) == (300, -1232.0)
