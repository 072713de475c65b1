"""The N > 1 host path on CPU: two gloo ranks shard tokens, process their own rows, and agree on
the max-over-ranks time; the union of the shards is exactly the single-process result."""
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
