"""Host logic of the multi-GPU path on CPU: world size 2 over gloo.

Rows are independent, so ranks split them with no data-path collective; the
only collective is the max over ranks of the step time.  These checks run the
float64 oracle on each rank's shard and compare with the full batch.
"""

import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from rotation_bit_quantization_b200 import workloads as wl


def _free_port():
    with socket.socket(socket.AF_INET, socket.SOCK_STREAM) as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist

    from oracle import butterfly as ob
    from oracle import quant as oq

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = wl.tiny(rows_x=37, rows_w=10)
        start, stop = wl.shard_rows(w.x.shape[0], world, rank)
        y = ob.forward(w.theta, w.x[start:stop].astype(np.float64))
        c, s, z = oq.quantize_pack(ob.forward(w.theta, w.w.astype(np.float64)).astype(np.float32), 2, 64)
        np.savez(os.path.join(out_dir, f"rank{rank}.npz"), y=y, start=start, stop=stop, c=c, s=s, z=z)
        # the step-time reduction bench.py uses: max over ranks
        t = torch.tensor([float(rank + 1) * 1.5], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        np.save(os.path.join(out_dir, f"max{rank}.npy"), t.numpy())
    finally:
        dist.destroy_process_group()


def test_shard_rows_covers_every_row_once():
    for total in (0, 1, 7, 2048, 11008):
        for world in (1, 2, 3, 8):
            spans = [wl.shard_rows(total, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == total
            for (a, b), (c, d) in zip(spans, spans[1:]):
                assert b == c and a <= b
            sizes = [b - a for a, b in spans]
            assert max(sizes) - min(sizes) <= 1
    with pytest.raises(ValueError):
        wl.shard_rows(10, 2, 2)


def test_two_ranks_gloo(tmp_path):
    world, port = 2, _free_port()
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True, start_method="spawn")
    from oracle import butterfly as ob

    w = wl.tiny(rows_x=37, rows_w=10)
    full = ob.forward(w.theta, w.x.astype(np.float64))
    parts = [np.load(tmp_path / f"rank{r}.npz") for r in range(world)]
    assert sum(int(p["stop"] - p["start"]) for p in parts) == 37
    stitched = np.concatenate([p["y"] for p in parts])
    assert np.array_equal(stitched, full)
    for p in parts[1:]:                          # replicated weight side: identical on every rank
        assert np.array_equal(p["c"], parts[0]["c"]) and np.array_equal(p["s"], parts[0]["s"])
    for r in range(world):
        assert float(np.load(tmp_path / f"max{r}.npy")[0]) == 3.0


# ---------------------------------------------------------------- backward split by layer

def test_shard_layers_covers_every_layer_once():
    for total in (0, 1, 5, 32, 33):
        for world in (1, 2, 3, 8):
            parts = [wl.shard_layers(total, world, r) for r in range(world)]
            flat = sorted(l for p in parts for l in p)
            assert flat == list(range(total))
            sizes = [len(p) for p in parts]
            assert max(sizes) - min(sizes) <= 1
    assert wl.shard_layers(32, 8, 3) == [3, 11, 19, 27]
    with pytest.raises(ValueError):
        wl.shard_layers(4, 2, 2)


def test_per_layer_angles_depend_on_the_layer_only():
    full = wl.backward_angles(6, 16)
    for world in (2, 3):
        for r in range(world):
            mine = wl.shard_layers(6, world, r)
            assert np.array_equal(wl.backward_angles(mine, 16), full[mine])


def test_per_rank_activation_seeding():
    # the transform bench gives every rank its own batch of the same shape and the same angles
    a, b = wl.act_4096(8, seed_offset=0), wl.act_4096(8, seed_offset=1)
    assert np.array_equal(a.theta, b.theta)
    assert not np.array_equal(a.x, b.x)
    assert np.array_equal(wl.act_4096(8, seed_offset=1).x, b.x)
    assert a.meta["outlier_channels"] == b.meta["outlier_channels"]


_BWD_LAYERS, _BWD_TOKENS, _BWD_M = 5, 12, 16


def _bwd_worker(rank, world, port, out_dir):
    import torch
    import torch.distributed as dist

    from oracle import butterfly as ob

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        mine = wl.shard_layers(_BWD_LAYERS, world, rank)
        thetas = wl.backward_angles(mine, _BWD_M)
        out = {}
        for k, l in enumerate(mine):
            w = wl.backward_layer_host(l, _BWD_TOKENS, _BWD_M)
            assert np.array_equal(w.theta, thetas[k])
            x = wl.f32_from_bf16_bits(w.x).astype(np.float64)
            _, dx, dth = ob.backward(thetas[k], x, w.dy.astype(np.float64))
            out[f"dth{l}"] = dth
            out[f"dx{l}"] = dx
        np.savez(os.path.join(out_dir, f"bwd{rank}.npz"), layers=np.array(mine, dtype=np.int64), **out)
        # the only collective: the max over ranks of the step time
        t = torch.tensor([10.0 - rank], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        np.save(os.path.join(out_dir, f"bmax{rank}.npy"), t.numpy())
    finally:
        dist.destroy_process_group()


def test_two_ranks_gloo_backward_by_layer(tmp_path):
    """Ranks take layers r, r + N, ...: the per-rank oracle dtheta and dX blocks reassemble
    into the single-process result over all layers, every layer exactly once."""
    world, port = 2, _free_port()
    mp.start_processes(_bwd_worker, args=(world, port, str(tmp_path)), nprocs=world, join=True, start_method="spawn")
    from oracle import butterfly as ob

    seen = []
    for r in range(world):
        p = np.load(tmp_path / f"bwd{r}.npz")
        for l in p["layers"].tolist():
            seen.append(l)
            w = wl.backward_layer_host(l, _BWD_TOKENS, _BWD_M)
            _, dx, dth = ob.backward(w.theta, wl.f32_from_bf16_bits(w.x).astype(np.float64), w.dy.astype(np.float64))
            assert np.array_equal(p[f"dth{l}"], dth)
            assert np.array_equal(p[f"dx{l}"], dx)
        assert float(np.load(tmp_path / f"bmax{r}.npy")[0]) == 10.0
    assert sorted(seen) == list(range(_BWD_LAYERS))
