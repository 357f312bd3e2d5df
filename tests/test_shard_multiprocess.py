"""The data-parallel partition on two CPU processes (gloo): the ranks' batch
slices tile the batch exactly, each rank's inputs equal the unsharded draw of
its rows, and the timing reduction takes the maximum over ranks."""
import os

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from quantized_recurrent_state_decode_b200 import inputs as I
from quantized_recurrent_state_decode_b200.shard import batch_slice, max_over_ranks


@pytest.mark.parametrize("B,world", [(256, 2), (7, 3), (1, 4), (0, 2), (1024, 8)])
def test_slices_tile_the_batch(B, world):
    seen = []
    for r in range(world):
        off, n = batch_slice(B, r, world)
        seen += list(range(off, off + n))
    assert seen == list(range(B))


def test_bad_partition_arguments():
    with pytest.raises(ValueError):
        batch_slice(8, 2, 2)


def _worker(rank, world, port, result_dir):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = I.WORKLOADS["gla_rtn_int8_b2h2_64"].with_batch(5)
        off, n = batch_slice(w.batch, rank, world)
        mine = I.step_inputs(w, 3, batch_offset=off, batch=n)
        full = I.step_inputs(w, 3)
        ok = all(torch.equal(mine[k], full[k][off:off + n]) for k in ("q", "k", "v", "gates"))
        S_mine = I.initial_state(w.__class__(**{**w.__dict__, "s0_std": 0.02}), off, n)
        m = max_over_ranks(float(rank + 1) * 1.5)
        torch.save({"ok": ok, "max": m, "n": n, "s0": tuple(S_mine.shape)},
                   os.path.join(result_dir, "r%d.pt" % rank))
    finally:
        dist.destroy_process_group()


def test_two_rank_gloo_partition(tmp_path):
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    world = 2
    mp.start_processes(_worker, args=(world, port, str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    res = [torch.load(os.path.join(tmp_path, "r%d.pt" % r)) for r in range(world)]
    assert all(r["ok"] for r in res)
    assert all(r["max"] == 3.0 for r in res)
    assert sum(r["n"] for r in res) == 5
