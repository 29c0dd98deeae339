"""The N>1 host logic of the replica bench on 2 gloo ranks (CPU): each rank gets
its own prompt batch with identical shapes, the timed interval is reduced by max,
and the whole-job throughput counts every rank's tokens."""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _worker(rank, world, port, out_dir):
    import datetime

    import torch.distributed as dist

    from learned_token_pruning_gate_b200 import dist as tgd
    from learned_token_pruning_gate_b200 import inputs as gen

    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = tgd.rank_workload(gen.scaled(gen.WORKLOADS["ragged_4"], 64), rank)
        inp = gen.make_inputs(w, with_qkv=False)
        local_ms = 10.0 + 5.0 * rank  # rank 1 is the slow one
        tgd.barrier("cpu")
        mx = tgd.max_over_ranks(local_ms, device="cpu")
        value = tgd.aggregate_throughput(w.total_tokens, 7, mx, world)
        np.savez(os.path.join(out_dir, f"r{rank}.npz"), h=inp.h.float().numpy(), mx=mx,
                 value=value, tokens=w.total_tokens, seed=w.seed)
    finally:
        dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_gloo_ranks(tmp_path):
    world = 2
    mp.start_processes(_worker, args=(world, _free_port(), str(tmp_path)), nprocs=world,
                       start_method="spawn", join=True)
    r0 = np.load(tmp_path / "r0.npz")
    r1 = np.load(tmp_path / "r1.npz")
    assert float(r0["mx"]) == float(r1["mx"]) == 15.0       # max over ranks
    assert int(r0["tokens"]) == int(r1["tokens"])            # weak scaling: same shapes
    assert int(r0["seed"]) != int(r1["seed"])                # ... different prompts
    assert r0["h"].shape == r1["h"].shape and not np.array_equal(r0["h"], r1["h"])
    expect = 2 * int(r0["tokens"]) * 7 / 0.015
    assert float(r0["value"]) == pytest.approx(expect) == float(r1["value"])
