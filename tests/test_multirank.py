"""The N > 1 plumbing of bench.py on CPU: two gloo ranks, as torchrun would
launch them (RANK / WORLD_SIZE / MASTER_* in the environment).  Every
(batch, head) slice is independent, so the ranks run replicas: the only
collective steps are the barrier and the max over ranks of the device time,
and each rank draws its own inputs."""
import importlib.util
import os
import socket

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench():
    spec = importlib.util.spec_from_file_location("bench_under_test", os.path.join(ROOT, "bench.py"))
    m = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(m)
    return m


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank: int, world: int, port: int, out_dir: str):
    os.environ.update(RANK=str(rank), LOCAL_RANK=str(rank), WORLD_SIZE=str(world),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch.distributed as dist
    b = _bench()
    r, local, w, pg = b.dist_setup(world)
    assert (r, local, w, pg) == (rank, rank, world, True)
    assert dist.get_backend() == "gloo"
    b.barrier(pg)
    # each rank reports a different "device time"; all must agree on the max
    mx = b.max_over_ranks(10.0 + rank, pg, "cpu")
    b.barrier(pg)
    dist.destroy_process_group()
    np.save(os.path.join(out_dir, f"rank{rank}.npy"), np.array([mx]))


def test_two_gloo_ranks_agree_on_the_max_time(tmp_path):
    import torch.multiprocessing as mp
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, str(tmp_path)), nprocs=2, join=True, start_method="spawn")
    got = [float(np.load(os.path.join(tmp_path, f"rank{r}.npy"))[0]) for r in range(2)]
    assert got == [11.0, 11.0]


def test_single_process_needs_no_process_group(monkeypatch):
    for k in ("RANK", "WORLD_SIZE", "LOCAL_RANK"):
        monkeypatch.delenv(k, raising=False)
    b = _bench()
    assert b.dist_setup(1) == (0, 0, 1, False)
    assert b.max_over_ranks(3.5, False, "cpu") == 3.5


def test_replicas_draw_distinct_inputs():
    """bench.py seeds rank r's replica with 1000 r: the ranks do not time the
    same tensors."""
    import synthetic
    a, _, _ = synthetic.qkv(0, 1, 1, 32, 32, 64, 4.0)
    b, _, _ = synthetic.qkv(1000, 1, 1, 32, 32, 64, 4.0)
    assert a.shape == b.shape and not np.allclose(a, b)
