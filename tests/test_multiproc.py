"""Host logic of the N > 1 bench path on CPU: two gloo ranks (world size 2, 127.0.0.1).

bench.py runs one full replica per GPU; nothing crosses ranks on the data path.  What the
ranks share is host logic, checked here without a GPU: the timed region is the slowest
rank's (all-reduce MAX), the job's value counts every rank's units over that time, each
rank draws its own input batch from its own seed while the weights are identical, and the
ranks leave the process group cleanly.
"""
import os
import socket

import numpy as np
import pytest

from depth_recurrent_attention_b200 import configs, inputs


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out_q):
    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    import bench
    cfg = configs.SMALL
    steps = 4
    ms_total = [10.0, 14.0][rank]               # the second rank is the slower one
    m = bench.max_over_ranks(ms_total, dist, torch.device("cpu"))
    units, value = bench.job_value(cfg, world, m / steps)
    spec = inputs.input_specs(cfg)[0]
    x = inputs.draw(spec, bench.rank_seed(cfg, rank), 0, 4096)
    w = inputs.draw(inputs.weight_specs(cfg)[0], cfg.seed, 0, 4096)
    out_q.put((rank, m, units, value, float(np.sum(x)), float(np.sum(w))))
    dist.barrier()
    dist.destroy_process_group()


def test_two_gloo_ranks():
    import torch.multiprocessing as mp
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(2):
        r = q.get(timeout=120)
        res[r[0]] = r
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    cfg = configs.SMALL
    for r in range(2):
        _, m, units, value, _, _ = res[r]
        assert m == 14.0                                   # max over ranks
        assert units == 2 * cfg.units                      # whole-job units
        assert value == pytest.approx(2 * cfg.units / (14.0 / 4 / 1e3))
    assert res[0][4] != res[1][4]                          # each rank its own batch
    assert res[0][5] == res[1][5]                          # shared weights


def test_single_rank_helpers():
    import bench
    cfg = configs.MEDIUM
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    units, value = bench.job_value(cfg, 1, 2.0)
    assert units == cfg.units and value == pytest.approx(cfg.units / 2e-3)
    assert bench.rank_seed(cfg, 0) == cfg.seed and bench.rank_seed(cfg, 3) != cfg.seed
