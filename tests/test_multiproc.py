"""Host logic of the N > 1 bench path on CPU: two gloo ranks (world size 2, 127.0.0.1).

bench.py runs one full replica per GPU; nothing crosses ranks on the data path.  What the
ranks share is host logic, checked here without a GPU: the timed region is the slowest
rank's (all-reduce MAX), the job's value counts every rank's units over that time, each
rank draws its own input batch from its own seed while the weights are identical, and the
ranks leave the process group cleanly.  The one exchange of the replicas, the all-reduce of
the [L][E] route counts before a bias-balance update, runs here on CPU tensors: every rank
gets the sum and computes the same update from it.
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


def _rank_counts(cfg, rank):
    """A rank's [L][E] route counts: each depth routes T k slots, spread unevenly."""
    rng = np.random.default_rng(100 + rank)
    c = np.zeros((cfg.depth, cfg.n_experts), np.int32)
    for l in range(cfg.depth):
        e = rng.integers(0, cfg.n_experts, cfg.tokens * cfg.top_k)
        np.add.at(c[l], e, 1)
    return c


def _worker(rank, world, port, out_q):
    import sys
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
    # route counts of this rank's batch, summed over the ranks, then the bias update from them
    from depth_recurrent_attention_b200.dreamer import allreduce_route_counts
    sys.path.insert(0, os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))),
                                    "oracle"))
    import oracle as O
    counts = allreduce_route_counts(torch.from_numpy(_rank_counts(cfg, rank)))
    bias0 = inputs.host_weights(configs.TINY)["bias"].astype(np.float64)
    tiny_counts = counts[:configs.TINY.depth, :configs.TINY.n_experts].numpy()
    new_b = O.bias_update(np.ascontiguousarray(tiny_counts), 0.01, bias0)
    out_q.put((rank, m, units, value, float(np.sum(x)), float(np.sum(w)), counts.numpy(), new_b))
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
        _, m, units, value, _, _, _, _ = res[r]
        assert m == 14.0                                   # max over ranks
        assert units == 2 * cfg.units                      # whole-job units
        assert value == pytest.approx(2 * cfg.units / (14.0 / 4 / 1e3))
    assert res[0][4] != res[1][4]                          # each rank its own batch
    assert res[0][5] == res[1][5]                          # shared weights
    total = _rank_counts(cfg, 0) + _rank_counts(cfg, 1)
    for r in range(2):                                     # the all-reduced route counts
        assert np.array_equal(res[r][6], total)
    assert np.array_equal(res[0][7], res[1][7])            # the same bias update everywhere


def test_single_rank_helpers():
    import bench
    cfg = configs.MEDIUM
    assert bench.max_over_ranks(3.5, None, None) == 3.5
    units, value = bench.job_value(cfg, 1, 2.0)
    assert units == cfg.units and value == pytest.approx(cfg.units / 2e-3)
    assert bench.rank_seed(cfg, 0) == cfg.seed and bench.rank_seed(cfg, 3) != cfg.seed
    # without a process group the count exchange leaves the counts as they are
    import torch
    from depth_recurrent_attention_b200.dreamer import allreduce_route_counts
    c = torch.arange(12, dtype=torch.int32).reshape(3, 4)
    assert torch.equal(allreduce_route_counts(c.clone()), c)
