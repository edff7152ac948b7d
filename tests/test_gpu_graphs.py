"""Repeated calls on the same buffers: the first runs the kernels directly, the second captures
them into a CUDA graph, later ones replay it (the form bench.py times).  Every call must give
the same output, bit for bit (the forward has no order-dependent floating-point atomics), and
the same route counts; a call with a trace (direct, with dumps between kernels) as well."""
import numpy as np
import pytest

from depth_recurrent_attention_b200 import configs, inputs

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("name,kw", [
    ("small", {}),
    ("small", dict(variant=2)),                       # expert attention on a third stream
    ("small", dict(n_proj_experts=8, depth=3)),       # grouped projections, tile tables
    ("small", dict(variant=1, depth=3)),
    ("medium", dict(depth=4)),
    ("large", dict(depth=2, batch=1, seq=2048)),
])
def test_graph_replay_equals_direct_run(cuda, name, kw):
    import torch
    from depth_recurrent_attention_b200.dreamer import Dreamer
    cfg = configs.CONFIGS[name].with_(**kw)
    W = inputs.device_weights(cfg)
    x0 = inputs.device_inputs(cfg)["x0"]
    dev = Dreamer(cfg, W)
    out = torch.empty_like(x0)
    outs, counts = [], []
    for _ in range(4):
        dev.forward(x0, x_out=out)
        outs.append(out.clone())
        counts.append(dev.route_counts(on_host=True).clone())
    tr = dict(y=torch.empty((cfg.depth, cfg.tokens, cfg.hidden), dtype=x0.dtype, device="cuda"))
    traced = dev.forward(x0, trace=tr)
    counts.append(dev.route_counts(on_host=True).clone())
    torch.cuda.synchronize()
    for i, o in enumerate(outs[1:] + [traced]):
        d = float((o.float() - outs[0].float()).abs().max())
        assert torch.equal(o, outs[0]), f"call {i + 1}: max-abs {d} from the first call"
    for c in counts[1:]:
        assert torch.equal(c, counts[0])
    dev.close()


def test_decode_graph_replay_equals_direct_run(cuda):
    import torch
    from depth_recurrent_attention_b200.dreamer import Dreamer
    cfg = configs.DECODE.with_(depth=4)
    W = inputs.device_weights(cfg)
    X = inputs.device_inputs(cfg)
    lens = torch.full((cfg.batch,), cfg.cache_len, dtype=torch.int32, device="cuda")
    dev = Dreamer(cfg, W)
    out = torch.empty_like(X["x0"])
    outs = []
    for _ in range(4):  # the same slot of every cache is rewritten with the same values
        dev.decode_step(X["x0"], X["k_cache"], X["v_cache"], lens, x_out=out)
        outs.append(out.clone())
    torch.cuda.synchronize()
    for i, o in enumerate(outs[1:]):
        assert torch.equal(o, outs[0]), f"call {i + 1}"
    dev.close()
