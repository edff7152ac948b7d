"""The bounded-wait path: a kernel whose wait expires sets the device error flag and winds
down, the call reports DREAMER_ERR_TIMEOUT, and the handle works again afterwards.

Runs the test-hook build of the library (the product's sources compiled with a 20 ms wait
limit and dreamer_test_inject): the injected call's first QKV projection GEMM issues no TMA
loads, so no operand ever arrives and its MMA issuer's wait on the first stage runs out.  No
MMA is issued and no copy is in flight when the CTAs exit, so nothing faults; every other
role sees the CTA's abort word and leaves its loop.
"""
import pytest

from depth_recurrent_attention_b200 import configs, inputs

pytestmark = pytest.mark.gpu


def test_expired_wait_returns_timeout_and_the_handle_recovers(cuda):
    import torch
    from depth_recurrent_attention_b200 import dreamer as D
    cfg = configs.SMALL.with_(depth=2)
    W = {k: inputs.to_device(v, "fp32" if k == "bias" else cfg.dtype)
         for k, v in inputs.host_weights(cfg).items()}
    x0 = inputs.to_device(inputs.host_inputs(cfg)["x0"], cfg.dtype)
    dev = D.Dreamer(cfg, W, lib_path=D.TESTHOOKS_PATH)
    ref = dev.forward(x0).clone()
    dev.route_counts(on_host=True)                  # synchronises; no error so far
    dev.test_inject(1)
    bad = dev.forward(x0)                           # enqueued; the error is found on the device
    with pytest.raises(D.DreamerError) as e:
        dev.route_counts(on_host=True)
    assert e.value.code == D.ERR_TIMEOUT
    del bad
    # the flag was cleared by the report: the handle and the context work again
    for _ in range(3):                              # direct, captured, replayed
        out = dev.forward(x0)
    counts = dev.route_counts(on_host=True)
    torch.cuda.synchronize()
    assert int(counts.sum()) == cfg.tokens * cfg.top_k * cfg.depth
    diff = float((out.float() - ref.float()).abs().max())
    assert torch.equal(out, ref), f"max-abs {diff}"
    dev.close()
