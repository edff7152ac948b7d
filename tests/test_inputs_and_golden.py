"""Seeded input generator (no method arithmetic) and the oracle's regression fixture."""
import json
import os

import numpy as np

import oracle as O
from depth_recurrent_attention_b200 import configs, inputs

HERE = os.path.dirname(os.path.abspath(__file__))


def test_splitmix64_published_first_outputs():
    # splitmix64 seeded with 0 starts 0xE220A8397B1DCDAF, 0x6E789E6AA1B965F4 (Vigna's
    # reference implementation of Steele/Lea/Flood's generator)
    r = inputs._raw(0, 0, 2)
    assert int(r[0]) == 0xE220A8397B1DCDAF and int(r[1]) == 0x6E789E6AA1B965F4


def test_random_access_and_statistics():
    key = inputs.stream_key(7, 3)
    full = inputs.normal(key, 0, 100001)
    assert np.array_equal(inputs.normal(key, 12345, 999), full[12345:13344])
    assert np.array_equal(inputs.normal(key, 1, 1), full[1:2])
    assert abs(full.mean()) < 0.01 and abs(full.std() - 1) < 0.01
    u = inputs.uniform(key, 0, 100000, 0.1)
    assert u.min() >= -0.1 and u.max() < 0.1 and abs(u.mean()) < 0.002


def test_bf16_rounding_is_nearest_even():
    x = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, 1.0 + 2 ** -9, -2.5], np.float32)
    bits = inputs.f32_to_bf16_bits(x)
    back = inputs.bf16_bits_to_f32(bits)
    # 1 + 2^-8 is a tie between 1 and 1 + 2^-7 -> even (1); 1 + 3*2^-8 -> 1 + 2^-6
    assert np.array_equal(back, np.array([1.0, 1.0, 1.0 + 2 ** -6, 1.0, -2.5], np.float32))


def test_weight_specs_follow_fan_in():
    cfg = configs.MEDIUM
    sp = {s.name: s for s in inputs.weight_specs(cfg)}
    assert sp["w_qkv"].shape == (8, 1024, 6144) and np.isclose(sp["w_qkv"].param, 1 / 32)
    assert sp["w2"].shape == (1024, 32, 1024) and np.isclose(sp["w2"].param, 1 / np.sqrt(32))
    assert sp["bias"].dtype == "fp32" and sp["k_E"].param == 1.0
    w = inputs.draw(sp["w_qkv"], cfg.seed, 0, 1 << 16)
    bits = inputs.f32_to_bf16_bits(w)
    assert np.array_equal(inputs.bf16_bits_to_f32(bits), w)      # exact bf16 values


def test_oracle_regression_fixture():
    with open(os.path.join(HERE, "golden", "tiny_oracle.json")) as f:
        g = json.load(f)
    cfg = configs.TINY
    r = O.Oracle(cfg, inputs.host_weights(cfg), threads=1).forward(
        inputs.host_inputs(cfg)["x0"])
    assert np.allclose(r["x_out"], np.array(g["x_out"]), rtol=1e-12, atol=1e-12)
    assert np.array_equal(r["idx"], np.array(g["idx"]))
    assert np.array_equal(r["counts"], np.array(g["counts"]))
