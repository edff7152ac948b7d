"""The algorithmic FLOP and byte counts behind the bench line's roofline fractions, pinned to
hand counts and to the workload table of the roofline accounting (small 0.55 GB, medium
16.6 GB, large 442 GB: perfect on-chip reuse inside a depth step, none across depths)."""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402
from depth_recurrent_attention_b200 import configs  # noqa: E402

# per depth, T = 2048 tokens:
#   QKV   2 T h 6h                       = 6 442 450 944
#   SA    4 h b s (s + 1) / 2            = 1 075 838 976   (causal half)
#   O     2 T 2h h                       = 2 147 483 648
#   EA    2 T h d_r + 2 T E d_r          =   201 326 592
#   FFN   4 T k h m                      = 1 073 741 824
# DA over all depths: 4 T h (1 + 2 + ... + 8) = 4 T h 36 = 150 994 944
SMALL_FLOPS = 8 * (6_442_450_944 + 1_075_838_976 + 2_147_483_648 + 201_326_592
                   + 1_073_741_824) + 150_994_944

# per depth (2-byte values, T = 2048, h = 512):
#   residual x read and written        4 T h     =  4 194 304
#   DA keys/values written             4 T h     =  4 194 304
#   SA keys/values written and read    8 T h     =  8 388 608
#   QKV and O weights                  (6 + 2) h^2 2 = 4 194 304
#   router query and keys              (h + E) d_r 2 =    98 304
#   expert weights (all 256 touched)   2 E h m 2     = 33 554 432
# DA re-reads of earlier depths: 4 T h (0 + 1 + ... + 7) = 117 440 512
SMALL_BYTES = 8 * (4_194_304 + 4_194_304 + 8_388_608 + 4_194_304 + 98_304
                   + 33_554_432) + 117_440_512


def test_small_totals_match_the_hand_count():
    st, f, b = bench.algorithmic(configs.SMALL)
    assert f == SMALL_FLOPS == 87_677_730_816
    assert b == SMALL_BYTES == 554_434_560
    assert st["qkv"][0] == 8 * 6_442_450_944
    assert st["da"] == (150_994_944, 117_440_512)


def test_workload_table_totals():
    """The roofline table's byte totals: medium 16.6 GB (DA 9.1), large 442 GB (DA 279)."""
    _, f, b = bench.algorithmic(configs.MEDIUM)
    assert round(b / 1e9, 1) == 16.6 and round(f / 1e12, 2) == 5.89
    st, f, b = bench.algorithmic(configs.LARGE)
    assert round(b / 1e9) == 442 and round(f / 1e12, 1) == 111.9
    T, h, L = configs.LARGE.tokens, configs.LARGE.hidden, configs.LARGE.depth
    da_bytes = st["da"][1] + 4 * T * h * L           # re-reads + the writes (in the qkv stage)
    assert round(da_bytes / 1e9) == 279


def test_untouched_experts_drop_their_weight_bytes():
    cfg = configs.SMALL
    counts = np.ones((cfg.depth, cfg.n_experts), np.int64)
    counts[3, 17] = 0
    counts[5, :4] = 0
    _, f, b = bench.algorithmic(cfg, counts)
    per_expert = 2 * cfg.hidden * cfg.expert_hidden * 2  # W1_e and W2_e, bf16
    assert f == SMALL_FLOPS
    assert b == SMALL_BYTES - 5 * per_expert


def test_da_window_and_no_da_arms():
    cfg = configs.SMALL
    T, h = cfg.tokens, cfg.hidden
    # window 2: depths attend to min(l + 1, 2) states, 1 + 2 * 7 = 15 in all; one earlier
    # depth re-read by each of depths 1..7
    st, _, _ = bench.algorithmic(cfg.with_(da_window=2))
    assert st["da"][0] == 4.0 * T * h * 15
    assert st["da"][1] == 2 * T * h * 2 * 7
    # without DA: half-width projections, no DA stage, no DA keys/values written
    st, f, b = bench.algorithmic(cfg.with_(variant=3))
    assert "da" not in st
    assert st["qkv"][0] == 8 * 2.0 * T * h * 3 * h
    assert st["o_proj"][0] == 8 * 2.0 * T * h * h
    assert f == SMALL_FLOPS - 150_994_944 - 8 * (3_221_225_472 + 1_073_741_824)
    assert b == SMALL_BYTES - 117_440_512 - 8 * (4_194_304 + 4 * h * h * 2)


def test_tensor_peak_follows_the_length_of_the_timed_loop():
    """Kernels timed inside a loop of a second or more run at the power cap: they are held to
    the sustained GEMM rate; shorter loops to the burst rate; the other rate is reported."""
    pk = dict(hbm=6650.0, tc=1590.0, tc_sust=1400.0, source="fallback")
    assert bench.tensor_peaks(pk, 2041.0) == (1400.0, 1590.0, "sustained")
    assert bench.tensor_peaks(pk, 1000.0) == (1400.0, 1590.0, "sustained")
    assert bench.tensor_peaks(pk, 150.9) == (1590.0, 1400.0, "burst")
    fb = bench.peaks()
    if fb["source"] == "fallback":
        assert (fb["hbm"], fb["tc"], fb["tc_sust"]) == (6650.0, 1590.0, 1400.0)


def test_reference_arm_line_on_a_tiny_workload():
    """The reference arm (the oracle on the host cores) prints the bench line's keys with
    impl "reference", a positive value, its own cpu_baseline and an e2e entry without copies."""
    import json
    import types
    cfg = configs.TINY
    args = types.SimpleNamespace(steps=2, warmup=1, gpus=1)
    line = bench.run_reference(args, cfg)
    json.dumps(line)
    assert line["impl"] == "reference" and line["value"] > 0 and line["unit"] == bench.UNIT
    assert line["config"]["workload"].startswith("tiny")
    cb = line["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == line["value"] and cb["cores"] >= 1
    assert "depths 0..3 of 4" in cb["sample"]
    assert line["e2e"]["h2d_bytes_per_step"] == 0 and line["e2e"]["value"] == line["value"]
