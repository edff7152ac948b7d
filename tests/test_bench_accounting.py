"""The algorithmic FLOP and byte counts behind the bench line's roofline fractions, pinned to
numbers worked out by hand for the small workload (b 4, s 512, h 512, 8x64, L 8, E 256, k 4,
m 64, d_r 64, bf16)."""
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

# per depth (2-byte values): norm 4 T h = 4 194 304; QKV T h 2 + 6h h 2 + T 6h 2 = 17 825 792;
# SA 8 T h = 8 388 608; O T 2h 2 + 2h h 2 + T h (2 + 4) = 11 534 336;
# EA T h 2 + h d_r 2 + E d_r 2 = 2 195 456; FFN (all 256 experts) 2 E h m 2 + T h 2 + 8 T h =
# 44 040 192.  DA over all depths: 8 (T h 2 + T h 2) + T 2h 2 (0 + 1 + ... + 7) = 150 994 944
SMALL_BYTES = 8 * (4_194_304 + 17_825_792 + 8_388_608 + 11_534_336 + 2_195_456
                   + 44_040_192) + 150_994_944


def test_small_totals_match_the_hand_count():
    st, f, b = bench.algorithmic(configs.SMALL)
    assert f == SMALL_FLOPS == 87_677_730_816
    assert b == SMALL_BYTES == 856_424_448
    assert st["qkv"][0] == 8 * 6_442_450_944
    assert st["da"] == (150_994_944, 150_994_944)


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
    # window 2: depths attend to min(l + 1, 2) states, 1 + 2 * 7 = 15 in all
    st, _, _ = bench.algorithmic(cfg.with_(da_window=2))
    assert st["da"][0] == 4.0 * T * h * 15
    assert st["da"][1] == 8 * 2 * T * h * 2 + 2 * T * h * 2 * 7
    # without DA: half-width projections, no DA stage
    st, f, _ = bench.algorithmic(cfg.with_(variant=3))
    assert "da" not in st
    assert st["qkv"][0] == 8 * 2.0 * T * h * 3 * h
    assert st["o_proj"][0] == 8 * 2.0 * T * h * h
    assert f == SMALL_FLOPS - 150_994_944 - 8 * (3_221_225_472 + 1_073_741_824)
