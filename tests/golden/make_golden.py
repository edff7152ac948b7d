"""Writes tests/golden/tiny_oracle.json from the CPU oracle alone.

The pages print no worked example with numbers (no tensor values, no scores), so the only
stored expected values are regression fixtures of the oracle on the seeded tiny workload
(b=1, s=16, h=64, 4x16 heads, L=4, E=16, k=2, m=16, fp32, seed 0).  Run from the repo root:
    python tests/golden/make_golden.py
"""
import json
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path[:0] = [ROOT, os.path.join(ROOT, "oracle")]

from depth_recurrent_attention_b200 import configs, inputs  # noqa: E402
import oracle as O  # noqa: E402


def main():
    cfg = configs.TINY
    o = O.Oracle(cfg, inputs.host_weights(cfg), threads=1)
    r = o.forward(inputs.host_inputs(cfg)["x0"])
    out = dict(
        workload="tiny fp32: b=1 s=16 h=64 H=4 d=16 L=4 E=16 k=2 m=16 d_r=16 seed=0",
        written_by="tests/golden/make_golden.py (oracle only)",
        x_out=[[float(v) for v in row] for row in r["x_out"]],
        idx=r["idx"].tolist(),
        counts=r["counts"].tolist(),
        min_margin=float(r["margin"].min()),
    )
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as f:
        json.dump(out, f, indent=1)
    print(path)


if __name__ == "__main__":
    main()
