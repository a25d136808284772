"""Write tests/golden/tiny_oracle.json: the fp64 oracle's output on the tiny workload.

Calls only the oracle (and the seeded input generator).  The stored values
anchor the oracle against later edits (tests/test_oracle_pins.py reproduces
them) and give the GPU test of the tiny fp32 workload a fixed expectation.
Run from the repository root:  python tests/golden/make_golden.py
"""
import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import oracle  # noqa: E402
from linear_vision_backbone_b200 import inputs  # noqa: E402


def main():
    wl = inputs.WORKLOADS["tiny"]
    d = inputs.make_inputs(wl)
    y = oracle.gla_fwd(d["q"], d["k"], d["v"], d["g"], d["z"], d["w"], gh=wl.gh, gw=wl.gw,
                       direction="LR")
    doc = {
        "what": "fp64 oracle output y [B,T,H,dv] of the tiny workload (B1 H1 8x8 d16 fp32 LR, seed 0)",
        "source": "oracle/gla_oracle.c oracle_gla_fwd_f64 via tests/golden/make_golden.py",
        "operator": "GTR article (shuwu5.cn/article/3124), 方法详解 §1: Key-only gated recurrence, "
                    "RMSNorm x SiLU output gate",
        "shape": list(y.shape),
        "y": [float.hex(float(v)) for v in y.ravel()],
    }
    with open(os.path.join(HERE, "tiny_oracle.json"), "w") as f:
        json.dump(doc, f, indent=0)


if __name__ == "__main__":
    main()
