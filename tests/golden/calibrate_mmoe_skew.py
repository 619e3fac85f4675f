"""Calibrate the zero-computation logit biases of the skewed MMOE workloads.

The MMOE page ("routing analysis") reports that the lightweight experts
(identity / zero / constant) take 44.6 % of the routing in early blocks and
23.4 % in late blocks. This script finds, for each share, the logit bias
added to those three experts for which the oracle's own top-2 routing of
the seeded `mmoe` inputs sends that share of the routed slots to them, by
bisection. It calls only the oracle and the input generator; its printed
values are MMOE_SKEW_BIAS (early) and MMOE_LATE_BIAS (late) in
mixture_experts_layer_33_b200/inputs.py.

    python tests/golden/calibrate_mmoe_skew.py
"""

import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from mixture_experts_layer_33_b200 import inputs as gen  # noqa: E402

TARGETS = {"early": 0.446, "late": 0.234}


def lightweight_share(cfg, hin, bias):
    b = np.array([bias if k != gen.HEAVY else 0.0 for k in cfg["kinds"]])
    z = oracle.router_logits(hin["x"], hin["W_r"], b, hin["z_prev"], cfg["gate_residual_scale"])
    idx = oracle.topk_token_choice(z, cfg["k"])
    return float(np.mean(idx >= cfg["E_heavy"]))


def calibrate(cfg, hin, target):
    lo, hi = -4.0, 4.0
    for _ in range(24):
        mid = 0.5 * (lo + hi)
        if lightweight_share(cfg, hin, mid) < target:
            lo = mid
        else:
            hi = mid
    return round(0.5 * (lo + hi), 4)


def main():
    cfg = gen.workload("mmoe")
    inp = gen.make_inputs(cfg, "cpu")
    hin = {k: gen.to_numpy_f32(inp[k]) for k in ("x", "W_r", "z_prev")}
    print(f"no bias: lightweight share {lightweight_share(cfg, hin, 0.0):.4f}")
    for name, target in TARGETS.items():
        bias = calibrate(cfg, hin, target)
        print(f"{name} ({target}): bias {bias}, lightweight share "
              f"{lightweight_share(cfg, hin, bias):.4f}")


if __name__ == "__main__":
    main()
