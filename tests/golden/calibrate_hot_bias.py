"""Find beta for the skewed B=64 workload (32 hot router rows get beta * u added, u ~ N(0,1/H)).

The workload asks that the hot experts receive about half of all selections.  A shared
bias on the hot rows shifts every hot logit of a token by the same s = beta * (u . x), which
is ~N(0, beta^2); as beta grows a layer's hot share tends to the fraction of its tokens with
s > 0 (those pick mostly hot experts, the others almost none).  On one layer that fraction is
a coin-flip count (28 of 64 on layer 0), so the share is taken over all 32 timed layers, each
with its own hot set and bias vector, where it tends to 1/2.  This script walks the grid
beta = 4, 8, 12, ... and prints the first beta whose hot share of the 32 x 64 x 16 selections
lies in [0.45, 0.55], using only the seeded generator and the CPU oracle's routing.  The value
is recorded as ``synth.HOT_BETA_B64`` and re-checked by ``tests/test_synth.py``.

Run:  python tests/golden/calibrate_hot_bias.py
"""
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
import oracle  # noqa: E402
import synth  # noqa: E402


def hot_share(beta: float, layer: int = 0) -> float:
    """Fraction of one layer's 64 x 16 selections that fall in its hot set."""
    w = synth.WORKLOADS["full_b64_skewed"]
    R = synth.router_weights(w, layer, beta)
    x = synth.tokens(w)
    _, idx, _ = oracle.route(R, x, w.dims.top_k)
    return float(np.isin(idx, synth.hot_set(w, layer)).mean())


def mean_hot_share(beta: float) -> float:
    w = synth.WORKLOADS["full_b64_skewed"]
    return float(np.mean([hot_share(beta, layer) for layer in range(w.layers)]))


def main():
    for beta in np.arange(4.0, 204.0, 4.0):
        share = mean_hot_share(beta)
        print(f"beta={beta:6.1f}  hot share over 32 layers={share:.4f}", flush=True)
        if 0.45 <= share <= 0.55:
            print(f"HOT_BETA_B64 = {beta}")
            return
    raise SystemExit("no beta on the grid reached the target share")


if __name__ == "__main__":
    main()
