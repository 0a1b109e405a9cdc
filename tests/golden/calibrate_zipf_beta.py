"""Derive the Zipf-bias multiplier beta of the wide (256-expert, top-10) layer.

The layer statement asks for a Zipf(s=1.1) router bias "so ~80% of hits land in
the top 64" experts.  The bias is b_e = -beta * s * ln(rank_e); with beta = 1
(the plain log-pmf) top-10 selection sharpens the distribution and ~98% of
hits land in the top 64, so beta is found by bisection on the seed-0 tokens
until the share is 0.80.  Calls only the oracle router and the input
generator; prints beta, which is stored as synth.WIDE_ZIPF_BETA.

    python tests/golden/calibrate_zipf_beta.py
"""
import dataclasses
import os
import sys

import numpy as np

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__)))))
import oracle  # noqa: E402
from quantized_routed_expert_04_b200 import synth  # noqa: E402


def share(beta, n_tokens=256):
    cfg = dataclasses.replace(synth.CONFIGS["wide"], zipf_beta=beta)
    W, b = synth.make_router(cfg)
    ranks = synth.zipf_ranks(cfg)
    x = synth.make_x(cfg, n_tokens, step=0)
    _, idx, _ = oracle.route(x, W, b, cfg.top_k)
    return float(np.mean(ranks[idx.reshape(-1)] <= 64))


def main():
    lo, hi = 0.0, 1.0
    for _ in range(12):
        mid = (lo + hi) / 2
        if share(mid) < 0.80:
            lo = mid
        else:
            hi = mid
    beta = round(hi * 256) / 256   # a short binary fraction
    print("beta = %.6f  share = %.4f  (beta=1: %.4f)" % (beta, share(beta), share(1.0)))


if __name__ == "__main__":
    main()
