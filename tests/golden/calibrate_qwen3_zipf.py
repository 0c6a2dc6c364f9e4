"""Re-derive the Zipf scale of the Qwen3-shaped layer's logit bias.

The workload asks for a log-Zipf(s=1.2) router bias that produces a max/mean
expert-load ratio of about 3.  Applied literally, s = 1.2 gives a far larger
ratio, so the bias is scaled by alpha, chosen here by bisection on seed 0 so
that max/mean of the per-expert assignment counts (before capacity) is 3.
Routing is computed by the oracle only.  Run: python tests/golden/calibrate_qwen3_zipf.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from routing_dispatch_expert_sigmoid_b200.workloads import WORKLOADS, make_inputs, to_numpy  # noqa: E402


def main():
    w = WORKLOADS["qwen3_prefill"].scaled(zipf_s=1.0)
    inp = make_inputs(w, seed=0)
    x, Wr = to_numpy(inp["x"]), to_numpy(inp["Wr"])
    log_rank = -to_numpy(inp["logit_bias"]).astype(np.float64)   # ln(rank_e) for s = 1
    logits = oracle.router_logits(x, Wr)

    def ratio(alpha):
        l32 = (logits - 1.2 * alpha * log_rank).astype(np.float32)
        idx, _ = oracle.gating(l32, w.k_max, w.gating)
        counts = oracle.capacity_dispatch(idx, w.E, w.capacity_factor)["counts"]
        return counts.max() / counts.mean(), counts

    lo, hi = 0.0, 1.0
    for _ in range(30):
        mid = 0.5 * (lo + hi)
        if ratio(mid)[0] < 3.0:
            lo = mid
        else:
            hi = mid
    r, counts = ratio(round(hi, 2))
    print(f"alpha={hi:.4f} (rounded {round(hi, 2)}): max/mean={r:.3f} "
          f"drops={np.maximum(counts - 1024, 0).sum() / counts.sum():.3f}")


if __name__ == "__main__":
    main()
