"""Find the draft-noise sigma of the single-stream Llama-3-vocabulary workload.

Bisects sigma until the mean over the K=5 positions of the oracle's acceptance
probability sum_v min(p_i(v), q_i(v)) is 0.75 +- 0.01 (the speculative decoding
blog measures 67-84% acceptance at K=5, section "The numbers: actual
measurement on Llama 3.1-70B").  Calls only the CPU oracle; prints the value
that speculative_sampling_b200/inputs.py stores as LLAMA_SINGLE_SIGMA.

    python -m oracle.calibrate_sigma
"""
import numpy as np

import oracle
from speculative_sampling_b200 import inputs

NAME = "llama3_single_b1_k5_v128256_bf16"


def mean_acceptance(sigma: float) -> float:
    x = inputs.generate(NAME, sigma=sigma)
    r = oracle.verify(x.target, x.draft, x.tokens, x.u_accept, x.u_resample, x.temperature)
    return float(np.mean(r["accept_prob"]))


def main(target: float = 0.75, tol: float = 0.01) -> float:
    lo, hi = 0.05, 5.0  # acceptance falls as sigma grows
    for _ in range(40):
        mid = 0.5 * (lo + hi)
        a = mean_acceptance(mid)
        if abs(a - target) <= tol / 4:
            break
        if a > target:
            lo = mid
        else:
            hi = mid
    mid = round(mid, 3)
    print(f"sigma={mid} mean_acceptance={mean_acceptance(mid):.4f}")
    return mid


if __name__ == "__main__":
    main()
