"""Write ``zero_share_beta.json``: the zero-expert selection offset per seed.

For the large-expert-count layer the bias input is U(-0.1, 0.1) plus one offset
beta on every zero expert, chosen so that about 30 % of all routing slots land
on zero experts (the share that the model card's 33-56B activated range
implies, see the card arithmetic test). beta is found by bisection on the
oracle's fp64 router: the logits are computed once, then only the selection is
repeated. Run:  python -m moe_synth.tune_zero_share [seeds...]
"""
import json
import sys

import numpy as np

import oracle
from moe_synth import BETA_FILE, CONFIGS, base_bias, beta_key, load_betas, make_router_inputs

TARGET = 0.30


def tune(shape, seed, lo=-4.0, hi=4.0, iters=40):
    x, w_r, _ = make_router_inputs(shape, seed, beta=0.0)
    logits = oracle.router_logits(x, w_r)
    b0 = base_bias(shape, seed).numpy()

    def share(beta):
        b = b0.copy()
        b[shape.n_routed:] += np.float32(beta)
        idx, _, _ = oracle.select(logits, b, shape.top_k)
        return float((idx >= shape.n_routed).mean())

    for _ in range(iters):
        mid = 0.5 * (lo + hi)
        if share(mid) < TARGET:
            lo = mid
        else:
            hi = mid
    beta = float(np.float32(0.5 * (lo + hi)))
    return beta, share(beta)


def main(seeds):
    shape = CONFIGS["large_e"]
    table = load_betas()
    for seed in seeds:
        beta, sh = tune(shape, seed)
        table[beta_key(shape, seed)] = {"beta": beta, "zero_share": sh}
        print(seed, beta, sh, flush=True)
    with open(BETA_FILE, "w") as f:
        json.dump(table, f, indent=1, sort_keys=True)


if __name__ == "__main__":
    main([int(s) for s in sys.argv[1:]] or [0, 1, 2])
